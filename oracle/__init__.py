"""CPU oracle (test infrastructure only; never imported by the product path)."""
from .oracle import *  # noqa: F401,F403
from . import oracle as core  # noqa: F401
