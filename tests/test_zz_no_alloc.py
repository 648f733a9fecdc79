"""The allocation-free forward (qlora_linear_fwd_noalloc) against the regular
one (qlora_linear_fwd), through the C ABI.

Some callers cannot allocate device memory at call time -- for example a
plugin inside a serving runtime that owns all of the GPU's memory and hands the
layer only its input and output buffers.  For them the library offers a
forward whose scratch is a fixed array inside the library itself.  This file
checks that it computes what the regular forward computes, on two calls in a
row (the array keeps the previous call's contents), and that sizes the array
cannot hold are refused before anything is launched.  It is named so that
pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from bit_nf4_quantized_20_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 5e-3, 1e-2


def _close(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g))
    bad = np.abs(g - r) > TOL_ABS + TOL_REL * np.abs(r)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} elements differ beyond tolerance"


def _largest_T_that_fits(N, K, r):
    import bit_nf4_quantized_20_b200 as q
    L = q.lib()
    lo, hi = 17, 1 << 16
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if L.qlora_workspace_bytes(1, mid, N, K, r) <= (4 << 20):
            lo = mid
        else:
            hi = mid - 1
    return lo


@pytest.mark.parametrize("T,N,K,r,s", [
    (16, 512, 512, 8, 2.0),       # decode-sized path
    (300, 384, 320, 24, 0.5),     # tensor-core path, ragged token tile and rank
    (4, 1024, 320, 16, 1.0),      # decode-sized, K not a multiple of 256 (per-tile GEMV)
    (16, 14336, 4096, 128, 1.0),  # 8B gate shape, 16 tokens, the largest rank
    (16, 4096, 14336, 100, 0.5),  # 8B down shape (56 k-units), a rank that is not a multiple of 16
    (None, 14336, 4096, 16, 2.0), # the largest token count whose scratch fits the array (partials near its end)
])
def test_noalloc_forward_matches_workspace_forward(T, N, K, r, s):
    import bit_nf4_quantized_20_b200 as q
    if T is None:
        T = _largest_T_that_fits(N, K, r)
        assert T > 16
    W, X, A, B, _ = inputs.layer_inputs(91, 0, 0, T, N, K, r, device="cuda")
    qw = q.quantize_nf4(W)
    ref = q.linear_fwd(X, qw, A, B, s)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        q.linear_fwd_noalloc(X, qw, A, B, s, out)
        q.noalloc_get_error()
        torch.cuda.synchronize()
        _close(out, ref)


def test_noalloc_status_query_reports_a_timeout_once():
    """A bounded wait that ran out is recorded in the fixed array's status
    word; qlora_noalloc_get_error reports it once, then the next forward
    computes and reports nothing."""
    import bit_nf4_quantized_20_b200 as q
    q.noalloc_get_error()
    q.wait_selftest(1000, noalloc=True)
    with pytest.raises(q.QLoraError) as e:
        q.noalloc_get_error()
    assert e.value.status == 7
    q.noalloc_get_error()
    W, X, A, B, _ = inputs.layer_inputs(91, 0, 0, 16, 512, 512, 8, device="cuda")
    qw = q.quantize_nf4(W)
    ref = q.linear_fwd(X, qw, A, B, 2.0)
    out = torch.empty_like(ref)
    q.linear_fwd_noalloc(X, qw, A, B, 2.0, out)
    q.noalloc_get_error()
    torch.cuda.synchronize()
    _close(out, ref)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    """14336 x 4096 at T = 4096, rank 64 needs more scratch than the fixed array."""
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200._lib import NF4Weight
    L = q.lib()
    assert L.qlora_workspace_bytes(1, 4096, 14336, 4096, 64) > (4 << 20)
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")   # never read: the call is refused first
    p = C.c_void_p(buf.data_ptr())
    w = NF4Weight()
    w.codes, w.scales, w.c2 = buf.data_ptr(), buf.data_ptr(), buf.data_ptr()
    w.rows, w.cols, w.blocksize, w.dq_block = 14336, 4096, 64, 256
    for i, v in enumerate(q.nf4_codebook()):
        w.codebook[i] = v
    st = L.qlora_linear_fwd_noalloc(p, 4096, C.byref(w), p, p, 64, 1.0, p, None)
    assert st == 4   # QLORA_ERR_WORKSPACE
