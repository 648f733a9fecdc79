"""The C-ABI library builds, loads and exports every symbol include/qlora.h
declares; host-only entry points and argument validation behave as documented.
No test here launches a kernel (it runs without a GPU)."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from bit_nf4_quantized_20_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")


@pytest.fixture(scope="module")
def L():
    from bit_nf4_quantized_20_b200 import build
    build.build()
    from bit_nf4_quantized_20_b200 import _lib
    return _lib.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QLORA_API[^;(]*?\b(qlora_\w+)\s*\(", text, flags=re.S)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for need in ["qlora_quantize_nf4", "qlora_dequantize", "qlora_linear_fwd", "qlora_linear_bwd",
                 "qlora_nf4_storage_bytes", "qlora_workspace_bytes", "qlora_get_error", "qlora_status_string"]:
        assert need in syms


def test_library_exports_every_declared_symbol(L):
    from bit_nf4_quantized_20_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (qlora_\w+)", out))
    for s in declared_symbols():
        assert s in exported, s
        assert hasattr(L, s)
    # nothing else leaks out under the qlora_ prefix
    assert exported == set(declared_symbols())


def test_status_strings_and_version(L):
    for code in range(8):
        assert L.qlora_status_string(code)
    assert b"sm_100a" in L.qlora_version()


def test_library_codebook_equals_oracle_codebook(L):
    """The library's own eq. 2 levels (bisection on erfc) match the oracle's
    (statistics.NormalDist) bit for bit."""
    buf = (C.c_float * 16)()
    assert L.qlora_nf4_codebook_eq2(buf) == 0
    got = np.array(list(buf), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), O.nf4_codebook().view(np.uint32))


@pytest.mark.parametrize("rows,cols", [(512, 512), (4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336),
                                       (3, 320), (22016, 8192)])
def test_storage_bytes_match_oracle(L, rows, cols):
    a, b, c = C.c_size_t(), C.c_size_t(), C.c_size_t()
    assert L.qlora_nf4_storage_bytes(rows, cols, 64, 256, C.byref(a), C.byref(b), C.byref(c)) == 0
    assert (a.value, b.value, c.value) == O.storage_bytes(rows, cols)


def test_storage_bytes_rejects(L):
    a, b, c = C.c_size_t(), C.c_size_t(), C.c_size_t()
    assert L.qlora_nf4_storage_bytes(4, 100, 64, 256, C.byref(a), C.byref(b), C.byref(c)) == 2
    assert L.qlora_nf4_storage_bytes(4, 128, 32, 256, C.byref(a), C.byref(b), C.byref(c)) == 2
    assert L.qlora_nf4_storage_bytes(4, 128, 64, 128, C.byref(a), C.byref(b), C.byref(c)) == 2
    assert L.qlora_nf4_storage_bytes(0, 128, 64, 256, C.byref(a), C.byref(b), C.byref(c)) == 1
    assert L.qlora_nf4_storage_bytes(4, 128, 64, 256, None, C.byref(b), C.byref(c)) == 1


def test_workspace_bytes(L):
    q = L.qlora_workspace_bytes(0, 0, 0, 0, 1)
    f = L.qlora_workspace_bytes(1, 4096, 4096, 4096, 16)
    b = L.qlora_workspace_bytes(2, 4096, 4096, 4096, 16)
    assert 256 <= q < f < b
    assert L.qlora_workspace_bytes(1, 4096, 4096, 4096, 0) == 0
    assert L.qlora_workspace_bytes(1, 4096, 4096, 4096, 129) == 0
    assert L.qlora_workspace_bytes(7, 16, 16, 64, 8) == 0
    # zero tokens is a valid (empty) call: the size query must not fault
    assert L.qlora_workspace_bytes(1, 0, 4096, 4096, 16) > 0
    assert L.qlora_workspace_bytes(2, 0, 4096, 4096, 16) > 0
    # grows with the token count
    assert L.qlora_workspace_bytes(2, 8192, 4096, 4096, 16) > b
    # the backward of the 8B gate shape: status header (256) and tile
    # counters (64 KiB), sU^T and dU^T (two planes each, 16 x 4096 BF16), dU's
    # hi | lo row planes (4096 x 128 BF16), B padded to 64 columns (14336 x 64
    # BF16), and the largest partial-sum buffer, here the fused dU/dB kernel's:
    # 3 x 9-tile blocks give 13 feature ranges and 11 token ranges of FP32 rows
    # of 16, 13 * 4096 * 64 + 11 * 14336 * 64 bytes
    parts = 13 * 4096 * 64 + 11 * 14336 * 64
    fixed = 256 + 65536 + 4 * 16 * 4096 * 2 + 4096 * 128 * 2 + 14336 * 64 * 2
    assert L.qlora_workspace_bytes(2, 4096, 14336, 4096, 16) == fixed + parts


def test_decode_workspace_fits_the_noalloc_scratch(L):
    """The allocation-free forward keeps its scratch in a fixed 4 MiB array; the
    decode shapes (1-16 tokens, rank up to 128) of the 8B and 65B projections
    must fit in it, split partials of the persistent GEMV included."""
    scratch = 4 << 20
    shapes = [(n, k) for (_, n, k) in inputs.LLAMA8B_PROJ] + [(8192, 8192), (22016, 8192), (8192, 22016)]
    for (n, k) in shapes:
        for T in (1, 4, 16):
            for r in (16, 64, 128):
                need = L.qlora_workspace_bytes(1, T, n, k, r)
                assert 0 < need <= scratch, (T, n, k, r, need)


def _weight(rows=128, cols=128, codes=0x1000, scales=0x2000, c2=0x3000, bs=64, dq=256):
    from bit_nf4_quantized_20_b200._lib import NF4Weight
    w = NF4Weight()
    w.codes, w.scales, w.c2 = codes, scales, c2
    w.rows, w.cols, w.blocksize, w.dq_block = rows, cols, bs, dq
    for i, v in enumerate(O.nf4_codebook()):
        w.codebook[i] = float(v)
    return w


FAKE = 0x10000   # never dereferenced: every call below fails validation first


def test_quantize_validation(L):
    from bit_nf4_quantized_20_b200._lib import NF4Weight
    cb = (C.c_float * 16)(*[float(v) for v in O.nf4_codebook()])
    out = _weight()
    ws, wsb = C.c_void_p(FAKE), 1 << 20
    q = L.qlora_quantize_nf4
    assert q(None, 128, 128, 64, 256, cb, C.byref(out), ws, wsb, None) == 1            # null input
    assert q(C.c_void_p(FAKE), 128, 100, 64, 256, cb, C.byref(out), ws, wsb, None) == 2  # cols % 64
    assert q(C.c_void_p(FAKE), 128, 128, 32, 256, cb, C.byref(out), ws, wsb, None) == 2  # blocksize
    assert q(C.c_void_p(FAKE + 2), 128, 128, 64, 256, cb, C.byref(out), ws, wsb, None) == 3  # misaligned
    bad = (C.c_float * 16)(*([0.0] * 16))
    assert q(C.c_void_p(FAKE), 128, 128, 64, 256, bad, C.byref(out), ws, wsb, None) == 1   # not ascending
    nan = (C.c_float * 16)(*[float("nan")] + [float(v) for v in O.nf4_codebook()[1:]])
    assert q(C.c_void_p(FAKE), 128, 128, 64, 256, nan, C.byref(out), ws, wsb, None) == 1
    assert q(C.c_void_p(FAKE), 128, 128, 64, 256, cb, C.byref(out), None, wsb, None) == 4  # no workspace
    assert q(C.c_void_p(FAKE), 128, 128, 64, 256, cb, C.byref(out), ws, 16, None) == 4     # too small
    empty = NF4Weight()
    assert q(C.c_void_p(FAKE), 128, 128, 64, 256, cb, C.byref(empty), ws, wsb, None) == 1  # no out buffers


def test_linear_validation(L):
    w = _weight()
    ws = C.c_void_p(FAKE)
    big = 1 << 30
    fwd = L.qlora_linear_fwd
    P = C.c_void_p(FAKE)
    assert fwd(None, 16, C.byref(w), P, P, 8, 2.0, P, ws, big, None) == 1
    assert fwd(P, 16, C.byref(w), P, P, 0, 2.0, P, ws, big, None) == 1       # r = 0
    assert fwd(P, 16, C.byref(w), P, P, 129, 2.0, P, ws, big, None) == 1     # r > 128
    assert fwd(P, 16, C.byref(w), P, P, 8, float("inf"), P, ws, big, None) == 1
    assert fwd(P, -1, C.byref(w), P, P, 8, 2.0, P, ws, big, None) == 1
    assert fwd(C.c_void_p(FAKE + 8), 16, C.byref(w), P, P, 8, 2.0, P, ws, big, None) == 3
    assert fwd(P, 16, C.byref(w), P, P, 8, 2.0, P, C.c_void_p(FAKE + 16), big, None) == 4  # ws not 256-aligned
    assert fwd(P, 16, C.byref(w), P, P, 8, 2.0, P, ws, 1024, None) == 4
    odd = _weight(rows=100)
    assert fwd(P, 16, C.byref(odd), P, P, 8, 2.0, P, ws, big, None) == 2     # N % 8
    bs = _weight(bs=128)
    assert fwd(P, 16, C.byref(bs), P, P, 8, 2.0, P, ws, big, None) == 2
    mis = _weight(codes=FAKE + 4)
    assert fwd(P, 16, C.byref(mis), P, P, 8, 2.0, P, ws, big, None) == 3
    bwd = L.qlora_linear_bwd
    assert bwd(P, P, 16, C.byref(w), P, P, 8, 2.0, P, None, P, ws, big, None) == 1
    assert bwd(P, P, 16, C.byref(w), P, P, 8, 2.0, P, P, C.c_void_p(FAKE + 2), ws, big, None) == 3
    assert bwd(P, P, 16, C.byref(w), P, P, 8, 2.0, P, P, P, ws, 64, None) == 4
    deq = L.qlora_dequantize
    assert deq(C.byref(w), None, None) == 1
    assert deq(C.byref(w), C.c_void_p(FAKE + 1), None) == 3


def test_merge_validation(L):
    """qlora_merge_adapter rejects bad arguments before touching the GPU."""
    w = _weight()
    P = C.c_void_p(FAKE)
    merge = L.qlora_merge_adapter
    assert merge(None, P, P, 8, 2.0, P, None) == 1
    assert merge(C.byref(w), None, P, 8, 2.0, P, None) == 1
    assert merge(C.byref(w), P, None, 8, 2.0, P, None) == 1
    assert merge(C.byref(w), P, P, 8, 2.0, None, None) == 1
    assert merge(C.byref(w), P, P, 0, 2.0, P, None) == 1            # r = 0
    assert merge(C.byref(w), P, P, 129, 2.0, P, None) == 1          # r > 128
    assert merge(C.byref(w), P, P, 8, float("nan"), P, None) == 1
    assert merge(C.byref(w), C.c_void_p(FAKE + 8), P, 8, 2.0, P, None) == 3   # A not 16-byte aligned
    assert merge(C.byref(w), P, C.c_void_p(FAKE + 1), 8, 2.0, P, None) == 3   # B not 2-byte aligned
    assert merge(C.byref(w), P, P, 8, 2.0, C.c_void_p(FAKE + 4), None) == 3   # output not 16-byte aligned
    assert merge(C.byref(_weight(bs=128)), P, P, 8, 2.0, P, None) == 2


def test_linear_fwd_zero_tokens_is_a_noop(L):
    """T == 0 launches nothing; the empty token buffers may be null."""
    w = _weight()
    P = C.c_void_p(FAKE)
    ws = C.c_void_p(FAKE)
    assert L.qlora_linear_fwd(None, 0, C.byref(w), P, P, 8, 2.0, None, ws, 1 << 30, None) == 0
    assert L.qlora_linear_fwd(None, 5, C.byref(w), P, P, 8, 2.0, None, ws, 1 << 30, None) == 1


def test_trace_attach_validation(L):
    from bit_nf4_quantized_20_b200._lib import TraceRec
    recs = (TraceRec * 4)()
    assert L.qlora_trace_attach(recs, 4, None) == 1
    cnt = C.c_int32(0)
    assert L.qlora_trace_attach(recs, 4, C.byref(cnt)) == 0
    assert L.qlora_trace_attach(None, 0, None) == 0
    assert L.qlora_kernel_name(6) == b"nf4_gemm_fwd"
    # the fused dU/dB kernel and the launch that sums its partials (the names
    # the bench's per-kernel map and the kernel-choice tests read)
    assert L.qlora_kernel_name(12) == b"lora_du+dB"
    assert L.qlora_kernel_name(14) == b"lora_du+dB_sum"
    assert L.qlora_kernel_name(15) == b"unknown"
    assert L.qlora_kernel_name(-1) == b"unknown"
    assert L.qlora_kernel_name(99) == b"unknown"


def test_product_fails_loudly_without_cuda():
    """No CPU fallback: the Python entry points refuse CPU tensors."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    with pytest.raises(ValueError):
        q.quantize_nf4(torch.zeros(64, 64, dtype=torch.bfloat16))


def test_saved_u_validation(L):
    """The saved-U forward and backward check their extra buffer before
    touching the GPU; its size query follows the documented layout."""
    w = _weight()
    P = C.c_void_p(FAKE)
    ws, big = C.c_void_p(FAKE), 1 << 30
    # two planes of r x ceil8(T) BF16, each rounded up to 256 bytes
    assert L.qlora_saved_u_bytes(4096, 16) == 2 * 16 * 4096 * 2
    assert L.qlora_saved_u_bytes(5, 3) == 2 * 256
    assert L.qlora_saved_u_bytes(0, 16) == 0
    assert L.qlora_saved_u_bytes(16, 0) == 0 and L.qlora_saved_u_bytes(16, 129) == 0
    fs = L.qlora_linear_fwd_save
    assert fs(P, 16, C.byref(w), P, P, 8, 2.0, P, None, ws, big, None) == 1                   # no u_save
    assert fs(P, 16, C.byref(w), P, P, 8, 2.0, P, C.c_void_p(FAKE + 8), ws, big, None) == 3   # misaligned
    assert fs(P, 16, C.byref(w), P, P, 8, 2.0, P, P, ws, 64, None) == 4                       # workspace
    assert fs(None, 0, C.byref(w), P, P, 8, 2.0, None, None, ws, big, None) == 0              # T == 0: no-op
    bs = L.qlora_linear_bwd_saved
    assert bs(P, P, 16, C.byref(w), P, P, 8, 2.0, None, P, P, P, ws, big, None) == 1
    assert bs(P, P, 16, C.byref(w), P, P, 8, 2.0, C.c_void_p(FAKE + 2), P, P, P, ws, big, None) == 3
    assert bs(P, P, 16, C.byref(w), P, P, 8, 2.0, P, P, P, P, ws, 64, None) == 4


def test_noalloc_validation_before_any_enqueue(L):
    """Bad outputs and oversized problems are refused by the allocation-free
    forward before it looks up its scratch array or enqueues anything (so these
    calls need no GPU)."""
    w = _weight()
    P = C.c_void_p(FAKE)
    na = L.qlora_linear_fwd_noalloc
    assert na(P, 16, C.byref(w), P, P, 8, 2.0, None, None) == 1                  # no output
    assert na(P, 16, C.byref(w), P, P, 8, 2.0, C.c_void_p(FAKE + 4), None) == 3  # misaligned output
    assert na(P, 16, C.byref(_weight(rows=100)), P, P, 8, 2.0, P, None) == 2      # N % 8
    big = _weight(rows=14336, cols=4096)
    assert na(P, 4096, C.byref(big), P, P, 64, 1.0, P, None) == 4                  # beyond the 4 MiB array
    assert na(None, 0, C.byref(w), P, P, 8, 2.0, None, None) == 0                 # T == 0: no-op


def test_wait_selftest_validation(L):
    P = C.c_void_p(FAKE)
    assert L.qlora_wait_selftest(C.c_void_p(FAKE + 16), 4096, 100, None) == 4   # not 256-byte aligned
    assert L.qlora_wait_selftest(P, 64, 100, None) == 4
    assert L.qlora_wait_selftest(P, 4096, 0, None) == 1
    assert L.qlora_wait_selftest(P, 4096, 2000001, None) == 1
    assert L.qlora_wait_selftest(None, 0, 0, None) == 1          # checked before the array's lookup


def test_quantize_ex_flags_validation(L):
    cb = (C.c_float * 16)(*[float(v) for v in O.nf4_codebook()])
    out = _weight()
    ws, wsb = C.c_void_p(FAKE), 1 << 20
    qx = L.qlora_quantize_nf4_ex
    assert qx(C.c_void_p(FAKE), 128, 128, 64, 256, cb, 2, C.byref(out), ws, wsb, None) == 1   # unknown flag
    assert qx(C.c_void_p(FAKE), 128, 100, 64, 256, cb, 1, C.byref(out), ws, wsb, None) == 2   # cols % 64
    assert qx(C.c_void_p(FAKE), 128, 128, 64, 256, cb, 1, C.byref(out), None, wsb, None) == 4


def test_adam_and_paged_validation(L):
    from bit_nf4_quantized_20_b200._lib import AdamHParams
    P = C.c_void_p(FAKE)
    h = AdamHParams(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    a = L.qlora_adam_step
    assert a(P, P, P, P, None, 0, C.byref(h), None) == 0              # nothing to do
    assert a(P, P, P, P, None, 10, None, None) == 1                   # no hyper-parameters
    assert a(None, P, P, P, None, 10, C.byref(h), None) == 1
    assert a(P, P, P, C.c_void_p(FAKE + 2), None, 10, C.byref(h), None) == 3
    assert a(P, P, P, P, C.c_void_p(FAKE + 8), 10, C.byref(h), None) == 3
    for bad in (AdamHParams(1e-3, 0.9, 0.999, 1e-8, 0.0, 0), AdamHParams(1e-3, 1.0, 0.999, 1e-8, 0.0, 1),
                AdamHParams(1e-3, 0.9, 0.999, 0.0, 0.0, 1), AdamHParams(float("nan"), 0.9, 0.999, 1e-8, 0.0, 1)):
        assert a(P, P, P, P, None, 10, C.byref(bad), None) == 1
    assert L.qlora_paged_alloc(0, C.byref(C.c_void_p())) == 1
    assert L.qlora_paged_alloc(16, None) == 1
    assert L.qlora_paged_free(None) == 0
    assert L.qlora_paged_prefetch(None, 16, 0, None) == 1


def test_decode_batch_validation(L):
    from bit_nf4_quantized_20_b200._lib import FwdProblem
    w = _weight()
    P = FAKE
    arr = (FwdProblem * 9)()
    for i in range(9):
        arr[i] = FwdProblem(P, C.pointer(w), P, P, 8, 2.0, P)
    ws = C.c_void_p(FAKE)
    assert L.qlora_decode_batch_workspace_bytes(2, arr, 4) > 0
    assert L.qlora_decode_batch_workspace_bytes(9, arr, 4) == 0          # at most 8 problems
    assert L.qlora_decode_batch_workspace_bytes(2, arr, 17) == 0         # decode-sized token counts only
    b = L.qlora_linear_fwd_decode_batch
    assert b(0, arr, 4, ws, 1 << 30, None) == 1
    assert b(9, arr, 4, ws, 1 << 30, None) == 1
    assert b(2, None, 4, ws, 1 << 30, None) == 1
    assert b(2, arr, 17, ws, 1 << 30, None) == 2
    assert b(2, arr, 4, ws, 64, None) == 4                               # workspace too small
    assert b(2, arr, 0, ws, 1 << 30, None) == 0                          # no tokens: nothing to do
    arr[1] = FwdProblem(P, C.pointer(w), P, P, 8, 2.0, None)             # a problem without output
    assert b(2, arr, 4, ws, 1 << 30, None) == 1
    odd = _weight(rows=100)
    arr[1] = FwdProblem(P, C.pointer(odd), P, P, 8, 2.0, P)              # N % 8 != 0
    assert b(2, arr, 4, ws, 1 << 30, None) == 2
