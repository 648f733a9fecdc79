"""QLoRA NF4 linear layer for B200 (sm_100a): Python entry points.

PyTorch supplies device memory and the current CUDA stream; every computation
runs in libqlora.so (include/qlora.h) through the ctypes binding in ``_lib``.
There is no CPU or PyTorch fallback: if the library is missing, or a tensor is
not on a CUDA device, the call raises.

    qw = quantize_nf4(w)                     # w: [N, K] bf16 on cuda
    y = linear_fwd(x, qw, A, B, s)           # x: [T, K], A: [r, K], B: [N, r]
    dx, dA, dB = linear_bwd(dy, x, qw, A, B, s)
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import OP_BWD, OP_FWD, OP_QUANTIZE, NF4Weight, QLoraError, check, lib

__all__ = ["QuantizedNF4", "nf4_codebook", "storage_bytes", "quantize_nf4", "dequantize", "merge_adapter",
           "linear_fwd", "linear_bwd", "linear_fwd_save", "linear_bwd_saved", "saved_u_bytes",
           "linear_fwd_noalloc", "noalloc_get_error", "wait_selftest", "workspace", "workspace_bytes",
           "get_error", "adam_step", "PagedBuffer", "quantize_nf4_into", "linear_fwd_decode_batch",
           "QLoraError", "lib"]


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> C.c_void_p:
    return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(name: str, t: torch.Tensor, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def nf4_codebook() -> list[float]:
    """The library's eq. 2 codebook (16 ascending fp32 levels in [-1, 1])."""
    buf = (C.c_float * 16)()
    check("qlora_nf4_codebook_eq2", lib().qlora_nf4_codebook_eq2(buf))
    return [float(v) for v in buf]


def storage_bytes(rows: int, cols: int, blocksize: int = 64, dq_block: int = 256):
    """(codes, scales, c2) bytes of a quantized rows x cols weight."""
    a, b, c = C.c_size_t(), C.c_size_t(), C.c_size_t()
    check("qlora_nf4_storage_bytes",
          lib().qlora_nf4_storage_bytes(rows, cols, blocksize, dq_block, C.byref(a), C.byref(b), C.byref(c)))
    return a.value, b.value, c.value


@dataclass
class QuantizedNF4:
    codes: torch.Tensor      # uint8 [rows*cols/2]
    scales: torch.Tensor     # uint8 [rows*cols/64], FP8-E4M3FN bytes
    c2: torch.Tensor         # float32 [ceil(rows*cols/16384)]
    rows: int
    cols: int
    codebook: list
    blocksize: int = 64
    dq_block: int = 256

    def struct(self) -> NF4Weight:
        s = NF4Weight()
        s.codes, s.scales, s.c2 = _ptr(self.codes), _ptr(self.scales), _ptr(self.c2)
        s.rows, s.cols, s.blocksize, s.dq_block = self.rows, self.cols, self.blocksize, self.dq_block
        for i, v in enumerate(self.codebook):
            s.codebook[i] = v
        return s

    @property
    def device(self):
        return self.codes.device

    def nbytes(self) -> int:
        return self.codes.numel() + self.scales.numel() + 4 * self.c2.numel()


def workspace_bytes(op: int, T: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes(op, T, N, K, r))


_WS: dict = {}


def workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    """A zeroed, 256-byte aligned workspace of at least nbytes on `device` (cached, grows)."""
    key = torch.device(device)
    ws = _WS.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 4096), dtype=torch.uint8, device=key)
        _WS[key] = ws
    return ws


def get_error(device=None) -> None:
    """Synchronize and raise if a kernel recorded a device-side failure."""
    dev = torch.device(device if device is not None else torch.cuda.current_device())
    ws = _WS.get(dev)
    if ws is None:
        return
    check("qlora_get_error", lib().qlora_get_error(C.c_void_p(ws.data_ptr()), _stream(dev)))


def quantize_nf4(w: torch.Tensor, codebook=None, blocksize: int = 64, dq_block: int = 256,
                 snap_to_dq_scale: bool = False) -> QuantizedNF4:
    """NF4 + double quantization of a BF16 weight w[rows, cols] on the GPU.
    snap_to_dq_scale: snap the codes against the double-quantized block scale
    (the one dequantization multiplies by) instead of the exact absmax."""
    _need_cuda("w", w)
    if w.dim() != 2:
        raise ValueError("w must be 2-D [rows, cols]")
    rows, cols = w.shape
    cb = list(nf4_codebook() if codebook is None else [float(v) for v in codebook])
    if len(cb) != 16:
        raise ValueError("codebook must have 16 entries")
    nc, ns, n2 = storage_bytes(rows, cols, blocksize, dq_block)
    dev = w.device
    codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    scales = torch.empty(ns, dtype=torch.uint8, device=dev)
    c2 = torch.empty(n2 // 4, dtype=torch.float32, device=dev)
    out = NF4Weight()
    out.codes, out.scales, out.c2 = codes.data_ptr(), scales.data_ptr(), c2.data_ptr()
    cbuf = (C.c_float * 16)(*cb)
    wsb = workspace_bytes(OP_QUANTIZE, 0, 0, 0, 1)
    ws = workspace(dev, wsb)
    flags = _lib.QUANT_SNAP_DQ_SCALE if snap_to_dq_scale else 0
    check("qlora_quantize_nf4_ex", lib().qlora_quantize_nf4_ex(
        C.c_void_p(w.data_ptr()), rows, cols, blocksize, dq_block, cbuf, flags, C.byref(out),
        C.c_void_p(ws.data_ptr()), ws.numel(), _stream(dev)))
    return QuantizedNF4(codes, scales, c2, rows, cols, cb, blocksize, dq_block)


def quantize_nf4_into(w: torch.Tensor, qw: QuantizedNF4, snap_to_dq_scale: bool = False) -> QuantizedNF4:
    """Quantize w again into the buffers of an existing QuantizedNF4 of the
    same shape and codebook (no allocation)."""
    _need_cuda("w", w)
    if tuple(w.shape) != (qw.rows, qw.cols) or w.device != qw.device:
        raise ValueError(f"w must be [{qw.rows}, {qw.cols}] on {qw.device}")
    out = qw.struct()
    cbuf = (C.c_float * 16)(*qw.codebook)
    ws = workspace(qw.device, workspace_bytes(OP_QUANTIZE, 0, 0, 0, 1))
    flags = _lib.QUANT_SNAP_DQ_SCALE if snap_to_dq_scale else 0
    check("qlora_quantize_nf4_ex", lib().qlora_quantize_nf4_ex(
        C.c_void_p(w.data_ptr()), qw.rows, qw.cols, qw.blocksize, qw.dq_block, cbuf, flags, C.byref(out),
        C.c_void_p(ws.data_ptr()), ws.numel(), _stream(qw.device)))
    return qw


def merge_adapter(qw: QuantizedNF4, A: torch.Tensor, B: torch.Tensor, s: float) -> torch.Tensor:
    """BF16(W' + s B A) [rows, cols]: the adapter folded into the dequantized
    weight for export (quantize_nf4 of the result gives an NF4 merged model)."""
    for name, t in (("A", A), ("B", B)):
        _need_cuda(name, t)
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor")
    r = A.shape[0]
    if A.dim() != 2 or A.shape[1] != qw.cols or tuple(B.shape) != (qw.rows, r):
        raise ValueError(f"A must be [r, {qw.cols}] and B [{qw.rows}, r]")
    out = torch.empty(qw.rows, qw.cols, dtype=torch.bfloat16, device=qw.device)
    st = qw.struct()
    check("qlora_merge_adapter", lib().qlora_merge_adapter(C.byref(st), C.c_void_p(A.data_ptr()),
                                                           C.c_void_p(B.data_ptr()), r, float(s),
                                                           C.c_void_p(out.data_ptr()), _stream(qw.device)))
    return out


def dequantize(qw: QuantizedNF4, out: torch.Tensor | None = None) -> torch.Tensor:
    """W' = BF16(RN32(codebook[code] * RN32(fp8 * c2))) as a [rows, cols] tensor."""
    if out is None:
        out = torch.empty(qw.rows, qw.cols, dtype=torch.bfloat16, device=qw.device)
    else:
        _check_out("out", out, (qw.rows, qw.cols), qw.device)
    s = qw.struct()
    check("qlora_dequantize", lib().qlora_dequantize(C.byref(s), C.c_void_p(out.data_ptr()), _stream(qw.device)))
    return out


def _check_linear(x, qw, A, B):
    for n, t in (("x", x), ("A", A), ("B", B)):
        _need_cuda(n, t)
    if x.dim() != 2 or x.shape[1] != qw.cols:
        raise ValueError(f"x must be [T, {qw.cols}]")
    r = A.shape[0]
    if tuple(A.shape) != (r, qw.cols) or tuple(B.shape) != (qw.rows, r):
        raise ValueError(f"A must be [r, {qw.cols}] and B [{qw.rows}, r]")
    for n, t in (("A", A), ("B", B), ("qw", qw.codes)):
        if t.device != x.device:
            raise ValueError(f"{n} is on {t.device}, x on {x.device}")
    return x.shape[0], r


def _check_out(name, t, shape, device):
    """An output buffer the kernels write: a contiguous bf16 CUDA tensor of
    exactly `shape` on `device` (the epilogues write every element of it)."""
    _need_cuda(name, t)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {list(shape)}, got {list(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def saved_u_bytes(T: int, r: int) -> int:
    """Bytes of the U = s x A^T planes the forward saves for the backward."""
    return int(lib().qlora_saved_u_bytes(T, r))


def linear_fwd(x: torch.Tensor, qw: QuantizedNF4, A: torch.Tensor, B: torch.Tensor, s: float,
               out: torch.Tensor | None = None) -> torch.Tensor:
    """y = x W'^T + s (x A^T) B^T (BF16), W' dequantized inside the kernel."""
    T, r = _check_linear(x, qw, A, B)
    dev = x.device
    if out is not None:
        _check_out("out", out, (T, qw.rows), dev)
    y = out if out is not None else torch.empty(T, qw.rows, dtype=torch.bfloat16, device=dev)
    ws = workspace(dev, workspace_bytes(OP_FWD, T, qw.rows, qw.cols, r))
    st = qw.struct()
    check("qlora_linear_fwd", lib().qlora_linear_fwd(
        C.c_void_p(x.data_ptr()), T, C.byref(st), C.c_void_p(A.data_ptr()), C.c_void_p(B.data_ptr()), r,
        float(s), C.c_void_p(y.data_ptr()), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(dev)))
    return y


def linear_fwd_save(x: torch.Tensor, qw: QuantizedNF4, A: torch.Tensor, B: torch.Tensor, s: float,
                    out: torch.Tensor | None = None, u_save: torch.Tensor | None = None):
    """The forward that also returns U = s x A^T (hi + lo BF16 planes, as a
    uint8 buffer of saved_u_bytes(T, r)) for linear_bwd_saved."""
    T, r = _check_linear(x, qw, A, B)
    dev = x.device
    if out is not None:
        _check_out("out", out, (T, qw.rows), dev)
    y = out if out is not None else torch.empty(T, qw.rows, dtype=torch.bfloat16, device=dev)
    nbytes = saved_u_bytes(T, r)
    if u_save is None:
        u_save = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _need_cuda("u_save", u_save, dtype=torch.uint8)
    if u_save.numel() < nbytes or u_save.device != dev:
        raise ValueError(f"u_save must hold {nbytes} bytes on {dev}")
    ws = workspace(dev, workspace_bytes(OP_FWD, T, qw.rows, qw.cols, r))
    st = qw.struct()
    check("qlora_linear_fwd_save", lib().qlora_linear_fwd_save(
        C.c_void_p(x.data_ptr()), T, C.byref(st), C.c_void_p(A.data_ptr()), C.c_void_p(B.data_ptr()), r,
        float(s), C.c_void_p(y.data_ptr()), C.c_void_p(u_save.data_ptr()), C.c_void_p(ws.data_ptr()), ws.numel(),
        _stream(dev)))
    return y, u_save


class DecodeBatch:
    """A prepared grouped decode-sized forward (qlora_linear_fwd_decode_batch):
    the argument structs are built once, so that repeated calls (or a CUDA
    graph capture) only cross the boundary.  problems: (x, qw, A, B, s, out)."""

    def __init__(self, problems):
        if not 1 <= len(problems) <= 8:
            raise ValueError("1 to 8 problems")
        T = None
        self._keep = []
        self.arr = (_lib.FwdProblem * len(problems))()
        for i, (x, qw, A, B, s, out) in enumerate(problems):
            Ti, r = _check_linear(x, qw, A, B)
            _check_out("out", out, (Ti, qw.rows), x.device)
            if T is None:
                T, self.device = Ti, x.device
            elif Ti != T or x.device != self.device:
                raise ValueError("every problem must have the same token count and device")
            st = qw.struct()
            self._keep.append((st, x, qw, A, B, out))
            self.arr[i] = _lib.FwdProblem(x.data_ptr(), C.pointer(st), A.data_ptr(), B.data_ptr(), r, float(s),
                                          out.data_ptr())
        self.n, self.T = len(problems), T
        need = int(lib().qlora_decode_batch_workspace_bytes(self.n, self.arr, T))
        if need == 0:
            raise ValueError("problems not supported by the grouped decode forward (T <= 16)")
        self.ws = workspace(self.device, need)

    def __call__(self):
        check("qlora_linear_fwd_decode_batch", lib().qlora_linear_fwd_decode_batch(
            self.n, self.arr, self.T, C.c_void_p(self.ws.data_ptr()), self.ws.numel(), _stream(self.device)))


def linear_fwd_decode_batch(problems) -> None:
    """Decode-sized forward (T <= 16) of several projections in one grouped
    call; problems: list of (x, qw, A, B, s, out), outputs written in place."""
    DecodeBatch(problems)()


def linear_fwd_noalloc(x: torch.Tensor, qw: QuantizedNF4, A: torch.Tensor, B: torch.Tensor, s: float,
                       out: torch.Tensor) -> torch.Tensor:
    """Forward through the entry point that uses the library's fixed device
    scratch instead of a workspace (for callers that cannot allocate device
    memory); `out` must be preallocated [T, N] bf16 on x's device."""
    T, r = _check_linear(x, qw, A, B)
    _check_out("out", out, (T, qw.rows), x.device)
    st = qw.struct()
    check("qlora_linear_fwd_noalloc", lib().qlora_linear_fwd_noalloc(
        C.c_void_p(x.data_ptr()), T, C.byref(st), C.c_void_p(A.data_ptr()), C.c_void_p(B.data_ptr()), r,
        float(s), C.c_void_p(out.data_ptr()), _stream(x.device)))
    return out


def noalloc_get_error(device=None) -> None:
    """Synchronize and raise if an allocation-free forward on `device` recorded
    a device-side failure (reads and clears the fixed array's status word)."""
    dev = torch.device(device if device is not None else torch.cuda.current_device())
    with torch.cuda.device(dev):
        check("qlora_noalloc_get_error", lib().qlora_noalloc_get_error(_stream(dev)))


def wait_selftest(limit_us: int, device=None, noalloc: bool = False) -> None:
    """Run the bounded-wait self-test kernel on `device` (its wait runs out
    after limit_us); the timeout is then reported by get_error(device), or by
    noalloc_get_error(device) when `noalloc` puts it in the allocation-free
    forward's fixed array."""
    dev = torch.device(device if device is not None else torch.cuda.current_device())
    with torch.cuda.device(dev):
        if noalloc:
            st = lib().qlora_wait_selftest(None, 0, int(limit_us), _stream(dev))
        else:
            ws = workspace(dev, 4096)
            st = lib().qlora_wait_selftest(C.c_void_p(ws.data_ptr()), ws.numel(), int(limit_us), _stream(dev))
    check("qlora_wait_selftest", st)


def _bwd_outs(outs, T, qw, r, dev):
    if outs is None:
        return (torch.empty(T, qw.cols, dtype=torch.bfloat16, device=dev),
                torch.empty(r, qw.cols, dtype=torch.bfloat16, device=dev),
                torch.empty(qw.rows, r, dtype=torch.bfloat16, device=dev))
    dx, dA, dB = outs
    _check_out("dx", dx, (T, qw.cols), dev)
    _check_out("dA", dA, (r, qw.cols), dev)
    _check_out("dB", dB, (qw.rows, r), dev)
    return dx, dA, dB


def linear_bwd(dy: torch.Tensor, x: torch.Tensor, qw: QuantizedNF4, A: torch.Tensor, B: torch.Tensor, s: float,
               outs=None):
    """(dX, dA, dB) of the layer for upstream gradient dy[T, N]."""
    T, r = _check_linear(x, qw, A, B)
    dev = x.device
    _check_out("dy", dy, (T, qw.rows), dev)
    dx, dA, dB = _bwd_outs(outs, T, qw, r, dev)
    ws = workspace(dev, workspace_bytes(OP_BWD, T, qw.rows, qw.cols, r))
    st = qw.struct()
    check("qlora_linear_bwd", lib().qlora_linear_bwd(
        C.c_void_p(dy.data_ptr()), C.c_void_p(x.data_ptr()), T, C.byref(st), C.c_void_p(A.data_ptr()),
        C.c_void_p(B.data_ptr()), r, float(s), C.c_void_p(dx.data_ptr()), C.c_void_p(dA.data_ptr()),
        C.c_void_p(dB.data_ptr()), C.c_void_p(ws.data_ptr()), ws.numel(), _stream(dev)))
    return dx, dA, dB


def linear_bwd_saved(dy: torch.Tensor, x: torch.Tensor, qw: QuantizedNF4, A: torch.Tensor, B: torch.Tensor,
                     s: float, u_saved: torch.Tensor, outs=None):
    """linear_bwd with U taken from linear_fwd_save's buffer instead of
    recomputed from x."""
    T, r = _check_linear(x, qw, A, B)
    dev = x.device
    _check_out("dy", dy, (T, qw.rows), dev)
    _need_cuda("u_saved", u_saved, dtype=torch.uint8)
    if u_saved.numel() < saved_u_bytes(T, r) or u_saved.device != dev:
        raise ValueError(f"u_saved must hold {saved_u_bytes(T, r)} bytes on {dev}")
    dx, dA, dB = _bwd_outs(outs, T, qw, r, dev)
    ws = workspace(dev, workspace_bytes(OP_BWD, T, qw.rows, qw.cols, r))
    st = qw.struct()
    check("qlora_linear_bwd_saved", lib().qlora_linear_bwd_saved(
        C.c_void_p(dy.data_ptr()), C.c_void_p(x.data_ptr()), T, C.byref(st), C.c_void_p(A.data_ptr()),
        C.c_void_p(B.data_ptr()), r, float(s), C.c_void_p(u_saved.data_ptr()), C.c_void_p(dx.data_ptr()),
        C.c_void_p(dA.data_ptr()), C.c_void_p(dB.data_ptr()), C.c_void_p(ws.data_ptr()), ws.numel(),
        _stream(dev)))
    return dx, dA, dB


# --------------------------------------------------------------------------
# the adapters' optimizer step, with its state optionally in unified memory
# --------------------------------------------------------------------------
class PagedBuffer:
    """`n` elements of unified ("paged") memory from qlora_paged_alloc: the
    driver keeps them on the GPU while there is room and pages them out to host
    memory under pressure.  `.ptr` is the address the kernels take; `.numpy()`
    views the same memory from the host (synchronize first).  Freed on delete."""

    _CT = {torch.float32: C.c_float, torch.bfloat16: C.c_uint16, torch.uint8: C.c_uint8}

    def __init__(self, n: int, dtype=torch.float32, device=None):
        if dtype not in self._CT:
            raise ValueError(f"unsupported dtype {dtype}")
        self.n, self.dtype = int(n), dtype
        self.device = torch.device(device if device is not None else torch.cuda.current_device())
        self.nbytes = max(16, self.n * torch.empty((), dtype=dtype).element_size())
        p = C.c_void_p()
        with torch.cuda.device(self.device):
            check("qlora_paged_alloc", lib().qlora_paged_alloc(self.nbytes, C.byref(p)))
        self.ptr = p.value

    def numpy(self):
        import numpy as np
        arr = (self._CT[self.dtype] * self.n).from_address(self.ptr)
        return np.ctypeslib.as_array(arr)

    def prefetch(self, to_host: bool = False):
        with torch.cuda.device(self.device):
            check("qlora_paged_prefetch", lib().qlora_paged_prefetch(C.c_void_p(self.ptr), self.nbytes,
                                                                     1 if to_host else 0, _stream(self.device)))

    def __del__(self):
        if getattr(self, "ptr", None):
            try:
                torch.cuda.synchronize(self.device)
                lib().qlora_paged_free(C.c_void_p(self.ptr))
            except Exception:
                pass
            self.ptr = None


def _addr(name, t, dtype, n, device):
    if isinstance(t, PagedBuffer):
        if t.dtype != dtype or t.n < n:
            raise ValueError(f"{name} must hold {n} {dtype}")
        return t.ptr
    _need_cuda(name, t, dtype=dtype)
    if t.numel() < n or t.device != device:
        raise ValueError(f"{name} must hold {n} elements on {device}")
    return t.data_ptr()


def adam_step(param, m, v, grad: torch.Tensor, param_bf16: torch.Tensor | None = None, *, step: int, lr: float,
              beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0) -> None:
    """One Adam step (decoupled weight decay) of the FP32 adapter parameters
    `param` with moments `m`, `v` (torch CUDA tensors or PagedBuffers) from the
    BF16 gradient `grad` (dA or dB); writes the BF16 copy of the new
    parameters to `param_bf16` if given.  Elementwise over grad.numel()."""
    n = grad.numel()
    dev = grad.device
    _need_cuda("grad", grad)
    ptrs = [_addr(nm, t, torch.float32, n, dev) for nm, t in (("param", param), ("m", m), ("v", v))]
    out = None
    if param_bf16 is not None:
        out = _addr("param_bf16", param_bf16, torch.bfloat16, n, dev)
    h = _lib.AdamHParams(lr, beta1, beta2, eps, weight_decay, int(step))
    check("qlora_adam_step", lib().qlora_adam_step(C.c_void_p(ptrs[0]), C.c_void_p(ptrs[1]), C.c_void_p(ptrs[2]),
                                                   C.c_void_p(grad.data_ptr()), C.c_void_p(out), n, C.byref(h),
                                                   _stream(dev)))
