"""The division-free snapping that the GPU quantizer uses, checked on the CPU.

For a block absmax c1 > 0 the code of w is #{j : RN32(w / c1) >= t_j}.  The
kernel instead forms, per block, B_j = the smallest BF16 value w with
w >= mid_j * c1 (or w > mid_j * c1), where mid_j is the real midpoint between
t_j and the fp32 value below it and the inequality is strict when that tie
rounds to the lower neighbour; then code = #{j : w >= B_j}.  This test states
that construction in NumPy and compares its codes with the oracle's IEEE
division on every BF16 weight |w| <= c1 for a spread of c1, for the eq. 2
codebook and an asymmetric one.  (The GPU kernel itself is compared with the
oracle on the full sweep in test_gpu_parity.py.)
"""
import numpy as np
import pytest

from oracle import oracle as O


def _nextdown(t):
    return np.nextafter(np.float32(t), np.float32(-np.inf), dtype=np.float32)


def _f32_round_up(p):
    f = np.float32(p)
    if float(f) < p:
        f = np.nextafter(f, np.float32(np.inf), dtype=np.float32)
    return f


def _boundary(c1, mid, incl):
    p = mid * float(c1)                       # exact in double
    u = int(np.float32(_f32_round_up(p)).view(np.uint32))
    if u & 0xFFFF:                            # up to the next BF16 value
        u = ((u + 0x10000) & 0xFFFF0000) if np.uint32(u).view(np.float32) > 0 else (u & 0xFFFF0000)
    b = np.uint32(u).view(np.float32)
    if not incl and float(b) == p:            # strictly above p
        if (u & 0x7FFFFFFF) == 0:
            u = 0x00010000
        else:
            u = (u + 0x10000) if b > 0 else (u - 0x10000)
        b = np.uint32(u & 0xFFFFFFFF).view(np.float32)
    return b


@pytest.mark.parametrize("codebook", ["eq2", "int4"])
def test_boundaries_reproduce_ieee_division_codes(codebook):
    if codebook == "eq2":
        cb = O.nf4_codebook().astype(np.float32)
    else:
        cb = np.array([(i - 8) / 8.0 for i in range(16)], dtype=np.float32)
    thr = O.snap_thresholds(cb).astype(np.float32)
    mid = [(float(t) + float(_nextdown(t))) * 0.5 for t in thr]
    incl = [(int(np.float32(t).view(np.uint32)) & 1) == 0 for t in thr]
    checked = 0
    for e in (1, 7, 100, 126, 127, 128, 200, 254):         # biased exponents of c1
        for m in range(0, 128, 17):
            cbits = (e << 7) | m
            c1 = np.uint32(cbits << 16).view(np.float32)
            B = np.array([_boundary(c1, mid[j], incl[j]) for j in range(15)], dtype=np.float32)
            w = np.arange(0, cbits + 1, dtype=np.uint32)
            w = np.concatenate([w, w | 0x8000])
            wf = (w << 16).view(np.float32)
            pad = (-w.size) % 64
            wb = np.concatenate([w, np.zeros(pad, np.uint32)]).astype(np.uint16).reshape(-1, 64)
            xq = O.normalise(wb, np.full(wb.shape[0], c1, np.float32)).reshape(-1)[:w.size]
            code_div = O.snap(xq, cb).reshape(-1)[:w.size]   # the oracle: IEEE division, nearest level
            code_bnd = (wf[:, None] >= B[None, :]).sum(axis=1)
            bad = np.flatnonzero(code_div != code_bnd)
            assert bad.size == 0, f"c1 bits {cbits:#06x}: w bits {int(w[bad[0]]):#06x}"
            checked += w.size
    assert checked > 1_000_000
