"""Pins for the CPU oracle: each check ties it to something other than itself.

The pages print no tensor values, so the oracle is pinned by closed forms,
invariants, brute force on tiny inputs, an independent number-format library
(ml_dtypes), an independent quantile routine (scipy), the pages' printed
storage and parameter counts, and exact finite differences.
"""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import scipy.special
import torch

from oracle import oracle as O
from bit_nf4_quantized_20_b200 import inputs

F32, F64 = np.float32, np.float64


# --------------------------------------------------------------------------
# eq. 2 codebook ("QLoRA: Efficient Fine-Tuning", Step 1)
# --------------------------------------------------------------------------

def test_codebook_shape_order_symmetry_ends():
    q = O.nf4_codebook()
    assert q.dtype == F32 and q.shape == (16,)
    assert np.all(np.diff(q.astype(F64)) > 0)                # strictly increasing
    assert q[0] == F32(-1.0) and q[15] == F32(1.0)            # normalised to [-1, 1]
    assert np.array_equal(q.view(np.uint32), (-q[::-1]).view(np.uint32))  # exact symmetry
    assert not np.any(q == 0)                                  # eq. 2 has no zero level


def test_codebook_equal_probability_mass():
    """Phi(q_i) - Phi(q_{i-1}) = 1/16: the levels sit at the centres of 16
    equal-probability intervals (eq. 2, 'equal-probability intervals')."""
    p = O.nf4_levels_eq2()
    cdf = np.array([O.normal_cdf(v) for v in p])
    assert np.allclose(cdf, (np.arange(1, 17) - 0.5) / 16, atol=1e-13, rtol=0)
    assert np.allclose(np.diff(cdf), 1 / 16, atol=1e-13, rtol=0)


def test_codebook_matches_scipy_ndtri():
    p = O.nf4_levels_eq2()
    ref = scipy.special.ndtri((np.arange(1, 17) - 0.5) / 16)
    assert np.allclose(p, ref, atol=1e-13, rtol=0)
    q = O.nf4_codebook()
    assert np.allclose(q.astype(F64), np.concatenate([-ref[8:][::-1], ref[8:]]) / ref[15], atol=1e-7)


def test_codebook_golden_fixture():
    """Regression fixture written by tests/golden/make_golden.py (oracle only)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nf4_codebook_eq2.txt")
    vals = []
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            vals.append(int(line.split()[0], 16))
    assert np.array_equal(np.array(vals, dtype=np.uint32), O.nf4_codebook().view(np.uint32))


# --------------------------------------------------------------------------
# nearest-level snapping ("snapped to the nearest NF4 quantile level")
# --------------------------------------------------------------------------

def _brute_nearest(v: float, q: np.ndarray) -> int:
    """argmin_j |v - q_j| in exact rational arithmetic, ties to the upper level."""
    best, bestd = 0, None
    fv = Fraction(float(v))
    for j in range(16):
        d = abs(fv - Fraction(float(q[j])))
        if bestd is None or d <= bestd:   # '<=' walks upward, so ties resolve to the larger j
            best, bestd = j, d
    return best


def test_thresholds_are_exact_midpoint_ceilings():
    q = [Fraction(float(v)) for v in O.nf4_codebook()]
    t = O.snap_thresholds(O.nf4_codebook())
    for j in range(15):
        tj = Fraction(float(t[j]))
        below = Fraction(float(np.nextafter(t[j], F32(-np.inf))))
        assert abs(tj - q[j + 1]) <= abs(tj - q[j])          # t_j snaps up
        assert abs(below - q[j]) < abs(below - q[j + 1])     # the fp32 below it snaps down
    assert t[7] == 0.0


def test_snap_equals_brute_force_nearest():
    q = O.nf4_codebook()
    t = O.snap_thresholds(q)
    rng = np.random.default_rng(7)
    cand = list(rng.uniform(-1, 1, 3000).astype(F32))
    for tj in t:                                   # every boundary and its fp32 neighbours
        for k in range(-3, 4):
            v = tj
            step = F32(np.inf) if k > 0 else F32(-np.inf)
            for _ in range(abs(k)):
                v = np.nextafter(v, step)
            cand.append(F32(v))
    cand += [F32(0.0), F32(-0.0), F32(1.0), F32(-1.0), F32(1e-45), F32(-1e-45)]
    cand += list(q) + [F32((float(q[j]) + float(q[j + 1])) / 2) for j in range(15)]
    cand = np.array(cand, dtype=F32)
    got = O.snap(cand, q)
    want = np.array([_brute_nearest(v, q) for v in cand])
    assert np.array_equal(got, want)
    # signed zero: -0.0 reaches the zero threshold, like +0.0
    assert O.snap(np.array([-0.0], F32), q)[0] == 8


def test_normalise_is_ieee_fp32_division():
    """RN32(w / c1) equals RN32(RN64(w / c1)): double rounding through binary64
    is innocuous for division (53 >= 2*24 + 2), so Python's float division is an
    independent check of the fp32 quotient."""
    rng = np.random.default_rng(3)
    w = inputs.bf16_bits(torch.from_numpy(rng.normal(0, 0.02, (4, 64)).astype(F32)).to(torch.bfloat16))
    c1 = O.block_absmax(w)
    got = O.normalise(w, c1)
    wf = O.bf16_bits_to_f32(w).reshape(-1, 64)
    for b in range(4):
        assert c1[b] == max(abs(float(v)) for v in wf[b])          # eq. 1 absmax
        for i in range(64):
            assert got[b, i] == F32(float(wf[b, i]) / float(c1[b]))


# --------------------------------------------------------------------------
# number formats against an independent implementation (ml_dtypes)
# --------------------------------------------------------------------------

def _dense_f32_sweep(lo, hi, n, seed):
    rng = np.random.default_rng(seed)
    return rng.uniform(lo, hi, n).astype(F32)


def test_bf16_rne_matches_ml_dtypes():
    x = np.concatenate([
        _dense_f32_sweep(-4, 4, 200000, 1),
        _dense_f32_sweep(-1e-36, 1e-36, 20000, 2),
        _dense_f32_sweep(-3e38, 3e38, 20000, 3),
    ])
    # exact ties: a bf16 value plus half a bf16 ulp
    base = np.arange(0x3F80, 0x4080, dtype=np.uint32) << 16
    ties = (base | 0x8000).view(F32)
    x = np.concatenate([x, ties, -ties]).astype(F32)
    got = O.f32_to_bf16_bits(x)
    want = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(got, want)
    tw = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, tw)


def test_e4m3_decode_matches_ml_dtypes():
    b = np.arange(256, dtype=np.uint8)
    finite = ~(((b & 0x7F) == 0x7F))
    got = O.e4m3_to_f32(b)
    want = b.view(ml_dtypes.float8_e4m3fn).astype(F32)
    assert np.array_equal(got[finite], want[finite])
    assert np.all(np.isnan(got[~finite]))


def test_e4m3_encode_matches_ml_dtypes_below_saturation():
    allv = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(F64)
    allv = np.unique(allv[np.isfinite(allv) & (allv >= 0)])
    mids = (allv[:-1] + allv[1:]) / 2                                 # exact ties
    near = np.concatenate([np.nextafter(mids.astype(F32), F32(0)), np.nextafter(mids.astype(F32), F32(1e9))])
    x = np.concatenate([allv.astype(F32), mids.astype(F32), near,
                        _dense_f32_sweep(0, 463.9, 300000, 4),
                        _dense_f32_sweep(0, 0.02, 100000, 5)]).astype(F32)
    x = x[x < 464.0]
    got = O.f32_to_e4m3(x)
    want = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got, want)
    assert np.array_equal(O.f32_to_e4m3(-x), want | 0x80)


def test_e4m3_saturates_at_448():
    x = np.array([464.0, 500.0, 1e6, 3e38], dtype=F32)
    assert np.all(O.f32_to_e4m3(x) == 0x7E)
    assert O.e4m3_to_f32(np.array([0x7E], np.uint8))[0] == 448.0


# --------------------------------------------------------------------------
# double quantization ("QLoRA & 4-bit Fine-Tuning", Innovation 2)
# --------------------------------------------------------------------------

def test_double_quantization_rule_and_error_bound():
    rng = np.random.default_rng(11)
    c1 = np.abs(rng.normal(0, 0.02, 1000)).astype(F32) + F32(0.01)
    f, c2 = O.double_quantize(c1)
    assert c2.shape == (4,)                                  # ceil(1000 / 256), last group short
    for g in range(4):
        part = c1[g * 256:(g + 1) * 256]
        assert c2[g] == F32(float(part.max()) / 448.0)       # fp32 RN of max/448 (innocuous double rounding)
        dec = O.e4m3_to_f32(f[g * 256:(g + 1) * 256]).astype(F64) * float(c2[g])
        # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal range
        assert np.all(np.abs(dec - part) <= 2.0 ** -4 * part + 1e-30)
        assert f[g * 256 + int(np.argmax(part))] == 0x7E     # the group max maps to 448


def test_double_quantization_zero_group():
    f, c2 = O.double_quantize(np.zeros(300, F32))
    assert np.all(f == 0) and np.all(c2 == 0)


# --------------------------------------------------------------------------
# quantize / dequantize as a whole
# --------------------------------------------------------------------------

def _w(rows, cols, seed, std=0.02):
    return inputs.bf16_bits(inputs.normal_bf16((rows, cols), std, seed))


def test_quantize_special_blocks():
    w = np.zeros((1, 256), np.uint16)                # block 0: all zero (+0.0)
    w[0, 64:128] = 0x8000                            # block 1: all -0.0
    w[0, 128 + 5] = 0x3F80                           # block 2: one-hot +1.0
    w[0, 192 + 9] = 0xBF80                           # block 3: one-hot -1.0
    codes, scales, c2 = O.quantize_nf4(w)
    c = O.unpack_codes(codes)
    assert np.all(c[:128] == 8)                      # w_hat = 0 snaps to the level just above 0
    assert c[128 + 5] == 15 and c[192 + 9] == 0
    assert np.all(np.delete(c[128:], [5, 64 + 9]) == 8)
    assert np.array_equal(scales, [0, 0, 0x7E, 0x7E])
    assert c2[0] == F32(1.0 / 448.0)
    wd = O.dequantize_nf4(codes, scales, c2, 1, 256)
    assert np.all(wd[0, :128] == 0) and wd[0, 128 + 5] == 0x3F80 and wd[0, 192 + 9] == 0xBF80


def test_dequant_error_bound():
    """|w - w'| <= c1 * (largest half-gap of the codebook + E4M3 and BF16 rounding)."""
    w = _w(64, 512, 5)
    codes, scales, c2 = O.quantize_nf4(w)
    wd = O.dequantize_nf4(codes, scales, c2, 64, 512)
    q = O.nf4_codebook().astype(F64)
    half_gap = np.max(np.diff(q)) / 2
    err = np.abs(O.bf16_bits_to_f32(wd).astype(F64) - O.bf16_bits_to_f32(w).astype(F64)).reshape(-1, 64)
    c1 = O.block_absmax(w).astype(F64)[:, None]
    assert np.all(err <= c1 * (half_gap + 2.0 ** -4 * 1.07 + 2.0 ** -8 * 1.07))


def test_quantize_codes_are_nearest_levels_brute_force():
    w = _w(2, 128, 9)
    codes, _, _ = O.quantize_nf4(w)
    c = O.unpack_codes(codes).reshape(-1, 64)
    wf = O.bf16_bits_to_f32(w).reshape(-1, 64)
    q = O.nf4_codebook()
    for b in range(wf.shape[0]):
        m = max(abs(float(v)) for v in wf[b])
        for i in range(64):
            assert c[b, i] == _brute_nearest(F32(float(wf[b, i]) / m), q)


def test_nf4_beats_uniform_4bit_tables_on_normal_weights():
    """"QLoRA & 4-bit Fine-Tuning" (Innovation 1) contrasts NF4 with uniform
    INT4 for normally distributed weights: through the same blockwise absmax
    + double quantization, eq. 2's levels give a lower round-trip error on
    N(0, 0.02^2) weights than the INT4 table (-1 .. 7/8, an exact zero) and
    than 16 evenly spaced levels on [-1, 1]."""
    rows, cols = 256, 4096
    wb = _bits((rows, cols), 0.02, 123)
    w = O.bf16_bits_to_f32(wb).astype(F64)

    def rms(cb):
        codes, scales, c2 = O.quantize_nf4(wb, cb)
        wd = O.bf16_bits_to_f32(O.dequantize_nf4(codes, scales, c2, rows, cols, cb)).astype(F64)
        return float(np.sqrt(((wd - w) ** 2).mean()))

    nf4 = rms(O.nf4_codebook().astype(np.float32))
    int4 = rms(np.array([(i - 8) / 8.0 for i in range(16)], np.float32))
    uni = rms(np.array([(2 * i - 15) / 15.0 for i in range(16)], np.float32))
    assert nf4 < 0.97 * int4 and nf4 < 0.97 * uni, (nf4, int4, uni)


def test_packing_low_nibble_is_even_element():
    assert np.array_equal(O.pack_codes(np.array([1, 2, 15, 0], np.uint8)), [0x21, 0x0F])
    assert np.array_equal(O.unpack_codes(np.array([0x21, 0x0F], np.uint8)), [1, 2, 15, 0])


def test_quantize_dequantize_idempotent():
    """Q(D(Q(W))) = Q(W) bit-exactly (codes, scale bytes, c2)."""
    w = _w(512, 512, 42)
    codes, scales, c2 = O.quantize_nf4(w)
    wd = O.dequantize_nf4(codes, scales, c2, 512, 512)
    codes2, scales2, c22 = O.quantize_nf4(wd)
    assert np.array_equal(codes, codes2)
    assert np.array_equal(scales, scales2)
    assert np.array_equal(c2.view(np.uint32), c22.view(np.uint32))


# --------------------------------------------------------------------------
# storage and parameter counts printed on the pages
# --------------------------------------------------------------------------

LLAMA8B = [(n, k) for (_, n, k) in inputs.LLAMA8B_PROJ]


def test_storage_overhead_0127_bits():
    """'What is QLoRA?': 0.5 -> 0.127 bits of scale overhead, 4.127 bits/param."""
    assert 32 / 64 == 0.5
    assert O.bits_per_param() == 4.126953125
    assert round(O.bits_per_param() - 4, 3) == 0.127
    assert round(0.5 - (O.bits_per_param() - 4), 2) == 0.37          # "saving about 0.37 bits"


def test_storage_llama8b_4_14_gb():
    """8.03e9 x 4.127 / 8 = 4.14 GB for the Llama 3.1 8B worked example."""
    assert round(8.03e9 * O.bits_per_param() / 8 / 1e9, 2) == 4.14
    assert round(8.03e9 * 2 / 1e9, 2) == 16.06                       # BF16 figure on the same page


def test_storage_32_layer_stack_exact():
    total_w, total_b = 0, 0
    for (n, k) in LLAMA8B:
        total_w += n * k
        total_b += sum(O.storage_bytes(n, k))
    total_w *= 32
    total_b *= 32
    assert total_w == 6_979_321_856
    assert total_b == 3_489_660_928 + 109_051_904 + 1_703_936 == 3_600_416_768
    assert total_b * 8 / total_w == O.bits_per_param()


def test_adapter_parameter_counts():
    """1,310,720 rank-16 adapter parameters per 8B block ('What is QLoRA?')."""
    per_block = O.lora_params(LLAMA8B, 16)
    assert per_block == 1_310_720
    assert round(per_block * 32 / 1e6, 1) == 41.9
    assert round(per_block * 32 * 16 / 1e9, 2) == 0.67                # fp32 + grads + Adam
    assert 4096 * 8 + 8 * 4096 == 65_536                              # rank-8 example, 4096 x 4096


def test_eq4_ratio():
    """eq. 4: r (m + n) / (m n) ~ r / min(m, n).  For 4096 x 4096 at r = 16 the
    exact value is 0.78 %, twice the page's '< 0.4 %' (recorded as a page error)."""
    assert O.lora_fraction(4096, 4096, 16) == 0.0078125
    assert abs(O.lora_fraction(8192, 4096, 8) - 8 / 4096) / (8 / 4096) < 0.51


# --------------------------------------------------------------------------
# eq. 3 forward and eq. 5 backward
# --------------------------------------------------------------------------

def _bits(shape, std, seed):
    return inputs.bf16_bits(inputs.normal_bf16(shape, std, seed))


def test_forward_brute_force_eq3():
    """h = W0 x + s B (A x) per token, as explicit scalar loops in the page's
    notation (W0 in R^{m x n}, A in R^{r x n}, B in R^{m x r}); odd sizes so a
    transposed operand cannot pass."""
    T, m, n, r, s = 3, 5, 7, 2, 1.75
    X, W, A, B = _bits((T, n), 1, 1), _bits((m, n), 0.1, 2), _bits((r, n), 0.3, 3), _bits((m, r), 0.2, 4)
    Y = O.linear_fwd(X, W, A, B, s)
    Xf, Wf, Af, Bf = (O.bf16_bits_to_f32(v).astype(F64) for v in (X, W, A, B))
    for t in range(T):
        ax = [sum(Af[i, j] * Xf[t, j] for j in range(n)) for i in range(r)]
        for o in range(m):
            h = sum(Wf[o, j] * Xf[t, j] for j in range(n)) + s * sum(Bf[o, i] * ax[i] for i in range(r))
            assert abs(Y[t, o] - h) <= 1e-12 * (1 + abs(h))


def test_forward_merged_weight_identity():
    """W' = W + s B A (the merged form): X (W + s B A)^T equals eq. 3."""
    T, m, n, r, s = 4, 6, 64, 3, 2.0
    X, W, A, B = _bits((T, n), 1, 5), _bits((m, n), 0.02, 6), _bits((r, n), 0.1, 7), _bits((m, r), 0.05, 8)
    Wm = O.bf16_bits_to_f32(W).astype(F64) + s * O.bf16_bits_to_f32(B).astype(F64) @ O.bf16_bits_to_f32(A).astype(F64)
    ref = O.bf16_bits_to_f32(X).astype(F64) @ Wm.T
    assert np.allclose(O.linear_fwd(X, W, A, B, s), ref, rtol=1e-12, atol=1e-12)
    # s = 0 (or B = 0) leaves the frozen layer alone
    zero = np.zeros_like(B)
    assert np.allclose(O.linear_fwd(X, W, A, zero, s), O.linear_fwd(X, W, A, B, 0.0), rtol=0, atol=1e-14)


def test_merge_adapter_elementwise_and_forward_identity():
    """merge_adapter = W' + s B A: element by element as an explicit sum over the
    rank, and X merged^T equals eq. 3's forward (the point of merging)."""
    T, m, n, r, s = 3, 5, 64, 3, 0.75
    X, W, A, B = _bits((T, n), 1, 15), _bits((m, n), 0.02, 16), _bits((r, n), 0.1, 17), _bits((m, r), 0.05, 18)
    M = O.merge_adapter(W, A, B, s)
    w, a, b = (O.bf16_bits_to_f32(v).astype(F64) for v in (W, A, B))
    for i in range(m):
        for k in range(n):
            ref = w[i, k] + s * sum(b[i, j] * a[j, k] for j in range(r))
            assert abs(M[i, k] - ref) <= 1e-15 * max(1.0, abs(ref))
    assert np.allclose(O.bf16_bits_to_f32(X).astype(F64) @ M.T, O.linear_fwd(X, W, A, B, s), rtol=1e-12, atol=1e-12)
    assert np.array_equal(O.merge_adapter(W, A, B, 0.0), w)


def test_backward_eq5_per_token_outer_products():
    """eq. 5: dL/dA = B^T g x^T and dL/dB = g (A x)^T per token (times s), summed."""
    T, m, n, r, s = 3, 5, 7, 2, 0.5
    X, W, A, B, dY = (_bits((T, n), 1, 11), _bits((m, n), 0.1, 12), _bits((r, n), 0.3, 13),
                      _bits((m, r), 0.2, 14), _bits((T, m), 1, 15))
    dX, dA, dB = O.linear_bwd(dY, X, W, A, B, s)
    Xf, Wf, Af, Bf, G = (O.bf16_bits_to_f32(v).astype(F64) for v in (X, W, A, B, dY))
    dA_ref = np.zeros((r, n))
    dB_ref = np.zeros((m, r))
    dX_ref = np.zeros((T, n))
    for t in range(T):
        g, x = G[t], Xf[t]
        btg = [sum(Bf[o, i] * g[o] for o in range(m)) for i in range(r)]
        ax = [sum(Af[i, j] * x[j] for j in range(n)) for i in range(r)]
        for i in range(r):
            for j in range(n):
                dA_ref[i, j] += s * btg[i] * x[j]
        for o in range(m):
            for i in range(r):
                dB_ref[o, i] += s * g[o] * ax[i]
        for j in range(n):
            dX_ref[t, j] = sum(g[o] * Wf[o, j] for o in range(m)) + s * sum(btg[i] * Af[i, j] for i in range(r))
    assert np.allclose(dA, dA_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(dB, dB_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(dX, dX_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("which", ["X", "A", "B"])
def test_backward_is_the_derivative_of_the_forward(which):
    """L = <dY, Y> is linear in each of X, A and B separately, so a central
    difference is exact up to rounding: dL/dV . D = (L(V + eD) - L(V - eD)) / 2e."""
    T, m, n, r, s = 6, 9, 64, 4, 2.0
    X, W, A, B, dY = (_bits((T, n), 1, 21), _bits((m, n), 0.02, 22), _bits((r, n), 0.1, 23),
                      _bits((m, r), 0.05, 24), _bits((T, m), 1, 25))
    dX, dA, dB = O.linear_bwd(dY, X, W, A, B, s)
    Xf, Wf, Af, Bf, G = (O.bf16_bits_to_f32(v).astype(F64) for v in (X, W, A, B, dY))

    def L(Xv, Av, Bv):
        Y = Xv @ Wf.T + s * (Xv @ Av.T) @ Bv.T
        return float(np.sum(G * Y))

    rng = np.random.default_rng(99)
    e = 1e-3
    if which == "X":
        D = rng.normal(size=Xf.shape)
        fd = (L(Xf + e * D, Af, Bf) - L(Xf - e * D, Af, Bf)) / (2 * e)
        an = float(np.sum(dX * D))
    elif which == "A":
        D = rng.normal(size=Af.shape)
        fd = (L(Xf, Af + e * D, Bf) - L(Xf, Af - e * D, Bf)) / (2 * e)
        an = float(np.sum(dA * D))
    else:
        D = rng.normal(size=Bf.shape)
        fd = (L(Xf, Af, Bf + e * D) - L(Xf, Af, Bf - e * D)) / (2 * e)
        an = float(np.sum(dB * D))
    assert abs(fd - an) <= 1e-8 * (1 + abs(an))


# --------------------------------------------------------------------------
# codebook variants ("QLoRA & 4-bit Fine-Tuning", Innovation 1 and 2)
# --------------------------------------------------------------------------

def test_codebook_with_zero_level():
    """eq. 2 with its negative level nearest zero replaced by an exact 0: still
    ascending, ends at -1 and +1, zero present, the other 15 entries eq. 2's."""
    z = O.nf4_codebook_with_zero()
    q = O.nf4_codebook()
    assert z.dtype == F32 and z.shape == (16,)
    assert np.all(np.diff(z.astype(F64)) > 0)
    assert z[7] == 0.0 and not np.signbit(z[7])
    keep = np.arange(16) != 7
    assert np.array_equal(z[keep].view(np.uint32), q[keep].view(np.uint32))
    assert z[0] == -1.0 and z[15] == 1.0
    # a zero weight in a non-zero block now dequantizes to exactly zero
    w = np.zeros((1, 64), np.uint16)
    w[0, 3] = 0x3C00                                   # one non-zero weight (2^-7)
    codes, scales, c2 = O.quantize_nf4(w, z)
    wd = O.dequantize_nf4(codes, scales, c2, 1, 64, z)
    assert np.all(wd[0, np.arange(64) != 3] == 0) and wd[0, 3] == 0x3C00


def _scale_of_bytes(scales, c2, dq=256):
    """s_b = RN32(fp8 * c2) with the FP8 bytes decoded by ml_dtypes."""
    f = np.asarray(scales, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(F32)
    return (f * np.asarray(c2, F32)[np.arange(f.size) // dq]).astype(F32)


def test_dq_scale_snapping_is_nearest_level_of_w_over_sb():
    """The variant that snaps against the double-quantized scale: each code is
    the level nearest RN32(w / s_b) (exact rational brute force, ties up), with
    s_b decoded independently; the scale bytes and c2 are the default's."""
    w = _w(4, 256, 19)
    for cb in (O.nf4_codebook(), O.nf4_codebook_with_zero()):
        codes, scales, c2 = O.quantize_nf4(w, cb, snap_to_dq_scale=True)
        codes0, scales0, c20 = O.quantize_nf4(w, cb)
        assert np.array_equal(scales, scales0) and np.array_equal(c2.view(np.uint32), c20.view(np.uint32))
        sb = _scale_of_bytes(scales, c2)
        c = O.unpack_codes(codes).reshape(-1, 64)
        wf = O.bf16_bits_to_f32(w).reshape(-1, 64)
        for b in range(wf.shape[0]):
            for i in range(64):
                v = F32(wf[b, i] / sb[b]) if sb[b] > 0 else F32(0.0)
                assert c[b, i] == _brute_nearest(v, cb)


def test_dq_scale_snapping_worked_example():
    """A group whose largest scale is 1.0 (c2 = RN32(1/448)) and a block with
    c1 = 0.9: 0.9 / c2 = 403.2 lies between the E4M3 values 384 and 416 and
    rounds to 416, so that block is dequantized with s_b = RN32(416 c2) =
    0.92857.. > c1.  A weight just above 0.9 t_14 (the threshold to the top
    level) snaps to level 15 against c1 but to level 14 against s_b."""
    q = O.nf4_codebook()
    t14 = float(O.snap_thresholds(q)[14])
    c2 = F32(F32(1.0) / F32(448.0))
    sb = F32(F32(416.0) * c2)
    w = np.zeros((1, 128), np.float32)
    w[0, 0] = 1.0                                     # block 0: c1 = 1.0, the group max
    w[0, 64] = 0.9                                    # block 1: c1 = 0.9 (BF16 0.8984375)
    c1 = float(ml_dtypes.bfloat16(0.9))
    # the smallest BF16 value above c1 * t14: reaches t14 against c1 ...
    x = ml_dtypes.bfloat16(c1 * t14)
    while float(x) < c1 * t14:
        x = np.nextafter(x, ml_dtypes.bfloat16(1.0))
    w[0, 65] = float(x)
    wb = w.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert float(x) / c1 >= t14 and float(x) / float(sb) < t14   # ... but not against s_b
    codes0, scales, c2g = O.quantize_nf4(wb, q)
    codes1, _, _ = O.quantize_nf4(wb, q, snap_to_dq_scale=True)
    assert c2g[0] == c2 and scales[1] == 0x7D                     # E4M3 0x7D = 1.625 * 2^8 = 416
    assert O.unpack_codes(codes0)[65] == 15 and O.unpack_codes(codes1)[65] == 14
    assert O.unpack_codes(codes0)[0] == O.unpack_codes(codes1)[0] == 15


def test_dq_scale_snapping_equals_default_when_scales_are_exact():
    """When every c1 is exactly an E4M3 multiple of c2 (here: powers of two
    with the group max 448 * 2^-12, so c2 = 2^-12), s_b == c1 and the variant
    gives the default's codes bit for bit."""
    rng = np.random.default_rng(5)
    w = rng.normal(0, 1, (4, 64 * 64)).astype(np.float32).reshape(-1, 64)
    w /= np.max(np.abs(w), axis=1, keepdims=True)                 # each block's absmax 1 ...
    w *= np.exp2(rng.integers(-20, -12, (w.shape[0], 1))).astype(np.float32)  # ... times 2^e
    w[0] *= 448.0 * 2.0 ** -12 / np.max(np.abs(w[0]))              # group max 448 * 2^-12
    wb = w.reshape(4, -1).astype(ml_dtypes.bfloat16).view(np.uint16)
    c1 = O.block_absmax(wb)
    _, scales, c2 = O.quantize_nf4(wb)
    assert np.array_equal(_scale_of_bytes(scales, c2), c1)
    assert np.array_equal(O.quantize_nf4(wb, snap_to_dq_scale=True)[0], O.quantize_nf4(wb)[0])


def test_dq_scale_snapping_lowers_the_round_trip_error():
    """Dequantization multiplies by s_b, so snapping against s_b picks, per
    weight, the level whose reconstruction is nearest: on N(0, 0.02^2) weights
    no weight's error grows and the RMS error falls, for each table."""
    rows, cols = 64, 4096
    wb = _bits((rows, cols), 0.02, 321)
    w = O.bf16_bits_to_f32(wb).astype(F64)
    tables = [O.nf4_codebook(), O.nf4_codebook_with_zero(), np.array([(i - 8) / 8.0 for i in range(16)], F32)]
    for cb in tables:
        errs = []
        for dq in (False, True):
            codes, scales, c2 = O.quantize_nf4(wb, cb, snap_to_dq_scale=dq)
            qv = cb.astype(F64)[O.unpack_codes(codes)].reshape(rows, cols)
            sb = _scale_of_bytes(scales, c2).astype(F64).repeat(64).reshape(rows, cols)
            errs.append(np.abs(qv * sb - w))        # reconstruction before the final BF16 rounding
        assert np.all(errs[1] <= errs[0] * (1 + 1e-6) + 1e-12)
        assert np.sqrt((errs[1] ** 2).mean()) < 0.999 * np.sqrt((errs[0] ** 2).mean())


# --------------------------------------------------------------------------
# the adapters' optimizer step (Adam with decoupled weight decay)
# --------------------------------------------------------------------------

def test_adam_first_step_is_lr_times_sign():
    """From zero moments the first step's bias-corrected m and v are g and g^2,
    so each parameter moves by lr g / (|g| + eps)."""
    g = _bits((1, 257), 0.3, 41)
    gf = O.bf16_bits_to_f32(g).astype(F64).reshape(-1)
    p0 = np.linspace(-1, 1, 257)
    p, m, v = O.adam_step(p0, np.zeros(257), np.zeros(257), g, 1, lr=1e-3, eps=1e-8)
    assert np.allclose(p, p0 - 1e-3 * gf / (np.abs(gf) + 1e-8), rtol=0, atol=1e-15)
    assert np.allclose(m, 0.1 * gf) and np.allclose(v, 0.001 * gf * gf)


def test_adam_constant_gradient_closed_form():
    """With the same gradient every step the bias-corrected moments stay g and
    g^2, so after t steps param = p0 - t lr g / (|g| + eps)."""
    g = _bits((1, 64), 0.5, 42)
    gf = O.bf16_bits_to_f32(g).astype(F64).reshape(-1)
    p, m, v = np.ones(64), np.zeros(64), np.zeros(64)
    for t in range(1, 26):
        p, m, v = O.adam_step(p, m, v, g, t, lr=2e-3, beta1=0.8, beta2=0.95, eps=1e-6)
    assert np.allclose(p, 1.0 - 25 * 2e-3 * gf / (np.abs(gf) + 1e-6), rtol=0, atol=1e-12)


def test_adam_weight_decay_alone_is_geometric():
    g = np.zeros(16, np.uint16)                       # BF16 +0.0 gradients
    p = np.full(16, 3.0)
    m, v = np.zeros(16), np.zeros(16)
    for t in range(1, 11):
        p, m, v = O.adam_step(p, m, v, g, t, lr=0.01, weight_decay=0.1)
    assert np.allclose(p, 3.0 * (1 - 0.01 * 0.1) ** 10, rtol=1e-15)


def test_adam_matches_torch_adamw():
    """Seven steps against torch.optim.AdamW (an independent implementation of
    the same published algorithm) in float64 on the CPU."""
    n = 1000
    p0 = np.random.default_rng(3).normal(0, 0.05, n)
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], lr=3e-3, betas=(0.85, 0.98), eps=1e-7, weight_decay=0.05)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 8):
        g = _bits((1, n), 0.02, 100 + t).reshape(-1)
        tp.grad = torch.from_numpy(O.bf16_bits_to_f32(g).astype(F64))
        opt.step()
        p, m, v = O.adam_step(p, m, v, g, t, lr=3e-3, beta1=0.85, beta2=0.98, eps=1e-7, weight_decay=0.05)
    assert np.allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-16)
