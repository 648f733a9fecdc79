"""CPU oracle for the QLoRA NF4 + double-quantized linear layer.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously-correct
statement of what the GPU library computes.  Only the test suite, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import
it; the product path never does and shares no code, table or helper with it.

Everything here is NumPy on the host.  Floating-point steps that the method
rounds (the fp32 division, the fp32 products, the BF16 and FP8 conversions) are
done in exactly that precision; the linear-layer forward and backward are done
in float64 from the BF16 inputs and the BF16 dequantized weight.

Sources (five web pages on QLoRA; cited by page title and the equation or
section the step comes from):

* "QLoRA: Efficient Fine-Tuning" (beta.fermi.ai wiki), Step 1, eq. 1 -- block
  absmax normalisation, alpha = 1; eq. 2 -- the NF4 levels
  q_i = Phi^-1((i - 1/2) / 2^k), i = 1..16; "snapped to the nearest NF4
  quantile level"; Step 2 -- double quantization of the scales to 8-bit floats
  in blocks of 256; Step 3, eq. 3 -- h = W0 x + B A x with W0 dequantized to
  BF16; the PEFT snippet -- scaling by lora_alpha / r; Step 4, eq. 5 -- the
  adapter gradients.
* "What is QLoRA?" (aquanode.io GPU glossary), "The three pieces" -- block size
  64, 0.5 -> 0.127 bits per parameter of scale overhead; "Worked example:
  Llama 3.1 8B" -- 4.127 bits/param, 1,310,720 rank-16 adapter parameters per
  block.
* "QLoRA & 4-bit Fine-Tuning" (prepfeed), "Innovation 2: Double Quantization"
  -- W ~ c1 * W_NF4, c1 quantized from FP32 to FP8 with a second scale c2.

Readings taken where the pages are silent or garbled (all documented in the
design notes; each is marked ``READING`` below):

* the codebook is eq. 2 normalised by its largest level, so that it spans
  [-1, 1] as eq. 1's normalised weights do; it is an input table;
* "nearest level" is exact: code = argmin_j |w_hat - q_j|, ties to the upper
  level.  Because w_hat is fp32 this equals counting the thresholds
  t_j = (smallest fp32 >= (q_j + q_{j+1}) / 2) that w_hat reaches;
* w_hat = RN32(w / c1) (IEEE fp32 division); an all-zero block gives w_hat = 0;
* the second-level scale is c2 = RN32(max(c1 over 256 scales) / 448) and the
  stored scale byte is FP8-E4M3FN(RN32(c1 / c2)), round-to-nearest-even with
  saturation at 448 (E4M3's largest finite value); c2 = 0 stores 0;
* dequantization is s_b = RN32(fp8(f_b) * c2), w' = BF16(RN32(q[code] * s_b));
* row-major flat order: blocks are 64 consecutive weights of a row (cols % 64
  == 0), DQ groups are 256 consecutive blocks (a trailing group may be short);
  two codes per byte, the even element in the low nibble;
* the LoRA term carries s = alpha / r: Y = X W'^T + s (X A^T) B^T, and the
  gradient through the frozen weight is dX = dY W' + s (dY B) A.
"""

from __future__ import annotations

import math
import statistics

import numpy as np

F32 = np.float32
F64 = np.float64

E4M3_MAX = 448.0          # largest finite OCP FP8 E4M3FN value: 1.75 * 2^8
BLOCKSIZE = 64            # "a scale constant for every block of 64 weights"
DQ_BLOCK = 256            # "8-bit floats with a block size of 256"


# ----------------------------------------------------------------------------
# Number formats, written from their definitions.
# ----------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """BF16 is the upper half of an IEEE binary32 word, so widening is exact."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(F32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to BF16, round-to-nearest, ties to even (finite inputs).

    Keep the upper 16 bits of the binary32 word after adding half an ulp of
    the result, where 'half' is 0x7FFF plus the kept lsb so exact halves go to
    the even neighbour.
    """
    u = np.asarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def e4m3_to_f32(byte: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal (m / 8 * 2^-6); there is no infinity and
    S.1111.111 is NaN.  Every finite value is exact in fp32.
    """
    b = np.asarray(byte, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return (sign * val).astype(F32)


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Encode fp32 to E4M3FN: round to nearest, ties to even, saturating.

    A finite value whose rounded magnitude would exceed 448 becomes +-448.
    The quantum is 2^(e-3) for |x| in [2^e, 2^(e+1)), e >= -6, and 2^-9 in the
    subnormal range below 2^-6.  Rounding is done on the exact quotient
    |x| / quantum (a power-of-two scaling, exact in float64).
    """
    v = np.asarray(x, dtype=F32).astype(F64)
    neg = np.signbit(v)
    a = np.abs(v)
    _, ex = np.frexp(a)                       # a = mant * 2^ex, mant in [0.5, 1)
    e = np.maximum(ex - 1, -6)                # unbiased exponent, floored at min normal
    quantum = np.exp2(e - 3.0)
    n = np.rint(a / quantum)                  # numpy rint: half to even
    r = np.minimum(n * quantum, E4M3_MAX)     # saturate at 448
    # encode the (now representable) magnitude
    _, rex = np.frexp(r)
    re = rex - 1
    sub = r < 2.0 ** -6
    mant_sub = np.rint(r / 2.0 ** -9)
    exp_field = np.where(sub, 0, re + 7)
    mant_norm = np.rint((r / np.exp2(re.astype(F64)) - 1.0) * 8.0)
    mant = np.where(sub, mant_sub, mant_norm)
    code = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(r == 0, 0, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


# ----------------------------------------------------------------------------
# "QLoRA: Efficient Fine-Tuning", Step 1, eq. 2: the NF4 levels.
# ----------------------------------------------------------------------------

def nf4_levels_eq2() -> np.ndarray:
    """q_i = Phi^-1((i - 1/2) / 2^k), i = 1..2^k, k = 4, in float64.

    Phi^-1 is the standard-normal quantile function from Python's statistics
    module (Wichura's algorithm AS241, accurate to about 1e-16).
    """
    nd = statistics.NormalDist(0.0, 1.0)
    k = 4
    return np.array([nd.inv_cdf((i - 0.5) / 2 ** k) for i in range(1, 2 ** k + 1)], dtype=F64)


def nf4_codebook() -> np.ndarray:
    """READING: eq. 2 normalised by its largest level, rounded to fp32.

    eq. 1 normalises each weight block to [-1, 1] before snapping, so the
    levels are divided by q_16 = Phi^-1(31/32).  Ascending; index 0..15 is
    i = 1..16.  The negative half is the exact negation of the positive half.
    """
    q = nf4_levels_eq2()
    pos = (q[8:] / q[15]).astype(F32)          # i = 9..16
    return np.concatenate([-pos[::-1], pos]).astype(F32)


def nf4_codebook_with_zero() -> np.ndarray:
    """READING: a variant of eq. 2 with an exact zero level.

    eq. 2 places no level at zero ("QLoRA: Efficient Fine-Tuning", Step 1), so
    a zero weight dequantizes to +-0.042 s.  The plainest table that keeps
    eq. 2's spacing and represents zero exactly replaces the negative level
    nearest zero, q_8, with 0: seven negative levels, zero, eight positive
    levels, all other entries equal to nf4_codebook()'s.  Ascending.
    """
    q = nf4_codebook().copy()
    q[7] = F32(0.0)
    return q


def snap_thresholds(codebook: np.ndarray) -> np.ndarray:
    """READING of "snapped to the nearest NF4 quantile level".

    t_j = the smallest fp32 value >= (q_j + q_{j+1}) / 2, j = 0..14, with the
    midpoint formed in float64.  For an fp32 w_hat, "w_hat >= t_j" then holds
    exactly when w_hat is at least as close to q_{j+1} as to q_j, so counting
    the thresholds reached gives the nearest level with ties going up.
    """
    q = np.asarray(codebook, dtype=F32).astype(F64)
    mid = (q[:-1] + q[1:]) / 2.0
    t = mid.astype(F32)                                    # round to nearest
    below = t.astype(F64) < mid
    t = np.where(below, np.nextafter(t, F32(np.inf)), t)   # ... then up if it went down
    return t.astype(F32)


# ----------------------------------------------------------------------------
# Quantization: eq. 1 absmax + nearest level, then double quantization.
# ----------------------------------------------------------------------------

def block_absmax(w_bits: np.ndarray, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """eq. 1 with alpha = 1: c1 = max |w| over each block of 64 (exact in fp32)."""
    w = bf16_bits_to_f32(w_bits).reshape(-1, blocksize)
    return np.max(np.abs(w), axis=1).astype(F32)


def normalise(w_bits: np.ndarray, c1: np.ndarray, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """eq. 1: w_hat = RN32(w / c1); READING: an all-zero block gives w_hat = 0."""
    w = bf16_bits_to_f32(w_bits).reshape(-1, blocksize)
    c = np.asarray(c1, dtype=F32)[:, None]
    safe = np.where(c > 0, c, F32(1.0)).astype(F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (w / safe).astype(F32)                 # IEEE fp32 division
    return np.where(c > 0, q, F32(0.0)).astype(F32)


def snap(w_hat: np.ndarray, codebook: np.ndarray) -> np.ndarray:
    """Nearest-level code in [0, 15]: the number of thresholds w_hat reaches."""
    t = snap_thresholds(codebook)
    flat = np.asarray(w_hat, dtype=F32).reshape(-1)
    codes = np.zeros(flat.shape, dtype=np.uint8)
    step = 1 << 20
    for s in range(0, flat.size, step):
        part = flat[s:s + step]
        codes[s:s + step] = (part[:, None] >= t[None, :]).sum(axis=1)
    return codes.reshape(np.shape(w_hat))


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte in flat order, the even element in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return (c[:, 0] | (c[:, 1] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


def double_quantize(c1: np.ndarray, dq_block: int = DQ_BLOCK):
    """Double quantization of the block scales (READING, see module header).

    Groups of 256 consecutive c1 in flat order: c2 = RN32(max / 448) in fp32,
    f = E4M3(RN32(c1 / c2)); a group whose scales are all zero stores c2 = 0
    and f = 0.  Returns (scale bytes uint8[n_blocks], c2 float32[n_groups]).
    """
    c1 = np.asarray(c1, dtype=F32)
    n = c1.size
    groups = (n + dq_block - 1) // dq_block
    c2 = np.zeros(groups, dtype=F32)
    f = np.zeros(n, dtype=np.uint8)
    for g in range(groups):
        part = c1[g * dq_block:(g + 1) * dq_block]
        c2g = (F32(np.max(part)) / F32(E4M3_MAX)).astype(F32)
        c2[g] = c2g
        if c2g > 0:
            ratio = (part / c2g).astype(F32)
            f[g * dq_block:(g + 1) * dq_block] = f32_to_e4m3(ratio)
    return f, c2


def quantize_nf4(w_bits: np.ndarray, codebook: np.ndarray | None = None,
                 blocksize: int = BLOCKSIZE, dq_block: int = DQ_BLOCK, snap_to_dq_scale: bool = False):
    """Quantize a BF16 weight W[rows, cols] (given as uint16 bit patterns).

    Returns (codes uint8[rows*cols/2], scales uint8[rows*cols/64], c2 fp32[...]).
    By default codes are snapped against the exact fp32 c1 (quantize first,
    then double-quantize the scales, in the order the prepfeed page describes
    them).  READING, variant: with snap_to_dq_scale the scales are
    double-quantized first and each block is normalised by the scale it will
    be dequantized with, s_b = RN32(fp8(f_b) * c2) (w_hat = 0 where s_b = 0),
    so that each code is the level nearest w / s_b.
    """
    if codebook is None:
        codebook = nf4_codebook()
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    assert w_bits.ndim == 2 and w_bits.shape[1] % blocksize == 0
    c1 = block_absmax(w_bits, blocksize)
    scales, c2 = double_quantize(c1, dq_block)
    divisor = block_scales(scales, c2, dq_block) if snap_to_dq_scale else c1
    codes = snap(normalise(w_bits, divisor, blocksize), codebook)
    return pack_codes(codes), scales, c2


def block_scales(scales: np.ndarray, c2: np.ndarray, dq_block: int = DQ_BLOCK) -> np.ndarray:
    """s_b = RN32(fp8(f_b) * c2_g): the scale each block is dequantized with."""
    f = e4m3_to_f32(scales)
    g = np.arange(f.size) // dq_block
    return (f * np.asarray(c2, dtype=F32)[g]).astype(F32)


def dequantize_nf4(codes: np.ndarray, scales: np.ndarray, c2: np.ndarray, rows: int, cols: int,
                   codebook: np.ndarray | None = None, blocksize: int = BLOCKSIZE,
                   dq_block: int = DQ_BLOCK) -> np.ndarray:
    """W' = BF16(RN32(q[code] * s_b)); returns uint16 BF16 bits [rows, cols]."""
    if codebook is None:
        codebook = nf4_codebook()
    q = np.asarray(codebook, dtype=F32)
    c = unpack_codes(codes).reshape(-1, blocksize)
    s = block_scales(scales, c2, dq_block)[:, None]
    w = (q[c] * s).astype(F32)
    return f32_to_bf16_bits(w).reshape(rows, cols)


# ----------------------------------------------------------------------------
# The layer: eq. 3 forward and eq. 5 backward, in float64.
# ----------------------------------------------------------------------------

def _f64(bits):
    return bf16_bits_to_f32(bits).astype(F64)


def linear_fwd(x_bits, w_deq_bits, a_bits, b_bits, s):
    """eq. 3 batched over tokens, with the PEFT scaling s = alpha / r.

    X[T, K], W'[N, K], A[r, K], B[N, r] (BF16 bits) -> Y[T, N] float64:
    Y = X W'^T + s (X A^T) B^T.
    """
    X, W, A, B = _f64(x_bits), _f64(w_deq_bits), _f64(a_bits), _f64(b_bits)
    U = X @ A.T
    return X @ W.T + float(s) * (U @ B.T)


def lora_adapter_grads(dy_bits, x_bits, a_bits, b_bits, s):
    """eq. 5 ("QLoRA: Efficient Fine-Tuning", Step 4) with the PEFT scaling,
    in float64: dU = s dY B; dB = s dY^T (X A^T); dA = dU^T X.

    Only the adapter gradients (they sum over every token; the gradient
    through the frozen weight is per token and lives in linear_bwd).
    Returns (dA[r, K], dB[N, r]).
    """
    dY, X, A, B = _f64(dy_bits), _f64(x_bits), _f64(a_bits), _f64(b_bits)
    s = float(s)
    U = X @ A.T
    dU = s * (dY @ B)
    dB = s * (dY.T @ U)
    dA = dU.T @ X
    return dA, dB


def linear_bwd(dy_bits, x_bits, w_deq_bits, a_bits, b_bits, s):
    """eq. 5 plus the gradient through the frozen weight, in float64.

    dU = s dY B; dX = dY W' + dU A; dB = s dY^T (X A^T); dA = dU^T X.
    Returns (dX[T, K], dA[r, K], dB[N, r]).  Row t of dX depends only on row t
    of dY, so dX of a subset of tokens is linear_bwd of those tokens' rows.
    """
    dY, W, A, B = _f64(dy_bits), _f64(w_deq_bits), _f64(a_bits), _f64(b_bits)
    dU = float(s) * (dY @ B)
    dX = dY @ W + dU @ A
    dA, dB = lora_adapter_grads(dy_bits, x_bits, a_bits, b_bits, s)
    return dX, dA, dB


# ----------------------------------------------------------------------------
# Storage and parameter counts ("What is QLoRA?", "The three pieces" and the
# Llama 3.1 8B worked example; "QLoRA: Efficient Fine-Tuning", eq. 4).
# ----------------------------------------------------------------------------

def merge_adapter(w_deq_bits, a_bits, b_bits, s):
    """The merged weight of "QLoRA: Efficient Fine-Tuning" Step 3 (h = W0 x + s B A x
    as one matrix): W'[N, K] + s B[N, r] A[r, K], in float64 from the BF16 dequantized
    weight and adapter.  Export rounds it to BF16 (and may quantize it again)."""
    w = _f64(w_deq_bits)
    a, b = _f64(a_bits), _f64(b_bits)
    return w + float(s) * (b @ a)


def storage_bytes(rows: int, cols: int, blocksize: int = BLOCKSIZE, dq_block: int = DQ_BLOCK):
    """(codes, scale bytes, c2 bytes) for one quantized weight."""
    n = rows * cols
    blocks = n // blocksize
    groups = (blocks + dq_block - 1) // dq_block
    return n // 2, blocks, 4 * groups


def bits_per_param(blocksize: int = BLOCKSIZE, dq_block: int = DQ_BLOCK) -> float:
    """4 code bits + one 8-bit scale per block + one fp32 c2 per DQ group."""
    return 4.0 + 8.0 / blocksize + 32.0 / (blocksize * dq_block)


def lora_params(shapes, r: int) -> int:
    """r (m + n) adapter parameters per adapted m x n weight (A is r x n, B is m x r)."""
    return sum(r * (m + n) for (m, n) in shapes)


def lora_fraction(m: int, n: int, r: int) -> float:
    """eq. 4, left-hand side: r (m + n) / (m n)."""
    return r * (m + n) / (m * n)


def normal_cdf(x: float) -> float:
    """Phi(x) = (1 + erf(x / sqrt 2)) / 2 -- used only to check eq. 2's spacing."""
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


# ----------------------------------------------------------------------------
# The adapters' optimizer step ("What is QLoRA?", "The three pieces": paged
# optimizers keep the optimizer state in unified memory; "Worked example":
# adapters in fp32 with gradients and Adam moments, 16 bytes each).
# ----------------------------------------------------------------------------

def adam_step(param, m, v, grad, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
              eps: float = 1e-8, weight_decay: float = 0.0):
    """One Adam step (Kingma & Ba, 2015, Algorithm 1) with decoupled weight
    decay (Loshchilov & Hutter, 2019), in float64:

        param <- param (1 - lr wd)
        m <- beta1 m + (1 - beta1) g;   v <- beta2 v + (1 - beta2) g^2
        param <- param - lr (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)

    READING: the pages name Adam and its fp32 moments but no formula or
    hyper-parameters; this is the published algorithm as written.  step counts
    from 1.  grad is given as BF16 bits (the layer's dA / dB); param, m, v as
    float arrays.  Returns (param, m, v) as new float64 arrays.
    """
    p = np.asarray(param, F64)
    m = np.asarray(m, F64)
    v = np.asarray(v, F64)
    g = bf16_bits_to_f32(grad).astype(F64).reshape(p.shape)
    p = p * (1.0 - lr * weight_decay)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    p = p - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p, m, v
