"""Every workload of the layer, at its full size, against the CPU oracle.

The Llama-3.1-8B block (seven projections, 4096 tokens, rank 16, s = 2) in the
launch configuration the bench times (the forward that saves U, the backward
that reuses it) and through the plain forward/backward; the 65B-shaped
projections (hidden 8192, ffn 22016) on 4 x 512 tokens at rank 64, s = 0.25;
the decode sweep (the seven 8B shapes at 1, 4 and 16 tokens, rank 64, s = 1);
and the code function over every (w, c1) pair of BF16 values.

Oracle values: quantize and dequantize bit for bit; the forward and the
gradient through the frozen weight on sampled tokens (each token's output row
is the oracle's forward of that token alone), the adapter gradients dA and dB
in full (they sum over every token).  Tolerance |gpu - oracle| <= 5e-3 +
1e-2 |oracle| per element.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from bit_nf4_quantized_20_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 5e-3, 1e-2


def Q():
    import bit_nf4_quantized_20_b200 as q
    return q


def bits(t):
    return inputs.bf16_bits(t)


def assert_close(name, gpu_bf16, ref64):
    g = O.bf16_bits_to_f32(bits(gpu_bf16)).astype(np.float64).reshape(ref64.shape)
    err = np.abs(g - ref64)
    tol = TOL_ABS + TOL_REL * np.abs(ref64)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu={g[i]!r} oracle={ref64[i]!r}")


def quantize_checked(W):
    """GPU quantize of W, bit-exact against the oracle; returns (qw, W' bits)."""
    q = Q()
    qw = q.quantize_nf4(W)
    torch.cuda.synchronize()
    wb = bits(W)
    codes, scales, c2 = O.quantize_nf4(wb)
    assert np.array_equal(qw.c2.cpu().numpy().view(np.uint32), c2.view(np.uint32)), "c2"
    assert np.array_equal(qw.scales.cpu().numpy(), scales), "scale bytes"
    assert np.array_equal(qw.codes.cpu().numpy(), codes), "codes"
    N, K = W.shape
    return qw, O.dequantize_nf4(codes, scales, c2, N, K)


def check_fwd_bwd_sampled(X, A, B, dY, wd, s, rows, y, dx, dA, dB):
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    idx = torch.from_numpy(rows).to(y.device)
    assert_close("Y[rows]", y[idx], O.linear_fwd(xb[rows], wd, ab, bb, s))
    rdx, _, _ = O.linear_bwd(dyb[rows], xb[rows], wd, ab, bb, s)
    assert_close("dX[rows]", dx[idx], rdx)
    rdA, rdB = O.lora_adapter_grads(dyb, xb, ab, bb, s)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)


# --------------------------------------------------------------------------
# Llama-3.1-8B block, T = 4096, rank 16, s = 2 (the bench's workload)
# --------------------------------------------------------------------------
ROWS_4096 = np.array([0, 1, 127, 128, 255, 256, 1000, 2047, 2048, 3333, 4094, 4095])


@pytest.mark.parametrize("proj", range(7), ids=[p[0] for p in inputs.LLAMA8B_PROJ])
def test_8b_block_projection_full_size(proj):
    """One projection of the block at T = 4096, r = 16, s = 2, seeded as the
    bench seeds it: forward with U saved, backward reusing it (the path the
    bench times), and the plain backward, which recomputes U from X."""
    q = Q()
    name, N, K = inputs.LLAMA8B_PROJ[proj]
    T, r, s = 4096, 16, 2.0
    W, X, A, B, dY = inputs.layer_inputs(1, 0, proj, T, N, K, r, device="cuda")
    qw, wd = quantize_checked(W)
    del W
    y, u = q.linear_fwd_save(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd_saved(dY, X, qw, A, B, s, u)
    q.get_error()
    torch.cuda.synchronize()
    check_fwd_bwd_sampled(X, A, B, dY, wd, s, ROWS_4096, y, dx, dA, dB)
    # the plain pair of calls gives the same forward bit for bit and a
    # backward within the rounding of the FP32 sums
    y2 = q.linear_fwd(X, qw, A, B, s)
    dx2, dA2, dB2 = q.linear_bwd(dY, X, qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    check_fwd_bwd_sampled(X, A, B, dY, wd, s, ROWS_4096[::3], y2, dx2, dA2, dB2)


# --------------------------------------------------------------------------
# 65B-shaped stack, layer by layer: T = 4 x 512, rank 64, s = 0.25
# --------------------------------------------------------------------------
@pytest.mark.parametrize("layer,proj", [(0, 0), (0, 4), (0, 6), (40, 0), (40, 4), (40, 6), (79, 0), (79, 4), (79, 6)],
                         ids=lambda v: str(v))
def test_65b_projection_full_size(layer, proj):
    """The three distinct shapes of a 65B-shaped layer (8192 <- 8192 for q, k,
    v, o; 22016 <- 8192 for gate, up; 8192 <- 22016 for down) on layers 0, 40
    and 79 of the 80-layer stack, seeded as the bench's layer-by-layer pass
    seeds them (weights and adapters per layer, tokens and gradients from
    layer 0)."""
    q = Q()
    name, N, K = inputs.LLAMA65B_PROJ[proj]
    T, r, s = 2048, 64, 0.25
    _, X, _, _, dY = inputs.layer_inputs(4, 0, proj, T, N, K, r, device="cuda")
    W = inputs.normal_bf16((N, K), 0.02, inputs.seed_of(4, layer, proj, "W"), "cuda")
    A = inputs.normal_bf16((r, K), (1.0 / K) ** 0.5, inputs.seed_of(4, layer, proj, "A"), "cuda")
    B = inputs.normal_bf16((N, r), 0.01, inputs.seed_of(4, layer, proj, "B"), "cuda")
    qw, wd = quantize_checked(W)
    del W
    y, u = q.linear_fwd_save(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd_saved(dY, X, qw, A, B, s, u)
    q.get_error()
    torch.cuda.synchronize()
    rows = np.array([0, 1, 255, 256, 511, 512, 1023, 1500, 2046, 2047])
    check_fwd_bwd_sampled(X, A, B, dY, wd, s, rows, y, dx, dA, dB)


# --------------------------------------------------------------------------
# decode sweep: the seven 8B shapes at T = 1, 4, 16, rank 64, s = 1
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def decode_set():
    """The decode sweep's seven projections, seeded as the bench seeds them:
    NF4 weights (quantize checked bit for bit), the oracle's W', adapters."""
    r = 64
    out = []
    for proj, (name, N, K) in enumerate(inputs.LLAMA8B_PROJ):
        W = inputs.normal_bf16((N, K), 0.02, inputs.seed_of(2, 0, proj, "W"), "cuda")
        qw, wd = quantize_checked(W)
        del W
        A = inputs.normal_bf16((r, K), (1.0 / K) ** 0.5, inputs.seed_of(2, 0, proj, "A"), "cuda")
        B = inputs.normal_bf16((N, r), 0.01, inputs.seed_of(2, 0, proj, "B"), "cuda")
        out.append((name, N, K, qw, wd, A, B))
    return out


@pytest.mark.parametrize("T", [1, 4, 16])
def test_decode_sweep(decode_set, T):
    """All seven projections of the decode sweep at one token count: every
    output element against the oracle, through the plain forward, the
    allocation-free one and the grouped call of all seven at once."""
    q = Q()
    s = 1.0
    xs, ys, ynas, ybs = [], [], [], []
    for proj, (name, N, K, qw, wd, A, B) in enumerate(decode_set):
        X = inputs.normal_bf16((T, K), 1.0, inputs.seed_of(2, T, proj, "X"), "cuda")
        xs.append(X)
        ys.append(q.linear_fwd(X, qw, A, B, s))
        ynas.append(torch.empty_like(ys[-1]))
        q.linear_fwd_noalloc(X, qw, A, B, s, ynas[-1])
        ybs.append(torch.full_like(ys[-1], float("nan")))
    q.linear_fwd_decode_batch([(xs[i], p[3], p[5], p[6], s, ybs[i]) for i, p in enumerate(decode_set)])
    q.get_error()
    q.noalloc_get_error()
    torch.cuda.synchronize()
    for proj, (name, N, K, qw, wd, A, B) in enumerate(decode_set):
        ref = O.linear_fwd(bits(xs[proj]), wd, bits(A), bits(B), s)
        assert_close(f"{name} Y T={T}", ys[proj], ref)
        assert_close(f"{name} Y noalloc T={T}", ynas[proj], ref)
        assert_close(f"{name} Y grouped T={T}", ybs[proj], ref)


# --------------------------------------------------------------------------
# the code function, exhaustively
# --------------------------------------------------------------------------
def _sweep_blocks(c1_lo, c1_hi):
    """Blocks holding c1 once (so it is the block's absmax) and 63 test weights:
    every BF16 w with |w| <= c1, both signs, for every c1 bit pattern in
    [c1_lo, c1_hi)."""
    all_w = np.arange(0, 0x7F80, dtype=np.uint16)     # non-negative finite BF16 patterns
    blocks = []
    for cb in range(c1_lo, c1_hi):
        mag = all_w[:cb + 1]
        ws = np.concatenate([mag, mag | 0x8000])
        pad = (-ws.size) % 63
        ws = np.concatenate([ws, np.zeros(pad, np.uint16)]).reshape(-1, 63)
        blk = np.empty((ws.shape[0], 64), np.uint16)
        blk[:, 0] = cb
        blk[:, 1:] = ws
        blocks.append(blk)
    allb = np.concatenate(blocks)
    pad = (-allb.shape[0]) % 256                       # whole double-quantization groups
    return np.concatenate([allb, np.zeros((pad, 64), np.uint16)]).reshape(-1, 64 * 256)


@pytest.mark.parametrize("part", range(8))
def test_code_function_every_bf16_pair(part):
    """The GPU quantizer's code against the oracle's for every pair (w, c1) of
    BF16 values with |w| <= c1 and c1 > 0 finite (c1 = 0x0001 .. 0x7F7F: every
    positive finite BF16 value, subnormals included), in eight slices of the c1
    range of about equal weight count (1.07e9 pairs in all)."""
    q = Q()
    # slice boundaries: the weight count of c1 = b grows like b, so cut the
    # bit-pattern range at equal areas (b^2 grows linearly)
    top = 0x7F80
    edges = [max(1, int(round(top * np.sqrt(i / 8)))) for i in range(9)]
    edges[-1] = top
    lo, hi = edges[part], edges[part + 1]
    allb = _sweep_blocks(lo, hi)
    step = 4096                                        # rows of 16384 weights per GPU call
    for a in range(0, allb.shape[0], step):
        chunk = np.ascontiguousarray(allb[a:a + step])
        w = torch.from_numpy(chunk.view(np.int16)).view(torch.bfloat16).cuda()
        qw = q.quantize_nf4(w)
        q.get_error()
        codes, _, _ = O.quantize_nf4(chunk)
        got = qw.codes.cpu().numpy()
        if not np.array_equal(got, codes):
            d = np.flatnonzero(got != codes)
            raise AssertionError(f"c1 in [{lo:#x}, {hi:#x}): {d.size} code bytes differ, first at {d[:4]}")
