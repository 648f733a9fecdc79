"""GPU path vs the CPU oracle, through the C ABI (ctypes binding).

Bit-exact for quantize (codes, FP8 scale bytes, c2) and dequantize; within
|gpu - oracle| <= 5e-3 + 1e-2 |oracle| per element for the forward and
backward (oracle in float64 from the same BF16 inputs and the BF16
dequantized weight).
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


def from_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def assert_close(name, gpu_bf16, ref64):
    g = O.bf16_bits_to_f32(bits(gpu_bf16)).astype(np.float64).reshape(ref64.shape)
    err = np.abs(g - ref64)
    tol = TOL_ABS + TOL_REL * np.abs(ref64)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu={g[i]!r} oracle={ref64[i]!r}")


def quantize_and_check(w_dev):
    q = Q()
    qw = q.quantize_nf4(w_dev)
    torch.cuda.synchronize()
    codes, scales, c2 = O.quantize_nf4(bits(w_dev))
    g_codes = qw.codes.cpu().numpy()
    g_scales = qw.scales.cpu().numpy()
    g_c2 = qw.c2.cpu().numpy()
    assert np.array_equal(g_c2.view(np.uint32), c2.view(np.uint32)), "c2 differs"
    assert np.array_equal(g_scales, scales), f"scale bytes differ at {np.flatnonzero(g_scales != scales)[:8]}"
    if not np.array_equal(g_codes, codes):
        d = np.flatnonzero(g_codes != codes)
        raise AssertionError(f"codes differ at {d.size} bytes, first {d[:8]}")
    return qw, (codes, scales, c2)


# --------------------------------------------------------------------------
# quantize / dequantize
# --------------------------------------------------------------------------

def test_quantize_dequantize_config0_bitexact():
    w = inputs.normal_bf16((512, 512), 0.02, inputs.seed_of(0, 0, 0, "W"), "cuda")
    qw, (codes, scales, c2) = quantize_and_check(w)
    wd = Q().dequantize(qw)
    torch.cuda.synchronize()
    ref = O.dequantize_nf4(codes, scales, c2, 512, 512)
    assert np.array_equal(bits(wd), ref)


def _special_weight(rows, cols, seed):
    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, (rows, cols)).astype(np.float32)
    flat = w.reshape(-1, 64)
    nb = flat.shape[0]
    flat[0] = 0.0                                       # all +0
    if nb > 1: flat[1] = -0.0                           # all -0
    if nb > 2: flat[2] = 0.0; flat[2, 17] = 3.0          # one-hot
    if nb > 3: flat[3] = rng.normal(0, 1e-38, 64)        # subnormal BF16 values
    if nb > 4: flat[4] = rng.normal(0, 1e37, 64)         # huge values
    if nb > 5: flat[5] = rng.normal(0, 1e-6, 64)         # scale in E4M3's subnormal range vs group max
    if nb > 6: flat[6] = np.linspace(-1, 1, 64)          # exact ties and levels
    if nb > 7: flat[7, :] = 1.0; flat[7, 5] = -1.0       # ties between +-c1
    return torch.from_numpy(w).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("rows,cols", [(3, 320), (5, 448), (64, 64 * 257), (1, 64), (17, 1024)])
def test_quantize_dequantize_ragged_and_special_bitexact(rows, cols):
    w = _special_weight(rows, cols, rows * 1000 + cols)
    qw, (codes, scales, c2) = quantize_and_check(w)
    wd = Q().dequantize(qw)
    torch.cuda.synchronize()
    assert np.array_equal(bits(wd), O.dequantize_nf4(codes, scales, c2, rows, cols))


def test_code_function_sweep_over_bf16_pairs():
    """Every BF16 weight w with |w| <= c1 against c1 = every BF16 mantissa at a
    spread of exponents (subnormal through near-max): the block holds c1 once
    (so it is the absmax) and 63 test weights."""
    c1_bits = []
    for e in [0, 1, 2, 7, 30, 100, 126, 127, 128, 129, 160, 200, 250, 253, 254]:   # biased exponents
        for m in range(128):
            b = (e << 7) | m
            if b != 0:
                c1_bits.append(b)
    blocks = []
    all_w = np.arange(0, 0x7F80, dtype=np.uint16)                  # non-negative finite BF16 patterns
    for cb in c1_bits:
        mag = all_w[all_w <= cb]
        ws = np.concatenate([mag, mag | 0x8000])
        pad = (-ws.size) % 63
        ws = np.concatenate([ws, np.zeros(pad, np.uint16)]).reshape(-1, 63)
        blk = np.empty((ws.shape[0], 64), np.uint16)
        blk[:, 0] = cb
        blk[:, 1:] = ws
        blocks.append(blk)
    allb = np.concatenate(blocks)
    pad = (-allb.shape[0]) % 256
    allb = np.concatenate([allb, np.zeros((pad, 64), np.uint16)])
    w = from_bits(allb.reshape(-1, 64 * 256)).cuda()
    qw = Q().quantize_nf4(w)
    torch.cuda.synchronize()
    codes, _, _ = O.quantize_nf4(allb.reshape(-1, 64 * 256))
    assert np.array_equal(qw.codes.cpu().numpy(), codes)


@pytest.mark.parametrize("N,K,r,s,a_std,b_std", [
    (512, 512, 8, 2.0, 0.1, 0.05),          # adapter term comparable to W'
    (1032, 768, 64, 0.25, 0.1, 0.05),       # ragged rows, large rank
    (4096, 4096, 16, 2.0, None, 0.01),      # 8B q shape, trained-adapter scale
])
def test_merge_adapter(N, K, r, s, a_std, b_std):
    """BF16(W' + s B A) on the GPU against the oracle's float64 merge.  The GPU
    forms d = sum_j B A in FP32 and fma(s, d, W') before rounding to BF16, so
    an element may differ from the oracle's value by one BF16 step (2^-7 |o|)
    plus the FP32 error of that arithmetic, 2^-24 (r + 2) (|W'| + s sum_j |B||A|)
    (which only matters where W' and s B A cancel)."""
    q = Q()
    W, _, A, B, _ = inputs.layer_inputs(95, 0, 0, 1, N, K, r, device="cuda", a_std=a_std, b_std=b_std)
    qw, (codes, scales, c2) = quantize_and_check(W)
    m = q.merge_adapter(qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    o = O.merge_adapter(wd, bits(A), bits(B), s)
    af, bf, wf = (O.bf16_bits_to_f32(v).astype(np.float64) for v in (bits(A), bits(B), wd))
    bound = 2.0 ** -7 * np.abs(o) + 2.0 ** -24 * (r + 2) * (np.abs(wf) + abs(s) * (np.abs(bf) @ np.abs(af)))
    g = bits(m).astype(np.uint32) << np.uint32(16)
    err = np.abs(g.view(np.float32).astype(np.float64) - o)
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} elements outside the bound; worst {np.max(err - bound)!r}"
    # the adapter really moved the weight (the term is not lost in rounding)
    assert (g != (wd.astype(np.uint32) << np.uint32(16))).mean() > 0.01


def test_nonfinite_weight_is_reported():
    q = Q()
    w = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    w[2, 7] = float("inf")
    q.quantize_nf4(w)
    with pytest.raises(q.QLoraError) as e:
        q.get_error()
    assert e.value.status == 6
    q.get_error()   # cleared


def test_stack_8b_32_layers_quantize_storage_roundtrip():
    """Every linear weight of a 32-layer Llama-3.1-8B-shaped stack (hidden 4096,
    ffn 14336, 8 KV heads of dim 128: 6.98e9 parameters), BF16 N(0, 0.02^2),
    quantized on the GPU.  Storage is exactly 4 + 0.127 bits per parameter
    ("What is QLoRA?"); dequantize then quantize gives back the same codes,
    scale bytes and c2 on every matrix; layer 0's seven matrices match the
    oracle bit for bit on their first, a middle and their last two 256-block
    groups (group-aligned, so each range quantizes on its own)."""
    q = Q()
    G = 64 * 256                     # weights per second-level group
    total_w = total_b = 0
    for layer in range(32):
        for i, (name, N, K) in enumerate(inputs.LLAMA8B_PROJ):
            W = inputs.normal_bf16((N, K), 0.02, inputs.seed_of(3, layer, i, "W"), "cuda")
            qw = q.quantize_nf4(W)
            qw2 = q.quantize_nf4(q.dequantize(qw))
            q.get_error()
            assert torch.equal(qw2.codes, qw.codes), f"layer {layer} {name}: codes"
            assert torch.equal(qw2.scales, qw.scales), f"layer {layer} {name}: scales"
            assert torch.equal(qw2.c2.view(torch.int32), qw.c2.view(torch.int32)), f"layer {layer} {name}: c2"
            n = N * K
            total_w += n
            total_b += qw.codes.numel() + qw.scales.numel() + 4 * qw.c2.numel()
            if layer == 0:
                w = bits(W).reshape(-1)
                g_codes, g_scales = qw.codes.cpu().numpy(), qw.scales.cpu().numpy()
                g_c2 = qw.c2.cpu().numpy().view(np.uint32)
                for a in (0, (n // 2) // G * G, n - 2 * G):
                    b = a + 2 * G
                    codes, scales, c2 = O.quantize_nf4(w[a:b].reshape(-1, 64))
                    assert np.array_equal(g_codes[a // 2:b // 2], codes), f"{name}: codes at {a}"
                    assert np.array_equal(g_scales[a // 64:b // 64], scales), f"{name}: scales at {a}"
                    assert np.array_equal(g_c2[a // G:b // G], c2.view(np.uint32)), f"{name}: c2 at {a}"
            del W, qw, qw2
    assert total_w == 32 * sum(N * K for (_, N, K) in inputs.LLAMA8B_PROJ)
    assert round(total_w / 1e9, 2) == 6.98
    assert total_b * 8 / total_w == O.bits_per_param()


# --------------------------------------------------------------------------
# forward / backward
# --------------------------------------------------------------------------

def run_layer(T, N, K, r, s, config=90, a_std=None, b_std=0.01, check_quant=True):
    W, X, A, B, dY = inputs.layer_inputs(config, 0, 0, T, N, K, r, device="cuda", a_std=a_std, b_std=b_std)
    q = Q()
    if check_quant:
        qw, (codes, scales, c2) = quantize_and_check(W)
    else:
        qw = q.quantize_nf4(W)
        codes, scales, c2 = O.quantize_nf4(bits(W))
    y = q.linear_fwd(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd(dY, X, qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    return (X, A, B, dY), wd, (y, dx, dA, dB)


def check_layer(T, N, K, r, s, **kw):
    (X, A, B, dY), wd, (y, dx, dA, dB) = run_layer(T, N, K, r, s, **kw)
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    assert_close("Y", y, O.linear_fwd(xb, wd, ab, bb, s))
    rdx, rdA, rdB = O.linear_bwd(dyb, xb, wd, ab, bb, s)
    assert_close("dX", dx, rdx)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)


def test_layer_config0():
    """512x512, 16 tokens, rank 8, s = 2; A ~ N(0, 1/512), B ~ N(0, 0.01^2)."""
    check_layer(16, 512, 512, 8, 2.0, config=0)


def test_layer_multi_tile_ragged():
    """Several weight tiles, two token tiles (one ragged), ragged rank."""
    check_layer(300, 384, 320, 24, 0.5)


@pytest.mark.parametrize("T,N,K,r,s", [
    (1, 64, 64, 1, 1.0),          # single token, rank 1
    (7, 136, 192, 16, 2.0),       # N not a multiple of the 128-row tile
    (33, 256, 128, 128, 0.25),    # maximum rank: two rank stages
    (257, 128, 256, 65, 1.0),     # ragged rank just over one stage, 2 token tiles
    (64, 1024, 4096, 64, 1.0),    # decode-like token count on an 8B k/v shape
])
def test_layer_edge_shapes(T, N, K, r, s):
    check_layer(T, N, K, r, s)


def test_layer_zero_tokens():
    q = Q()
    W = inputs.normal_bf16((128, 128), 0.02, 1, "cuda")
    qw = q.quantize_nf4(W)
    X = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    A = inputs.normal_bf16((8, 128), 0.1, 2, "cuda")
    B = inputs.normal_bf16((128, 8), 0.1, 3, "cuda")
    y = q.linear_fwd(X, qw, A, B, 2.0)
    dx, dA, dB = q.linear_bwd(torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"), X, qw, A, B, 2.0)
    torch.cuda.synchronize()
    assert y.shape == (0, 128) and dx.shape == (0, 128)
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


def test_layer_8b_q_projection_full_size_sampled():
    """T = 4096 tokens on the 4096 x 4096 q projection, rank 16, s = 2: the
    launch configuration of the bench.  Quantize is checked in full; Y and dX on
    sampled tokens (every output feature); dA and dB in full."""
    T, N, K, r, s = 4096, 4096, 4096, 16, 2.0
    (X, A, B, dY), wd, (y, dx, dA, dB) = run_layer(T, N, K, r, s, config=1)
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    rows = np.array([0, 1, 255, 256, 1000, 2047, 2048, 3333, 4094, 4095])
    assert_close("Y[rows]", y[torch.from_numpy(rows).cuda()], O.linear_fwd(xb[rows], wd, ab, bb, s))
    Xf, Wf, Af, Bf, G = (O.bf16_bits_to_f32(v).astype(np.float64) for v in (xb, wd, ab, bb, dyb))
    dU = s * (G @ Bf)
    assert_close("dX[rows]", dx[torch.from_numpy(rows).cuda()], G[rows] @ Wf + dU[rows] @ Af)
    assert_close("dA", dA, dU.T @ Xf)
    assert_close("dB", dB, s * (G.T @ (Xf @ Af.T)))


def test_backward_graph_capture_matches_eager():
    """The backward forks dB/dA onto a second stream and joins it back; captured
    in a CUDA graph and replayed it gives the eager results bit for bit, and a
    forward queued right after it on the same stream sees the finished dA/dB."""
    q = Q()
    T, N, K, r, s = 512, 1024, 768, 16, 2.0
    W, X, A, B, dY = inputs.layer_inputs(91, 0, 0, T, N, K, r, device="cuda")
    qw = q.quantize_nf4(W)
    ref = q.linear_bwd(dY, X, qw, A, B, s)
    torch.cuda.synchronize()
    outs = tuple(torch.empty_like(t) for t in ref)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        q.linear_bwd(dY, X, qw, A, B, s, outs=outs)   # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for t in outs:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        q.linear_bwd(dY, X, qw, A, B, s, outs=outs)
    g.replay()
    # the adapter gradients are complete once the stream reaches the next call
    y_dA = q.linear_fwd(X, qw, outs[1], B, s)
    q.get_error()
    torch.cuda.synchronize()
    for name, a, b in zip(("dX", "dA", "dB"), outs, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), name
    y_ref = q.linear_fwd(X, qw, ref[1], B, s)
    torch.cuda.synchronize()
    assert torch.equal(y_dA.view(torch.int16), y_ref.view(torch.int16))
    del g


@pytest.mark.parametrize("name,N,K", [("q", 8192, 8192), ("down", 8192, 22016)])
def test_layer_65b_shapes_full_size_sampled(name, N, K):
    """A 65B-shaped projection (hidden 8192, ffn 22016; the q/k/v/o and down
    shapes), fwd + bwd on 4 x 512 = 2048 tokens, rank 64, s = 0.25, as in the
    layer-by-layer run.  Quantize in full; Y and dX on sampled tokens (every
    output feature); dA and dB in full."""
    T, r, s = 2048, 64, 0.25
    i = {"q": 0, "down": 6}[name]
    W, X, A, B, dY = inputs.layer_inputs(4, 0, i, T, N, K, r, device="cuda")
    q = Q()
    qw, (codes, scales, c2) = quantize_and_check(W)
    del W
    y = q.linear_fwd(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd(dY, X, qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    rows = np.array([0, 1, 511, 512, 1023, 1500, 2046, 2047])
    assert_close("Y[rows]", y[torch.from_numpy(rows).cuda()], O.linear_fwd(xb[rows], wd, ab, bb, s))
    Xf, Wf, Af, Bf, G = (O.bf16_bits_to_f32(v).astype(np.float64) for v in (xb, wd, ab, bb, dyb))
    dU = s * (G @ Bf)
    assert_close("dX[rows]", dx[torch.from_numpy(rows).cuda()], G[rows] @ Wf + dU[rows] @ Af)
    assert_close("dA", dA, dU.T @ Xf)
    assert_close("dB", dB, s * (G.T @ (Xf @ Af.T)))


@pytest.mark.parametrize("T,N,K", [
    (1, 1024, 4096),      # 8B k/v projection, single token
    (4, 4096, 4096),      # 8B q/o projection
    (9, 4096, 14336),     # 8B down projection: 56 k-units, 7-CTA cluster, 9..16-token variant
    (16, 14336, 4096),    # 8B gate/up projection
    (3, 40, 320),         # ragged rows and a k-unit with a missing block
    (5, 1032, 768),       # last 16-row tile half empty (table-lookup kernel)
    (13, 2048, 2560),     # 9..16 tokens, one k-unit per split, ten splits
    (2, 40000, 1792),     # seven k-units in three splits of 2, 2 and 3 units
    (2, 113664, 512),     # enough rows that each tile is one item (no split partials)
])
def test_decode_forward(T, N, K):
    """Decode-sized forward (T <= 16): rank 64, s = 1, as in the decode sweep."""
    r, s = 64, 1.0
    W, X, A, B, _ = inputs.layer_inputs(2, 0, 0, T, N, K, r, device="cuda")
    q = Q()
    qw, (codes, scales, c2) = quantize_and_check(W)
    y = q.linear_fwd(X, qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    assert_close("Y", y, O.linear_fwd(bits(X), wd, bits(A), bits(B), s))


# equally spaced 4-bit levels ("QLoRA & 4-bit Fine-Tuning", Innovation 1: the
# INT4 contrast to NF4); not symmetric (-1 .. 7/8), so the kernels take their
# general 16-entry lookup instead of the sign-symmetric one
INT4_LEVELS = [(i - 8) / 8.0 for i in range(16)]


@pytest.mark.parametrize("T,N,K,r,s", [(300, 384, 320, 24, 0.5), (4, 1024, 4096, 64, 1.0), (16, 512, 512, 8, 2.0)])
def test_layer_asymmetric_codebook(T, N, K, r, s):
    q = Q()
    W, X, A, B, dY = inputs.layer_inputs(93, 0, 0, T, N, K, r, device="cuda")
    cb = np.array(INT4_LEVELS, dtype=np.float32)
    qw = q.quantize_nf4(W, codebook=[float(v) for v in cb])
    torch.cuda.synchronize()
    codes, scales, c2 = O.quantize_nf4(bits(W), cb)
    assert np.array_equal(qw.codes.cpu().numpy(), codes)
    assert np.array_equal(qw.scales.cpu().numpy(), scales)
    wd = O.dequantize_nf4(codes, scales, c2, N, K, cb)
    assert np.array_equal(bits(q.dequantize(qw)), wd)
    y = q.linear_fwd(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd(dY, X, qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    assert_close("Y", y, O.linear_fwd(xb, wd, ab, bb, s))
    rdx, rdA, rdB = O.linear_bwd(dyb, xb, wd, ab, bb, s)
    assert_close("dX", dx, rdx)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)
