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


@pytest.mark.parametrize("T", [4046, 3900])
def test_layer_half_tiles_in_last_round(T):
    """1280 x 1280 at about 4000 tokens: 80 tiles of 256 x 256 on both GEMMs,
    so on 74 CTA pairs the last round's six tiles run as 128-token halves; at
    T = 3900 the second half of the last token tile lies wholly past T."""
    check_layer(T, 1280, 1280, 16, 2.0)


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
    # each token's gradient row is the oracle's backward of that token alone;
    # the adapter gradients sum over every token
    rdx, _, _ = O.linear_bwd(dyb[rows], xb[rows], wd, ab, bb, s)
    assert_close("dX[rows]", dx[torch.from_numpy(rows).cuda()], rdx)
    rdA, rdB = O.lora_adapter_grads(dyb, xb, ab, bb, s)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)


def test_backward_graph_capture_matches_eager():
    """The backward (its dB/dA grid a programmatic dependent of the dX GEMM),
    captured in a CUDA graph and replayed, gives the eager results bit for bit,
    and a forward queued right after it on the same stream sees the finished
    dA/dB."""
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
    # each token's gradient row is the oracle's backward of that token alone;
    # the adapter gradients sum over every token
    rdx, _, _ = O.linear_bwd(dyb[rows], xb[rows], wd, ab, bb, s)
    assert_close("dX[rows]", dx[torch.from_numpy(rows).cuda()], rdx)
    rdA, rdB = O.lora_adapter_grads(dyb, xb, ab, bb, s)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)


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


# --------------------------------------------------------------------------
# the forward that saves U and the backward that reuses it
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T,N,K,r,s", [
    (16, 512, 512, 8, 2.0),       # the tiny layer; decode-sized forward with U saved
    (1, 64, 64, 1, 1.0),          # one token, rank 1
    (5, 1032, 768, 64, 1.0),      # decode-sized, ragged last row tile
    (300, 384, 320, 24, 0.5),     # two token tiles (one ragged), ragged rank
    (33, 256, 128, 128, 0.25),    # maximum rank
    (257, 128, 256, 65, 1.0),     # rank just over one 64-wide stage
    (7, 136, 192, 16, 2.0),       # N not a multiple of the weight tile
])
def test_layer_saved_u(T, N, K, r, s):
    q = Q()
    W, X, A, B, dY = inputs.layer_inputs(92, 0, 0, T, N, K, r, device="cuda")
    qw, (codes, scales, c2) = quantize_and_check(W)
    y, u = q.linear_fwd_save(X, qw, A, B, s)
    assert u.numel() == q.saved_u_bytes(T, r)
    dx, dA, dB = q.linear_bwd_saved(dY, X, qw, A, B, s, u)
    q.get_error()
    torch.cuda.synchronize()
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    assert_close("Y", y, O.linear_fwd(xb, wd, ab, bb, s))
    rdx, rdA, rdB = O.linear_bwd(dyb, xb, wd, ab, bb, s)
    assert_close("dX", dx, rdx)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)
    # the saved planes hold sU = s X A^T as hi + lo: about 16 significant bits
    Tp = (T + 7) // 8 * 8
    plane = u.numel() // 2
    hi = u[:r * Tp * 2].view(torch.bfloat16).float().reshape(r, Tp)
    lo = u[plane:plane + r * Tp * 2].view(torch.bfloat16).float().reshape(r, Tp)
    got = (hi + lo).double().cpu().numpy()[:, :T]
    ref = float(s) * (O.bf16_bits_to_f32(xb).astype(np.float64) @ O.bf16_bits_to_f32(ab).astype(np.float64).T).T
    assert np.all(np.abs(got - ref) <= 1e-3 + 2.0 ** -14 * np.abs(ref))


def _launched_kernels(fn):
    """Names of the library kernels that fn() launches (the trace hook, without events)."""
    import ctypes as C
    from bit_nf4_quantized_20_b200 import _lib
    recs = (_lib.TraceRec * 64)()
    count = C.c_int32(0)
    lib = _lib.lib()
    _lib.check("qlora_trace_attach", lib.qlora_trace_attach(recs, 64, C.byref(count)))
    try:
        fn()
    finally:
        lib.qlora_trace_attach(None, 0, None)
    return [lib.qlora_kernel_name(recs[i].kernel).decode() for i in range(min(count.value, 64))]


@pytest.mark.parametrize("T,N,K,r,s,one_read", [
    (2500, 3080, 256, 24, 0.5, True),   # blocks of 2 token tiles x 2 feature chunks; ragged T and N
    (3000, 4104, 128, 13, 2.0, True),   # 2 x 3 blocks, rank 13
    (2500, 4104, 64, 36, 1.0, True),    # hi and lo planes of 64 rows each (N = 128), three stages
    (513, 4104, 192, 1, 1.0, True),     # rank 1; one token in the last tile
    (1300, 4104, 64, 8, 1.0, True),     # three token tiles a block
    (300, 384, 320, 24, 0.5, False),    # partial sums would outweigh the second read of dY
    (257, 1024, 128, 65, 1.0, False),   # rank above 64
])
def test_layer_saved_u_one_read_of_dy(T, N, K, r, s, one_read):
    """Both backwards with dU and dB from one read of dY (block partial sums,
    then a launch that sums them), against the oracle: the saved-U one, and
    the plain one, which first computes sU.  Shapes where the partial sums do
    not pay off, or the rank is above 64, run dU and dB as two launches (saved)
    or in the two paired grids (plain) instead."""
    q = Q()
    W, X, A, B, dY = inputs.layer_inputs(93, 0, 0, T, N, K, r, device="cuda")
    qw, (codes, scales, c2) = quantize_and_check(W)
    y, u = q.linear_fwd_save(X, qw, A, B, s)
    names = _launched_kernels(lambda: q.linear_bwd_saved(dY, X, qw, A, B, s, u))
    plain = _launched_kernels(lambda: q.linear_bwd(dY, X, qw, A, B, s))
    torch.cuda.synchronize()
    if one_read:
        assert "lora_du+dB" in names and "lora_du+dB_sum" in names and "lora_dB" not in names, names
        assert plain[:3] == ["lora_u", "lora_du+dB", "lora_du+dB_sum"] and "lora_u+du" not in plain, plain
    else:
        assert "lora_du+dB" not in names and "lora_dB" in names and "lora_du" in names, names
        assert "lora_u+du" in plain and "lora_du+dB" not in plain, plain
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    rdx, rdA, rdB = O.linear_bwd(dyb, xb, wd, ab, bb, s)
    for bwd in (lambda: q.linear_bwd_saved(dY, X, qw, A, B, s, u), lambda: q.linear_bwd(dY, X, qw, A, B, s)):
        dx, dA, dB = bwd()
        q.get_error()
        torch.cuda.synchronize()
        assert_close("dX", dx, rdx)
        assert_close("dA", dA, rdA)
        assert_close("dB", dB, rdB)


def test_backward_saved_graph_capture_matches_eager():
    """The saved-U backward (its adapter-gradient grid a programmatic
    dependent of the dX GEMM), captured in a CUDA graph on a non-default
    stream, gives the eager results bit for bit."""
    q = Q()
    T, N, K, r, s = 512, 1024, 768, 16, 2.0
    W, X, A, B, dY = inputs.layer_inputs(94, 0, 0, T, N, K, r, device="cuda")
    qw = q.quantize_nf4(W)
    _, u = q.linear_fwd_save(X, qw, A, B, s)
    ref = q.linear_bwd_saved(dY, X, qw, A, B, s, u)
    torch.cuda.synchronize()
    outs = tuple(torch.empty_like(t) for t in ref)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        q.linear_bwd_saved(dY, X, qw, A, B, s, u, outs=outs)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for t in outs:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        q.linear_bwd_saved(dY, X, qw, A, B, s, u, outs=outs)
    g.replay()
    q.get_error()
    torch.cuda.synchronize()
    for name, a, b in zip(("dX", "dA", "dB"), outs, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), name
    del g


# --------------------------------------------------------------------------
# failure detection and argument checks on a GPU
# --------------------------------------------------------------------------
def test_bounded_wait_runs_out_and_is_reported():
    """A wait on a barrier that nothing arrives on gives up after its limit
    (here 2 ms), the status word reports QLORA_ERR_TIMEOUT once, and the
    context stays usable: a forward right after it is correct."""
    import time
    q = Q()
    q.get_error()                              # start clean
    t0 = time.perf_counter()
    q.wait_selftest(2000)
    with pytest.raises(q.QLoraError) as e:
        q.get_error()
    assert e.value.status == 7                 # QLORA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    q.get_error()                              # the word was cleared
    check_layer(16, 512, 512, 8, 2.0, config=0)


def test_wrong_output_buffers_are_refused_before_launch():
    q = Q()
    T, N, K, r = 32, 256, 128, 8
    W, X, A, B, dY = inputs.layer_inputs(96, 0, 0, T, N, K, r, device="cuda")
    qw = q.quantize_nf4(W)
    bad = [torch.empty(T, N + 8, dtype=torch.bfloat16, device="cuda"),   # too wide
           torch.empty(T - 1, N, dtype=torch.bfloat16, device="cuda"),   # too short
           torch.empty(T, N, dtype=torch.float32, device="cuda")]        # wrong dtype
    for out in bad:
        with pytest.raises(ValueError):
            q.linear_fwd(X, qw, A, B, 1.0, out=out)
        with pytest.raises(ValueError):
            q.linear_fwd_noalloc(X, qw, A, B, 1.0, out)
    with pytest.raises(ValueError):
        q.linear_bwd(dY, X, qw, A, B, 1.0, outs=(torch.empty(T, K + 8, dtype=torch.bfloat16, device="cuda"),
                                                torch.empty(r, K, dtype=torch.bfloat16, device="cuda"),
                                                torch.empty(N, r, dtype=torch.bfloat16, device="cuda")))


# --------------------------------------------------------------------------
# codebook variants ("QLoRA & 4-bit Fine-Tuning", Innovations 1 and 2)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("table", ["eq2", "eq2_zero", "int4"])
@pytest.mark.parametrize("rows,cols", [(512, 512), (17, 1024), (64, 64 * 257)])
def test_quantize_snapped_to_dq_scale_bitexact(table, rows, cols):
    """Codes snapped against the double-quantized block scale: codes, scale
    bytes and c2 bit for bit against the oracle, special blocks included, and
    the dequantization of those codes too."""
    q = Q()
    cb = {"eq2": O.nf4_codebook(), "eq2_zero": O.nf4_codebook_with_zero(),
          "int4": np.array(INT4_LEVELS, np.float32)}[table]
    w = _special_weight(rows, cols, 7 * rows + cols)
    qw = q.quantize_nf4(w, codebook=[float(v) for v in cb], snap_to_dq_scale=True)
    torch.cuda.synchronize()
    codes, scales, c2 = O.quantize_nf4(bits(w), cb, snap_to_dq_scale=True)
    assert np.array_equal(qw.c2.cpu().numpy().view(np.uint32), c2.view(np.uint32))
    assert np.array_equal(qw.scales.cpu().numpy(), scales)
    got = qw.codes.cpu().numpy()
    assert np.array_equal(got, codes), f"{np.count_nonzero(got != codes)} code bytes differ"
    wd = q.dequantize(qw)
    torch.cuda.synchronize()
    assert np.array_equal(bits(wd), O.dequantize_nf4(codes, scales, c2, rows, cols, cb))


@pytest.mark.parametrize("T,N,K,r,s", [(300, 384, 320, 24, 0.5), (4, 1024, 4096, 64, 1.0), (16, 512, 512, 8, 2.0),
                                       (2, 1032, 768, 16, 1.0)])
def test_layer_codebook_with_zero_level(T, N, K, r, s):
    """eq. 2 with an exact zero level through every kernel: quantize and
    dequantize bit for bit, the tensor-core forward/backward (T > 16) or the
    decode forward (T <= 16), the saved-U pair, and the adapter merge."""
    q = Q()
    cb = O.nf4_codebook_with_zero()
    W, X, A, B, dY = inputs.layer_inputs(97, 0, 0, T, N, K, r, device="cuda")
    qw = q.quantize_nf4(W, codebook=[float(v) for v in cb])
    torch.cuda.synchronize()
    codes, scales, c2 = O.quantize_nf4(bits(W), cb)
    assert np.array_equal(qw.codes.cpu().numpy(), codes)
    assert np.array_equal(qw.scales.cpu().numpy(), scales)
    wd = O.dequantize_nf4(codes, scales, c2, N, K, cb)
    assert np.array_equal(bits(q.dequantize(qw)), wd)
    y = q.linear_fwd(X, qw, A, B, s)
    y2, u = q.linear_fwd_save(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd_saved(dY, X, qw, A, B, s, u)
    m = q.merge_adapter(qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    ref = O.linear_fwd(xb, wd, ab, bb, s)
    assert_close("Y", y, ref)
    assert_close("Y saved", y2, ref)
    rdx, rdA, rdB = O.linear_bwd(dyb, xb, wd, ab, bb, s)
    assert_close("dX", dx, rdx)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)
    o = O.merge_adapter(wd, ab, bb, s)
    af, bf, wf = (O.bf16_bits_to_f32(v).astype(np.float64) for v in (ab, bb, wd))
    bound = 2.0 ** -7 * np.abs(o) + 2.0 ** -24 * (r + 2) * (np.abs(wf) + abs(s) * (np.abs(bf) @ np.abs(af)))
    got = O.bf16_bits_to_f32(bits(m)).astype(np.float64)
    assert np.all(np.abs(got - o) <= bound)


@pytest.mark.parametrize("T,N,K", [(1, 4096, 4096), (4, 1024, 4096), (16, 4096, 14336), (300, 384, 320),
                                   (4096, 1024, 4096)])
def test_large_adapter_activation(T, N, K):
    """Token rows aligned with rows of A (x = 64 A_j K^{1/2} in distribution),
    so that U = s x A^T reaches ~64 in a few columns while B ~ N(0, 0.01^2):
    the rank-r term is then as large as the base term and partly cancels it,
    and rounding U to one BF16 value would put outputs near zero outside the
    tolerance.  Upstream gradients aligned with columns of B likewise make dU
    large for the backward."""
    q = Q()
    r, s = 64, 1.0
    W, X, A, B, dY = inputs.layer_inputs(98, 0, 0, T, N, K, r, device="cuda")
    Xf, dYf = X.float(), dY.float()
    for t in range(min(T, 8)):
        Xf[t] = A[t % r].float() * (K ** 0.5) * 1.5
        dYf[t] = B[:, t % r].float() * 300.0
    X, dY = Xf.to(torch.bfloat16), dYf.to(torch.bfloat16)
    qw, (codes, scales, c2) = quantize_and_check(W)
    y = q.linear_fwd(X, qw, A, B, s)
    y2, u = q.linear_fwd_save(X, qw, A, B, s)
    dx, dA, dB = q.linear_bwd_saved(dY, X, qw, A, B, s, u)
    dx2, _, _ = q.linear_bwd(dY, X, qw, A, B, s)
    q.get_error()
    torch.cuda.synchronize()
    wd = O.dequantize_nf4(codes, scales, c2, N, K)
    xb, ab, bb, dyb = bits(X), bits(A), bits(B), bits(dY)
    rows = np.unique(np.concatenate([np.arange(min(T, 8)), [T - 1, T // 2]]))
    idx = torch.from_numpy(rows).cuda()
    ref = O.linear_fwd(xb[rows], wd, ab, bb, s)
    U = O.bf16_bits_to_f32(xb[rows]).astype(np.float64) @ O.bf16_bits_to_f32(ab).astype(np.float64).T
    assert np.abs(U).max() > 1.4 * K ** 0.5        # the stress really is there (U ~ N(0, 1) otherwise)
    assert_close("Y", y[idx], ref)
    assert_close("Y saved", y2[idx], ref)
    rdx, _, _ = O.linear_bwd(dyb[rows], xb[rows], wd, ab, bb, s)
    assert_close("dX", dx[idx], rdx)
    assert_close("dX plain", dx2[idx], rdx)
    rdA, rdB = O.lora_adapter_grads(dyb, xb, ab, bb, s)
    assert_close("dA", dA, rdA)
    assert_close("dB", dB, rdB)


# --------------------------------------------------------------------------
# the adapters' optimizer step, with device and unified ("paged") state
# --------------------------------------------------------------------------
def _adam_inputs(n, seed):
    g = torch.Generator().manual_seed(seed)
    p0 = (torch.randn(n, generator=g) * 0.05).float()
    grads = [inputs.normal_bf16((n,), 0.02, seed + 1 + t) for t in range(4)]
    return p0, grads


def _adam_oracle(p0, grads, hp):
    p, m, v = p0.double().numpy(), np.zeros(p0.numel()), np.zeros(p0.numel())
    for t, g in enumerate(grads, start=1):
        p, m, v = O.adam_step(p, m, v, bits(g), t, **hp)
    return p, m, v


HP = dict(lr=2e-3, beta1=0.9, beta2=0.99, eps=1e-8, weight_decay=0.01)


def _check_adam(p, m, v, ref, grads):
    """FP32 arithmetic against the float64 oracle: each step rounds a few
    times, so m and v may differ by a few FP32 ulps of the magnitudes summed
    into them (|m| itself may cancel to near zero), and p by a few ulps of
    itself and of the updates applied."""
    rp, rm, rv = ref
    p, m, v = (np.asarray(a, np.float64) for a in (p, m, v))
    ulp = 2.0 ** -23
    mag_m = np.zeros_like(rm)
    for g in grads:                     # the same recursion on |g|: what m's terms add up to
        mag_m = HP["beta1"] * mag_m + (1 - HP["beta1"]) * np.abs(O.bf16_bits_to_f32(bits(g)).astype(np.float64))
    steps = len(grads)
    assert np.all(np.abs(m - rm) <= 4 * steps * ulp * mag_m + 1e-30)
    assert np.all(np.abs(v - rv) <= 4 * steps * ulp * rv + 1e-30)
    assert np.all(np.abs(p - rp) <= 6 * steps * ulp * (np.abs(rp) + HP["lr"]))


@pytest.mark.parametrize("n", [1_310_720 + 5, 7, 64 * 4096])
def test_adam_step_matches_oracle(n):
    """Four steps on FP32 state in device memory against the float64 oracle;
    the BF16 parameter copy is the round-to-nearest-even of the FP32 result."""
    q = Q()
    p0, grads = _adam_inputs(n, 11 + n % 97)
    p, m, v = p0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    for t, g in enumerate(grads, start=1):
        q.adam_step(p, m, v, g.cuda(), pb, step=t, **HP)
    torch.cuda.synchronize()
    _check_adam(p.cpu().numpy(), m.cpu().numpy(), v.cpu().numpy(), _adam_oracle(p0, grads, HP), grads)
    assert torch.equal(pb.view(torch.int16), p.to(torch.bfloat16).view(torch.int16))


def test_adam_step_on_paged_state():
    """The same steps with parameters and moments in unified memory, paged out
    to the host before every step (the kernel's first touch brings them back):
    bit-identical to the device-memory run, and readable from the host."""
    q = Q()
    n = 1_310_720
    p0, grads = _adam_inputs(n, 5)
    pd, md, vd = p0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    pp, mp, vp = (q.PagedBuffer(n) for _ in range(3))
    torch.cuda.synchronize()
    pp.numpy()[:] = p0.numpy()
    mp.numpy()[:] = 0.0
    vp.numpy()[:] = 0.0
    for t, g in enumerate(grads, start=1):
        gd = g.cuda()
        q.adam_step(pd, md, vd, gd, step=t, **HP)
        for b in (pp, mp, vp):
            b.prefetch(to_host=True)
        q.adam_step(pp, mp, vp, gd, step=t, **HP)
    torch.cuda.synchronize()
    for dev_t, paged in ((pd, pp), (md, mp), (vd, vp)):
        assert np.array_equal(dev_t.cpu().numpy().view(np.uint32), paged.numpy().view(np.uint32))
    _check_adam(pp.numpy(), mp.numpy(), vp.numpy(), _adam_oracle(p0, grads, HP), grads)


@pytest.mark.parametrize("T", [1, 7, 16])
def test_decode_grouped_mixed_shapes_and_codebooks(T):
    """The grouped decode forward over problems of different shapes (ragged
    rows and k-units), ranks, scales and codebooks (sign-symmetric eq. 2 and the
    asymmetric INT4 table in one call), each against the oracle."""
    q = Q()
    specs = [(40, 320, 8, 0.5, None), (1032, 768, 64, 1.0, INT4_LEVELS), (4096, 4096, 16, 2.0, None),
             (136, 192, 100, 0.25, None), (2048, 14336, 128, 1.0, INT4_LEVELS)]
    probs, refs = [], []
    for i, (N, K, r, s, cb) in enumerate(specs):
        W, X, A, B, _ = inputs.layer_inputs(99, i, 0, T, N, K, r, device="cuda")
        table = np.array(cb if cb is not None else O.nf4_codebook(), np.float32)
        qw = q.quantize_nf4(W, codebook=[float(v) for v in table])
        codes, scales, c2 = O.quantize_nf4(bits(W), table)
        assert np.array_equal(qw.codes.cpu().numpy(), codes)
        wd = O.dequantize_nf4(codes, scales, c2, N, K, table)
        y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        probs.append((X, qw, A, B, s, y))
        refs.append(O.linear_fwd(bits(X), wd, bits(A), bits(B), s))
    q.linear_fwd_decode_batch(probs)
    q.get_error()
    torch.cuda.synchronize()
    for i, (p, ref) in enumerate(zip(probs, refs)):
        assert_close(f"problem {i}", p[5], ref)
