// gemv_nf4.cu -- the forward at decode-sized token counts (T <= 16), bound by
// HBM bandwidth on the 4.127-bit weights ("What is QLoRA?": NF4 converted to
// BF16 on the fly for each matrix multiplication):
//
//   Y[T, N] = X[T, K] W'[N, K]^T + U'[T, r] B[N, r]^T,   U' = s X A^T
//
// (U' as two BF16 planes, hi = bf16(v) and lo = bf16(v - hi), whose products
// with B are added as two MMA chains: the rank-r term keeps ~16 bits of U'.)
//
// Each lane dequantizes whole 64-weight blocks straight into mma.sync A
// fragments (no shared-memory tiles): the MMA's M is 16 weight rows and its N
// is 8 tokens (a second MMA for tokens 8-15), and lane (g, t) of a warp owns
// block t of a 256-wide k-unit for rows g and g + 8 of the warp's 16-row tile.
// The MMA's k-slots are permuted consistently for both operands (a sum does
// not depend on the order of its terms): slot 2t+j of k16-step i holds
// k = 64t + 4i + j and slot 2t+8+j holds k = 64t + 4i + 2 + j, so the four
// codes a lane feeds one MMA per row are four consecutive codes of its block,
// and its X fragments are eight consecutive bytes of one token row.
//
// Two kernels share that per-lane work and differ in how they spread it:
//
// nf4_gemv_kernel (any K that is a multiple of 64): every lane copies its own
// blocks (32 code bytes, the aligned word holding its scale byte, and its c2)
// with cp.async into a private ring of GD items in shared memory.  A CTA is
// one 16-row tile; its S warps split the k-units, and their accumulators are
// added in warp order through shared memory by warp 0, which adds the rank-r
// term B U'^T as extra MMA k-steps and writes BF16 Y.  S is the largest split
// count whose grid of N/16 CTAs is resident in one wave.
//
// nf4_gemv_persist_kernel (K a multiple of 256, the default): persistent
// stream-K over all 16 x 256 units, described where it is defined.
//
// Both are launched with programmatic dependent launch: the first units of
// the weight stream are requested while the preceding kernel (the one
// computing U') still runs; X, U' and Y are touched only after
// griddepcontrol.wait.
//
// lora_u_decode_kernel computes U' itself for these token counts: a cluster of
// 8 CTAs per 16 columns of U' splits K, each CTA requests its whole slice of A
// (and, after the dependency wait, of X) at once, and the partial sums meet
// in rank 0's shared memory.

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int GD = 3;              // units in the per-warp ring
constexpr int kGemvMaxWarps = 8;   // warps per CTA (k-splits of one 16-row tile)
// one item of one warp: codes [2 rows][2 halves][32 lanes][16 B], then per row
// [32 lanes] scale words and [32 lanes] c2
constexpr int kItemBytes = 2048 + 512;

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// cp.async with a source size: bytes past src_bytes are zero-filled (0 reads nothing)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint32_t ldg_pair_bf16(const uint16_t *p, int64_t i0, int64_t i1, bool v0, bool v1) {
  const uint32_t lo = v0 ? static_cast<uint32_t>(__ldg(p + i0)) : 0u;
  const uint32_t hi = v1 ? static_cast<uint32_t>(__ldg(p + i1)) : 0u;
  return lo | (hi << 16);
}

}  // namespace

// Fragments of one item for lane (g, t): weight rows r0 = 16 * tile + g and
// r0 + 8 are the MMA's A operand (M = 16 rows), X is the B operand (N = 8
// tokens, a second MMA for tokens 8-15).  Accumulator: c0/c1 = (row r0, tokens
// 2t, 2t + 1), c2/c3 = (row r0 + 8, tokens 2t, 2t + 1).

// rank-r term for 16-row tile `tile`: v += B U'^T (k16-steps over r), once
// with U''s hi plane and once with its lo plane (columns ldu / 2 on)
template <int TT>
__device__ __forceinline__ void gemv_lora(const GemvParams &p, int64_t tile, int g, int t, float (&v)[TT / 8][4]) {
  const int64_t r0 = tile * 16 + g, r1 = r0 + 8;
  const bool v0 = r0 < p.N, v1 = r1 < p.N;
  const int rv = p.r;
  const int64_t lo_off = p.ldu / 2;
  for (int j0 = 0; j0 < rv; j0 += 16) {
    const int ja = j0 + 2 * t, jb = j0 + 2 * t + 8;
    const uint32_t a0 = ldg_pair_bf16(p.B, r0 * rv + ja, r0 * rv + ja + 1, v0 && ja < rv, v0 && ja + 1 < rv);
    const uint32_t a1 = ldg_pair_bf16(p.B, r1 * rv + ja, r1 * rv + ja + 1, v1 && ja < rv, v1 && ja + 1 < rv);
    const uint32_t a2 = ldg_pair_bf16(p.B, r0 * rv + jb, r0 * rv + jb + 1, v0 && jb < rv, v0 && jb + 1 < rv);
    const uint32_t a3 = ldg_pair_bf16(p.B, r1 * rv + jb, r1 * rv + jb + 1, v1 && jb < rv, v1 && jb + 1 < rv);
#pragma unroll
    for (int h = 0; h < TT / 8; ++h) {
      const int tok = 8 * h + g;
      uint32_t b0 = 0u, b1 = 0u, l0 = 0u, l1 = 0u;
      if (tok < p.T) {
        const uint16_t *ur = p.u + static_cast<int64_t>(tok) * p.ldu;   // each plane zero-padded past r
        b0 = *reinterpret_cast<const uint32_t *>(ur + ja);
        b1 = *reinterpret_cast<const uint32_t *>(ur + jb);
        l0 = *reinterpret_cast<const uint32_t *>(ur + lo_off + ja);
        l1 = *reinterpret_cast<const uint32_t *>(ur + lo_off + jb);
      }
      mma16816(v[h], a0, a1, a2, a3, b0, b1);
      mma16816(v[h], a0, a1, a2, a3, l0, l1);
    }
  }
}

// Y = BF16(v) for the rows and tokens of tile `tile` that exist
template <int TT>
__device__ __forceinline__ void gemv_store(const GemvParams &p, int64_t tile, int g, int t, const float (&v)[TT / 8][4]) {
  const int64_t r0 = tile * 16 + g, r1 = r0 + 8;
  const bool v0 = r0 < p.N, v1 = r1 < p.N;
#pragma unroll
  for (int h = 0; h < TT / 8; ++h) {
    const int ta = 8 * h + 2 * t, tb = ta + 1;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v[h][0], v[h][1]);   // row r0, tokens ta, tb
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v[h][2], v[h][3]);   // row r1
    if (v0 && ta < p.T) p.y[static_cast<int64_t>(ta) * p.N + r0] = __bfloat16_as_ushort(lo.x);
    if (v0 && tb < p.T) p.y[static_cast<int64_t>(tb) * p.N + r0] = __bfloat16_as_ushort(lo.y);
    if (v1 && ta < p.T) p.y[static_cast<int64_t>(ta) * p.N + r1] = __bfloat16_as_ushort(hi.x);
    if (v1 && tb < p.T) p.y[static_cast<int64_t>(tb) * p.N + r1] = __bfloat16_as_ushort(hi.y);
  }
}

// X fragments of k16-steps 4c .. 4c + 3 for the lane's token rows (8 registers per token half)
template <int NH>
__device__ __forceinline__ void load_x_chunk(const uint16_t *const (&xrow)[NH], bool kv, int c, uint32_t (&xf)[NH][8]) {
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if (kv) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4 *>(xrow[h]) + 2 * c);
      const uint4 v1 = __ldg(reinterpret_cast<const uint4 *>(xrow[h]) + 2 * c + 1);
      xf[h][0] = v0.x; xf[h][1] = v0.y; xf[h][2] = v0.z; xf[h][3] = v0.w;
      xf[h][4] = v1.x; xf[h][5] = v1.y; xf[h][6] = v1.z; xf[h][7] = v1.w;
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) xf[h][q] = 0u;
    }
  }
}

template <int TT, bool SYM>
__global__ void __launch_bounds__(kGemvMaxWarps * 32) nf4_gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(16) uint8_t gsm[];
  constexpr int NH = TT / 8;   // token halves
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int S = p.splits;
  const int64_t tile = blockIdx.x;
  const int64_t KB = p.K / 64;
  const int u_beg = warp * p.upw;
  const int nu = max(0, min(p.units, u_beg + p.upw) - u_beg);
  const uint32_t ring = smem_u32(gsm) + warp * GD * kItemBytes;
  const uintptr_t scales_addr = reinterpret_cast<uintptr_t>(p.scales);
  const int64_t r0 = tile * 16 + g;
  bool rok[2];
  int64_t rowblk[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    rok[h] = r0 + 8 * h < p.N;
    rowblk[h] = (r0 + 8 * h) * KB;
  }

  // unit u_beg + i into ring slot i % GD (one commit group per unit, empty past the end)
  auto issue = [&](int i) {
    if (i < nu) {
      const int64_t kb = static_cast<int64_t>(u_beg + i) * 4 + t;
      const uint32_t base = ring + (i % GD) * kItemBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool ok = kb < KB && rok[h];
        const int64_t blk = ok ? rowblk[h] + kb : 0;
        const uint32_t d = base + h * 1024 + lane * 16;
        const uint8_t *src = p.codes + blk * 32;
        cp_async16(d, src, ok ? 16u : 0u);
        cp_async16(d + 512, src + 16, ok ? 16u : 0u);
        const uint32_t da = base + 2048 + h * 256 + lane * 4;
        cp_async4(da, reinterpret_cast<const void *>((scales_addr + blk) & ~static_cast<uintptr_t>(3)), ok ? 4u : 0u);
        cp_async4(da + 128, p.c2 + (blk >> 8), ok ? 4u : 0u);
      }
    }
    cp_async_commit();
  };

#pragma unroll 1
  for (int i = 0; i < GD - 1; ++i) issue(i);   // the weights do not depend on the preceding kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  grid_dep_wait();                               // X, U' and Y may

  // token rows this lane feeds to the MMA (rows past T repeat row T - 1; their
  // accumulator columns are never stored)
  const uint16_t *xrow0[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) xrow0[h] = p.x + static_cast<int64_t>(min(8 * h + g, p.T - 1)) * p.K + 64 * t;
  float acc[NH][4], acc2[NH][4];   // even / odd k16-steps (two independent MMA chains)
#pragma unroll
  for (int h = 0; h < NH; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = acc2[h][e] = 0.f;
#pragma unroll 1
  for (int i = 0; i < nu; ++i) {
    issue(i + GD - 1);
    const int u = u_beg + i;
    const bool kv = static_cast<int64_t>(u) * 256 + 64 * t < p.K;   // false past K (codes zero-filled too)
    const uint16_t *xrow[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) xrow[h] = xrow0[h] + static_cast<int64_t>(u) * 256;
    uint32_t xf[NH][8], xn[NH][8];
    load_x_chunk<NH>(xrow, kv, 0, xf);
    cp_async_wait<GD - 1>();      // this lane's copies of unit i have landed
    const uint32_t base = ring + (i % GD) * kItemBytes;
    float scale[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t sword = lds32(base + 2048 + h * 256 + lane * 4);
      const float c2v = __uint_as_float(lds32(base + 2048 + h * 256 + 128 + lane * 4));
      const int64_t blk = rowblk[h] + static_cast<int64_t>(u) * 4 + t;
      const uint32_t fbyte = (sword >> (8u * static_cast<uint32_t>((scales_addr + blk) & 3u))) & 0xffu;
      scale[h] = __fmul_rn(e4m3_to_float(fbyte), c2v);
    }
    // four chunks of 16 codes per row (k16-steps 4c .. 4c + 3); X of the next chunk is loaded ahead
    if constexpr (SYM) {
      const Lut8 l0 = make_lut8(p.codebook, scale[0]);
      const Lut8 l1 = make_lut8(p.codebook, scale[1]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < 3) load_x_chunk<NH>(xrow, kv, c + 1, xn);
        const uint2 w0 = lds64(base + (c >> 1) * 512 + lane * 16 + (c & 1) * 8);
        const uint2 w1 = lds64(base + 1024 + (c >> 1) * 512 + lane * 16 + (c & 1) * 8);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          uint32_t a[4], b[4];
          lut8_lookup8(l0, e ? w0.y : w0.x, a[0], a[1], a[2], a[3]);
          lut8_lookup8(l1, e ? w1.y : w1.x, b[0], b[1], b[2], b[3]);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            mma16816(acc[h], a[0], b[0], a[1], b[1], xf[h][4 * e], xf[h][4 * e + 1]);
            mma16816(acc2[h], a[2], b[2], a[3], b[3], xf[h][4 * e + 2], xf[h][4 * e + 3]);
          }
        }
        if (c < 3) {
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) xf[h][q] = xn[h][q];
        }
      }
    } else {
      const Lut16 l0 = make_lut16(p.codebook, scale[0]);
      const Lut16 l1 = make_lut16(p.codebook, scale[1]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < 3) load_x_chunk<NH>(xrow, kv, c + 1, xn);
        const uint2 w0 = lds64(base + (c >> 1) * 512 + lane * 16 + (c & 1) * 8);
        const uint2 w1 = lds64(base + 1024 + (c >> 1) * 512 + lane * 16 + (c & 1) * 8);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t s0 = (k & 2) ? w0.y : w0.x, s1 = (k & 2) ? w1.y : w1.x;
          uint32_t a0, a2, a1, a3;
          lut16_lookup4(l0, (k & 1) ? (s0 >> 16) : s0, a0, a2);
          lut16_lookup4(l1, (k & 1) ? (s1 >> 16) : s1, a1, a3);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            if (k & 1) mma16816(acc2[h], a0, a1, a2, a3, xf[h][2 * k], xf[h][2 * k + 1]);
            else mma16816(acc[h], a0, a1, a2, a3, xf[h][2 * k], xf[h][2 * k + 1]);
          }
        }
        if (c < 3) {
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) xf[h][q] = xn[h][q];
        }
      }
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int h = 0; h < NH; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] += acc2[h][e];

  // the warps' partial sums over their k-units, added in warp order by warp 0;
  // each warp's slot is the start of its own ring, whose copies have all landed
  if (S > 1) {
    if (warp > 0) {
      float4 *red = reinterpret_cast<float4 *>(gsm + warp * GD * kItemBytes);
#pragma unroll
      for (int h = 0; h < NH; ++h) red[h * 32 + lane] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
    }
    __syncthreads();
    if (warp == 0) {
      for (int w2 = 1; w2 < S; ++w2) {
        const float4 *red = reinterpret_cast<const float4 *>(gsm + w2 * GD * kItemBytes);
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float4 o = red[h * 32 + lane];
          acc[h][0] += o.x; acc[h][1] += o.y; acc[h][2] += o.z; acc[h][3] += o.w;
        }
      }
    }
  }
  if (warp == 0) {
    gemv_lora<TT>(p, tile, g, t, acc);
    gemv_store<TT>(p, tile, g, t, acc);
  }
}

// ---------------------------------------------------------------------------
// Persistent GEMV for K a multiple of 256: the same per-code work as the kernel
// above (each lane converts whole 64-weight blocks with a per-block register
// table of BF16(RN32(codebook[j] * scale)), so W' is the dequantization's to
// the bit), with the work spread for bandwidth rather than one CTA per tile.
//
// The 16 x 256 units are numbered tile-major (unit = tile * KU + k-unit) and
// cut into C equal contiguous ranges, one per CTA, each cut again into
// contiguous chunks, one per warp.  A warp streams its chunk through a private
// cp.async ring of kPGD units (the 16 x 128-byte code tile stored with a
// 128-byte swizzle, so that each lane's 32-byte block loads without bank
// conflicts) and keeps one tile's sums at a time.  When a tile ends:
//   - a tile inside the warp's chunk is finished by the warp: rank-r term
//     B U'^T, then BF16 Y;
//   - a tile shared with other warps of the CTA leaves its sums in the warp's
//     shared-memory slot (slot 0 for the chunk's first tile, 1 for its last);
//     the last of those warps to arrive (a shared-memory counter) adds the
//     slots in warp order and, if the tile lies inside the CTA's range,
//     finishes it;
//   - a tile shared with another CTA leaves the CTA's sum in the split
//     workspace (slot 0 / 1 as above, per CTA); the last CTA to arrive (a
//     workspace counter per tile, zeroed again after use) adds them in CTA
//     order and finishes the tile.
// Every sum is taken in a fixed order, so a launch's result does not depend on
// timing.  No thread waits on another warp or CTA.  U' (from the preceding
// kernel) is copied to shared memory once per CTA after the dependency wait.
// ---------------------------------------------------------------------------
// A CTA is 8 warps with about 86 KB of shared memory and 32K registers, so that
// two CTAs fit on an SM: those of one launch, or one of this launch and one of
// the next (which then requests its weights while this one runs).
#ifndef QLORA_PERSIST_CTAS_PER_SM
#define QLORA_PERSIST_CTAS_PER_SM 2
#endif
constexpr int kPWarps = 8;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kPGD = 4;                            // units per warp ring (3 in flight)
constexpr int kPStage = 2048 + 64 + 64;            // codes [16][128] swizzled, scale words [16], c2 [16]
constexpr int kPRing = kPWarps * kPGD * kPStage;
constexpr int kPSlotFloats = 16 * 16;              // one tile's sums: [T <= 16][16 rows]
constexpr int kPUBytes = 16 * 256 * 2;             // U' [T <= 16][ldu <= 256] BF16 (hi and lo planes)
constexpr int kPSmem = kPRing + kPWarps * 2 * kPSlotFloats * 4 + kPWarps * 2 * 4 + kPUBytes;
constexpr int kPCtasPerSm = QLORA_PERSIST_CTAS_PER_SM;

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// lane (g, t) values of one tile's sums in a [T][16] float array: v[h][e] is
// (row g + 8 (e >> 1), token 8 h + 2 t + (e & 1))
template <int NH, typename F>
__device__ __forceinline__ void for_tile_values(int T, int g, int t, F &&f) {
#pragma unroll
  for (int h = 0; h < NH; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = 8 * h + 2 * t + (e & 1), row = g + 8 * (e >> 1);
      if (tok < T) f(h, e, tok * 16 + row);
    }
}

template <int TT, bool SYM>
__global__ void __launch_bounds__(kPThreads, 2) nf4_gemv_persist_kernel(const GemvParams p) {
  extern __shared__ __align__(128) uint8_t psm[];
  constexpr int NH = TT / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  float *slots = reinterpret_cast<float *>(psm + kPRing);                          // [warp][2][kPSlotFloats]
  // one counter per (first contributing warp, that warp's slot) of each shared tile
  uint32_t *scnt = reinterpret_cast<uint32_t *>(psm + kPRing + kPWarps * 2 * kPSlotFloats * 4);   // [warp][2]
  uint16_t *su = reinterpret_cast<uint16_t *>(psm + kPRing + kPWarps * 2 * kPSlotFloats * 4 + kPWarps * 2 * 4);
  const uint32_t ring = smem_u32(psm) + warp * (kPGD * kPStage);
  const int KU = p.units;
  const int64_t KB = p.K / 64, rowbytes = p.K / 2;
  const int64_t U = static_cast<int64_t>(p.tiles) * KU, C = gridDim.x;
  // this CTA's units [ub, ue) and this warp's chunk [wb, we)
  auto cta_begin = [&](int64_t c) { return c * U / C; };
  const int64_t ub = cta_begin(blockIdx.x), ue = cta_begin(blockIdx.x + 1), n = ue - ub;
  const int64_t weff = min(static_cast<int64_t>(kPWarps), n);
  auto warp_begin = [&](int64_t w) { return ub + w * n / weff; };
  const int64_t wb = warp < weff ? warp_begin(warp) : ue, we = warp < weff ? warp_begin(warp + 1) : ue;
  auto owner_warp = [&](int64_t x) { return ((x - ub + 1) * weff - 1) / n; };
  auto owner_cta = [&](int64_t x) { return ((x + 1) * C - 1) / U; };

  if (threadIdx.x < 2 * kPWarps) scnt[threadIdx.x] = 0u;
  // Even warps walk their chunk forwards and odd warps backwards, so that of
  // two neighbouring warps sharing a tile one reaches it first, and a CTA's
  // last warp (odd) starts with the tile it may share with the next CTA.
  const bool rev = (warp & 1) != 0;
  const int64_t cnt = we - wb;
  const int64_t x0 = rev ? we - 1 : wb;
  auto step = [&](int64_t &tl, int &uu) {
    if (!rev) {
      if (++uu == KU) {
        uu = 0;
        ++tl;
      }
    } else if (--uu < 0) {
      uu = KU - 1;
      --tl;
    }
  };

  // the next unit into ring slot `slot`: lane L copies 16-byte chunks L + 32 j of
  // the code tile (row L / 8 + 4 j, column L % 8), lanes 0-15 the scale words and
  // lanes 16-31 the c2 of rows 0-15 (one commit group per unit, empty past the end)
  const int crow = lane >> 3, ccol = lane & 7;
  int64_t inext = 0, itile = x0 / KU;
  int iu = static_cast<int>(x0 - itile * KU);
  auto issue = [&](int slot) {
    if (inext < cnt) {
      const uint32_t st = ring + slot * kPStage;
      const int64_t n0 = itile * 16;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = crow + 4 * j;
        const bool ok = n0 + row < p.N;
        const uint8_t *src = p.codes + (ok ? (n0 + row) * rowbytes + static_cast<int64_t>(iu) * 128 + ccol * 16 : 0);
        cp_async16(st + row * 128 + ((ccol ^ (row & 7)) << 4), src, ok ? 16u : 0u);
      }
      const int row = lane & 15;
      const bool ok = n0 + row < p.N;
      const int64_t blk = ok ? (n0 + row) * KB + 4 * static_cast<int64_t>(iu) : 0;
      if (lane < 16) cp_async4(st + 2048 + row * 4, p.scales + blk, ok ? 4u : 0u);
      else cp_async4(st + 2112 + row * 4, p.c2 + (blk >> 8), ok ? 4u : 0u);
      step(itile, iu);
    }
    ++inext;
    cp_async_commit();
  };

#pragma unroll 1
  for (int s = 0; s < kPGD - 1; ++s) issue(s);   // the weights do not depend on the preceding kernel
  __syncthreads();                                        // the shared counters are zero
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  grid_dep_wait();   // X, U', Y and the split workspace may
  // U' into shared memory, once for all the CTA's rank-r terms
  {
    const int words = p.T * static_cast<int>(p.ldu) / 8;
    for (int i = threadIdx.x; i < words; i += kPThreads)
      reinterpret_cast<uint4 *>(su)[i] = reinterpret_cast<const uint4 *>(p.u)[i];
  }
  __syncthreads();
  GemvParams pl = p;   // the rank-r term reads U' from shared memory
  pl.u = su;

  float acc[NH][4], acc2[NH][4];   // even / odd k16-steps (two independent MMA chains)
#pragma unroll
  for (int h = 0; h < NH; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = acc2[h][e] = 0.f;
  // token rows this lane feeds to the MMA (rows past T repeat row T - 1; their
  // accumulator columns are never stored)
  const uint16_t *xrow0[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) xrow0[h] = p.x + static_cast<int64_t>(min(8 * h + g, p.T - 1)) * p.K + 64 * t;

  int64_t tile = x0 / KU;
  int u = static_cast<int>(x0 - tile * KU);
  int slot = 0;
  bool seg_start = true;
  const int64_t brow_bytes = 2 * static_cast<int64_t>(p.r) * 16;   // one tile's rows of B
#pragma unroll 1
  for (int64_t i = 0; i < cnt; ++i) {
    issue((slot + kPGD - 1) % kPGD);
    if (seg_start) {
      // the tile's rows of B, for whichever warp finishes it
      const int64_t off = static_cast<int64_t>(lane) * 128;
      if (off < brow_bytes && tile * 16 + off / (2 * p.r) < p.N)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t *>(p.B) + tile * brow_bytes + off));
      seg_start = false;
    }
    const uint16_t *xrow[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) xrow[h] = xrow0[h] + static_cast<int64_t>(u) * 256;
    uint32_t xf[NH][8], xn[NH][8];
    load_x_chunk<NH>(xrow, true, 0, xf);
    cp_async_wait<kPGD - 1>();   // this lane's copies of the unit have landed
    __syncwarp();                // and every lane's
    const uint32_t st = ring + slot * kPStage;
    // block t of rows g and g + 8: its scale, and its 32 code bytes (chunks 2t, 2t + 1)
    float scale[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t sword = lds32(st + 2048 + (g + 8 * h) * 4);
      const float c2v = __uint_as_float(lds32(st + 2112 + (g + 8 * h) * 4));
      scale[h] = __fmul_rn(e4m3_to_float((sword >> (8 * t)) & 0xffu), c2v);
    }
    const uint32_t r0a = st + g * 128, r1a = st + (g + 8) * 128;
    const uint4 q0[2] = {lds128(r0a + (((2 * t) ^ g) << 4)), lds128(r0a + (((2 * t + 1) ^ g) << 4))};
    const uint4 q1[2] = {lds128(r1a + (((2 * t) ^ g) << 4)), lds128(r1a + (((2 * t + 1) ^ g) << 4))};
    __syncwarp();   // every lane has read the slot before it is refilled
    slot = (slot + 1) % kPGD;
    // four chunks of 16 codes per row (k16-steps 4c .. 4c + 3); X of the next chunk is loaded ahead
    if constexpr (SYM) {
      const Lut8 l0 = make_lut8(p.codebook, scale[0]);
      const Lut8 l1 = make_lut8(p.codebook, scale[1]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < 3) load_x_chunk<NH>(xrow, true, c + 1, xn);
        const uint4 &v0 = q0[c >> 1], &v1 = q1[c >> 1];
        const uint32_t w0[2] = {(c & 1) ? v0.z : v0.x, (c & 1) ? v0.w : v0.y};
        const uint32_t w1[2] = {(c & 1) ? v1.z : v1.x, (c & 1) ? v1.w : v1.y};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          uint32_t a[4], b[4];
          lut8_lookup8(l0, w0[e], a[0], a[1], a[2], a[3]);
          lut8_lookup8(l1, w1[e], b[0], b[1], b[2], b[3]);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            mma16816(acc[h], a[0], b[0], a[1], b[1], xf[h][4 * e], xf[h][4 * e + 1]);
            mma16816(acc2[h], a[2], b[2], a[3], b[3], xf[h][4 * e + 2], xf[h][4 * e + 3]);
          }
        }
        if (c < 3) {
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) xf[h][q] = xn[h][q];
        }
      }
    } else {
      const Lut16 l0 = make_lut16(p.codebook, scale[0]);
      const Lut16 l1 = make_lut16(p.codebook, scale[1]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < 3) load_x_chunk<NH>(xrow, true, c + 1, xn);
        const uint4 &v0 = q0[c >> 1], &v1 = q1[c >> 1];
        const uint32_t w0[2] = {(c & 1) ? v0.z : v0.x, (c & 1) ? v0.w : v0.y};
        const uint32_t w1[2] = {(c & 1) ? v1.z : v1.x, (c & 1) ? v1.w : v1.y};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t s0 = w0[k >> 1], s1 = w1[k >> 1];
          uint32_t a0, a2, a1, a3;
          lut16_lookup4(l0, (k & 1) ? (s0 >> 16) : s0, a0, a2);
          lut16_lookup4(l1, (k & 1) ? (s1 >> 16) : s1, a1, a3);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            if (k & 1) mma16816(acc2[h], a0, a1, a2, a3, xf[h][2 * k], xf[h][2 * k + 1]);
            else mma16816(acc[h], a0, a1, a2, a3, xf[h][2 * k], xf[h][2 * k + 1]);
          }
        }
        if (c < 3) {
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) xf[h][q] = xn[h][q];
        }
      }
    }

    if (i + 1 == cnt || (rev ? u == 0 : u + 1 == KU)) {
      seg_start = true;
      // the end of this warp's part of the tile
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[h][e] += acc2[h][e];
          acc2[h][e] = 0.f;
        }
      const int64_t t0 = tile * KU, t1 = t0 + KU;   // the tile's units
      if (t0 >= wb && t1 <= we) {
        gemv_lora<TT>(pl, tile, g, t, acc);
        gemv_store<TT>(p, tile, g, t, acc);
      } else {
        float *mine = slots + (warp * 2 + (t0 <= wb ? 0 : 1)) * kPSlotFloats;
        for_tile_values<NH>(p.T, g, t, [&](int h, int e, int i) { mine[i] = acc[h][e]; });
        const int64_t wf = owner_warp(max(ub, t0)), wl = owner_warp(min(ue, t1) - 1);
        __threadfence_block();
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atomicAdd(scnt + 2 * wf + (t0 <= warp_begin(wf) ? 0 : 1), 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == static_cast<uint32_t>(wl - wf)) {
          // the CTA's last warp on this tile: its sum over the CTA's warps, in warp order
          __threadfence_block();
          float sum[NH][4];
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) sum[h][e] = 0.f;
          for (int64_t w2 = wf; w2 <= wl; ++w2) {
            const float *src = slots + (w2 * 2 + (t0 <= warp_begin(w2) ? 0 : 1)) * kPSlotFloats;
            for_tile_values<NH>(p.T, g, t, [&](int h, int e, int i) { sum[h][e] += src[i]; });
          }
          if (t0 >= ub && t1 <= ue) {
            gemv_lora<TT>(pl, tile, g, t, sum);
            gemv_store<TT>(p, tile, g, t, sum);
          } else {
            // shared with another CTA: leave the CTA's sum in the workspace
            float *gp = p.part + (static_cast<int64_t>(blockIdx.x) * 2 + (t0 <= ub ? 0 : 1)) * kPSlotFloats;
            for_tile_values<NH>(p.T, g, t, [&](int h, int e, int i) { gp[i] = sum[h][e]; });
            __threadfence();
            __syncwarp();
            uint32_t gold = 0;
            if (lane == 0) gold = atomicAdd(p.counters + tile, 1u);
            gold = __shfl_sync(0xffffffffu, gold, 0);
            const int64_t cf = owner_cta(t0), cl = owner_cta(t1 - 1);
            if (gold == static_cast<uint32_t>(cl - cf)) {
              // the last CTA on this tile: the CTAs' sums in CTA order
              __threadfence();
              float tot[NH][4];
#pragma unroll
              for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int e = 0; e < 4; ++e) tot[h][e] = 0.f;
              for (int64_t c2 = cf; c2 <= cl; ++c2) {
                const float *src = p.part + (c2 * 2 + (t0 <= cta_begin(c2) ? 0 : 1)) * kPSlotFloats;
                for_tile_values<NH>(p.T, g, t, [&](int h, int e, int i) { tot[h][e] += __ldcg(src + i); });
              }
              gemv_lora<TT>(pl, tile, g, t, tot);
              gemv_store<TT>(p, tile, g, t, tot);
              if (lane == 0) p.counters[tile] = 0u;   // zero again for the next call
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
    }
    step(tile, u);
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// U' = s X A^T for T <= 16 tokens, as BF16 hi and lo planes.  Grid:
// 8 x (plane / 16) CTAs in clusters of 8; cluster c owns columns 16c .. 16c + 15
// of each plane (A rows past r arrive as zeros, so the padding columns come
// out zero), rank k owns the k-th slice of the contraction.  Four warps split the slice; each runs mma.sync with
// A = X [tokens][k] and B = A^T.
// ---------------------------------------------------------------------------
constexpr int kUCluster = 8;
constexpr int kUThreads = 128;

template <int TT>
__global__ void __launch_bounds__(kUThreads, 1) lora_u_decode_kernel(const LoraUDecodeParams p) {
  extern __shared__ __align__(16) uint8_t usm[];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int cg = blockIdx.x / kUCluster;
  const int pitch = p.kc + 8;                      // BF16 elements per shared row (conflict-free fragments)
  uint16_t *sa = reinterpret_cast<uint16_t *>(usm);            // [16 j][pitch]
  uint16_t *sx = sa + 16 * pitch;                              // [TT tok][pitch]
  float4 *red = reinterpret_cast<float4 *>(sx + TT * pitch);   // [4 warps][2][32]
  const int64_t kbeg = static_cast<int64_t>(rank) * p.kc;
  const int64_t klen = max(static_cast<int64_t>(0), min(static_cast<int64_t>(p.kc), p.K - kbeg));
  const int chunks = static_cast<int>(p.kc / 8);               // 16-byte pieces per row

  // A rows 16cg .. 16cg + 15 of this slice (static: requested before the dependency wait)
  for (int c = threadIdx.x; c < 16 * chunks; c += kUThreads) {
    const int j = c / chunks, q = c % chunks;
    const int64_t jr = static_cast<int64_t>(cg) * 16 + j;
    const bool ok = jr < p.r && 8 * q < klen;
    const uint16_t *src = ok ? p.A + jr * p.K + kbeg + 8 * q : p.A;
    const uint32_t d = smem_u32(sa + j * pitch + 8 * q);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(ok ? 16 : 0) : "memory");
  }
  grid_dep_wait();   // X may be written by the preceding kernel, U' read by it
  for (int c = threadIdx.x; c < TT * chunks; c += kUThreads) {
    const int tok = c / chunks, q = c % chunks;
    const bool ok = tok < p.T && 8 * q < klen;
    const uint16_t *src = ok ? p.x + static_cast<int64_t>(tok) * p.K + kbeg + 8 * q : p.x;
    const uint32_t d = smem_u32(sx + tok * pitch + 8 * q);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(ok ? 16 : 0) : "memory");
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int steps = p.kc / 16;
  for (int st = warp; st < steps; st += 4) {
    const int k0 = st * 16;
    auto ld32 = [&](const uint16_t *row, int k) { return *reinterpret_cast<const uint32_t *>(row + k); };
    const uint32_t a0 = ld32(sx + g * pitch, k0 + 2 * t);
    const uint32_t a2 = ld32(sx + g * pitch, k0 + 2 * t + 8);
    const uint32_t a1 = TT == 16 ? ld32(sx + (g + 8) * pitch, k0 + 2 * t) : 0u;
    const uint32_t a3 = TT == 16 ? ld32(sx + (g + 8) * pitch, k0 + 2 * t + 8) : 0u;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const uint16_t *arow = sa + (nt * 8 + g) * pitch;
      mma16816(acc[nt], a0, a1, a2, a3, ld32(arow, k0 + 2 * t), ld32(arow, k0 + 2 * t + 8));
    }
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) red[(warp * 2 + nt) * 32 + lane] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float4 v = red[nt * 32 + lane];
      for (int w = 1; w < 4; ++w) {
        const float4 o = red[(w * 2 + nt) * 32 + lane];
        v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
      }
      red[nt * 32 + lane] = v;   // this CTA's partial sum, in warp 0's slots
    }
  }
  cluster_arrive_wait();
  if (rank == 0 && warp == 0) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float4 v = red[nt * 32 + lane];
      for (uint32_t k = 1; k < kUCluster; ++k) {
        const uint32_t ra = mapa_shared(smem_u32(&red[nt * 32 + lane]), k);
        float4 o;
        asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(o.x), "=f"(o.y), "=f"(o.z), "=f"(o.w)
                     : "r"(ra)
                     : "memory");
        v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
      }
      // fragment: (token g, columns 2t, 2t+1) and (token g + 8, ...); the hi
      // plane, then the lo plane p.plane columns on
      const int64_t col = static_cast<int64_t>(cg) * 16 + nt * 8 + 2 * t;
      auto put = [&](int tok, float a, float b) {
        const __nv_bfloat162 hi = __floats2bfloat162_rn(p.alpha * a, p.alpha * b);
        const __nv_bfloat162 lo =
            __floats2bfloat162_rn(p.alpha * a - __low2float(hi), p.alpha * b - __high2float(hi));
        uint16_t *row = p.u + static_cast<int64_t>(tok) * p.ldu;
        *reinterpret_cast<__nv_bfloat162 *>(row + col) = hi;
        *reinterpret_cast<__nv_bfloat162 *>(row + p.plane + col) = lo;
      };
      if (g < p.T) put(g, v.x, v.y);
      if (TT == 16 && g + 8 < p.T) put(g + 8, v.z, v.w);
    }
  }
  cluster_arrive_wait();   // the peers keep their shared memory until rank 0 has read it
}

int gemv_smem_bytes(int splits) { return splits * GD * kItemBytes; }

namespace {

// CTAs of `splits` warps that one SM holds at once (cached per kernel and split count)
template <int TT, bool SYM>
int gemv_occupancy(int splits) {
  static std::atomic<int> occ[64][kGemvMaxWarps + 1];   // per device; 0 = not yet known
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (ensure_smem_optin(reinterpret_cast<const void *>(nf4_gemv_kernel<TT, SYM>), gemv_smem_bytes(kGemvMaxWarps)) !=
      cudaSuccess)
    return -1;
  int known = occ[dev][splits].load(std::memory_order_relaxed);
  if (known == 0) {
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, nf4_gemv_kernel<TT, SYM>, 32 * splits,
                                                      gemv_smem_bytes(splits)) != cudaSuccess)
      return -1;
    known = o > 0 ? o : -1;
    occ[dev][splits].store(known, std::memory_order_relaxed);
  }
  return known;
}

// The most k-splits per 16-row tile whose grid still fits in one wave (all
// tiles resident at once); one split if even that does not fit.
template <int TT, bool SYM>
cudaError_t gemv_plan(int64_t N, int64_t K, int num_sms, GemvPlan &pl) {
  pl.units = static_cast<int>((K + 255) / 256);
  pl.tiles = static_cast<int>((N + 15) / 16);
  int best = 1;
  for (int s = 1; s <= kGemvMaxWarps && s <= pl.units; ++s) {
    const int upw = (pl.units + s - 1) / s;
    const int splits = (pl.units + upw - 1) / upw;
    if (splits != s) continue;
    const int occ = gemv_occupancy<TT, SYM>(s);
    if (occ < 0) return cudaErrorInvalidConfiguration;
    if (static_cast<int64_t>(occ) * num_sms >= pl.tiles) best = s;
  }
  pl.upw = (pl.units + best - 1) / best;
  pl.splits = (pl.units + pl.upw - 1) / pl.upw;
  return cudaSuccess;
}

template <int TT, bool SYM>
cudaError_t launch_t(GemvParams p, int num_sms, cudaStream_t st, bool pdl) {
  GemvPlan pl;
  cudaError_t e = gemv_plan<TT, SYM>(p.N, p.K, num_sms, pl);
  if (e != cudaSuccess) return e;
  p.units = pl.units;
  p.upw = pl.upw;
  p.splits = pl.splits;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.tiles), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(32 * pl.splits), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(gemv_smem_bytes(pl.splits));
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, nf4_gemv_kernel<TT, SYM>, p);
}

}  // namespace

int lora_u_decode_smem_bytes(int64_t K, int T) {
  const int64_t kc = ((K + kUCluster - 1) / kUCluster + 63) / 64 * 64;
  const int tt = T > 8 ? 16 : 8;
  return static_cast<int>((16 + tt) * (kc + 8) * 2 + 4 * 2 * 32 * 16);
}

namespace {
template <int TT>
cudaError_t launch_u(const LoraUDecodeParams &p, int smem, cudaStream_t st, bool pdl) {
  cudaError_t e = ensure_smem_optin(reinterpret_cast<const void *>(lora_u_decode_kernel<TT>), kLoraUDecodeMaxSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(kUCluster * (p.plane / 16)), 1, 1);
  cfg.blockDim = dim3(kUThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = kUCluster;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, lora_u_decode_kernel<TT>, p);
}
}  // namespace

cudaError_t launch_lora_u_decode(const LoraUDecodeParams &p_in, cudaStream_t st, bool pdl) {
  LoraUDecodeParams p = p_in;
  if (p.T < 1 || p.T > 16 || p.r < 1 || p.plane % 16 != 0 || p.plane < p.r || p.ldu < 2 * p.plane ||
      p.ldu % 8 != 0 || p.K % 64 != 0)
    return cudaErrorInvalidValue;
  p.kc = static_cast<int>(((p.K + kUCluster - 1) / kUCluster + 63) / 64 * 64);
  const int smem = lora_u_decode_smem_bytes(p.K, p.T);
  if (smem > kLoraUDecodeMaxSmem) return cudaErrorInvalidValue;
  return p.T > 8 ? launch_u<16>(p, smem, st, pdl) : launch_u<8>(p, smem, st, pdl);
}

int gemv_persist_ctas(int64_t N, int64_t K, int num_sms, int max_tiles) {
  if (K % 256 != 0 || K <= 0 || N <= 0) return 0;
  const int64_t tiles = (N + 15) / 16, units = tiles * (K / 256);
  if (tiles > max_tiles || units > (int64_t(1) << 40)) return 0;
  // one whole tile per CTA when the tiles fit in the resident CTAs (no tile is
  // then shared between CTAs), otherwise every resident CTA with an equal share
  const int64_t slots = std::min<int64_t>(static_cast<int64_t>(num_sms) * kPCtasPerSm, kPersistMaxCtas);
  return static_cast<int>(tiles <= slots ? tiles : std::min<int64_t>(units, slots));
}

size_t gemv_persist_partials_bytes(int64_t N, int64_t K, int max_tiles) {
  if (gemv_persist_ctas(N, K, kPersistMaxCtas, max_tiles) == 0) return 0;
  return static_cast<size_t>(kPersistMaxCtas) * 2 * kPSlotFloats * sizeof(float);
}

namespace {
template <int TT, bool SYM>
cudaError_t launch_persist(const GemvParams &p, int num_sms, cudaStream_t st, bool pdl) {
  cudaError_t e = ensure_smem_optin(reinterpret_cast<const void *>(nf4_gemv_persist_kernel<TT, SYM>), kPSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.ctas), 1, 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = kPSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, nf4_gemv_persist_kernel<TT, SYM>, p);
}
}  // namespace

cudaError_t launch_gemv(const GemvParams &p_in, int num_sms, cudaStream_t st, bool pdl) {
  const GemvParams &p = p_in;
  if (p.T < 1 || p.T > 16 || p.N % 8 != 0 || p.K % 64 != 0 || num_sms < 1) return cudaErrorInvalidValue;
  const bool t16 = p.T > 8;
  if (p.ctas > 0) {
    GemvParams q = p;
    q.units = static_cast<int>(p.K / 256);
    q.tiles = static_cast<int>((p.N + 15) / 16);
    q.ctas = std::min(p.ctas, num_sms * kPCtasPerSm);
    if (p.K % 256 != 0 || !q.part || !q.counters || p.ldu > 256 || p.ldu % 8 != 0) return cudaErrorInvalidValue;
    if (q.sym) return t16 ? launch_persist<16, true>(q, num_sms, st, pdl) : launch_persist<8, true>(q, num_sms, st, pdl);
    return t16 ? launch_persist<16, false>(q, num_sms, st, pdl) : launch_persist<8, false>(q, num_sms, st, pdl);
  }
  if (p.sym) return t16 ? launch_t<16, true>(p, num_sms, st, pdl) : launch_t<8, true>(p, num_sms, st, pdl);
  return t16 ? launch_t<16, false>(p, num_sms, st, pdl) : launch_t<8, false>(p, num_sms, st, pdl);
}

}  // namespace qlora
