// decode.cu -- the forward at decode-sized token counts (T <= 16), for one
// projection or several at once, bound by HBM bandwidth on the 4.127-bit
// weights ("What is QLoRA?": NF4 converted to BF16 on the fly for each matrix
// multiplication; "QLoRA: Efficient Fine-Tuning", Step 3 eq. 3):
//
//   Y_p[T, N_p] = X_p W'_p^T + U'_p B_p^T,   U'_p = s_p X_p A_p^T   (p = each projection)
//
// decode_u_kernel computes every U'_p (as BF16 hi + lo planes); then
// decode_gemv_kernel streams every weight once.
//
// decode_gemv_kernel.  Work is cut into units of 32 weight rows x 256 codes (4
// blocks of 64 per row, 4 KB of codes), numbered problem by problem, tile
// (32 rows) by tile, and split into contiguous ranges: one per CTA, then one per
// warp (stream-K).  Each warp streams its range through a private ring of four
// 4 KB slots, each filled by ONE tensor-memory-access copy (a [32 rows x 128 B]
// box with the 128-byte swizzle, so that every lane's 32-byte block reads
// without bank conflicts) completing on the slot's mbarrier.
//
// The MMA is mma.sync.m16n8k16 with the weights as M (16 rows) and the tokens
// as N (8; a second MMA for tokens 8-15): lane (g, t) dequantizes block t of
// rows g, g + 8 (first half of the tile) and g + 16, g + 24 (second half)
// straight into A fragments, so the lookups write the MMA's operand registers
// directly and one X fragment (B, a contiguous half of one 16-byte load) serves
// both halves.  The k-slots of each MMA are permuted identically for both
// operands (a sum does not depend on the order of its terms): lane t's slots
// {2t, 2t+1, 2t+8, 2t+9} hold four consecutive codes of its block, and its X
// fragment holds the matching eight bytes of token row g.  W' is the dequantization's to the bit: each block's 16 (or 8, for a
// sign-symmetric codebook) BF16(RN32(q_j * s_b)) values are built in registers
// and the codes select them with byte permutes.
//
// When a warp ends a tile: a tile inside its range is finished by it (the
// rank-r term U' B^T as extra MMAs over the hi and the lo plane of U', then
// BF16 Y); a tile shared with other warps of the CTA leaves its sums in the
// warp's shared-memory slot and the last warp to arrive adds the slots in warp
// order; a tile shared with other CTAs leaves the CTA's sums in the workspace
// and the last CTA to arrive adds them in CTA order.  Every sum is taken in a
// fixed order, so results do not depend on timing; no thread waits on another.
//
// Launched as a programmatic dependent: the first ring fills are requested
// before griddepcontrol.wait (the weights are static); X, U', the workspace and
// Y are touched only after it.

#include <algorithm>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int DT = 32;                      // weight rows per tile
constexpr int DUC = 256;                    // codes per row per unit (4 blocks)
constexpr int DW = kDecodeWarps;            // warps per CTA (two CTAs per SM)
constexpr int DS = 3;                       // ring slots per warp
constexpr int SLOT_BYTES = DT * DUC / 2;    // 4096
constexpr int RED_FLOATS = 16 * DT;         // one tile's sums: [16 tokens][32 rows]
constexpr int OFF_RING = 0;
constexpr int OFF_BAR = OFF_RING + DW * DS * SLOT_BYTES;
constexpr int OFF_RED = OFF_BAR + DW * DS * 8;
constexpr int OFF_CNT = OFF_RED + DW * 2 * RED_FLOATS * 4;
constexpr int DECODE_SMEM = OFF_CNT + DW * 2 * 4;
constexpr int DECODE_SMEM_ALLOC = DECODE_SMEM + 1024;   // the ring is 1 KB aligned (swizzle atoms)

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// Position of a unit: problem, 32-row tile within it, 256-code k-unit.
struct UnitPos {
  int p;
  int64_t tile;
  int ku;
};

__device__ __forceinline__ void advance(const DecodeArgs &a, UnitPos &u) {
  if (++u.ku == a.prob[u.p].kus) {
    u.ku = 0;
    if (++u.tile == a.prob[u.p].tiles) {
      u.tile = 0;
      ++u.p;
    }
  }
}

__device__ __forceinline__ UnitPos locate(const DecodeArgs &a, int64_t g) {
  int p = 0;
  while (p + 1 < a.n && g >= a.prob[p + 1].unit0) ++p;
  const int64_t rel = g - a.prob[p].unit0;
  UnitPos u;
  u.p = p;
  u.tile = rel / a.prob[p].kus;
  u.ku = static_cast<int>(rel - u.tile * a.prob[p].kus);
  return u;
}

// the tile's global index (counters) and its first unit
__device__ __forceinline__ int64_t tile_gid(const DecodeArgs &a, const UnitPos &u) {
  return a.prob[u.p].tile0 + u.tile;
}
__device__ __forceinline__ int64_t tile_first_unit(const DecodeArgs &a, const UnitPos &u) {
  return a.prob[u.p].unit0 + u.tile * a.prob[u.p].kus;
}

// lane (g, t)'s values of one tile's sums in a [16 tokens][32 rows] float array:
// v[h][b][e] is (row 16 h + g + 8 (e >> 1), token 8 b + 2 t + (e & 1))
template <int NB, typename F>
__device__ __forceinline__ void for_tile_values(int T, int g, int t, F &&f) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = 8 * b + 2 * t + (e & 1), row = 16 * h + g + 8 * (e >> 1);
        if (tok < T) f(h, b, e, tok * DT + row);
      }
}

__device__ __forceinline__ uint32_t ldg_pair_bf16(const uint16_t *p, int64_t i, bool v0, bool v1) {
  const uint32_t lo = v0 ? static_cast<uint32_t>(__ldg(p + i)) : 0u;
  const uint32_t hi = v1 ? static_cast<uint32_t>(__ldg(p + i + 1)) : 0u;
  return lo | (hi << 16);
}

// Finish a tile: v += B U'^T (hi plane, then lo plane of U'), then Y = BF16(v).
template <int NB>
__device__ __forceinline__ void finish_tile(const DecodeArgs &a, const UnitPos &u, int g, int t,
                                            float (&v)[2][NB][4]) {
  grid_dep_wait();   // U' comes from the preceding kernel (returns at once after the first call)
  grid_dep_launch();
  const DecodeProblem &P = a.prob[u.p];
  const int T = a.T;
  const int64_t row0 = u.tile * DT;
  const int rv = P.r;
  const int64_t plane = P.ldu / 2;
  for (int j0 = 0; j0 < rv; j0 += 16) {
    const int ja = j0 + 2 * t, jb = ja + 8;
    // B (as the A operand): rows 16 h + g and 16 h + g + 8, rank slots ja, jb
    uint32_t ar[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int64_t n = row0 + 16 * h + g + 8 * q;
        const bool ok = n < P.N;
        const uint16_t *br = P.B + (ok ? n : 0) * rv;
        ar[h][q] = ldg_pair_bf16(br, ja, ok && ja < rv, ok && ja + 1 < rv);
        ar[h][2 + q] = ldg_pair_bf16(br, jb, ok && jb < rv, ok && jb + 1 < rv);
      }
    // U' (as the B operand): token 8 b + g, rank slots ja, jb, hi then lo plane
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int tok = 8 * b + g;
      uint32_t uh0 = 0u, uh1 = 0u, ul0 = 0u, ul1 = 0u;
      if (tok < T) {
        const uint16_t *ur = P.u + static_cast<int64_t>(tok) * P.ldu;   // planes zero-padded past r
        uh0 = *reinterpret_cast<const uint32_t *>(ur + ja);
        uh1 = *reinterpret_cast<const uint32_t *>(ur + jb);
        ul0 = *reinterpret_cast<const uint32_t *>(ur + plane + ja);
        ul1 = *reinterpret_cast<const uint32_t *>(ur + plane + jb);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mma16816(v[h][b], ar[h][0], ar[h][1], ar[h][2], ar[h][3], uh0, uh1);
        mma16816(v[h][b], ar[h][0], ar[h][1], ar[h][2], ar[h][3], ul0, ul1);
      }
    }
  }
  // c0, c1: row 16 h + g, tokens 2t, 2t + 1; c2, c3: row 16 h + g + 8
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int64_t n = row0 + 16 * h + g + 8 * q;
      if (n >= P.N) continue;
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = 8 * b + 2 * t + e;
          if (tok < T) P.y[static_cast<int64_t>(tok) * P.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v[h][b][2 * q + e]));
        }
    }
}

// The scales of block column kb of rows row0 + 8 j + g (0 past the matrix):
// the E4M3 bytes and the second-level scales, loaded ahead of their use.
struct ScalePre {
  uint32_t f[4];
  float c2[4];
};

__device__ __forceinline__ ScalePre load_scales(const DecodeProblem &P, int64_t row0, int64_t kb, int g) {
  ScalePre sp;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t n = row0 + 8 * j + g;
    const bool ok = kb < P.kb && n < P.N;
    const int64_t blk = ok ? n * P.kb + kb : 0;
    sp.f[j] = ok ? static_cast<uint32_t>(__ldg(P.scales + blk)) : 0u;
    sp.c2[j] = ok ? __ldg(P.c2 + (blk >> 8)) : 0.f;
  }
  return sp;
}

template <bool SYM, bool T16>
__global__ void __launch_bounds__(DW * 32, 2) decode_gemv_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  const uint32_t base = (smem_u32(dsm_raw) + 1023u) & ~1023u;
  uint8_t *gbase = dsm_raw + (base - smem_u32(dsm_raw));
  float *slots = reinterpret_cast<float *>(gbase + OFF_RED);       // [warp][2][RED_FLOATS]
  uint32_t *scnt = reinterpret_cast<uint32_t *>(gbase + OFF_CNT);  // [warp][2]
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const int g = static_cast<int>(lane >> 2), t = static_cast<int>(lane & 3);
  const uint32_t ring = base + OFF_RING + warp * (DS * SLOT_BYTES);
  const uint32_t bars = base + OFF_BAR + warp * (DS * 8);
  const int T = a.T;

  // this CTA's units [ub, ue) and this warp's [wb, we)
  const int64_t U = a.units, C = gridDim.x;
  auto cta_begin = [&](int64_t c) { return c * U / C; };
  const int64_t ub = cta_begin(blockIdx.x), ue = cta_begin(blockIdx.x + 1), n_cta = ue - ub;
  const int64_t weff = min(static_cast<int64_t>(DW), n_cta);
  auto warp_begin = [&](int64_t w) { return ub + w * n_cta / weff; };
  const int64_t wb = warp < weff ? warp_begin(warp) : ue, we = warp < weff ? warp_begin(warp + 1) : ue;
  auto owner_warp = [&](int64_t x) { return ((x - ub + 1) * weff - 1) / n_cta; };
  auto owner_cta = [&](int64_t x) { return ((x + 1) * C - 1) / U; };
  const int cnt = static_cast<int>(we - wb);

  if (threadIdx.x < 2 * DW) scnt[threadIdx.x] = 0u;
  if (lane == 0) {
    for (int s = 0; s < DS; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();

  // ring fills: unit wb + i into slot i % DS (lane 0; one box per unit)
  UnitPos ip = cnt > 0 ? locate(a, wb) : UnitPos{0, 0, 0};
  int inext = 0;
  auto issue = [&]() {
    if (inext < cnt) {
      if (lane == 0) {
        const int s = inext % DS;
        const uint32_t bar = bars + 8 * s;
        mbar_arrive_expect_tx(bar, SLOT_BYTES);
        tma_load_2d(ring + s * SLOT_BYTES, &a.codes_map[ip.p], bar, ip.ku * (DUC / 2),
                    static_cast<int32_t>(ip.tile * DT));
      }
      advance(a, ip);
    }
    ++inext;
  };
  if (lane == 0 && cnt > 0) tma_prefetch_desc(&a.codes_map[ip.p]);
#pragma unroll 1
  for (int s = 0; s < DS; ++s) issue();   // the weights do not depend on the preceding kernel
  UnitPos cur = cnt > 0 ? locate(a, wb) : UnitPos{0, 0, 0};
  // the first unit's scales (static too)
  ScalePre sp = load_scales(a.prob[cur.p], cur.tile * DT, static_cast<int64_t>(cur.ku) * 4 + t, g);
  __syncthreads();                          // the shared counters are zero
  // X, Y and the workspace may depend on earlier kernels.  After a decode U'
  // kernel (which lets this grid start only once everything before it has
  // completed) only U' may still be in flight, and it is read after its own
  // wait in finish_tile; otherwise wait here.
  if (!a.early_start) {
    grid_dep_wait();
    grid_dep_launch();
  }

  constexpr int NB = T16 ? 2 : 1;   // token halves (MMA N = 8 each)
  float cb[16];
  float acc[2][NB][4];
  auto clear_acc = [&]() {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][b][e] = 0.f;
  };
  clear_acc();

  int cb_p = -1;
  bool ok = true;
  int64_t t0 = 0, t1 = 0;   // the current tile's first and end unit
  if (cnt > 0) {
    t0 = tile_first_unit(a, cur);
    t1 = t0 + a.prob[cur.p].kus;
  }
#pragma unroll 1
  for (int i = 0; i < cnt; ++i) {
    const DecodeProblem &P = a.prob[cur.p];
    if (cur.p != cb_p) {
#pragma unroll
      for (int q = 0; q < 16; ++q) cb[q] = P.codebook[q];
      cb_p = cur.p;
    }
    const int64_t kb = static_cast<int64_t>(cur.ku) * 4 + t;      // this lane's block column
    const bool kv = kb < P.kb;
    // X fragments: token g (and g + 8) at the block's 64 k, eight 16-byte chunks.
    // Lanes past the last token read token T - 1 (their output columns are never
    // stored), and a block past K reads block 0 (its W' is exactly zero: its
    // scale is zero), so every load is unconditional.
    uint4 x0[8], x1[8];
    {
      const int64_t kbx = kv ? kb : 0;
      const uint4 *xp = reinterpret_cast<const uint4 *>(P.x + static_cast<int64_t>(min(g, T - 1)) * P.K + kbx * 64);
#pragma unroll
      for (int m = 0; m < 8; ++m) x0[m] = __ldg(xp + m);
      if (T16) {
        const uint4 *xq =
            reinterpret_cast<const uint4 *>(P.x + static_cast<int64_t>(min(g + 8, T - 1)) * P.K + kbx * 64);
#pragma unroll
        for (int m = 0; m < 8; ++m) x1[m] = __ldg(xq + m);
      } else {
#pragma unroll
        for (int m = 0; m < 8; ++m) x1[m] = x0[m];   // unused
      }
    }
    // this unit's block tables from the prefetched scales, then the next unit's scales
    BlockLut<SYM> lut[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) lut[j].make(cb, __fmul_rn(e4m3_to_float(sp.f[j]), sp.c2[j]));
    UnitPos nx = cur;
    advance(a, nx);
    if (i + 1 < cnt) sp = load_scales(a.prob[nx.p], nx.tile * DT, static_cast<int64_t>(nx.ku) * 4 + t, g);
    // the unit's codes: block t of rows g + 8 j (128-byte swizzle: 16-byte chunk c of
    // row r sits at chunk c ^ (r & 7), and r & 7 == g)
    const int s = i % DS;
    const bool landed = mbar_wait(bars + 8 * s, static_cast<uint32_t>((i / DS) & 1), a.status);
    if (!__all_sync(0xffffffffu, landed)) {   // warp-uniform decision
      ok = false;
      break;
    }
    const uint32_t slot = ring + s * SLOT_BYTES;
    uint4 cw[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t ra = slot + (8 * j + g) * 128;
      cw[j][0] = lds128(ra + (((2 * t) ^ g) << 4));
      cw[j][1] = lds128(ra + (((2 * t + 1) ^ g) << 4));
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint4 xa = x0[m], xb = x1[m];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // rows 16 h + g (j = 2 h) and 16 h + g + 8 (j = 2 h + 1)
        uint32_t p[2][4];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 &c = cw[2 * h + q][m >> 2];
          const uint32_t w = (m & 3) == 0 ? c.x : (m & 3) == 1 ? c.y : (m & 3) == 2 ? c.z : c.w;
          lut[2 * h + q].lookup8(w, p[q][0], p[q][1], p[q][2], p[q][3]);
        }
        // codes 8m .. 8m + 3 of the block with x[k .. k + 3], then 8m + 4 .. 8m + 7
        mma16816(acc[h][0], p[0][0], p[1][0], p[0][1], p[1][1], xa.x, xa.y);
        mma16816(acc[h][0], p[0][2], p[1][2], p[0][3], p[1][3], xa.z, xa.w);
        if (T16) {
          mma16816(acc[h][NB - 1], p[0][0], p[1][0], p[0][1], p[1][1], xb.x, xb.y);
          mma16816(acc[h][NB - 1], p[0][2], p[1][2], p[0][3], p[1][3], xb.z, xb.w);
        }
      }
    }
    // every lane has read the slot: refill it with the unit DS ahead
    __syncwarp();
    fence_proxy_async_smem();
    issue();

    const int64_t gi = wb + i;
    if (gi + 1 == t1 || i + 1 == cnt) {
      // the end of this warp's part of the tile
      if (t0 >= wb && t1 <= we) {
        finish_tile<NB>(a, cur, g, t, acc);
      } else {
        float *mine = slots + (warp * 2 + (t0 <= wb ? 0 : 1)) * RED_FLOATS;
        for_tile_values<NB>(T, g, t, [&](int h, int b, int e, int idx) { mine[idx] = acc[h][b][e]; });
        const int64_t wf = owner_warp(max(ub, t0)), wl = owner_warp(min(ue, t1) - 1);
        __threadfence_block();
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atomicAdd(scnt + 2 * wf + (t0 <= warp_begin(wf) ? 0 : 1), 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == static_cast<uint32_t>(wl - wf)) {
          // the CTA's last warp on this tile: its sum over the CTA's warps, in warp order
          __threadfence_block();
          float sum[2][NB][4];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
              for (int e = 0; e < 4; ++e) sum[h][b][e] = 0.f;
          for (int64_t w2 = wf; w2 <= wl; ++w2) {
            const float *src = slots + (w2 * 2 + (t0 <= warp_begin(w2) ? 0 : 1)) * RED_FLOATS;
            for_tile_values<NB>(T, g, t, [&](int h, int b, int e, int idx) { sum[h][b][e] += src[idx]; });
          }
          if (t0 >= ub && t1 <= ue) {
            finish_tile<NB>(a, cur, g, t, sum);
          } else {
            // shared with another CTA: leave the CTA's sum in the workspace
            float *gp = a.part + (static_cast<int64_t>(blockIdx.x) * 2 + (t0 <= ub ? 0 : 1)) * RED_FLOATS;
            for_tile_values<NB>(T, g, t, [&](int h, int b, int e, int idx) { gp[idx] = sum[h][b][e]; });
            __syncwarp();
            uint32_t gold = 0;
            const int64_t tg = tile_gid(a, cur);
            if (lane == 0) {
              asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
                           : "=r"(gold)
                           : "l"(a.counters + tg)
                           : "memory");
            }
            gold = __shfl_sync(0xffffffffu, gold, 0);
            const int64_t cf = owner_cta(t0), cl = owner_cta(t1 - 1);
            if (gold == static_cast<uint32_t>(cl - cf)) {
              // the last CTA on this tile: the CTAs' sums in CTA order
              __syncwarp();
              float tot[2][NB][4];
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                  for (int e = 0; e < 4; ++e) tot[h][b][e] = 0.f;
              for (int64_t c2i = cf; c2i <= cl; ++c2i) {
                const float *src = a.part + (c2i * 2 + (t0 <= cta_begin(c2i) ? 0 : 1)) * RED_FLOATS;
                for_tile_values<NB>(T, g, t, [&](int h, int b, int e, int idx) { tot[h][b][e] += __ldcg(src + idx); });
              }
              finish_tile<NB>(a, cur, g, t, tot);
              if (lane == 0) a.counters[tg] = 0u;   // zero again for the next call
            }
          }
        }
      }
      clear_acc();
      if (i + 1 < cnt) {
        t0 = t1;
        t1 = t0 + a.prob[nx.p].kus;
      }
    }
    cur = nx;
  }
  if (!ok) {
    // a wait ran out: let this warp's copies in flight land before the CTA exits
    for (int k = 0; k < DS; ++k) {
      const int i2 = inext - 1 - k;
      if (i2 < 0 || i2 >= cnt) continue;
      mbar_wait(bars + 8 * (i2 % DS), static_cast<uint32_t>((i2 / DS) & 1), a.status);
    }
  }
  // warps that finished no tile have not waited yet
  grid_dep_wait();
  grid_dep_launch();
}

// ---------------------------------------------------------------------------
// U'_p = s_p X_p A_p^T for every problem, T <= 16, as BF16 hi + lo planes.
// Grid: for each problem, 16 x (plane_p / 16) CTAs in clusters of 16; cluster
// c of problem p owns columns 16c .. 16c + 15 of each of its planes (A rows
// past r arrive as zeros, so the padding columns come out zero) and rank k of
// the cluster the k-th sixteenth of the contraction.  Four warps split the slice, each
// running mma.sync with A = X [tokens][k] and B = A^T; the partial sums meet
// in rank 0's shared memory through distributed shared memory.
// ---------------------------------------------------------------------------
constexpr int kUCluster = 16;   // CTAs per cluster (a non-portable size, opted in at launch)
constexpr int kUThreads = 128;

__device__ __forceinline__ int u_problem(const DecodeUArgs &a, int cluster) {
  int p = 0;
  while (p + 1 < a.n && cluster >= a.prob[p + 1].cluster0) ++p;
  return p;
}

template <bool T16>
__global__ void __launch_bounds__(kUThreads, 1) decode_u_kernel(const __grid_constant__ DecodeUArgs args) {
  extern __shared__ __align__(16) uint8_t usm[];
  constexpr int TT = T16 ? 16 : 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x / kUCluster;
  const int pi = u_problem(args, cluster);
  const DecodeUProblem &p = args.prob[pi];
  const int cg = cluster - p.cluster0;
  const int kc = p.kc;
  const int pitch = kc + 8;                                    // BF16 elements per shared row (conflict-free fragments)
  uint16_t *sa = reinterpret_cast<uint16_t *>(usm);            // [16 j][pitch]
  uint16_t *sx = sa + 16 * pitch;                              // [TT tok][pitch]
  float4 *red = reinterpret_cast<float4 *>(usm + args.red_off);   // [4 warps][2][32]
  const int64_t kbeg = static_cast<int64_t>(rank) * kc;
  const int64_t klen = max(static_cast<int64_t>(0), min(static_cast<int64_t>(kc), p.K - kbeg));
  const int chunks = kc / 8;                                   // 16-byte pieces per row

  // A rows 16 cg .. 16 cg + 15 of this slice (static: requested before the dependency wait)
  for (int c = threadIdx.x; c < 16 * chunks; c += kUThreads) {
    const int j = c / chunks, q = c % chunks;
    const int64_t jr = static_cast<int64_t>(cg) * 16 + j;
    const bool ok = jr < p.r && 8 * q < klen;
    const uint16_t *src = ok ? p.A + jr * p.K + kbeg + 8 * q : p.A;
    const uint32_t d = smem_u32(sa + j * pitch + 8 * q);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(ok ? 16 : 0) : "memory");
  }
  grid_dep_wait();   // X may be written by the preceding kernel, U' read by it
  // every kernel before this one has now completed: the GEMV that follows may
  // start (and read X, the weights and its workspace) while U' is computed
  grid_dep_launch();
  for (int c = threadIdx.x; c < TT * chunks; c += kUThreads) {
    const int tok = c / chunks, q = c % chunks;
    const bool ok = tok < args.T && 8 * q < klen;
    const uint16_t *src = ok ? p.x + static_cast<int64_t>(tok) * p.K + kbeg + 8 * q : p.x;
    const uint32_t d = smem_u32(sx + tok * pitch + 8 * q);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(ok ? 16 : 0) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int steps = kc / 16;
  for (int st = warp; st < steps; st += 4) {
    const int k0 = st * 16;
    auto ld32 = [&](const uint16_t *row, int k) { return *reinterpret_cast<const uint32_t *>(row + k); };
    const uint32_t a0 = ld32(sx + g * pitch, k0 + 2 * t);
    const uint32_t a2 = ld32(sx + g * pitch, k0 + 2 * t + 8);
    const uint32_t a1 = T16 ? ld32(sx + (g + 8) * pitch, k0 + 2 * t) : 0u;
    const uint32_t a3 = T16 ? ld32(sx + (g + 8) * pitch, k0 + 2 * t + 8) : 0u;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const uint16_t *arow = sa + (nt * 8 + g) * pitch;
      mma16816(acc[nt], a0, a1, a2, a3, ld32(arow, k0 + 2 * t), ld32(arow, k0 + 2 * t + 8));
    }
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
    red[(warp * 2 + nt) * 32 + lane] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
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
      // plane, then the lo plane plane columns on
      const int64_t col = static_cast<int64_t>(cg) * 16 + nt * 8 + 2 * t;
      auto put = [&](int tok, float x0, float x1) {
        const __nv_bfloat162 hi = __floats2bfloat162_rn(p.alpha * x0, p.alpha * x1);
        const __nv_bfloat162 lo =
            __floats2bfloat162_rn(p.alpha * x0 - __low2float(hi), p.alpha * x1 - __high2float(hi));
        uint16_t *row = p.u + static_cast<int64_t>(tok) * p.ldu;
        *reinterpret_cast<__nv_bfloat162 *>(row + col) = hi;
        *reinterpret_cast<__nv_bfloat162 *>(row + p.plane + col) = lo;
      };
      if (g < args.T) put(g, v.x, v.y);
      if (T16 && g + 8 < args.T) put(g + 8, v.z, v.w);
    }
  }
  cluster_arrive_wait();   // the peers keep their shared memory until rank 0 has read it
}

}  // namespace

int decode_u_kc(int64_t K) { return static_cast<int>(((K + kUCluster - 1) / kUCluster + 63) / 64 * 64); }

// Clusters of 16 CTAs need an opt-in per kernel and device.
cudaError_t ensure_cluster16_optin(const void *fn) {
  static std::mutex mu;
  static std::pair<const void *, int> done[64];
  static int n_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].first == fn && done[i].second == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  if (n_done < 64) done[n_done++] = {fn, dev};
  return cudaSuccess;
}

int decode_u_smem_bytes(int64_t K_max, int T) {
  const int kc = decode_u_kc(K_max);
  const int tt = T > 8 ? 16 : 8;
  return (16 + tt) * (kc + 8) * 2 + 4 * 2 * 32 * 16;
}

cudaError_t launch_decode_u(const DecodeUArgs &a_in, cudaStream_t st, bool pdl) {
  DecodeUArgs a = a_in;
  if (a.T < 1 || a.T > 16 || a.n < 1 || a.n > kDecodeMaxProblems) return cudaErrorInvalidValue;
  int clusters = 0;
  int64_t kmax = 0;
  for (int i = 0; i < a.n; ++i) {
    DecodeUProblem &p = a.prob[i];
    if (p.r < 1 || p.plane % 16 != 0 || p.plane < p.r || p.ldu < 2 * p.plane || p.ldu % 8 != 0 || p.K % 64 != 0)
      return cudaErrorInvalidValue;
    p.cluster0 = clusters;
    clusters += static_cast<int>(p.plane / 16);
    kmax = std::max<int64_t>(kmax, p.K);
  }
  for (int i = 0; i < a.n; ++i) a.prob[i].kc = decode_u_kc(a.prob[i].K);   // K / 8 per cluster rank
  const int smem = decode_u_smem_bytes(kmax, a.T);                          // sized for the longest
  a.red_off = smem - 4 * 2 * 32 * 16;
  if (smem > kDecodeUMaxSmem) return cudaErrorInvalidValue;
  const bool t16 = a.T > 8;
  const void *fn = t16 ? reinterpret_cast<const void *>(decode_u_kernel<true>)
                       : reinterpret_cast<const void *>(decode_u_kernel<false>);
  cudaError_t e = ensure_smem_optin(fn, kDecodeUMaxSmem);
  if (e != cudaSuccess) return e;
  e = ensure_cluster16_optin(fn);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(kUCluster * clusters), 1, 1);
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
  return t16 ? cudaLaunchKernelEx(&cfg, decode_u_kernel<true>, a) : cudaLaunchKernelEx(&cfg, decode_u_kernel<false>, a);
}

int decode_gemv_ctas(int64_t units, int num_sms) {
  // every resident CTA (two per SM), but no fewer than one unit per warp: the
  // time of a small problem is the latency of one unit
  const int64_t slots = std::min<int64_t>(2 * static_cast<int64_t>(num_sms), kDecodeMaxCtas);
  int64_t c = std::min<int64_t>((units + DW - 1) / DW, slots);
  return static_cast<int>(c < 1 ? 1 : c);
}

size_t decode_gemv_partials_bytes() { return static_cast<size_t>(kDecodeMaxCtas) * 2 * RED_FLOATS * sizeof(float); }

cudaError_t launch_decode_gemv(DecodeArgs &a, int num_sms, cudaStream_t st, bool pdl) {
  if (a.T < 1 || a.T > 16 || a.n < 1 || a.n > kDecodeMaxProblems || !a.part || !a.counters) return cudaErrorInvalidValue;
  int64_t units = 0, tiles = 0;
  bool sym = true;
  for (int i = 0; i < a.n; ++i) {
    DecodeProblem &p = a.prob[i];
    if (p.N % 8 != 0 || p.K % 64 != 0 || p.ldu % 8 != 0 || p.ldu / 2 < ((p.r + 15) / 16) * 16)
      return cudaErrorInvalidValue;
    p.kb = p.K / 64;
    p.kus = static_cast<int>((p.K + DUC - 1) / DUC);
    p.tiles = (p.N + DT - 1) / DT;
    p.unit0 = units;
    p.tile0 = tiles;
    units += p.tiles * p.kus;
    tiles += p.tiles;
    sym = sym && p.sym;
  }
  if (tiles > kDecodeMaxTiles) return cudaErrorInvalidValue;
  a.units = units;
  const int ctas = decode_gemv_ctas(units, num_sms);
  const bool t16 = a.T > 8;
  const void *fn = sym ? (t16 ? reinterpret_cast<const void *>(decode_gemv_kernel<true, true>)
                              : reinterpret_cast<const void *>(decode_gemv_kernel<true, false>))
                       : (t16 ? reinterpret_cast<const void *>(decode_gemv_kernel<false, true>)
                              : reinterpret_cast<const void *>(decode_gemv_kernel<false, false>));
  cudaError_t e = ensure_smem_optin(fn, DECODE_SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  cfg.blockDim = dim3(DW * 32, 1, 1);
  cfg.dynamicSmemBytes = DECODE_SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = pdl ? 1 : 0;
  if (sym) {
    return t16 ? cudaLaunchKernelEx(&cfg, decode_gemv_kernel<true, true>, a)
               : cudaLaunchKernelEx(&cfg, decode_gemv_kernel<true, false>, a);
  }
  return t16 ? cudaLaunchKernelEx(&cfg, decode_gemv_kernel<false, true>, a)
             : cudaLaunchKernelEx(&cfg, decode_gemv_kernel<false, false>, a);
}

}  // namespace qlora
