// dudb.cu -- the two adapter-gradient products that stream dY, from one read
// of it ("QLoRA: Efficient Fine-Tuning", Step 4 eq. 5, with the forward's sU =
// s X A^T cached):
//
//   dU = s dY B      [T, r]   contraction over the N output features
//   dB = dY^T (sU)   [N, r]   contraction over the T tokens
//
// Each CTA owns a block of dY -- tt 128-token tiles by nn 128-feature chunks --
// and reads each of its 128 x 128 tiles from HBM once.  The tile, staged in
// shared memory by TMA as two 128B-swizzled boxes [128 t][64 n], is the A
// operand of both tcgen05 MMAs: K-major (rows t, contraction n) for dU and
// MN-major (rows n in two 64-feature halves, contraction t) for dB.  All the
// block's accumulators stay in tensor memory for the whole block: dU for each
// token tile (64 columns: B's rows arrive as an MN-major [n][j] operand whose
// columns past r read as zeros), dB for each feature chunk (the hi and lo
// planes of sU, r rounded up to rb = 16, 32 or 64 rows each, stacked into one
// N = 2 rb operand: one MMA per step, the two halves of the accumulator summed
// when it is drained).  The sU planes of the block's tokens are loaded once,
// B's rows of a feature chunk once per chunk (two buffers); the loop runs over
// feature chunks, and over the block's token tiles inside each chunk.
//
// The block's dU rows are partial sums over its features and its dB rows over
// its tokens: both go to the workspace in FP32 -- each chunk's dB rows as soon
// as the chunk is complete, while the next chunk's MMAs run -- and
// dudb_finish_kernel, the next launch, sums them in block order (so the result
// does not depend on timing) and writes dU (hi | lo row planes for the dX GEMM,
// transposed hi and lo planes for dA) and dB.
//
// Launched as a programmatic dependent: the prologue overlaps the previous
// kernel; every global access comes after griddepcontrol.wait, and the finish
// launch is let start at once (it waits for this grid before reading).
//
// Warps: 0 TMA producer, 1 tensor-memory allocation + MMA issue, 2-5 epilogue.

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace qlora {

using namespace gemm;

namespace {

constexpr int DT = 128;                         // tokens per tile (the dU MMA's M)
constexpr int DN = 128;                         // features per chunk (the dB MMA's M)
constexpr int TILE_BYTES = DT * DN * 2;         // 32 KiB: two boxes [128 t][64 n]
constexpr int BOX_BYTES = TILE_BYTES / 2;
constexpr int UB = 64;                          // dU accumulator columns (B's rows, 64 wide)
constexpr int BT_BYTES = DN * UB * 2;           // 16 KiB: two boxes [64 n][64 j]
constexpr int kThreads = 192;
constexpr int kBarBytes = 8 * (2 * kDudbMaxStages + 4 + 2 + kDudbMaxChunks) + 8;
constexpr int kFixed = 2 * BT_BYTES + kBarBytes + 1024;   // + alignment slack for the swizzle atoms
constexpr int kSmemBudget = 220 * 1024;

int su_bytes(int tt, int rb) { return tt * 4 * rb * 128; }   // tt tiles x two 64-token halves x {hi, lo} boxes [rb j][64 t]

__device__ __forceinline__ void st_global_f4(float *p, const float (&v)[4]) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// Columns c0 .. c0 + 15 of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_load16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  tmem_ld_32x32b_x16(taddr, r);
  tc_wait_ld();
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// One row of partial sums (r4 columns, a multiple of 4) from tensor memory to
// the workspace; the loads are warp-collective, the stores only for valid rows.
__device__ __forceinline__ void drain_row(uint32_t taddr, bool have, bool valid, float *dst, int r4) {
#pragma unroll 1
  for (int c0 = 0; c0 < r4; c0 += 16) {
    float v[16];
    if (have) {
      tmem_load16(taddr + static_cast<uint32_t>(c0), v);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.f;
    }
    if (valid) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (c0 + 4 * g < r4) {
          const float w[4] = {v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]};
          st_global_f4(dst + c0 + 4 * g, w);
        }
      }
    }
  }
}

// v += sum over k < n of src[k * stride] (float4), in k order, eight loads in
// flight at a time.
__device__ __forceinline__ void sum_partials(const float *src, int64_t stride, int n, float (&v)[4]) {
  int k = 0;
  for (; k + 8 <= n; k += 8) {
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldcg(reinterpret_cast<const float4 *>(src + (k + u) * stride));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      v[0] += x[u].x;
      v[1] += x[u].y;
      v[2] += x[u].z;
      v[3] += x[u].w;
    }
  }
  for (; k < n; ++k) {
    const float4 x = __ldcg(reinterpret_cast<const float4 *>(src + k * stride));
    v[0] += x.x;
    v[1] += x.y;
    v[2] += x.z;
    v[3] += x.w;
  }
}

// The same for a dB accumulator: columns c and rb + c (the hi and lo planes'
// products) summed.
__device__ __forceinline__ void drain_row_pair(uint32_t taddr, int rb, bool have, bool valid, float *dst, int r4) {
#pragma unroll 1
  for (int c0 = 0; c0 < r4; c0 += 16) {
    float v[16], w[16];
    if (have) {
      tmem_load16(taddr + static_cast<uint32_t>(c0), v);
      tmem_load16(taddr + static_cast<uint32_t>(rb + c0), w);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = w[j] = 0.f;
    }
    if (valid) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (c0 + 4 * g < r4) {
          const float x[4] = {v[4 * g] + w[4 * g], v[4 * g + 1] + w[4 * g + 1], v[4 * g + 2] + w[4 * g + 2],
                              v[4 * g + 3] + w[4 * g + 3]};
          st_global_f4(dst + c0 + 4 * g, x);
        }
      }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    dudb_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_su_hi, const __grid_constant__ CUtensorMap tm_su_lo,
                const DuDbArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int NS = a.stages, TT = a.tt, RB = a.rb;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t su_box = static_cast<uint32_t>(RB) * 128u;   // one [RB j][64 t] box
  const uint32_t su0 = base + static_cast<uint32_t>(NS) * TILE_BYTES;
  const uint32_t bt0 = su0 + static_cast<uint32_t>(TT) * 4u * su_box;
  const uint32_t bar0 = bt0 + 2 * BT_BYTES;
  auto stage = [&](int s) { return base + static_cast<uint32_t>(s) * TILE_BYTES; };
  // token tile i, 64-token half h: the hi box [RB j][64 t], the lo box right after it
  auto su = [&](int i, int h) { return su0 + static_cast<uint32_t>(i * 2 + h) * 2u * su_box; };
  auto btile = [&](int b) { return bt0 + static_cast<uint32_t>(b) * BT_BYTES; };
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kDudbMaxStages + s); };
  auto b_full = [&](int b) { return bar0 + 8u * (2 * kDudbMaxStages + b); };
  auto b_empty = [&](int b) { return bar0 + 8u * (2 * kDudbMaxStages + 2 + b); };
  const uint32_t su_full = bar0 + 8u * (2 * kDudbMaxStages + 4);
  const uint32_t acc_bar = su_full + 8u;
  auto chunk_bar = [&](int c) { return acc_bar + 8u + 8u * c; };
  const uint32_t tmem_slot = acc_bar + 8u + 8u * kDudbMaxChunks;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const int tr = static_cast<int>(blockIdx.x) % a.t_ranges;
  const int nr = static_cast<int>(blockIdx.x) / a.t_ranges;
  const int t_tiles = static_cast<int>((a.T + DT - 1) / DT);
  const int n_chunks = static_cast<int>((a.N + DN - 1) / DN);
  const int tt_n = min(TT, t_tiles - tr * TT);     // >= 1: t_ranges = ceil(t_tiles / tt)
  const int nn_n = min(a.nn, n_chunks - nr * a.nn);
  const int64_t t_base = static_cast<int64_t>(tr) * TT * DT;
  const int64_t n_base = static_cast<int64_t>(nr) * a.nn * DN;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_full(b), 1);
      mbar_init(b_empty(b), 1);
    }
    mbar_init(su_full, 1);
    mbar_init(acc_bar, 1);
    for (int c = 0; c < nn_n; ++c) mbar_init(chunk_bar(c), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, static_cast<uint32_t>(a.tmem_cols));
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_dy);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_su_hi);
    tma_prefetch_desc(&tm_su_lo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_u32(tmem_slot);
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      // the sU planes of the block's tokens, once
      mbar_arrive_expect_tx(su_full, static_cast<uint32_t>(tt_n) * 4u * su_box);
      for (int i = 0; i < tt_n; ++i)
        for (int p = 0; p < 2; ++p)
          for (int h = 0; h < 2; ++h)
            tma_load_2d(su(i, h) + p * su_box, p ? &tm_su_lo : &tm_su_hi, su_full,
                        static_cast<int32_t>(t_base + i * DT + h * 64), 0);                  // [RB j][64 t]
      int issued = 0, b_issued = 0;
      bool ok = true;
      for (int c = 0; c < nn_n && ok; ++c) {
        const int b = c & 1;
        if (s_abort || !mbar_wait(b_empty(b), ((c >> 1) & 1) ^ 1, a.status)) {
          ok = false;
          break;
        }
        const int32_t n0 = static_cast<int32_t>(n_base + c * DN);
        mbar_arrive_expect_tx(b_full(b), BT_BYTES);
        tma_load_2d(btile(b), &tm_b, b_full(b), 0, n0);                                     // [64 n][64 j]
        tma_load_2d(btile(b) + BT_BYTES / 2, &tm_b, b_full(b), 0, n0 + 64);
        b_issued = c + 1;
        for (int i = 0; i < tt_n; ++i) {
          const int st = c * tt_n + i;
          const int s = st % NS;
          const uint32_t ph = (st / NS) & 1;
          if (s_abort || !mbar_wait(empty(s), ph ^ 1, a.status)) {
            ok = false;
            break;
          }
          const int32_t t0 = static_cast<int32_t>(t_base + i * DT);
          mbar_arrive_expect_tx(full(s), TILE_BYTES);
          tma_load_2d(stage(s), &tm_dy, full(s), n0, t0);                                    // [128 t][64 n]
          tma_load_2d(stage(s) + BOX_BYTES, &tm_dy, full(s), n0 + 64, t0);
          issued = st + 1;
        }
      }
      if (!ok) {
        s_abort = 1;
        // every copy in flight lands before the CTA can exit
        for (int st = max(0, issued - NS); st < issued; ++st) mbar_wait(full(st % NS), (st / NS) & 1, a.status);
        for (int c = max(0, b_issued - 2); c < b_issued; ++c) mbar_wait(b_full(c & 1), (c >> 1) & 1, a.status);
        mbar_wait(su_full, 0, a.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      const uint32_t idesc_u = idesc_bf16_f32(DT, UB, false, true);
      const uint32_t idesc_b = idesc_bf16_f32(DN, static_cast<uint32_t>(2 * RB), true, false);
      bool ok = mbar_wait(su_full, 0, a.status);
      int c = 0;
      for (; c < nn_n && ok; ++c) {
        const int b = c & 1;
        if (!mbar_wait(b_full(b), (c >> 1) & 1, a.status)) {
          ok = false;
          break;
        }
        const uint32_t d_b = tmem + static_cast<uint32_t>(TT * UB + c * 2 * RB);
        for (int i = 0; i < tt_n; ++i) {
          const int st = c * tt_n + i;
          const int s = st % NS;
          if (!mbar_wait(full(s), (st / NS) & 1, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_u = tmem + static_cast<uint32_t>(i * UB);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // dU: the tile K-major (16 features a step, box kk / 4), B's rows MN-major
            const uint64_t ad = smem_desc_sw128(stage(s) + (kk >> 2) * BOX_BYTES + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(btile(b) + (kk >> 2) * (BT_BYTES / 2) + (kk & 3) * 2048,
                                                BT_BYTES / 2, 1024);
            tc_mma_ss(d_u, ad, bd, idesc_u, (c > 0 || kk > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // dB: the tile MN-major (features in two 64-wide boxes, 16 tokens a
            // step), the stacked hi | lo sU planes K-major (N = 2 RB)
            const uint64_t ad = smem_desc_sw128(stage(s) + kk * 2048, BOX_BYTES, 1024);
            const uint64_t bd = smem_desc_sw128(su(i, kk >> 2) + (kk & 3) * 32, 16, 1024);
            tc_mma_ss(d_b, ad, bd, idesc_b, (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty(s));
        }
        if (!ok) break;
        tc_commit(b_empty(b));
        tc_commit(chunk_bar(c));
      }
      if (!ok) {
        s_abort = 1;
        // the epilogue does not wait out its limit on chunks that were never computed
        for (; c < nn_n; ++c) tc_commit(chunk_bar(c));
      }
      tc_commit(acc_bar);   // also drains: arrives once everything issued has completed
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: row `row` of each accumulator per thread ----------------
    const int q = warp & 3;   // tensor-memory lane quarter
    const int row = q * 32 + static_cast<int>(lane);
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int r4 = (a.R + 3) & ~3;
    // dB rows of each feature chunk as soon as the chunk is complete
    for (int c = 0; c < nn_n; ++c) {
      const bool okc = mbar_wait(chunk_bar(c), 0, a.status);
      const bool have = __all_sync(0xffffffffu, okc && !s_abort);   // tcgen05.ld is warp-collective
      tc_fence_after();
      const int64_t n = n_base + static_cast<int64_t>(c) * DN + row;
      drain_row_pair(trow + static_cast<uint32_t>(TT * UB + c * 2 * RB), RB, have, n < a.N,
                     a.part_b + (static_cast<int64_t>(tr) * a.N + n) * r4, r4);
    }
    const bool oka = mbar_wait(acc_bar, 0, a.status);
    const bool have = __all_sync(0xffffffffu, oka && !s_abort);
    tc_fence_after();
    for (int i = 0; i < tt_n; ++i) {
      const int64_t t = t_base + static_cast<int64_t>(i) * DT + row;
      drain_row(trow + static_cast<uint32_t>(i * UB), have, t < a.T,
                a.part_u + (static_cast<int64_t>(nr) * a.T + t) * r4, r4);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(a.tmem_cols));
  }
}

// The blocks' partial sums, summed in block order.  Items: for each token t,
// r64 / 4 groups of 4 dU columns (groups past r write the zero padding of the
// row planes); then for each feature n, (r + 3) / 4 groups of 4 dB columns.
// Consecutive threads take consecutive groups of a row, so that the partial
// reads coalesce.
__global__ void __launch_bounds__(256) dudb_finish_kernel(const DuDbArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int r4 = (a.R + 3) & ~3;
  const int gu = static_cast<int>(a.ocols >> 2), gb = r4 >> 2;
  const int64_t nu = a.T * gu, total = nu + a.N * gb;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (i < nu) {
      const int64_t t = i / gu;
      const int c0 = static_cast<int>(i - t * gu) * 4;
      if (c0 < r4) sum_partials(a.part_u + t * r4 + c0, a.T * r4, a.n_ranges, v);
      uint16_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = c0 + e < a.R ? a.s * v[e] : 0.f;
        const __nv_bfloat16 hb = __float2bfloat16_rn(x);
        const __nv_bfloat16 lb = __float2bfloat16_rn(x - __bfloat162float(hb));
        hi[e] = *reinterpret_cast<const uint16_t *>(&hb);
        lo[e] = *reinterpret_cast<const uint16_t *>(&lb);
        if (c0 + e < a.R) {
          a.duT_hi[static_cast<int64_t>(c0 + e) * a.ldt + t] = hi[e];
          a.duT_lo[static_cast<int64_t>(c0 + e) * a.ldt + t] = lo[e];
        }
      }
      *reinterpret_cast<uint2 *>(a.du_hi + t * a.ldo + c0) =
          make_uint2(hi[0] | (static_cast<uint32_t>(hi[1]) << 16), hi[2] | (static_cast<uint32_t>(hi[3]) << 16));
      *reinterpret_cast<uint2 *>(a.du_lo + t * a.ldo + c0) =
          make_uint2(lo[0] | (static_cast<uint32_t>(lo[1]) << 16), lo[2] | (static_cast<uint32_t>(lo[3]) << 16));
    } else {
      const int64_t j = i - nu;
      const int64_t n = j / gb;
      const int c0 = static_cast<int>(j - n * gb) * 4;
      sum_partials(a.part_b + n * r4 + c0, a.N * r4, a.t_ranges, v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (c0 + e < a.R) {
          const __nv_bfloat16 b = __float2bfloat16_rn(v[e]);
          a.dB[n * a.R + c0 + e] = *reinterpret_cast<const uint16_t *>(&b);
        }
      }
    }
  }
}

bool dudb_geom(int64_t T, int64_t N, int r, int num_sms, DuDbGeom &g) {
  if (T <= 0 || N <= 0 || r < 1 || r > kDudbMaxRank || num_sms <= 0) return false;
  const int rb = r <= 16 ? 16 : r <= 32 ? 32 : 64;
  const int64_t t_tiles = (T + DT - 1) / DT, n_chunks = (N + DN - 1) / DN;
  const double r4 = static_cast<double>((r + 3) & ~3);
  bool found = false;
  double best = 0.0;
  for (int tt0 = 1; tt0 <= 8 && tt0 <= t_tiles; ++tt0) {
    const int64_t t_ranges = (t_tiles + tt0 - 1) / tt0;
    const int tt = static_cast<int>((t_tiles + t_ranges - 1) / t_ranges);   // the same ranges, balanced
    int stages = (kSmemBudget - kFixed - su_bytes(tt, rb)) / TILE_BYTES;
    if (stages > kDudbMaxStages) stages = kDudbMaxStages;
    if (stages < 2) continue;
    int64_t nn_max = (512 - tt * UB) / (2 * rb);   // tensor-memory columns
    if (nn_max > kDudbMaxChunks) nn_max = kDudbMaxChunks;
    if (nn_max > n_chunks) nn_max = n_chunks;
    for (int64_t nn0 = 1; nn0 <= nn_max; ++nn0) {
      const int64_t n_ranges = (n_chunks + nn0 - 1) / nn0;
      const int64_t nn = (n_chunks + n_ranges - 1) / n_ranges;   // the same ranges, balanced
      const int64_t waves = (t_ranges * n_ranges + num_sms - 1) / num_sms;
      // the largest block's dY bytes times the waves, plus the partial sums
      // written and read back
      const double cost = static_cast<double>(waves) * tt * nn * TILE_BYTES * num_sms +
                          2.0 * 4.0 * r4 * (static_cast<double>(n_ranges) * T + static_cast<double>(t_ranges) * N);
      if (found && cost >= best) continue;
      found = true;
      best = cost;
      g.tt = tt;
      g.nn = static_cast<int>(nn);
      g.t_ranges = static_cast<int>(t_ranges);
      g.n_ranges = static_cast<int>(n_ranges);
      g.rb = rb;
      g.stages = stages;
      g.smem = stages * TILE_BYTES + su_bytes(tt, rb) + kFixed;
      int cols = 32;
      while (cols < tt * UB + static_cast<int>(nn) * 2 * rb) cols *= 2;
      g.tmem_cols = cols;
    }
  }
  // the partial sums, written and read back, must cost less than the second
  // read of dY that they replace
  return found && static_cast<double>(dudb_partials_bytes(g, T, N, r)) <= static_cast<double>(T) * N;
}

size_t dudb_part_u_bytes(const DuDbGeom &g, int64_t T, int r) {
  const size_t b = static_cast<size_t>(g.n_ranges) * static_cast<size_t>(T) * static_cast<size_t>((r + 3) & ~3) * 4;
  return (b + 255) & ~static_cast<size_t>(255);
}

size_t dudb_partials_bytes(const DuDbGeom &g, int64_t T, int64_t N, int r) {
  return dudb_part_u_bytes(g, T, r) +
         static_cast<size_t>(g.t_ranges) * static_cast<size_t>(N) * static_cast<size_t>((r + 3) & ~3) * 4;
}

cudaError_t launch_dudb(const DuDbArgs &a, const CUtensorMap &tm_dy, const CUtensorMap &tm_b,
                        const CUtensorMap &tm_su_hi, const CUtensorMap &tm_su_lo, cudaStream_t st, bool pdl) {
  if (a.T <= 0 || a.N <= 0 || a.R < 1 || a.R > kDudbMaxRank) return cudaErrorInvalidValue;
  if (a.rb != (a.R <= 16 ? 16 : a.R <= 32 ? 32 : 64)) return cudaErrorInvalidValue;
  if (a.stages < 2 || a.stages > kDudbMaxStages || a.tt < 1 || a.nn < 1 || a.nn > kDudbMaxChunks)
    return cudaErrorInvalidValue;
  if (a.tt * UB + a.nn * 2 * a.rb > a.tmem_cols || a.tmem_cols > 512) return cudaErrorInvalidValue;
  const int64_t t_tiles = (a.T + DT - 1) / DT, n_chunks = (a.N + DN - 1) / DN;
  // every CTA of the grid owns at least one tile and one chunk
  if (a.t_ranges != (t_tiles + a.tt - 1) / a.tt || a.n_ranges != (n_chunks + a.nn - 1) / a.nn)
    return cudaErrorInvalidValue;
  const int smem = a.stages * TILE_BYTES + su_bytes(a.tt, a.rb) + kFixed;
  if (smem > kSmemBudget) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_optin(reinterpret_cast<const void *>(dudb_kernel), kSmemBudget);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.t_ranges * a.n_ranges), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, dudb_kernel, tm_dy, tm_b, tm_su_hi, tm_su_lo, a);
}

cudaError_t launch_dudb_finish(const DuDbArgs &a, cudaStream_t st, bool pdl, int num_sms) {
  if (a.T <= 0 || a.N <= 0 || a.R < 1 || a.R > kDudbMaxRank) return cudaErrorInvalidValue;
  if (a.ocols % 4 != 0 || a.ocols < ((a.R + 3) & ~3) || a.ocols > a.ldo || a.ldo % 4 != 0 || a.ldt < a.T)
    return cudaErrorInvalidValue;
  const int64_t total = a.T * (a.ocols >> 2) + a.N * (((a.R + 3) & ~3) >> 2);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 8 * static_cast<int64_t>(num_sms)) blocks = 8 * static_cast<int64_t>(num_sms);
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, dudb_finish_kernel, a);
}

}  // namespace qlora
