// skinny_tc.cu -- the rank-r GEMMs of the LoRA adapter on the 5th-generation
// tensor cores ("QLoRA: Efficient Fine-Tuning", Step 3 eq. 3 and Step 4 eq. 5):
//
//   U  = s X A^T      [T, r]   P = X  [t][k] (K-major),            Q = A     [j][k] (K-major)
//   dU = s dY B       [T, r]   P = dY [t][n] (K-major),            Q = B     [n][j] (MN-major)
//   dB = dY^T (sU)    [N, r]   P = dY [t][n] as [c][m] (MN-major), Q = sU^T  [j][t] planes (K-major)
//   dA = dU^T X       [r, K]   P = X  [t][k] as [c][m] (MN-major), Q = dU^T  [j][t] planes (K-major)
//
// C[M, R] = alpha * sum_c P(m, c) Q(c, j): the large operand P streams from HBM
// through a TMA pipeline in 128-row tiles (the MMA's M), the rank-r operand Q
// (R rounded up to NB = 16, 32, 64 or 128 columns, the MMA's N; rows past R
// arrive as zeros) rides along, and the FP32 accumulator sits in tensor
// memory.  U and dU are also written transposed as two BF16 planes hi = bf16(v),
// lo = bf16(v - hi), which dB and dA take as two MMAs into one accumulator.
// The contraction is split across CTAs so that the grid fills the GPU in one
// wave (two CTAs per SM).  With `cluster` set, the splits of a row tile form
// one thread-block cluster (at most 8 CTAs, co-scheduled): each CTA leaves its
// FP32 partial tile in its own shared memory, and after a cluster barrier
// every CTA sums its share of the tile's rows over the cluster's CTAs, in
// split order, through distributed shared memory and writes them out.
// Otherwise each split writes an FP32 partial tile to the workspace and the
// last CTA of a row tile (a workspace counter, reset by that CTA) sums the
// partials in split order and writes the outputs.
//
// Launched as a programmatic dependent: the prologue (barriers, tensor memory,
// descriptor prefetch) overlaps the previous kernel, and every global access
// comes after griddepcontrol.wait -- except in a launch whose inputs all come
// from kernels that had completed before its predecessor let it start
// (dep_late: dU beside dB, the adapter gradients after the dX GEMM), which
// waits only before it exits, so that it runs beside its predecessor, and
// lets its own dependent start at once (that dependent is the next kernel of
// the same layer call, which touches nothing the predecessor writes and reads
// this launch's outputs only after its own wait).
//
// Warps: 0 TMA producer, 1 tensor-memory allocation + MMA issue, 2-5 epilogue.

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace qlora {

using namespace gemm;

namespace {

constexpr int TBM = 128;                 // rows of P per CTA (MMA M)
constexpr int TBK = 64;                  // contraction per stage
constexpr int TMAX_STAGES = 8;
constexpr int P_BYTES = TBM * TBK * 2;   // 16 KiB
constexpr int TNUM_THREADS = 192;
constexpr int kBarBytes = 8 * (2 * TMAX_STAGES + 1) + 8;   // full[], empty[], accumulator, tensor-memory slot
constexpr int kFixedSmem = kBarBytes + 1024;               // + alignment slack for the 1 KiB swizzle atoms
constexpr int kTwoPerSmBudget = 110 * 1024;
// row pitch (floats) of a CTA's partial tile in shared memory in cluster mode:
// 16-byte aligned rows, offset by 4 floats to spread the banks
template <int NB>
constexpr int RED_PITCH = NB + 4;
constexpr int kOnePerSmBudget = 220 * 1024;

// Columns c0 .. c0 + CW - 1 of row m: v[j] is the un-scaled accumulator.
template <int CW>
__device__ __forceinline__ void emit_chunk(const SkinnyTcArgs &a, int64_t m, int c0, const float (&v)[CW]) {
  if (a.row_hi) {
    uint16_t *h = a.row_hi + m * a.ldo + c0;
    uint16_t *l = a.row_lo ? a.row_lo + m * a.ldo + c0 : nullptr;
#pragma unroll
    for (int g = 0; g < CW; g += 8) {
      uint32_t w[4], wl[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float x0 = (c0 + g + e < a.R) ? a.alpha * v[g + e] : 0.f;
        const float x1 = (c0 + g + e + 1 < a.R) ? a.alpha * v[g + e + 1] : 0.f;
        const __nv_bfloat162 hh = __floats2bfloat162_rn(x0, x1);
        w[e / 2] = *reinterpret_cast<const uint32_t *>(&hh);
        const __nv_bfloat162 ll = __floats2bfloat162_rn(x0 - __low2float(hh), x1 - __high2float(hh));
        wl[e / 2] = *reinterpret_cast<const uint32_t *>(&ll);
      }
      *reinterpret_cast<uint4 *>(h + g) = make_uint4(w[0], w[1], w[2], w[3]);
      if (l) *reinterpret_cast<uint4 *>(l + g) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    }
  }
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const int c = c0 + j;
    if (c < a.R) {
      const float x = a.alpha * v[j];
      const __nv_bfloat16 hb = __float2bfloat16_rn(x);
      const uint16_t hu = *reinterpret_cast<const uint16_t *>(&hb);
      if (a.t_hi) {
        a.t_hi[static_cast<int64_t>(c) * a.ldt + m] = hu;
        const __nv_bfloat16 lb = __float2bfloat16_rn(x - __bfloat162float(hb));
        a.t_lo[static_cast<int64_t>(c) * a.ldt + m] = *reinterpret_cast<const uint16_t *>(&lb);
      }
      if (a.row) a.row[m * a.R + c] = hu;
      if (a.tr) a.tr[static_cast<int64_t>(c) * a.M + m] = hu;
    }
  }
}

template <int CW>
__device__ __forceinline__ void tmem_load_chunk(uint32_t taddr, float (&v)[CW]) {
  uint32_t r[CW];
  if constexpr (CW == 16) {
    tmem_ld_32x32b_x16(taddr, r);
  } else {
    tmem_ld_32x32b_x32(taddr, r);
  }
  tc_wait_ld();
#pragma unroll
  for (int j = 0; j < CW; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void st_shared_f4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

}  // namespace

// One CTA of one product: 128-row tile m_tile, contraction split `split`.
template <int NB>
__device__ __forceinline__ void skinny_tc_body(const CUtensorMap *tm_p, const CUtensorMap *tm_q0,
                                               const CUtensorMap *tm_q1, const SkinnyTcArgs &a, int m_tile,
                                               int split) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr int CW = NB < 32 ? NB : 32;                  // epilogue chunk (columns)
  constexpr uint32_t TMEM_COLS = NB < 32 ? 32u : static_cast<uint32_t>(NB);
  constexpr uint32_t Q_BYTES = NB * TBK * 2;
  const int NS = a.stages;
  const uint32_t stage_bytes = P_BYTES + a.nq * Q_BYTES;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bar0 = base + NS * stage_bytes;
  auto stage_p = [&](int s) { return base + s * stage_bytes; };
  auto stage_q = [&](int s, int qi) { return base + s * stage_bytes + P_BYTES + qi * Q_BYTES; };
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (TMAX_STAGES + s); };
  const uint32_t acc_bar = bar0 + 8 * (2 * TMAX_STAGES);
  const uint32_t tmem_slot = acc_bar + 8;
  __shared__ int s_last;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(m_tile) * TBM;
  const int64_t cbeg = static_cast<int64_t>(split) * a.c_per_split;
  const int64_t cend = min(a.C, cbeg + a.c_per_split);
  const int nst = static_cast<int>((cend - cbeg + TBK - 1) / TBK);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(acc_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tm_p);
    tma_prefetch_desc(tm_q0);
    if (a.nq > 1) tma_prefetch_desc(tm_q1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_u32(tmem_slot);
  if (!a.dep_late) grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int st = 0; st < nst; ++st) {
        const int s = st % NS;
        const uint32_t ph = (st / NS) & 1;
        if (s_abort || !mbar_wait(empty(s), ph ^ 1, a.status)) {
          s_abort = 1;
          break;
        }
        const int32_t c0 = static_cast<int32_t>(cbeg + static_cast<int64_t>(st) * TBK);
        mbar_arrive_expect_tx(full(s), stage_bytes);
        if (!a.p_col) {
          tma_load_2d(stage_p(s), tm_p, full(s), c0, static_cast<int32_t>(m0));                      // [128 m][64 c]
        } else {
          tma_load_2d(stage_p(s), tm_p, full(s), static_cast<int32_t>(m0), c0);                      // m 0-63
          tma_load_2d(stage_p(s) + P_BYTES / 2, tm_p, full(s), static_cast<int32_t>(m0) + 64, c0);   // m 64-127
        }
        for (int qi = 0; qi < a.nq; ++qi) {
          const CUtensorMap *tq = qi ? tm_q1 : tm_q0;
          if (!a.q_cj) {
            tma_load_2d(stage_q(s, qi), tq, full(s), c0, 0);                                          // [NB j][64 c]
          } else {
            for (int h = 0; h < NB / 64; ++h)
              tma_load_2d(stage_q(s, qi) + h * (TBK * 128), tq, full(s), h * 64, c0);                 // [64 c][64 j]
          }
        }
        issued = st + 1;
      }
      if (s_abort) {
        for (int st = max(0, issued - NS); st < issued; ++st)
          mbar_wait(full(st % NS), (st / NS) & 1, a.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(TBM, static_cast<uint32_t>(NB), a.p_col != 0, a.q_cj != 0);
      bool ok = true;
      for (int st = 0; st < nst; ++st) {
        const int s = st % NS;
        const uint32_t ph = (st / NS) & 1;
        if (!mbar_wait(full(s), ph, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = !a.p_col ? smem_desc_sw128(stage_p(s) + kk * 32, 16, 1024)
                                       : smem_desc_sw128(stage_p(s) + kk * 2048, P_BYTES / 2, 1024);
          for (int qi = 0; qi < a.nq; ++qi) {
            const uint64_t bd = !a.q_cj ? smem_desc_sw128(stage_q(s, qi) + kk * 32, 16, 1024)
                                        : smem_desc_sw128(stage_q(s, qi) + kk * 2048, TBK * 128, 1024);
            tc_mma_ss(tmem, ad, bd, idesc, (st > 0 || kk > 0 || qi > 0) ? 1u : 0u);
          }
        }
        tc_commit(empty(s));
      }
      if (!ok) s_abort = 1;
      tc_commit(acc_bar);   // also drains: arrives once everything issued has completed
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: row m of the tile per thread ----------------
    const int q = warp & 3;                       // tensor-memory lane quarter
    const int row = q * 32 + static_cast<int>(lane);
    const int64_t m = m0 + row;
    const bool fail = !mbar_wait(acc_bar, 0, a.status) || s_abort;
    // tcgen05.ld is warp-collective: the decision must be uniform within the warp
    const bool have = __all_sync(0xffffffffu, !fail && nst > 0);
    tc_fence_after();
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int pw = (a.R + 3) & ~3;      // partial row width (the R meaningful columns, float4 granular)
    float v[CW];
    if (a.cluster && a.splits > 1) {
      // this CTA's partial rows into its own shared memory (the drained stage
      // ring), read by every CTA of the cluster after the cluster barrier
      const uint32_t red_row = base + static_cast<uint32_t>(row) * static_cast<uint32_t>(RED_PITCH<NB> * 4);
#pragma unroll 1
      for (int c0 = 0; c0 < NB; c0 += CW) {
        if (have) {
          tmem_load_chunk<CW>(trow + c0, v);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int g = 0; g < CW; g += 4)
          st_shared_f4(red_row + static_cast<uint32_t>(c0 + g) * 4u, v[g], v[g + 1], v[g + 2], v[g + 3]);
      }
    } else if (a.splits > 1) {
#pragma unroll 1
      for (int c0 = 0; c0 < NB; c0 += CW) {
        if (have) {
          tmem_load_chunk<CW>(trow + c0, v);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = 0.f;
        }
        if (m < a.M) {
          float4 *dst = reinterpret_cast<float4 *>(a.partials + (static_cast<int64_t>(split) * a.M + m) * pw + c0);
#pragma unroll
          for (int g = 0; g < CW / 4; ++g)
            if (c0 + 4 * g < pw) dst[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
      }
      // the epilogue's partial writes, ordered before one thread's GPU-scope
      // release by the CTA barrier (the release is cumulative)
      named_bar_sync(1, 128);
      if (threadIdx.x == 64) {
        uint32_t old;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.counters + m_tile) : "memory");
        s_last = (old == static_cast<uint32_t>(a.splits - 1)) ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (s_last) {
        // (the acquiring atomic above, then the CTA barrier, order the other
        // splits' partials before these reads)
        if (m < a.M) {
#pragma unroll 1
          for (int c0 = 0; c0 < NB; c0 += CW) {
#pragma unroll
            for (int j = 0; j < CW; ++j) v[j] = 0.f;
            // the splits' partials in groups (64 floats of loads in flight per
            // thread), each group's loads issued together, summed in split order
            constexpr int G = 64 / CW;
            constexpr int NV = CW / 4;
            for (int sp0 = 0; sp0 < a.splits; sp0 += G) {
              float4 t4[G][NV];
#pragma unroll
              for (int gi = 0; gi < G; ++gi) {
                const int sp = sp0 + gi;
                const float4 *src =
                    reinterpret_cast<const float4 *>(a.partials + (static_cast<int64_t>(sp) * a.M + m) * pw + c0);
#pragma unroll
                for (int g = 0; g < NV; ++g)
                  t4[gi][g] = (sp < a.splits && c0 + 4 * g < pw) ? __ldcg(src + g) : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
              for (int gi = 0; gi < G; ++gi) {
#pragma unroll
                for (int g = 0; g < NV; ++g) {
                  v[4 * g] += t4[gi][g].x;
                  v[4 * g + 1] += t4[gi][g].y;
                  v[4 * g + 2] += t4[gi][g].z;
                  v[4 * g + 3] += t4[gi][g].w;
                }
              }
            }
            emit_chunk<CW>(a, m, c0, v);
          }
        }
        if (threadIdx.x == 64) a.counters[m_tile] = 0u;
      }
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < NB; c0 += CW) {
        if (have) {   // warp-uniform
          tmem_load_chunk<CW>(trow + c0, v);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = 0.f;
        }
        if (m < a.M) emit_chunk<CW>(a, m, c0, v);
      }
    }
    // the rest of a padded row of the hi / lo planes (columns NB .. ocols - 1) is zero
    if (a.row_hi && m < a.M && (a.splits == 1 || (s_last && !a.cluster))) {
      for (int64_t c = NB; c < a.ocols; c += 8) {
        *reinterpret_cast<uint4 *>(a.row_hi + m * a.ldo + c) = make_uint4(0u, 0u, 0u, 0u);
        if (a.row_lo) *reinterpret_cast<uint4 *>(a.row_lo + m * a.ldo + c) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }

  if (a.cluster && a.splits > 1) {
    // every CTA of the cluster has its partial rows in shared memory
    cluster_arrive_wait();
    // this CTA's rows: [split * rows_per, +rows_per) of the tile, in 8-column
    // groups (only the groups that hold any of the R columns), consecutive
    // threads on consecutive rows so that the transposed outputs coalesce
    const int rows_per = (TBM + a.splits - 1) / a.splits;
    const int r0 = split * rows_per;
    const int nrows = min(rows_per, TBM - r0);
    const int groups = (a.R + 7) / 8;
    for (int i = static_cast<int>(threadIdx.x); i < nrows * groups; i += TNUM_THREADS) {
      const int rl = r0 + i % nrows, c0 = (i / nrows) * 8;
      const int64_t mg = m0 + rl;
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
      const uint32_t local = base + static_cast<uint32_t>(rl) * static_cast<uint32_t>(RED_PITCH<NB> * 4) +
                             static_cast<uint32_t>(c0) * 4u;
      for (int k = 0; k < a.splits; ++k) {   // split order: the sum does not depend on timing
        const uint32_t remote = mapa_shared(local, static_cast<uint32_t>(k));
        const float4 x0 = ld_dsmem_f4(remote), x1 = ld_dsmem_f4(remote + 16u);
        acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
        acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
      }
      if (mg < a.M) {
        emit_chunk<8>(a, mg, c0, acc);
        // the rest of a padded row of the hi / lo planes is zero
        if (a.row_hi && c0 == 8 * (groups - 1)) {
          for (int64_t c = 8 * groups; c < a.ocols; c += 8) {
            *reinterpret_cast<uint4 *>(a.row_hi + mg * a.ldo + c) = make_uint4(0u, 0u, 0u, 0u);
            if (a.row_lo) *reinterpret_cast<uint4 *>(a.row_lo + mg * a.ldo + c) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
    }
    // no CTA leaves (and frees its shared memory) while another still reads it
    cluster_arrive_wait();
  }
  if (a.dep_late) grid_dep_wait();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int NB>
__global__ void __launch_bounds__(TNUM_THREADS, 2)
    skinny_tc_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q0,
                     const __grid_constant__ CUtensorMap tm_q1, const SkinnyTcArgs a) {
  skinny_tc_body<NB>(&tm_p, &tm_q0, &tm_q1, a, static_cast<int>(blockIdx.x), static_cast<int>(blockIdx.y));
}

// Two independent products in one grid (the first ctas0 CTAs run product 0):
// their ramp-up and split-reduction tails overlap instead of following each other.
template <int NB>
__global__ void __launch_bounds__(TNUM_THREADS, 2)
    skinny_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_p0, const __grid_constant__ CUtensorMap tm_q00,
                          const __grid_constant__ CUtensorMap tm_q10, const __grid_constant__ CUtensorMap tm_p1,
                          const __grid_constant__ CUtensorMap tm_q01, const __grid_constant__ CUtensorMap tm_q11,
                          const SkinnyTcArgs a0, const SkinnyTcArgs a1) {
  const int mt0 = static_cast<int>((a0.M + TBM - 1) / TBM);
  const int n0 = mt0 * a0.splits;
  const int b = static_cast<int>(blockIdx.x);
  if (b < n0) {
    skinny_tc_body<NB>(&tm_p0, &tm_q00, &tm_q10, a0, b % mt0, b / mt0);
  } else {
    const int mt1 = static_cast<int>((a1.M + TBM - 1) / TBM);
    skinny_tc_body<NB>(&tm_p1, &tm_q01, &tm_q11, a1, (b - n0) % mt1, (b - n0) / mt1);
  }
}

// One thread writes 8 consecutive outputs (one 16-byte store); ldd is a
// multiple of 8.
__global__ void pad_cols_kernel(const uint16_t *__restrict__ src, int64_t rows, int cols, uint16_t *__restrict__ dst,
                                int ldd) {
  const int per_row = ldd >> 3;
  const int64_t n = rows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / per_row;
    const int c0 = static_cast<int>(i - r * per_row) << 3;
    const uint16_t *s = src + r * cols;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c0 + 2 * e;
      const uint32_t lo = c < cols ? s[c] : 0u;
      const uint32_t hi = c + 1 < cols ? s[c + 1] : 0u;
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(dst + r * ldd + c0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

namespace {
int tc_nb(int R, bool q_cj) {
  if (q_cj) return R <= 64 ? 64 : 128;
  return R <= 16 ? 16 : R <= 32 ? 32 : R <= 64 ? 64 : 128;
}
// Pipeline depth and CTAs per SM for a tile width; returns the CTAs per SM.
int tc_stages(int nb, int nq, SkinnyTcGeom &g) {
  const int stage = P_BYTES + nq * nb * TBK * 2;
  int per_sm = 2;
  int stages = (kTwoPerSmBudget - kFixedSmem) / stage;
  if (stages < 3) {
    per_sm = 1;
    stages = (kOnePerSmBudget - kFixedSmem) / stage;
  }
  if (stages > TMAX_STAGES) stages = TMAX_STAGES;
  g.nb = nb;
  g.stages = stages;
  g.smem = stages * stage + kFixedSmem;
  g.splits = 1;
  g.c_per_split = TBK;
  return per_sm;
}
// Contraction splits for `slots` CTAs over the 128-row tiles of an M x C product.
void tc_splits(int64_t M, int64_t C, int64_t slots, SkinnyTcGeom &g, int max_splits = 0) {
  if (M <= 0 || C <= 0) return;
  const int64_t m_tiles = (M + TBM - 1) / TBM;
  int64_t s = slots / m_tiles;
  if (max_splits > 0 && s > max_splits) s = max_splits;
  const int64_t cap = (C + 2 * TBK - 1) / (2 * TBK);      // at least two stages per split
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  int64_t per = (C + s - 1) / s;
  per = (per + TBK - 1) / TBK * TBK;
  g.c_per_split = per;
  g.splits = static_cast<int>((C + per - 1) / per);
}
}  // namespace

SkinnyTcGeom skinny_tc_geom(int64_t M, int64_t C, int R, int nq, bool q_cj, int num_sms) {
  SkinnyTcGeom g;
  const int per_sm = tc_stages(tc_nb(R, q_cj), nq, g);
  // one wave: m_tiles x splits <= the CTAs the GPU holds at once
  if (num_sms > 0) tc_splits(M, C, static_cast<int64_t>(per_sm) * num_sms, g, kSkinnyMaxClusterSplits);
  return g;
}

void skinny_tc_pair_geom(int64_t M0, int64_t C0, bool q_cj0, int nq0, int64_t M1, int64_t C1, bool q_cj1, int nq1,
                         int R, int num_sms, SkinnyTcGeom &g0, SkinnyTcGeom &g1, int max_splits) {
  const int nb = tc_nb(R, q_cj0) > tc_nb(R, q_cj1) ? tc_nb(R, q_cj0) : tc_nb(R, q_cj1);
  const int per0 = tc_stages(nb, nq0, g0);
  const int per1 = tc_stages(nb, nq1, g1);
  // the grid is launched with the larger of the two shared-memory footprints
  const int per_sm = per0 < per1 ? per0 : per1;
  if (num_sms <= 0) return;
  // one wave for both, the slots shared in proportion to the bytes each streams
  const int64_t slots = static_cast<int64_t>(per_sm) * num_sms;
  const double b0 = static_cast<double>(M0) * C0, b1 = static_cast<double>(M1) * C1;
  int64_t s0 = b0 + b1 > 0 ? static_cast<int64_t>(slots * b0 / (b0 + b1) + 0.5) : slots / 2;
  if (s0 < 1) s0 = 1;
  if (s0 > slots - 1) s0 = slots - 1;
  tc_splits(M0, C0, s0, g0, max_splits);
  tc_splits(M1, C1, slots - s0, g1, max_splits);
}

void skinny_tc_share_geom(int64_t M0, int64_t C0, bool q_cj0, int nq0, int64_t M1, int64_t C1, bool q_cj1, int nq1,
                          int R, int num_sms, SkinnyTcGeom &g0, SkinnyTcGeom &g1) {
  const int per0 = tc_stages(tc_nb(R, q_cj0), nq0, g0);
  const int per1 = tc_stages(tc_nb(R, q_cj1), nq1, g1);
  if (num_sms <= 0) return;
  const int64_t slots = static_cast<int64_t>(per0 < per1 ? per0 : per1) * num_sms;
  const double b0 = static_cast<double>(M0) * C0, b1 = static_cast<double>(M1) * C1;
  int64_t s0 = b0 + b1 > 0 ? static_cast<int64_t>(slots * b0 / (b0 + b1) + 0.5) : slots / 2;
  if (s0 < 1) s0 = 1;
  if (s0 > slots - 1) s0 = slots - 1;
  tc_splits(M0, C0, s0, g0, kSkinnyMaxClusterSplits);
  tc_splits(M1, C1, slots - s0, g1, kSkinnyMaxClusterSplits);
}

size_t skinny_tc_partials_bytes(const SkinnyTcGeom &g, int64_t M, int R) {
  if (g.splits <= 1 || M <= 0) return 0;
  return static_cast<size_t>(g.splits) * static_cast<size_t>(M) * static_cast<size_t>((R + 3) & ~3) * sizeof(float);
}

namespace {
template <int NB>
cudaError_t launch_nb(const SkinnyTcArgs &a, const CUtensorMap &tm_p, const CUtensorMap &tm_q0,
                      const CUtensorMap &tm_q1, cudaStream_t st, bool pdl) {
  cudaError_t e = ensure_smem_optin(reinterpret_cast<const void *>(skinny_tc_kernel<NB>), kOnePerSmBudget);
  if (e != cudaSuccess) return e;
  const int stage = P_BYTES + a.nq * NB * TBK * 2;
  const bool cluster = a.cluster && a.splits > 1;
  // the partial tile of cluster mode lives in the (drained) stage ring
  if (cluster && (a.splits > kSkinnyMaxClusterSplits || a.stages * stage < TBM * RED_PITCH<NB> * 4))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((a.M + TBM - 1) / TBM), static_cast<unsigned>(a.splits), 1);
  cfg.blockDim = dim3(TNUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(a.stages * stage + kFixedSmem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (cluster) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = static_cast<unsigned>(a.splits);
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, skinny_tc_kernel<NB>, tm_p, tm_q0, tm_q1, a);
}
}  // namespace

cudaError_t launch_skinny_tc(const SkinnyTcArgs &a, const CUtensorMap &tm_p, const CUtensorMap &tm_q0,
                             const CUtensorMap &tm_q1, cudaStream_t st, bool pdl) {
  if (a.M <= 0 || a.C <= 0 || a.R <= 0) return cudaSuccess;
  if (a.stages < 1 || a.stages > TMAX_STAGES || a.splits < 1 || (a.nq != 1 && a.nq != 2))
    return cudaErrorInvalidValue;
  if (a.q_cj && a.nb < 64) return cudaErrorInvalidValue;
  switch (a.nb) {
    case 16: return launch_nb<16>(a, tm_p, tm_q0, tm_q1, st, pdl);
    case 32: return launch_nb<32>(a, tm_p, tm_q0, tm_q1, st, pdl);
    case 64: return launch_nb<64>(a, tm_p, tm_q0, tm_q1, st, pdl);
    case 128: return launch_nb<128>(a, tm_p, tm_q0, tm_q1, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

namespace {
template <int NB>
cudaError_t launch_pair_nb(const SkinnyTcArgs &a0, const CUtensorMap *m0, const SkinnyTcArgs &a1,
                           const CUtensorMap *m1, cudaStream_t st, bool pdl) {
  cudaError_t e = ensure_smem_optin(reinterpret_cast<const void *>(skinny_tc_pair_kernel<NB>), kOnePerSmBudget);
  if (e != cudaSuccess) return e;
  const int smem0 = a0.stages * (P_BYTES + a0.nq * NB * TBK * 2) + kFixedSmem;
  const int smem1 = a1.stages * (P_BYTES + a1.nq * NB * TBK * 2) + kFixedSmem;
  const int64_t n0 = (a0.M + TBM - 1) / TBM * a0.splits, n1 = (a1.M + TBM - 1) / TBM * a1.splits;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n0 + n1), 1, 1);
  cfg.blockDim = dim3(TNUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem0 > smem1 ? smem0 : smem1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, skinny_tc_pair_kernel<NB>, m0[0], m0[1], m0[2], m1[0], m1[1], m1[2], a0, a1);
}
}  // namespace

cudaError_t launch_skinny_tc_pair(const SkinnyTcArgs &a0, const CUtensorMap *maps0, const SkinnyTcArgs &a1,
                                  const CUtensorMap *maps1, cudaStream_t st, bool pdl) {
  if (a0.M <= 0 || a0.C <= 0 || a1.M <= 0 || a1.C <= 0 || a0.R <= 0) return cudaErrorInvalidValue;
  if (a0.cluster || a1.cluster) return cudaErrorInvalidValue;   // one grid of both products: no cluster mode
  if (a0.nb != a1.nb) return cudaErrorInvalidValue;
  for (const SkinnyTcArgs *a : {&a0, &a1})
    if (a->stages < 1 || a->stages > TMAX_STAGES || a->splits < 1 || (a->nq != 1 && a->nq != 2))
      return cudaErrorInvalidValue;
  if ((a0.q_cj || a1.q_cj) && a0.nb < 64) return cudaErrorInvalidValue;
  switch (a0.nb) {
    case 16: return launch_pair_nb<16>(a0, maps0, a1, maps1, st, pdl);
    case 32: return launch_pair_nb<32>(a0, maps0, a1, maps1, st, pdl);
    case 64: return launch_pair_nb<64>(a0, maps0, a1, maps1, st, pdl);
    case 128: return launch_pair_nb<128>(a0, maps0, a1, maps1, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_pad_cols(const uint16_t *src, int64_t rows, int cols, uint16_t *dst, int ldd, cudaStream_t st,
                            int num_sms) {
  if (ldd % 8 != 0 || (reinterpret_cast<uintptr_t>(dst) & 15u)) return cudaErrorInvalidValue;
  const int64_t n = rows * (ldd / 8);
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4 * static_cast<int64_t>(num_sms)) blocks = 4 * static_cast<int64_t>(num_sms);
  if (blocks < 1) blocks = 1;
  pad_cols_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(src, rows, cols, dst, ldd);
  return cudaGetLastError();
}

}  // namespace qlora
