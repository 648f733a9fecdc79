// skinny.cu -- the rank-r GEMMs of the LoRA adapter ("QLoRA: Efficient
// Fine-Tuning", Step 3 eq. 3 and Step 4 eq. 5):
//
//   U  = s X A^T      [T, r]   contraction over K   (P = X  [t][k],  Q = A  [j][k])
//   dU = s dY B       [T, r]   contraction over N   (P = dY [t][n],  Q = B  [n][j])
//   dB = dY^T (sU)    [N, r]   contraction over T   (P = dY [t][n] read as [c][m], Q = sU [t][j])
//   dA = (dU)^T X     [r, K]   contraction over T   (P = X  [t][k] read as [c][m], Q = dU [t][j])
//
// All four are C[M, R] = alpha * sum_c P(m, c) Q(c, j) with R = r <= 128: one
// operand is a large activation read once from HBM, the other is rank r.  They
// run on mma.sync m16n8k16 (BF16 in, FP32 accumulate) with cp.async double
// buffering.  U and dU are stored as two BF16 planes hi = bf16(v), lo =
// bf16(v - hi) so that dB and dA, which sum T products, see them to ~16
// significant bits (Q = hi + lo), while the fused GEMM reads the hi plane.
//
// The contraction may be split across CTAs; each split writes an FP32 partial
// tile and the last CTA to finish a 64-row tile (a per-tile counter in the
// workspace) sums the partials in split order, writes the output and resets
// the counter to zero.

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int SBM = 64;    // rows (m) per CTA
constexpr int SBC = 64;    // contraction per stage
constexpr int ST = 128;    // threads
constexpr int SST = 4;     // cp.async pipeline stages

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <bool PCOL, bool QCJ, bool TWOQ, int RP>
struct Layout {
  // P tile: PCOL ? [c][m] : [m][c], rows of 64 + 8 pad BF16
  static constexpr int P_PITCH = 72;
  static constexpr int P_BYTES = 64 * P_PITCH * 2;
  // Q tile: QCJ ? [c][j] rows of RP + 8 : [j][c] rows of 64 + 8
  static constexpr int Q_PITCH = QCJ ? (RP + 8) : 72;
  static constexpr int Q_ROWS = QCJ ? 64 : RP;
  static constexpr int Q_BYTES = Q_ROWS * Q_PITCH * 2;
  static constexpr int NQ = TWOQ ? 2 : 1;
  static constexpr int STAGE_BYTES = P_BYTES + NQ * Q_BYTES;
  static constexpr int ACC_PITCH = RP + 4;
  static constexpr int ACC_BYTES = SBM * ACC_PITCH * 4;
  static constexpr int SMEM = (SST * STAGE_BYTES > ACC_BYTES ? SST * STAGE_BYTES : ACC_BYTES) + 16;
};

template <bool PCOL, bool QCJ, bool TWOQ, int RP>
__global__ void __launch_bounds__(ST) skinny_kernel(const SkinnyParams p, int out_mode, int q_ncols,
                                                    int q_vec) {
  using L = Layout<PCOL, QCJ, TWOQ, RP>;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_last;
  // a kernel launched after this one with programmatic dependent launch may
  // start now; it waits (griddepcontrol.wait) before reading what we write
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_tile = blockIdx.x;
  const int split = blockIdx.y;
  const int64_t m0 = static_cast<int64_t>(m_tile) * SBM;
  const int64_t cbeg = static_cast<int64_t>(split) * p.c_per_split;
  const int64_t cend = min(p.C, cbeg + p.c_per_split);
  const int nstages = static_cast<int>((cend - cbeg + SBC - 1) / SBC);

  auto load_stage = [&](int buf, int64_t c0) {
    const uint32_t pb = sbase + buf * L::STAGE_BYTES;
    // P tile: 64 rows x 8 chunks of 8 BF16
    for (int idx = tid; idx < 64 * 8; idx += ST) {
      const int row = idx >> 3, ch = idx & 7;
      int64_t m, c;
      if (PCOL) { c = c0 + row; m = m0 + ch * 8; } else { m = m0 + row; c = c0 + ch * 8; }
      bool ok;
      if (PCOL) ok = (c < cend) && (m + 8 <= p.M);
      else ok = (m < p.M) && (c + 8 <= cend);
      const uint16_t *src = p.P + (ok ? (PCOL ? c * p.ldp + m : m * p.ldp + c) : 0);
      cp_async16(pb + (row * L::P_PITCH + ch * 8) * 2, src, ok);
    }
    // Q tile(s)
    for (int qi = 0; qi < L::NQ; ++qi) {
      const uint16_t *Q = qi ? p.Q1 : p.Q0;
      const uint32_t qb = pb + L::P_BYTES + qi * L::Q_BYTES;
      if (QCJ) {
        // rows c, RP/8 chunks along j
        constexpr int CH = RP / 8;
        if (q_vec) {
          for (int idx = tid; idx < 64 * CH; idx += ST) {
            const int row = idx / CH, ch = idx % CH;
            const int64_t c = c0 + row;
            const int j = ch * 8;
            const bool ok = (c < cend) && (j + 8 <= q_ncols);
            cp_async16(qb + (row * L::Q_PITCH + j) * 2, Q + (ok ? c * p.ldq + j : 0), ok);
          }
        } else {
          for (int idx = tid; idx < 64 * RP; idx += ST) {
            const int row = idx / RP, j = idx % RP;
            const int64_t c = c0 + row;
            const uint16_t v = (c < cend && j < q_ncols) ? Q[c * p.ldq + j] : static_cast<uint16_t>(0);
            *reinterpret_cast<uint16_t *>(smem + (qb - sbase) + (row * L::Q_PITCH + j) * 2) = v;
          }
        }
      } else {
        // rows j, 8 chunks along c
        for (int idx = tid; idx < RP * 8; idx += ST) {
          const int j = idx >> 3, ch = idx & 7;
          const int64_t c = c0 + ch * 8;
          const bool ok = (j < q_ncols) && (c + 8 <= cend);
          cp_async16(qb + (j * L::Q_PITCH + ch * 8) * 2, Q + (ok ? static_cast<int64_t>(j) * p.ldq + c : 0), ok);
        }
      }
    }
  };

  constexpr int NT = RP / 8;
  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  // SST-deep cp.async pipeline; one commit group per stage slot (possibly empty)
#pragma unroll
  for (int i = 0; i < SST - 1; ++i) {
    if (i < nstages) load_stage(i, cbeg + static_cast<int64_t>(i) * SBC);
    cp_async_commit();
  }
  for (int st = 0; st < nstages; ++st) {
    const int buf = st % SST;
    {
      const int nxt = st + SST - 1;
      if (nxt < nstages) load_stage(nxt % SST, cbeg + static_cast<int64_t>(nxt) * SBC);
      cp_async_commit();
    }
    cp_async_wait<SST - 1>();
    __syncthreads();
    const uint32_t pb = sbase + buf * L::STAGE_BYTES;
#pragma unroll
    for (int k16 = 0; k16 < 4; ++k16) {
      uint32_t a[4];
      {
        const int i = lane >> 3, r = lane & 7;
        if (PCOL) {
          const int crow = k16 * 16 + r + ((i >> 1) << 3);
          const int mcol = warp * 16 + ((i & 1) << 3);
          ldsm_x4_t(pb + (crow * L::P_PITCH + mcol) * 2, a[0], a[1], a[2], a[3]);
        } else {
          const int mrow = warp * 16 + (lane & 15);
          const int ccol = k16 * 16 + ((lane >> 4) << 3);
          ldsm_x4(pb + (mrow * L::P_PITCH + ccol) * 2, a[0], a[1], a[2], a[3]);
        }
      }
#pragma unroll
      for (int qi = 0; qi < L::NQ; ++qi) {
        const uint32_t qb = pb + L::P_BYTES + qi * L::Q_BYTES;
#pragma unroll
        for (int jp = 0; jp < RP / 16; ++jp) {
          uint32_t b0, b1, b2, b3;
          const int i = lane >> 3, r = lane & 7;
          if (QCJ) {
            const int crow = k16 * 16 + r + ((i & 1) << 3);
            const int jcol = jp * 16 + ((i >> 1) << 3);
            ldsm_x4_t(qb + (crow * L::Q_PITCH + jcol) * 2, b0, b1, b2, b3);
          } else {
            const int jrow = jp * 16 + r + ((i >> 1) << 3);
            const int ccol = k16 * 16 + ((i & 1) << 3);
            ldsm_x4(qb + (jrow * L::Q_PITCH + ccol) * 2, b0, b1, b2, b3);
          }
          mma_bf16(acc[2 * jp], a, b0, b1);
          mma_bf16(acc[2 * jp + 1], a, b2, b3);
        }
      }
    }
    __syncthreads();
  }

  // accumulators -> shared tile [64][RP]
  float *acc_s = reinterpret_cast<float *>(smem);
  {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = warp * 16 + g, col = nt * 8 + 2 * t;
      acc_s[row * L::ACC_PITCH + col] = acc[nt][0];
      acc_s[row * L::ACC_PITCH + col + 1] = acc[nt][1];
      acc_s[(row + 8) * L::ACC_PITCH + col] = acc[nt][2];
      acc_s[(row + 8) * L::ACC_PITCH + col + 1] = acc[nt][3];
    }
  }
  __syncthreads();

  const int rows = static_cast<int>(min(static_cast<int64_t>(SBM), p.M - m0));
  if (p.splits > 1) {
    float *part = p.partials + (static_cast<int64_t>(split) * p.M + m0) * RP;
    for (int idx = tid; idx < rows * RP; idx += ST) {
      const int row = idx / RP, col = idx % RP;
      part[idx] = acc_s[row * L::ACC_PITCH + col];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const uint32_t old = atomicAdd(p.counters + m_tile, 1u);
      s_last = (old == static_cast<uint32_t>(p.splits - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int idx = tid; idx < rows * RP; idx += ST) {
      const int row = idx / RP, col = idx % RP;
      float v = 0.f;
      for (int s = 0; s < p.splits; ++s) {
        v += __ldcg(p.partials + (static_cast<int64_t>(s) * p.M + m0) * RP + idx);
      }
      acc_s[row * L::ACC_PITCH + col] = v;
    }
    if (tid == 0) p.counters[m_tile] = 0u;
    __syncthreads();
  }

  // write-out
  if (out_mode == OUT_HILO) {
    const int ocols = static_cast<int>(p.ocols);
    for (int idx = tid; idx < rows * ocols; idx += ST) {
      const int row = idx / ocols, col = idx % ocols;
      const float v = (col < p.R && col < RP) ? p.alpha * acc_s[row * L::ACC_PITCH + col] : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const int64_t o = (m0 + row) * p.ldo + col;
      p.out0[o] = *reinterpret_cast<const uint16_t *>(&hi);
      if (p.out1) {
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        p.out1[o] = *reinterpret_cast<const uint16_t *>(&lo);
      }
    }
  } else if (out_mode == OUT_ROW) {
    for (int idx = tid; idx < rows * p.R; idx += ST) {
      const int row = idx / p.R, col = idx % p.R;
      const __nv_bfloat16 v = __float2bfloat16_rn(p.alpha * acc_s[row * L::ACC_PITCH + col]);
      p.out0[(m0 + row) * p.R + col] = *reinterpret_cast<const uint16_t *>(&v);
    }
  } else {
    for (int idx = tid; idx < rows * p.R; idx += ST) {
      const int col = idx / rows, row = idx % rows;
      const __nv_bfloat16 v = __float2bfloat16_rn(p.alpha * acc_s[row * L::ACC_PITCH + col]);
      p.out0[static_cast<int64_t>(col) * p.M + m0 + row] = *reinterpret_cast<const uint16_t *>(&v);
    }
  }
}

template <bool PCOL, bool QCJ, bool TWOQ, int RP>
cudaError_t launch_t(const SkinnyParams &p, int out_mode, int q_ncols, int q_vec, cudaStream_t st) {
  using L = Layout<PCOL, QCJ, TWOQ, RP>;
  auto kern = skinny_kernel<PCOL, QCJ, TWOQ, RP>;
  cudaError_t e = ensure_smem_optin(reinterpret_cast<const void *>(kern), L::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t m_tiles = (p.M + SBM - 1) / SBM;
  dim3 grid(static_cast<unsigned>(m_tiles), static_cast<unsigned>(p.splits));
  kern<<<grid, ST, L::SMEM, st>>>(p, out_mode, q_ncols, q_vec);
  return cudaGetLastError();
}

template <bool PCOL, bool QCJ, bool TWOQ>
cudaError_t launch_rp(const SkinnyParams &p, int out_mode, int q_ncols, int q_vec, cudaStream_t st) {
  if (p.R <= 16) return launch_t<PCOL, QCJ, TWOQ, 16>(p, out_mode, q_ncols, q_vec, st);
  if (p.R <= 32) return launch_t<PCOL, QCJ, TWOQ, 32>(p, out_mode, q_ncols, q_vec, st);
  if (p.R <= 64) return launch_t<PCOL, QCJ, TWOQ, 64>(p, out_mode, q_ncols, q_vec, st);
  return launch_t<PCOL, QCJ, TWOQ, 128>(p, out_mode, q_ncols, q_vec, st);
}

}  // namespace

static int rp_of(int R) { return R <= 16 ? 16 : R <= 32 ? 32 : R <= 64 ? 64 : 128; }

int skinny_splits(int64_t M, int64_t C, int num_sms) {
  if (M <= 0 || C <= 0 || num_sms <= 0) return 1;
  const int64_t m_tiles = (M + SBM - 1) / SBM;
  int64_t want = (2 * static_cast<int64_t>(num_sms) + m_tiles - 1) / m_tiles;
  const int64_t cap = (C + 255) / 256;        // at least four stages per split
  int64_t s = want < cap ? want : cap;
  if (s < 1) s = 1;
  // normalise so that every split is non-empty
  int64_t per = (C + s - 1) / s;
  per = (per + SBC - 1) / SBC * SBC;
  s = (C + per - 1) / per;
  return static_cast<int>(s < 1 ? 1 : s);
}

size_t skinny_partials_bytes(int64_t M, int64_t C, int R, int num_sms) {
  const int s = skinny_splits(M, C, num_sms);
  if (s <= 1) return 0;
  return static_cast<size_t>(s) * static_cast<size_t>(M) * static_cast<size_t>(rp_of(R)) * sizeof(float);
}

cudaError_t launch_skinny(const SkinnyParams &p_in, bool p_col, bool q_cj, int out_mode, cudaStream_t st) {
  SkinnyParams p = p_in;
  if (p.M <= 0 || p.R <= 0) return cudaSuccess;
  const bool two = p.Q1 != nullptr;
  // columns of Q that exist in memory: padded planes have ldq >= RP
  const int q_ncols = q_cj ? static_cast<int>(p.ldq >= rp_of(p.R) ? rp_of(p.R) : p.R) : p.R;
  const int q_vec = q_cj ? (((p.ldq % 8) == 0 && (q_ncols % 8) == 0 &&
                             (reinterpret_cast<uintptr_t>(p.Q0) % 16) == 0) ? 1 : 0)
                         : 1;
  if (p_col && q_cj && two) return launch_rp<true, true, true>(p, out_mode, q_ncols, q_vec, st);
  if (!p_col && !q_cj && !two) return launch_rp<false, false, false>(p, out_mode, q_ncols, q_vec, st);
  if (!p_col && q_cj && !two) return launch_rp<false, true, false>(p, out_mode, q_ncols, q_vec, st);
  return cudaErrorInvalidValue;
}

}  // namespace qlora
