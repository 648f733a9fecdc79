// gemv_nf4.cu -- the forward at decode-sized token counts (T <= 16), bound by
// HBM bandwidth on the 4.127-bit weights ("What is QLoRA?": NF4 converted to
// BF16 on the fly for each matrix multiplication):
//
//   Y[T, N] = X[T, K] W'[N, K]^T + U'[T, r] B[N, r]^T,   U' = BF16(s X A^T)
//
// Each lane dequantizes whole 64-weight blocks straight into mma.sync B
// fragments (no shared-memory staging): lane (g, t) of a warp owns block t of a
// 256-wide k-unit for weight row g of an 8-row group.  The MMA's k-slots are
// permuted consistently for both operands (a sum does not depend on the order
// of its terms): slot 2t+j of k16-step i holds k = 64t + 4i + j and slot
// 2t+8+j holds k = 64t + 4i + 2 + j, so the four codes a lane feeds one MMA
// are four consecutive codes of its block, and the X fragments are eight
// consecutive bytes of one token row.
//
// Work split: a CTA (8 warps) owns 8*RG weight rows and a range of k-units,
// one unit per warp at a time; the CTAs that share a row tile form a thread
// block cluster and their partial sums are added in rank order through
// distributed shared memory by rank 0, which adds the rank-r term and writes
// BF16 Y.  Launched with programmatic dependent launch: the weight stream
// starts while the kernel computing U' still runs; U' is read only after
// griddepcontrol.wait.

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int GW = 8;              // warps per CTA
constexpr int kMaxRank = 128;
constexpr int GT = GW * 32;

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// a block as loaded; its scale is formed at use so that loads never wait
struct Blk {
  uint4 c0, c1;
  uint32_t fbyte;
  float c2;
};

template <int TT, int RG, bool SYM>
__global__ void __launch_bounds__(GT, 2) nf4_gemv_kernel(const GemvParams p) {
  __shared__ float s_red[GW][TT][8 * RG];
  __shared__ float s_part[TT][8 * RG];
  __shared__ __align__(16) uint16_t s_B[8 * RG][kMaxRank + 8];
  __shared__ __align__(16) uint16_t s_U[TT][kMaxRank + 8];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int S = p.splits;
  const int split = static_cast<int>(cluster_rank());
  const int rt = blockIdx.x / S;
  const int64_t row0 = static_cast<int64_t>(rt) * 8 * RG;
  const int64_t kblocks = p.K / 64;

  float cb[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) cb[i] = p.codebook[i];

  float acc[RG][4];
#pragma unroll
  for (int r = 0; r < RG; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;

  auto load_blk = [&](int u, int rg) -> Blk {
    Blk b;
    const int64_t n = row0 + rg * 8 + g;
    const int64_t kb = static_cast<int64_t>(u) * 4 + t;
    if (u < p.units && n < p.N && kb < kblocks) {
      const int64_t blk = n * kblocks + kb;
      const uint8_t *cp = p.codes + blk * 32;
      b.c0 = ldg_stream(cp);
      b.c1 = ldg_stream(cp + 16);
      b.fbyte = __ldg(p.scales + blk);
      b.c2 = __ldg(p.c2 + (blk >> 8));
    } else {
      b.c0 = make_uint4(0, 0, 0, 0);
      b.c1 = b.c0;
      b.fbyte = 0u;
      b.c2 = 0.f;
    }
    return b;
  };

  // Units of this warp: u_j = (split * upw + j) * GW + warp.  The codes of
  // unit j + 1 are requested before unit j is computed (two register sets).
  auto unit_of = [&](int j) { return (split * p.upw + j) * GW + warp; };
  Blk cur[RG], nxt[RG];
  {
    const int u0 = unit_of(0);
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) cur[rg] = load_blk(u0 < p.units ? u0 : p.units, rg);
  }
  for (int j = 0; j < p.upw; ++j) {
    const int u = unit_of(j);
    if (u >= p.units) break;
    const int un = unit_of(j + 1);
    const bool more = (j + 1 < p.upw) && (un < p.units);
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) nxt[rg] = load_blk(more ? un : p.units, rg);
    // X fragments for this unit: token rows g (and g + 8), k = 64t .. 64t + 63
    uint32_t xa[32], xb[TT == 16 ? 32 : 1];
    {
      const int64_t k0 = static_cast<int64_t>(u) * 256 + 64 * t;
      const bool kv = k0 < p.K;
      if (g < p.T && kv) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + static_cast<int64_t>(g) * p.K + k0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = __ldg(src + q);
          xa[4 * q] = v.x; xa[4 * q + 1] = v.y; xa[4 * q + 2] = v.z; xa[4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) xa[q] = 0u;
      }
      if (TT == 16) {
        if (g + 8 < p.T && kv) {
          const uint4 *src = reinterpret_cast<const uint4 *>(p.x + static_cast<int64_t>(g + 8) * p.K + k0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 v = __ldg(src + q);
            xb[4 * q] = v.x; xb[4 * q + 1] = v.y; xb[4 * q + 2] = v.z; xb[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < (TT == 16 ? 32 : 1); ++q) xb[q] = 0u;
        }
      }
    }
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) {
      const float scale = __fmul_rn(e4m3_to_float(cur[rg].fbyte), cur[rg].c2);
      const uint32_t w[8] = {cur[rg].c0.x, cur[rg].c0.y, cur[rg].c0.z, cur[rg].c0.w,
                             cur[rg].c1.x, cur[rg].c1.y, cur[rg].c1.z, cur[rg].c1.w};
      if (SYM) {
        const Lut8 lut = make_lut8(cb, scale);
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const uint32_t mag = mag_index8(w[h]);
          uint32_t b0, b1, b2, b3;
          lut8_lookup4(lut, w[h], mag, b0, b1);
          lut8_lookup4(lut, w[h] >> 16, mag >> 16, b2, b3);
          const int i = 2 * h;
          mma16816(acc[rg], xa[2 * i], (TT == 16) ? xb[2 * i] : 0u, xa[2 * i + 1], (TT == 16) ? xb[2 * i + 1] : 0u,
                   b0, b1);
          mma16816(acc[rg], xa[2 * i + 2], (TT == 16) ? xb[2 * i + 2] : 0u, xa[2 * i + 3],
                   (TT == 16) ? xb[2 * i + 3] : 0u, b2, b3);
        }
      } else {
        const Lut16 lut = make_lut16(cb, scale);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          uint32_t b0, b1;
          lut16_lookup4(lut, (i & 1) ? (w[i >> 1] >> 16) : w[i >> 1], b0, b1);
          const uint32_t a1 = (TT == 16) ? xb[2 * i] : 0u;
          const uint32_t a3 = (TT == 16) ? xb[2 * i + 1] : 0u;
          mma16816(acc[rg], xa[2 * i], a1, xa[2 * i + 1], a3, b0, b1);
        }
      }
    }
#pragma unroll
    for (int rg = 0; rg < RG; ++rg) cur[rg] = nxt[rg];
  }

  // accumulator fragment: c0/c1 = (token g, rows 2t, 2t+1), c2/c3 = (token g+8, ...)
#pragma unroll
  for (int rg = 0; rg < RG; ++rg) {
    const int r0 = rg * 8 + 2 * t;
    if (g < TT) {
      s_red[warp][g][r0] = acc[rg][0];
      s_red[warp][g][r0 + 1] = acc[rg][1];
    }
    if (TT == 16) {
      s_red[warp][(g + 8) % TT][r0] = acc[rg][2];
      s_red[warp][(g + 8) % TT][r0 + 1] = acc[rg][3];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < TT * 8 * RG; idx += GT) {
    const int tok = idx / (8 * RG), row = idx % (8 * RG);
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < GW; ++w) v += s_red[w][tok][row];
    s_part[tok][row] = v;
  }
  if (S > 1) cluster_sync();
  else __syncthreads();

  if (split == 0) {
    // rank-r term sum_j U'[tok, j] B[n, j] from shared memory: this CTA's rows of
    // B (independent of the preceding kernel) first, U' after the dependency wait
    const int nrows = static_cast<int>(min(static_cast<int64_t>(8 * RG), p.N - row0));
    const int rv = p.r;
    const uint16_t *bsrc = p.B + row0 * rv;
    const int nb = nrows * rv;
    if ((rv % 8) == 0) {
      for (int c = threadIdx.x; c < nb / 8; c += GT) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(bsrc) + c);
        const int e = c * 8, row = e / rv, j = e % rv;
        *reinterpret_cast<uint4 *>(&s_B[row][j]) = v;
      }
    } else {
      for (int e = threadIdx.x; e < nb; e += GT) s_B[e / rv][e % rv] = bsrc[e];
    }
    grid_dep_wait();   // U' is written by the preceding kernel
    const int ucols = static_cast<int>((rv + 7) / 8 * 8);      // the U' plane is zero-padded to ldu >= this
    for (int c = threadIdx.x; c < p.T * (ucols / 8); c += GT) {
      const int tok = c / (ucols / 8), j = (c % (ucols / 8)) * 8;
      *reinterpret_cast<uint4 *>(&s_U[tok][j]) =
          __ldg(reinterpret_cast<const uint4 *>(p.u + static_cast<int64_t>(tok) * p.ldu + j));
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < TT * 8 * RG; idx += GT) {
      const int tok = idx / (8 * RG), row = idx % (8 * RG);
      const int64_t n = row0 + row;
      if (tok >= p.T || row >= nrows) continue;
      float v = 0.f;
      for (int r = 0; r < S; ++r) v += (r == 0) ? s_part[tok][row] : ld_dsmem_f32(&s_part[tok][row], r);
      float l = 0.f;
      for (int jj = 0; jj < rv; ++jj) {
        l = fmaf(__uint_as_float(static_cast<uint32_t>(s_U[tok][jj]) << 16),
                 __uint_as_float(static_cast<uint32_t>(s_B[row][jj]) << 16), l);
      }
      const __nv_bfloat16 o = __float2bfloat16_rn(v + l);
      p.y[static_cast<int64_t>(tok) * p.N + n] = *reinterpret_cast<const uint16_t *>(&o);
    }
  }
  if (S > 1) cluster_sync();   // peers keep their shared memory alive until rank 0 has read it
}

template <int TT, int RG, bool SYM>
cudaError_t launch_tr(const GemvParams &p, int row_tiles, cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(row_tiles * p.splits), 1, 1);
  cfg.blockDim = dim3(GT, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = static_cast<unsigned>(p.splits);
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, nf4_gemv_kernel<TT, RG, SYM>, p);
}

}  // namespace

GemvPlan gemv_plan(int64_t N, int64_t K, int num_sms) {
  GemvPlan pl;
  pl.units = static_cast<int>((K + 255) / 256);
  // 16-row tiles (8-row tiles for small N); split k over a cluster only when the
  // row tiles alone cannot give every SM two CTAs
  pl.rg = 2;
  int64_t tiles = (N + 15) / 16;
  if (tiles < 2 * static_cast<int64_t>(num_sms)) {
    pl.rg = 1;
    tiles = (N + 7) / 8;
  }
  int splits = 1;
  while (splits < 8 && tiles * splits < 2 * static_cast<int64_t>(num_sms) &&
         pl.units >= GW * (splits + 1)) {
    ++splits;
  }
  // every split gets whole rounds of GW units; at most 8 CTAs per cluster
  pl.upw = (pl.units + GW * splits - 1) / (GW * splits);
  pl.splits = (pl.units + GW * pl.upw - 1) / (GW * pl.upw);
  pl.row_tiles = static_cast<int>(tiles);
  return pl;
}

cudaError_t launch_gemv(const GemvParams &p_in, const GemvPlan &pl, cudaStream_t st, bool pdl) {
  GemvParams p = p_in;
  p.units = pl.units;
  p.upw = pl.upw;
  p.splits = pl.splits;
  const bool t16 = p.T > 8;
  if (p.sym) {
    if (pl.rg == 2) return t16 ? launch_tr<16, 2, true>(p, pl.row_tiles, st, pdl) : launch_tr<8, 2, true>(p, pl.row_tiles, st, pdl);
    return t16 ? launch_tr<16, 1, true>(p, pl.row_tiles, st, pdl) : launch_tr<8, 1, true>(p, pl.row_tiles, st, pdl);
  }
  if (pl.rg == 2) return t16 ? launch_tr<16, 2, false>(p, pl.row_tiles, st, pdl) : launch_tr<8, 2, false>(p, pl.row_tiles, st, pdl);
  return t16 ? launch_tr<16, 1, false>(p, pl.row_tiles, st, pdl) : launch_tr<8, 1, false>(p, pl.row_tiles, st, pdl);
}

}  // namespace qlora
