// gemm_fwd_2sm.cu -- the forward of the fused NF4 layer on CTA pairs, with the
// dequantized weight tile in tensor memory:
//
//   Y[T, N] = X[T, K] W'[N, K]^T + (s X A^T)[T, r] B[N, r]^T
//
// ("QLoRA: Efficient Fine-Tuning", Step 3 eq. 3 and Step 4; W' is "converted to
// BF16 on the fly for each matrix multiplication", "What is QLoRA?".)  The
// rank-r operand s X A^T arrives as two BF16 planes, hi and lo = bf16(v - hi),
// each its own run of 64-wide stages against the same B rows.
//
// A cluster of two CTAs on two SMs owns a 256-weight-row x 256-token tile.  The
// MMA is tcgen05.mma.cta_group::2 with A read from TENSOR memory: each CTA's
// dequantization threads write their 128 weight rows of a 64-wide stage
// straight into that CTA's tensor memory (tcgen05.st, one lane per row), so the
// dequantized weights never touch shared memory; B (128 tokens per CTA) is
// TMA-loaded into shared memory.  Tensor memory (512 columns):
//   columns   0..255  the FP32 accumulator, 128 rows x 256 tokens
//   columns 256..511  eight A stages of 32 columns (64 BF16 per row)
// With one accumulator the epilogue drains it (tcgen05.ld -> BF16 -> a
// swizzled shared-memory tile) before the next tile's first MMA; the MMA pipe
// restarts with the A and B rings already full, and the tile goes to global
// memory by TMA store while the next tile runs.  When the last round of tiles
// would leave most pairs idle, its tiles run as 128-token halves (N = 128).
//
// Warp roles (576 threads per CTA, one CTA per SM, persistent over tiles):
//   warps 0-3   epilogue (warp q reads accumulator lanes 32q..32q+31)
//   warps 4-15  dequantization in three groups of four warps; group g fills the
//               stages it with it % 3 == g, thread t of a group row t of the tile
//   warp 16     TMA loads of this CTA's token half (X, then the sU planes)
//   warp 17     paired tensor-memory allocation; on the even CTA, the MMA issue
// Barriers: full[s] (even CTA) counts both CTAs' TMA bytes and dequantization
// warps; empty[s] and acc_full are signalled in both CTAs by a multicast
// tcgen05.commit; acc_empty (even CTA) counts both CTAs' epilogue warps.  Every
// wait is bounded; after a timeout each role stops issuing work and drains
// what it issued, and both CTAs meet at the final cluster barrier before the
// tensor memory is freed.

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace qlora {

using namespace gemm;

namespace {

constexpr int PM = 128;                        // weight rows per CTA (256 per pair)
constexpr int PN = 256;                        // tokens per tile
constexpr int HN = 128;                        // tokens loaded by each CTA
constexpr int BK = 64;
constexpr int STAGES = 8;
constexpr int B_BYTES = HN * BK * 2;           // 16 KiB
constexpr int A_COLS = BK / 2;                 // tensor-memory columns of one A stage
constexpr int ACC_COLS = PN;
constexpr int TMEM_COLS = 512;
static_assert(ACC_COLS + STAGES * A_COLS == TMEM_COLS, "tensor memory budget");
constexpr int NUM_THREADS = 576;
constexpr int DQ_GROUPS = 3;
constexpr int EPI_COLS = 32;                   // accumulator columns per tcgen05.ld
constexpr int OUT_BOX_BYTES = PN * 128;        // 256 tokens x 64 features, BF16 (stored as two 128-token boxes)
constexpr int EPI_BAR = 1, EPI_ANY_BAR = 2;    // named barriers of the epilogue warps

constexpr int OFF_B = 0;
constexpr int OFF_OUT = OFF_B + STAGES * B_BYTES;
constexpr int OFF_BAR = OFF_OUT + 2 * OUT_BOX_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 3;       // full[S], empty[S], acc_full, acc_empty, drain
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

// full[s]: the leader's TMA producer (arrive.expect_tx for both CTAs' bytes)
// + 2 x 4 dequantization warps
constexpr uint32_t FULL_ARRIVALS = 1 + 8;
constexpr uint32_t ACC_EMPTY_ARRIVALS = 8;     // 2 x 4 epilogue warps

struct Smem {
  uint32_t base;
  __device__ uint32_t b(int s) const { return base + OFF_B + s * B_BYTES; }
  __device__ uint32_t out(int box) const { return base + OFF_OUT + box * OUT_BOX_BYTES; }
  __device__ uint32_t full(int s) const { return base + OFF_BAR + 8 * s; }
  __device__ uint32_t empty(int s) const { return base + OFF_BAR + 8 * (STAGES + s); }
  __device__ uint32_t acc_full() const { return base + OFF_BAR + 8 * (2 * STAGES); }
  __device__ uint32_t acc_empty() const { return base + OFF_BAR + 8 * (2 * STAGES + 1); }
  __device__ uint32_t drain() const { return base + OFF_BAR + 8 * (2 * STAGES + 2); }
  __device__ uint32_t tmem_slot() const { return base + OFF_BAR + 8 * NUM_BARS; }
};

// One block of 64 codes -> 32 BF16x2 words, k order (word j = weights 2j, 2j+1).
template <bool SYM>
__device__ __forceinline__ void dequant_block(const float (&cb)[16], const BlockIn &in, uint32_t (&v)[32]) {
  BlockLut<SYM> lut;
  lut.make(cb, __fmul_rn(e4m3_to_float(in.fbyte), in.c2));
  const uint32_t w[8] = {in.c0.x, in.c0.y, in.c0.z, in.c0.w, in.c1.x, in.c1.y, in.c1.z, in.c1.w};
#pragma unroll
  for (int c = 0; c < 8; ++c) lut.lookup8(w[c], v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// Up to 64 BF16 values of a row (zero-padded past n_valid) -> 32 words.
__device__ __forceinline__ void load_row64(const uint16_t *src, int n_valid, bool aligned16, uint32_t (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int e0 = c * 8;
    if (aligned16 && e0 + 8 <= n_valid) {
      const uint4 q = *reinterpret_cast<const uint4 *>(src + e0);
      v[4 * c] = q.x;
      v[4 * c + 1] = q.y;
      v[4 * c + 2] = q.z;
      v[4 * c + 3] = q.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (e0 + 2 * i < n_valid) ? static_cast<uint32_t>(src[e0 + 2 * i]) : 0u;
        const uint32_t hi = (e0 + 2 * i + 1 < n_valid) ? static_cast<uint32_t>(src[e0 + 2 * i + 1]) : 0u;
        v[4 * c + i] = lo | (hi << 16);
      }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(NUM_THREADS, 1)
    nf4_gemm_fwd_2sm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_lact,
                            const __grid_constant__ CUtensorMap tmap_act_h,
                            const __grid_constant__ CUtensorMap tmap_lact_h, const __grid_constant__ CUtensorMap tmap_out,
                            const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem sm;
  sm.base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0: leader (issues the MMAs), 1: peer
  const bool leader = rank == 0;
  const int ksteps = p.k_main + p.k_lora;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(sm.full(s), FULL_ARRIVALS);
      mbar_init(sm.empty(s), 1);
    }
    mbar_init(sm.acc_full(), 1);
    mbar_init(sm.acc_empty(), ACC_EMPTY_ARRIVALS);
    mbar_init(sm.drain(), 1);
    fence_mbar_init();
  }
  if (warp == 16 && lane == 0) {
    tma_prefetch_desc(&tmap_act);
    tma_prefetch_desc(&tmap_lact);
    if (p.units > p.units_full) {
      tma_prefetch_desc(&tmap_act_h);
      tma_prefetch_desc(&tmap_lact_h);
    }
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmap_out);
  if (warp == 17) {
    tmem_alloc_pair(sm.tmem_slot(), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive_wait();   // the leader's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = ld_shared_u32(sm.tmem_slot());
  const uint32_t tmem_a = tmem_base + ACC_COLS;
  auto lead = [&](uint32_t local_addr) { return mapa_shared(local_addr, 0); };

  if (warp == 17) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (leader && lane == 0) {
      // The issuing thread shares its scheduler and ALU pipe with three
      // dequantization warps, so a stage costs it as few instructions as
      // possible: the ring position, the phase, the stage's barrier and
      // tensor-memory addresses and the low word of its B descriptor are
      // advanced incrementally (the descriptor's address field cannot carry
      // out: shared addresses stay below 256 KiB); slice kk adds kk * 8
      // columns to A and 32 bytes (2 in the field) to B.
      const uint32_t idesc_full = idesc_bf16_f32(2 * PM, PN, false, false);
      const uint32_t idesc_half = idesc_bf16_f32(2 * PM, PN / 2, false, false);
      const uint64_t bdesc0 = smem_desc_sw128(sm.b(0), 16, 1024);
      const uint32_t b_lo0 = static_cast<uint32_t>(bdesc0), b_hi = static_cast<uint32_t>(bdesc0 >> 32);
      // 16-wide K slices of the last rank-r stage of a plane that hold any of
      // the r columns (the slices past them multiply zeros and are skipped)
      const int nk_tail = min(4, (p.r - (p.k_lora_plane - 1) * BK + 15) / 16);
      int s = 0, tc = 0;
      uint32_t ph = 0, ad = tmem_a, b_lo = b_lo0, fb = sm.full(0), eb = sm.empty(0);
      bool ok = true;
      auto advance = [&]() {
        ad += A_COLS;
        b_lo += B_BYTES >> 4;
        fb += 8;
        eb += 8;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
          ad = tmem_a;
          b_lo = b_lo0;
          fb = sm.full(0);
          eb = sm.empty(0);
        }
      };
      for (int u = cluster_id; u < p.units && ok; u += num_clusters, ++tc) {
        const uint32_t idesc = unit_of(p, u).ntok == PN ? idesc_full : idesc_half;
        if (!mbar_wait(sm.acc_empty(), (tc & 1) ^ 1, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < p.k_main; ++ks) {
          if (!mbar_wait(fb, ph, p.status)) { ok = false; break; }
          tc_fence_after();
          tc_mma_ts_pair_lo(tmem_base, ad, b_lo, b_hi, idesc, ks > 0 ? 1u : 0u);
          tc_mma_ts_pair_lo(tmem_base, ad + 8, b_lo + 2, b_hi, idesc, 1u);
          tc_mma_ts_pair_lo(tmem_base, ad + 16, b_lo + 4, b_hi, idesc, 1u);
          tc_mma_ts_pair_lo(tmem_base, ad + 24, b_lo + 6, b_hi, idesc, 1u);
          tc_commit_pair_mc(eb, 0x3);
          advance();
        }
        for (int pl = 0; pl < 2 && ok; ++pl) {
          for (int l = 0; l < p.k_lora_plane; ++l) {
            const int nk = l == p.k_lora_plane - 1 ? nk_tail : 4;
            if (!mbar_wait(fb, ph, p.status)) { ok = false; break; }
            tc_fence_after();
            for (int kk = 0; kk < nk; ++kk)
              tc_mma_ts_pair_lo(tmem_base, ad + kk * 8, b_lo + kk * 2, b_hi, idesc, 1u);
            tc_commit_pair_mc(eb, 0x3);
            advance();
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(sm.acc_full(), 0x3);
      }
      if (!ok) s_abort = 1;
      tc_commit_pair_mc(sm.drain(), 0x1);     // every MMA issued so far has completed
      mbar_wait(sm.drain(), 0, p.status);
    }
    __syncwarp();
  } else if (warp == 16) {
    // ---------------- TMA producer: this CTA's token half ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true, dep_done = false;
      for (int u = cluster_id; u < p.units && ok; u += num_clusters) {
        const Unit w = unit_of(p, u);
        const bool half = w.ntok != PN;              // each CTA loads 64 of 128 tokens
        const int t0 = w.tok0 + static_cast<int>(rank) * (w.ntok / 2);
        const CUtensorMap *m_act = half ? &tmap_act_h : &tmap_act;
        const CUtensorMap *m_lact = half ? &tmap_lact_h : &tmap_lact;
        const uint32_t bytes = 2u * static_cast<uint32_t>(half ? B_BYTES / 2 : B_BYTES);
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (s_abort || !mbar_wait(sm.empty(s), ph ^ 1, p.status)) { ok = false; break; }
          // the leader arms its full barrier for both CTAs' bytes; the peer's
          // load only completes transactions on it
          const uint32_t fb = lead(sm.full(s));
          if (leader) mbar_arrive_expect_tx(sm.full(s), bytes);
          if (ks < p.k_main) {
            tma_load_2d_pair(sm.b(s), m_act, fb, ks * BK, t0);
          } else {
            // the rank-r planes are the preceding kernel's output
            if (!dep_done) {
              grid_dep_wait();
              grid_dep_launch();
              dep_done = true;
            }
            tma_load_2d_pair(sm.b(s), m_lact, fb, (ks - p.k_main) * BK, t0);
          }
        }
      }
      if (!dep_done) {
        grid_dep_wait();
        grid_dep_launch();
      }
      if (!ok) {
        s_abort = 1;
        // loads still in flight land in this CTA's shared memory; give them time to
        // finish (their completion is counted in the leader's barrier, which this
        // CTA cannot wait on)
        const uint64_t t_end = globaltimer() + 2000000ull;
        while (globaltimer() < t_end) {
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- dequantization: three groups, rotating stages ----------------
    const int grp = (warp - 4) >> 2;                 // group g fills stages it % 3 == g
    const int tid = threadIdx.x - 128 - 128 * grp;   // 0..127: the tile row, and its TMEM lane
    float cb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) cb[i] = p.codebook[i];
    const int64_t kblocks = p.K / 64;
    // this warp's lane quadrant (warp % 4 == tid / 32)
    const uint32_t t_lane = tmem_a + (static_cast<uint32_t>(tid & ~31) << 16);
    const bool lora_aligned = (p.r % 8) == 0;
    int it_base = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += num_clusters) {
      const int m_pair = unit_of(p, u).m_pair;
      const int64_t n = static_cast<int64_t>(m_pair) * 2 * PM + static_cast<int64_t>(rank) * PM + tid;
      const bool row_ok = n < p.N;
      auto fetch = [&](int ks) -> BlockIn { return load_block(p, n * kblocks + ks, row_ok && ks < p.k_main); };
      auto produce = [&](int ks, BlockIn &buf) -> bool {
        const int it = it_base + ks;
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (s_abort || !mbar_wait(sm.empty(s), ph ^ 1, p.status)) return false;
        uint32_t v[32];
        if (ks < p.k_main) {
          if (p.sym) dequant_block<true>(cb, buf, v);
          else dequant_block<false>(cb, buf, v);
        } else {
          // rank-r stage: the same B rows for the hi and the lo plane of sU
          const int l = (ks - p.k_main) % p.k_lora_plane;
          const int nv = row_ok ? max(0, min(BK, p.r - l * BK)) : 0;
          load_row64(p.lora + (row_ok ? n : 0) * p.r + l * BK, nv, lora_aligned, v);
        }
        tmem_st_32x32b_x32(t_lane + s * A_COLS, v);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead(sm.full(s)));
        buf = fetch(ks + 2 * DQ_GROUPS);
        return true;
      };
      // this group's stages of the tile: ks0, ks0 + 3, ks0 + 6, ... (two
      // register buffers, each refilled in place six stages ahead)
      const int ks0 = (grp - (it_base % DQ_GROUPS) + DQ_GROUPS) % DQ_GROUPS;
      BlockIn r0 = fetch(ks0), r1 = fetch(ks0 + DQ_GROUPS);
      for (int ks = ks0; ks < ksteps && ok; ks += 2 * DQ_GROUPS) {
        ok = produce(ks, r0);
        if (ok && ks + DQ_GROUPS < ksteps) ok = produce(ks + DQ_GROUPS, r1);
      }
      it_base += ksteps;
    }
    if (!ok) s_abort = 1;
  } else {
    // ---------------- epilogue (warps 0-3) ----------------
    // Lane l of warp q holds feature m = 32q + l of the CTA's 128; features
    // 0-63 go to staging box 0, 64-127 to box 1, each [256 tokens][64
    // features] with the 128-byte swizzle (16-byte chunk c of row t at chunk
    // c ^ (t & 7)).  Lanes 2i and 2i + 1 swap one value so that each writes a
    // BF16 pair of adjacent features: the even lane for token j, the odd lane
    // for token j + 4 (j & 4 == 0); the two rows of one store instruction then
    // fall in complementary halves of the 32 banks.
    const int q = warp;
    const bool odd = (lane & 1) != 0;
    const int fm = 32 * (q & 1) + static_cast<int>(lane & ~1u);   // even feature within the box
    const uint32_t chunk = static_cast<uint32_t>(fm >> 3);
    const uint32_t lane_base =
        sm.out(q >> 1) + (odd ? 4u * 128u : 0u) + static_cast<uint32_t>((fm & 7) >> 1) * 4u;
    uint32_t xo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xo[i] = (chunk ^ static_cast<uint32_t>(i + (odd ? 4 : 0))) << 4;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int tc = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += num_clusters, ++tc) {
      const Unit w = unit_of(p, u);
      const int nch = w.ntok / EPI_COLS;             // accumulator chunks (8, or 4 for a half tile)
      const bool fail = s_abort || !mbar_wait(sm.acc_full(), tc & 1, p.status);
      // the previous tile's TMA store has finished reading the staging tile
      if (threadIdx.x == 0) tma_store_wait_read<0>();
      if (named_bar_any(EPI_ANY_BAR, 128, fail)) { ok = false; break; }
      tc_fence_after();
      uint32_t ra[EPI_COLS], rb[EPI_COLS];
      tmem_ld_32x32b_x32(t_row, ra);
      tc_wait_ld();
      reg_fence(ra);
      auto emit = [&](const uint32_t (&r)[EPI_COLS], int ch) {
        const uint32_t row_base = lane_base + static_cast<uint32_t>(ch * EPI_COLS) * 128u;
#pragma unroll
        for (int j0 = 0; j0 < EPI_COLS; j0 += 8) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = j0 + i;
            const float own_lo = __uint_as_float(r[j]), own_hi = __uint_as_float(r[j + 4]);
            const float recv = __shfl_xor_sync(0xffffffffu, odd ? own_lo : own_hi, 1);
            const uint32_t w = odd ? pack_bf16x2(recv, own_hi) : pack_bf16x2(own_lo, recv);
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(row_base + static_cast<uint32_t>(j) * 128u + xo[i]),
                         "r"(w)
                         : "memory");
          }
        }
      };
#pragma unroll 1
      for (int ch = 0; ch < nch; ch += 2) {
        // the load of the next chunk is in flight while this one is stored
        tmem_ld_32x32b_x32(t_row + (ch + 1) * EPI_COLS, rb);
        emit(ra, ch);
        tc_wait_ld();
        reg_fence(rb);
        if (ch + 2 < nch) {
          tmem_ld_32x32b_x32(t_row + (ch + 2) * EPI_COLS, ra);
        } else {
          // every accumulator column is in registers: release it to the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead(sm.acc_empty()));
        }
        emit(rb, ch + 1);
        if (ch + 2 < nch) {
          tc_wait_ld();
          reg_fence(ra);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(EPI_BAR, 128);
      if (threadIdx.x == 0) {
        // boxes of 128 tokens x 64 features; a 128-token box of the staging
        // tile starts 16 KiB on, a whole number of swizzle atoms
        const int feat0 = w.m_pair * 2 * PM + static_cast<int>(rank) * PM;
        for (int th = 0; th < w.ntok / 128; ++th)
          for (int b = 0; b < 2; ++b)
            tma_store_2d(&tmap_out, sm.out(b) + th * 128 * 128, feat0 + 64 * b, w.tok0 + 128 * th);
        tma_store_commit();
      }
    }
    if (threadIdx.x == 0) tma_store_wait_all<0>();
    if (!ok) s_abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  cluster_arrive_wait();   // both CTAs are done with the pair's tensor memory
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

int gemm_fwd_2sm_smem_bytes() { return SMEM_ALLOC; }

}  // namespace qlora
