// gemm_dx_2sm.cu -- the gradient through the frozen weight, fused NF4
// dequantization + tcgen05 GEMM on CTA pairs (2-SM UMMA, cta_group::2):
//
//   dX[T, K] = dY[T, N] W'[N, K] + (s dY B)[T, r] A[r, K]
//
// ("QLoRA: Efficient Fine-Tuning", Step 4: the backward pass needs the
// gradient with respect to the input through W', which is dequantized on the
// fly as in the forward, "What is QLoRA?".)  The rank-r operand dU = s dY B
// arrives as two BF16 planes, hi and lo = bf16(v - hi), each its own run of
// 64-wide stages against the same A columns.
//
// A cluster of two CTAs on two SMs owns a 256-column (of W, i.e. of dX) x
// 256-token tile.  The contraction runs over the N rows of W, so each CTA's A
// operand is W'^T: its dequantization threads turn 128 64-weight blocks (64
// rows of W x two 64-column blocks) into an MN-major, 128-byte-swizzled
// shared-memory tile; TMA loads this CTA's 128 tokens of dY (then of the dU
// planes) as the B half; the even CTA issues tcgen05.mma.cta_group::2 (M = 256,
// N = 256) accumulating each CTA's 128 columns x 256 tokens in its own tensor
// memory, two accumulators of 256 columns so that the epilogue of one tile
// overlaps the next tile's MMAs.  When the last round of tiles would leave
// most pairs idle, its tiles run as 128-token halves (N = 128).
//
// Warp roles (576 threads per CTA, one CTA per SM, persistent over tiles):
//   warps 0-3   epilogue: tensor memory -> BF16 -> global memory, a pair of columns
//               per 32-bit store (each store instruction writes 64 contiguous bytes
//               for each of two tokens)
//   warps 4-15  dequantization in three groups of four warps; group g fills the
//               pipeline stages it with it % 3 == g
//   warp 16     TMA loads of this CTA's token half (dY, then the dU planes)
//   warp 17     paired tensor-memory allocation; on the even CTA, the MMA issue
// Pipeline barriers: full[s] lives in the even CTA and counts both CTAs' TMA
// bytes (armed by the even CTA) and both CTAs' dequantization warps; empty[s]
// and acc_full are signalled in both CTAs by a multicast tcgen05.commit;
// acc_empty (even CTA) counts both CTAs' epilogue warps.  Every wait is
// bounded; after a timeout each role stops issuing work, drains what it
// issued, and both CTAs meet at the final cluster barrier before the tensor
// memory is freed.

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace qlora {

using namespace gemm;

namespace {

constexpr int PM = 128;                        // columns of W per CTA (256 per pair)
constexpr int PN = 256;                        // tokens per tile
constexpr int HN = 128;                        // tokens loaded by each CTA
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int A_BYTES = PM * BK * 2;           // 16 KiB
constexpr int B_BYTES = HN * BK * 2;           // 16 KiB
constexpr int EPI_ROWS = 32;
constexpr int NUM_THREADS = 576;
constexpr int DQ_GROUPS = 3;
constexpr int TMEM_COLS = 512;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 5;       // full[S], empty[S], acc_full[2], acc_empty[2], drain
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

// full[s]: the leader's TMA producer (arrive.expect_tx for both CTAs' bytes)
// + 2 x 4 dequantization warps
constexpr uint32_t FULL_ARRIVALS = 1 + 8;
// acc_empty: 2 x 4 epilogue warps
constexpr uint32_t ACC_EMPTY_ARRIVALS = 8;

struct Smem {
  uint32_t base;
  __device__ uint32_t a(int s) const { return base + OFF_A + s * A_BYTES; }
  __device__ uint32_t b(int s) const { return base + OFF_B + s * B_BYTES; }
  __device__ uint32_t full(int s) const { return base + OFF_BAR + 8 * s; }
  __device__ uint32_t empty(int s) const { return base + OFF_BAR + 8 * (STAGES + s); }
  __device__ uint32_t acc_full(int i) const { return base + OFF_BAR + 8 * (2 * STAGES + i); }
  __device__ uint32_t acc_empty(int i) const { return base + OFF_BAR + 8 * (2 * STAGES + 2 + i); }
  __device__ uint32_t drain() const { return base + OFF_BAR + 8 * (2 * STAGES + 4); }
  __device__ uint32_t tmem_slot() const { return base + OFF_BAR + 8 * NUM_BARS; }
};

}  // namespace

__global__ void __launch_bounds__(NUM_THREADS, 1)
    nf4_gemm_dx_2sm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_lact,
                           const __grid_constant__ CUtensorMap tmap_act_h,
                           const __grid_constant__ CUtensorMap tmap_lact_h, const GemmParams p) {
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.acc_full(i), 1);
      mbar_init(sm.acc_empty(i), ACC_EMPTY_ARRIVALS);
    }
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
  if (warp == 17) {
    tmem_alloc_pair(sm.tmem_slot(), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_arrive_wait();   // the leader's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = ld_shared_u32(sm.tmem_slot());
  auto lead = [&](uint32_t local_addr) { return mapa_shared(local_addr, 0); };

  if (warp == 17) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (leader && lane == 0) {
      // The issuing thread shares its scheduler and ALU pipe with three
      // dequantization warps, so a stage costs it as few instructions as
      // possible: the ring position, the phase, the stage's barrier addresses
      // and the low words of its descriptors are advanced incrementally (the
      // address fields cannot carry out: shared addresses stay below 256
      // KiB); slice kk adds 4096 bytes to A (MN-major: 16 rows of the
      // contraction) and 32 bytes to B (K-major), i.e. 256 and 2 in the fields.
      const uint32_t idesc_full = idesc_bf16_f32(2 * PM, PN, true, false);
      const uint32_t idesc_half = idesc_bf16_f32(2 * PM, PN / 2, true, false);
      const uint64_t adesc0 = smem_desc_sw128(sm.a(0), 1024, 2048);
      const uint64_t bdesc0 = smem_desc_sw128(sm.b(0), 16, 1024);
      const uint32_t a_lo0 = static_cast<uint32_t>(adesc0), a_hi = static_cast<uint32_t>(adesc0 >> 32);
      const uint32_t b_lo0 = static_cast<uint32_t>(bdesc0), b_hi = static_cast<uint32_t>(bdesc0 >> 32);
      // 16-wide K slices of the last rank-r stage of a plane that hold any of
      // the r rows of A (the slices past them multiply zeros and are skipped)
      const int nk_tail = min(4, (p.r - (p.k_lora_plane - 1) * BK + 15) / 16);
      int s = 0, tc = 0;
      uint32_t ph = 0, a_lo = a_lo0, b_lo = b_lo0, fb = sm.full(0), eb = sm.empty(0);
      bool ok = true;
      auto advance = [&]() {
        a_lo += A_BYTES >> 4;
        b_lo += B_BYTES >> 4;
        fb += 8;
        eb += 8;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
          a_lo = a_lo0;
          b_lo = b_lo0;
          fb = sm.full(0);
          eb = sm.empty(0);
        }
      };
      for (int u = cluster_id; u < p.units && ok; u += num_clusters, ++tc) {
        const uint32_t idesc = unit_of(p, u).ntok == PN ? idesc_full : idesc_half;
        const int acc = tc & 1;
        const uint32_t acc_phase = (tc >> 1) & 1;
        if (!mbar_wait(sm.acc_empty(acc), acc_phase ^ 1, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * PN);
        for (int ks = 0; ks < p.k_main; ++ks) {
          if (!mbar_wait(fb, ph, p.status)) { ok = false; break; }
          tc_fence_after();
          tc_mma_ss_pair_lo(d, a_lo, a_hi, b_lo, b_hi, idesc, ks > 0 ? 1u : 0u);
          tc_mma_ss_pair_lo(d, a_lo + 256, a_hi, b_lo + 2, b_hi, idesc, 1u);
          tc_mma_ss_pair_lo(d, a_lo + 512, a_hi, b_lo + 4, b_hi, idesc, 1u);
          tc_mma_ss_pair_lo(d, a_lo + 768, a_hi, b_lo + 6, b_hi, idesc, 1u);
          tc_commit_pair_mc(eb, 0x3);
          advance();
        }
        for (int pl = 0; pl < 2 && ok; ++pl) {
          for (int l = 0; l < p.k_lora_plane; ++l) {
            const int nk = l == p.k_lora_plane - 1 ? nk_tail : 4;
            if (!mbar_wait(fb, ph, p.status)) { ok = false; break; }
            tc_fence_after();
            for (int kk = 0; kk < nk; ++kk)
              tc_mma_ss_pair_lo(d, a_lo + kk * 256, a_hi, b_lo + kk * 2, b_hi, idesc, 1u);
            tc_commit_pair_mc(eb, 0x3);
            advance();
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(sm.acc_full(acc), 0x3);
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
    // Thread t of a group dequantizes block (row ks * 64 + t % 64 of W, column
    // block t / 64 of the CTA's two) into row t % 64 of the MN-major tile half
    // t / 64: 128-byte rows, 8-row swizzle atoms of 1 KiB, the two halves'
    // atoms interleaved.
    const int grp = (warp - 4) >> 2;                 // group g fills stages it % 3 == g
    const int tid = threadIdx.x - 128 - 128 * grp;   // 0..127
    const int rho = tid & 63, h = tid >> 6;
    float cb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) cb[i] = p.codebook[i];
    const int64_t kblocks = p.K / 64;
    const uint32_t row_off = static_cast<uint32_t>(((rho >> 3) * 2 + h) * 1024 + (rho & 7) * 128);
    const uint32_t phase = static_cast<uint32_t>(rho & 7);
    int it_base = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += num_clusters) {
      const int m_pair = unit_of(p, u).m_pair;
      const int64_t col0 = static_cast<int64_t>(m_pair) * 2 * PM + static_cast<int64_t>(rank) * PM;
      const int64_t kb = col0 / 64 + h;              // this thread's column block of W
      const bool kb_ok = kb < kblocks;
      auto fetch = [&](int ks) -> BlockIn {
        const int64_t n = static_cast<int64_t>(ks) * BK + rho;
        return load_block(p, n * kblocks + kb, ks < p.k_main && n < p.N && kb_ok);
      };
      auto produce = [&](int ks, BlockIn &buf) -> bool {
        const int it = it_base + ks;
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (s_abort || !mbar_wait(sm.empty(s), ph ^ 1, p.status)) return false;
        const uint32_t row_addr = sm.a(s) + row_off;
        if (ks < p.k_main) {
          if (p.sym) dequant_row<true>(cb, buf, row_addr, phase);
          else dequant_row<false>(cb, buf, row_addr, phase);
        } else {
          // rank-r stage: row j of A (64 columns of the CTA's block) for the hi
          // and the lo plane of dU alike
          const int j = ((ks - p.k_main) % p.k_lora_plane) * BK + rho;
          const int64_t k0 = kb * 64;
          const int nv = (j < p.r && kb_ok) ? 64 : 0;
          const uint16_t *src = p.lora + static_cast<int64_t>(j < p.r ? j : 0) * p.K + (kb_ok ? k0 : 0);
          copy_row(src, nv, true, row_addr, phase);
        }
        fence_proxy_async_smem();
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
    const int q = warp;
    int tc = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += num_clusters, ++tc) {
      const Unit w = unit_of(p, u);
      const int acc = tc & 1;
      const uint32_t acc_phase = (tc >> 1) & 1;
      const bool fail = s_abort || !mbar_wait(sm.acc_full(acc), acc_phase, p.status);
      if (named_bar_any(2, 128, fail)) { ok = false; break; }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * PN);
      const int m_local = q * 32 + static_cast<int>(lane);
      const int col_base = w.m_pair * 2 * PM + static_cast<int>(rank) * PM;
      // lanes 2i and 2i + 1 hold columns c and c + 1 (c even); after one exchange
      // the even lane stores both columns of token j, the odd lane those of j + 1
      const int64_t col = static_cast<int64_t>(col_base) + (m_local & ~1);
      const bool odd = (lane & 1) != 0;
      const int nch = w.ntok / EPI_ROWS;             // accumulator chunks (8, or 4 for a half tile)
      for (int ch = 0; ch < nch; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + ch * EPI_ROWS, r);
        tc_wait_ld();
        reg_fence(r);
        if (ch == nch - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead(sm.acc_empty(acc)));
        }
        const int64_t tok0 = static_cast<int64_t>(w.tok0) + ch * EPI_ROWS;
        if (tok0 >= p.T) continue;   // uniform
#pragma unroll
        for (int j = 0; j < EPI_ROWS; j += 2) {
          const float a = __uint_as_float(r[j]), b = __uint_as_float(r[j + 1]);
          const float recv = __shfl_xor_sync(0xffffffffu, odd ? a : b, 1);
          const int64_t tok = tok0 + j + (odd ? 1 : 0);
          // the row stride is a multiple of 8: an even column below it has its pair too
          if (tok < p.T && col < p.K) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(odd ? recv : a, odd ? b : recv);
            *reinterpret_cast<__nv_bfloat162 *>(p.out + tok * p.ldo + col) = v;
          }
        }
      }
    }
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

int gemm_dx_2sm_smem_bytes() { return SMEM_ALLOC; }

}  // namespace qlora
