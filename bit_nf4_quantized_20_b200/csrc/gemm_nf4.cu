// gemm_nf4.cu -- fused NF4 dequantization + tcgen05 GEMM for the QLoRA linear
// layer, forward and backward-dX.
//
// Forward ("QLoRA: Efficient Fine-Tuning", Step 3, eq. 3, with the PEFT
// alpha/r scaling):   Y[T, N] = X[T, K] W'[N, K]^T + (s X A^T)[T, r] B[N, r]^T
// Backward dX (gradient through the frozen weight, Step 4):
//                     dX[T, K] = dY[T, N] W'[N, K] + (s dY B)[T, r] A[r, K]
// W' = BF16(RN32(codebook[code] * RN32(fp8(scale) * c2))) is produced in shared
// memory by dequantization warps and never written to global memory ("converted
// to BF16 on the fly for each matrix multiplication", "What is QLoRA?").
//
// Tiling: the weight side is the MMA's M operand (128 weight rows: output
// features in the forward, input features in the backward), the tokens are the
// N operand (256 per tile); the accumulator tile (features x tokens) lives in
// tensor memory, double-buffered (2 x 256 columns), and the epilogue transposes
// it through shared memory into row-major Y / dX with TMA stores.
//
// Warp roles (320 threads, one CTA per SM, persistent over tiles):
//   warps 0-3  epilogue (tensor-memory lane quarters 0-3)
//   warps 4-7  A producers: dequantize one 64-weight block per thread per stage
//              into a 128-byte-swizzled BF16 tile (K-major forward, MN-major
//              backward), or copy the LoRA matrix for the extra rank-r stages
//   warp 8     B producer: TMA loads of X / dY (and of the s*U / dU operand)
//   warp 9     tensor-memory allocation + single-thread tcgen05.mma issue
// Every mbarrier wait is bounded; on a timeout the CTA records the status bit,
// stops issuing work, drains what it issued and frees tensor memory.

#include "common.cuh"
#include "gemm_common.cuh"
#include "kernels.h"

namespace qlora {

using namespace gemm;

namespace {

constexpr int BM = 128;           // weight rows per tile (MMA M)
constexpr int BN = 256;           // tokens per tile (MMA N)
constexpr int BK = 64;            // contraction per pipeline stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KiB
constexpr int B_BYTES = BN * BK * 2;          // 32 KiB
constexpr int EPI_ROWS = 32;                  // tokens per epilogue store
constexpr int EPI_BYTES = EPI_ROWS * BM * 2;  // 8 KiB
constexpr int NUM_THREADS = 320;
constexpr int TMEM_COLS = 512;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_EPI = OFF_B + STAGES * B_BYTES;
constexpr int OFF_BAR = OFF_EPI + 2 * EPI_BYTES;
// barriers: fullA[S], fullB[S], empty[S], accFull[2], accEmpty[2], drain, tmem slot
constexpr int NUM_BARS = 3 * STAGES + 5;
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment

struct Smem {
  uint32_t base;  // 1024-aligned shared address
  __device__ uint32_t a(int s) const { return base + OFF_A + s * A_BYTES; }
  __device__ uint32_t b(int s) const { return base + OFF_B + s * B_BYTES; }
  __device__ uint32_t epi(int i) const { return base + OFF_EPI + i * EPI_BYTES; }
  __device__ uint32_t full_a(int s) const { return base + OFF_BAR + 8 * s; }
  __device__ uint32_t full_b(int s) const { return base + OFF_BAR + 8 * (STAGES + s); }
  __device__ uint32_t empty(int s) const { return base + OFF_BAR + 8 * (2 * STAGES + s); }
  __device__ uint32_t acc_full(int i) const { return base + OFF_BAR + 8 * (3 * STAGES + i); }
  __device__ uint32_t acc_empty(int i) const { return base + OFF_BAR + 8 * (3 * STAGES + 2 + i); }
  __device__ uint32_t drain() const { return base + OFF_BAR + 8 * (3 * STAGES + 4); }
  __device__ uint32_t tmem_slot() const { return base + OFF_BAR + 8 * NUM_BARS; }
};

}  // namespace

__global__ void __launch_bounds__(NUM_THREADS, 1)
    nf4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_lact,
                    const __grid_constant__ CUtensorMap tmap_out, const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem sm;
  sm.base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const bool bwd = p.mode != 0;
  const int ksteps = p.k_main + p.k_lora;
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(sm.full_a(s), 128);
      mbar_init(sm.full_b(s), 1);
      mbar_init(sm.empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.acc_full(i), 1);
      mbar_init(sm.acc_empty(i), 4);
    }
    mbar_init(sm.drain(), 1);
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmap_act);
    tma_prefetch_desc(&tmap_lact);
    tma_prefetch_desc(&tmap_out);
  }
  if (warp == 9) {
    tmem_alloc(sm.tmem_slot(), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ld_shared_u32(sm.tmem_slot());

  if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, bwd, false);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tc) {
        const int acc = tc & 1;
        const uint32_t acc_phase = (tc >> 1) & 1;
        if (!mbar_wait(sm.acc_empty(acc), acc_phase ^ 1, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(sm.full_a(s), ph, p.status) || !mbar_wait(sm.full_b(s), ph, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          int nk = 4;
          if (ks >= p.k_main) {
            const int rem = p.r - (ks - p.k_main) * BK;
            nk = min(4, (rem + 15) / 16);
          }
          for (int kk = 0; kk < nk; ++kk) {
            uint64_t adesc;
            if (!bwd) {
              adesc = smem_desc_sw128(sm.a(s) + kk * 32, 16, 1024);       // K-major
            } else {
              adesc = smem_desc_sw128(sm.a(s) + kk * 4096, 1024, 2048);   // MN-major
            }
            const uint64_t bdesc = smem_desc_sw128(sm.b(s) + kk * 32, 16, 1024);
            tc_mma_ss(d_tmem, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(sm.empty(s));
        }
        if (!ok) break;
        tc_commit(sm.acc_full(acc));
      }
      if (!ok) atomicExch(const_cast<int *>(&s_abort), 1);
      // drain: wait until every MMA this thread issued has completed
      tc_commit(sm.drain());
      mbar_wait(sm.drain(), 0, p.status);
    }
    __syncwarp();
  } else if (warp == 8) {
    // ---------------- B producer (TMA) ----------------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int n_tile = tile / p.m_tiles;
        const int t0 = n_tile * BN;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (s_abort || !mbar_wait(sm.empty(s), ph ^ 1, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(sm.full_b(s), B_BYTES);
          if (ks < p.k_main) {
            tma_load_2d(sm.b(s), &tmap_act, sm.full_b(s), ks * BK, t0);
          } else {
            tma_load_2d(sm.b(s), &tmap_lact, sm.full_b(s), (ks - p.k_main) * BK, t0);
          }
        }
      }
      if (!ok) {
        atomicExch(const_cast<int *>(&s_abort), 1);
        // let every load still in flight land before the CTA can exit
        for (int i = max(0, it - STAGES); i < it; ++i) mbar_wait(sm.full_b(i % STAGES), (i / STAGES) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- A producers (dequantize / LoRA copy) ----------------
    const int tid = threadIdx.x - 128;  // 0..127
    float cb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) cb[i] = p.codebook[i];
    const int64_t kblocks = p.K / 64;   // quantization blocks per weight row
    // shared-memory row of this thread inside an A stage, and its swizzle phase
    uint32_t row_off, phase;
    if (!bwd) {
      row_off = (tid >> 3) * 1024 + (tid & 7) * 128;
      phase = tid & 7;
    } else {
      const int rho = tid & 63, h = tid >> 6;   // 8 consecutive lanes: 8 swizzle phases
      row_off = ((rho >> 3) * 2 + h) * 1024 + (rho & 7) * 128;
      phase = rho & 7;
    }
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m_tile = tile % p.m_tiles;
      // block coordinates for stage ks
      auto block_of = [&](int ks, int64_t &blk) -> bool {
        int64_t n, kb;
        if (!bwd) {
          n = static_cast<int64_t>(m_tile) * BM + tid;
          kb = ks;
        } else {
          n = static_cast<int64_t>(ks) * BK + (tid & 63);
          kb = static_cast<int64_t>(m_tile) * (BM / 64) + (tid >> 6);
        }
        blk = n * kblocks + kb;
        return n < p.N && kb < kblocks;
      };
      // Codes and scales are prefetched four stages ahead into four fixed
      // register buffers; each buffer is refilled in place right after it is
      // consumed (no register moves of loads still in flight).
      auto fetch = [&](int ks) -> BlockIn {
        int64_t blk = 0;
        const bool v = ks < p.k_main && block_of(ks, blk);
        return load_block(p, blk, v);
      };
      auto produce = [&](int ks, BlockIn &buf) -> bool {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        ++it;
        if (s_abort || !mbar_wait(sm.empty(s), ph ^ 1, p.status)) return false;
        const uint32_t row_addr = sm.a(s) + row_off;
        if (ks < p.k_main) {
          if (p.sym) dequant_row<true>(cb, buf, row_addr, phase);
          else dequant_row<false>(cb, buf, row_addr, phase);
        } else {
          const int l = ks - p.k_main;
          if (!bwd) {
            // B[N, r] rows: lora columns 64l .. 64l+63 of weight row n
            const int64_t n = static_cast<int64_t>(m_tile) * BM + tid;
            const int nv = (n < p.N) ? max(0, min(BK, p.r - l * BK)) : 0;
            const uint16_t *src = p.lora + (n < p.N ? n : 0) * p.r + l * BK;
            copy_row(src, nv, (p.r % 8) == 0, row_addr, phase);
          } else {
            // A[r, K] rows j = 64l + rho, columns k0 .. k0+63
            const int j = l * BK + (tid & 63);
            const int64_t k0 = static_cast<int64_t>(m_tile) * BM + (tid >> 6) * 64;
            const int nv = (j < p.r && k0 < p.K) ? 64 : 0;
            const uint16_t *src = p.lora + static_cast<int64_t>(j < p.r ? j : 0) * p.K + (k0 < p.K ? k0 : 0);
            copy_row(src, nv, true, row_addr, phase);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(sm.full_a(s));
        buf = fetch(ks + 4);
        return true;
      };
      BlockIn r0 = fetch(0), r1 = fetch(1), r2 = fetch(2), r3 = fetch(3);
      for (int ks = 0; ks < ksteps && ok; ks += 4) {
        ok = produce(ks, r0);
        if (ok && ks + 1 < ksteps) ok = produce(ks + 1, r1);
        if (ok && ks + 2 < ksteps) ok = produce(ks + 2, r2);
        if (ok && ks + 3 < ksteps) ok = produce(ks + 3, r3);
      }
    }
    if (!ok) atomicExch(const_cast<int *>(&s_abort), 1);
  } else {
    // ---------------- epilogue (warps 0-3) ----------------
    const int q = warp;  // lane quarter
    const bool issuer = (threadIdx.x == 0);
    int tc = 0, chunk_count = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tc) {
      const int m_tile = tile % p.m_tiles;
      const int n_tile = tile / p.m_tiles;
      const int acc = tc & 1;
      const uint32_t acc_phase = (tc >> 1) & 1;
      const bool fail = s_abort || !mbar_wait(sm.acc_full(acc), acc_phase, p.status);
      if (named_bar_any(2, 128, fail)) { ok = false; break; }   // uniform across the 4 warps
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const int m_local = q * 32 + static_cast<int>(lane);
      for (int ch = 0; ch < BN / EPI_ROWS; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + ch * EPI_ROWS, r);
        tc_wait_ld();
        if (ch == BN / EPI_ROWS - 1) {
          // all of this warp's tensor-memory reads for the tile are done
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sm.acc_empty(acc));
        }
        // chunks wholly past the last token have nothing to store (uniform branch)
        if (static_cast<int64_t>(n_tile) * BN + ch * EPI_ROWS >= p.T) continue;
        const int buf = chunk_count & 1;
        if (issuer) tma_store_wait_read<1>();
        named_bar_sync(1, 128);
        const uint32_t stg = sm.epi(buf);
#pragma unroll
        for (int j = 0; j < EPI_ROWS; ++j) {
          const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[j]));
          st_shared_u16(stg + (j * BM + m_local) * 2, *reinterpret_cast<const uint16_t *>(&v));
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (issuer) {
          tma_store_2d(&tmap_out, stg, m_tile * BM, n_tile * BN + ch * EPI_ROWS);
          tma_store_commit();
        }
        ++chunk_count;   // staging buffers alternate over stored chunks only
      }
    }
    if (!ok) atomicExch(const_cast<int *>(&s_abort), 1);
    if (issuer) tma_store_wait_all<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

int gemm_smem_bytes() { return SMEM_ALLOC; }

}  // namespace qlora
