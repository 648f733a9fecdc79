// common.cuh -- device helpers shared by the sm_100a kernels of the QLoRA
// NF4 linear-layer library: status word, bounded mbarrier waits, TMA and
// tcgen05 (5th-generation tensor core / tensor memory) PTX wrappers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

// ---------------------------------------------------------------------------
// Status word at the start of every workspace (see qlora_get_error).
// ---------------------------------------------------------------------------
enum : uint32_t {
  DEV_NONFINITE = 1u,   // quantize saw an Inf/NaN weight
  DEV_TIMEOUT = 2u,     // a bounded wait ran out
};

// Workspace header: status word + per-kernel completion counters.
struct WsHeader {
  uint32_t status;
  uint32_t pad_[63];
};
constexpr size_t kWsHeaderBytes = 256;
constexpr size_t kWsCounterBytes = 64 * 1024;   // 16384 tile counters

// A wait that has not completed after this many nanoseconds gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most limit_ns
// (kWaitLimitNs unless a caller asks for less).  Returns false (and records
// DEV_TIMEOUT) if it never does.
// Waiting threads are suspended between probes (try_wait's time hint) and
// read the global timer only every 64 probes, so that long waits (the
// epilogue waiting for a whole tile) take few issue slots.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t *status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 1000u)) return true;
    if ((i & 63u) == 0) {
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
        set_status(status, DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// The same bounded wait with cluster-scope acquire: for barriers that receive
// release.cluster arrivals from another CTA of the cluster.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint32_t *status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 63u) == 0 && globaltimer() - t0 > kWaitLimitNs) {
      set_status(status, DEV_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library waits for the
// preceding kernel of its stream (griddepcontrol.wait) before it completes
// and before it touches anything that kernel writes, so a kernel completes
// only after everything before it.  It lets its own dependents launch
// (griddepcontrol.launch_dependents) only after that wait -- so that a kernel
// that starts early can rely on everything before its predecessor having
// completed -- with one exception: a rank-r launch whose inputs were all
// complete before its predecessor started (it waits only before exiting)
// lets its dependent start at once; that dependent is the next kernel of the
// same layer call and reads this launch's outputs only after its own wait.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Proxy fences
// ---------------------------------------------------------------------------
// Generic-proxy shared-memory writes -> visible to the async proxy (TMA store,
// tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int32_t c0,
                                            int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}

__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (BF16 inputs, FP32 accumulate).
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05 ops of this thread complete.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Ties registers filled by an asynchronous tcgen05.ld to this point of the
// program: placed after tcgen05.wait::ld, no use of them is moved above it.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 32 consecutive columns: thread i gets lane (base+i), cols c..c+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 32 lanes x 32 bits, 32 consecutive columns: thread i writes lane (base+i), cols c..c+31.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
      "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]),
      "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Wait until every tcgen05.st of this thread has completed.
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Thread block clusters and the 2-SM (cta_group::2) forms
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_arrive_wait() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// Arrive on an mbarrier of any CTA of the cluster (shared::cluster address).
// Release at CTA scope, the form cluster pipelines use for a producer's own
// shared-memory writes (a cluster-scope release costs a full memory barrier).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_bar),
               "r"(bytes)
               : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// the pair leader's mbarrier (2-SM form, no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, uint32_t leader_bar,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

// D (+)= A * B^T across a CTA pair, issued by the leader (even rank) only,
// kind::f16 (BF16 inputs, FP32 accumulate), D in both CTAs' tensor memory:
// each CTA holds 128 of A's 256 rows and half of B's rows (the N operand).
//   _ts: A in tensor memory (each CTA's 128 rows in its lanes 0..127 at column
//        a_tmem, K-major, two BF16 per 32-bit column, the lower k in the low
//        half), B from shared memory;
//   _ss: A and B from shared memory.
// Shared-memory descriptors are passed as 32-bit halves: only the low half,
// which holds the start address, changes from stage to stage, so a stage
// costs the issuing thread 32-bit adds.
__device__ __forceinline__ void tc_mma_ts_pair_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                                  uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_mma_ss_pair_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                                  uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 ad, {%1, %2};\n\t"
      "mov.b64 bd, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], ad, bd, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once each) on the mbarrier at the same offset in every CTA of
// `cta_mask` when all prior tcgen05 ops of this thread complete.
__device__ __forceinline__ void tc_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}

// ---------------------------------------------------------------------------
// UMMA descriptors (shared-memory matrix descriptor and instruction descriptor)
// ---------------------------------------------------------------------------
// Shared-memory descriptor, 128-byte swizzle (layout type 2), version 1.
//   bits  0-13 start address >> 4
//   bits 16-29 leading-dimension byte offset >> 4
//   bits 32-45 stride-dimension byte offset >> 4
//   bits 46-47 version (1 on sm_100)
//   bits 49-51 base offset (0: atoms 1024-byte aligned)
//   bits 61-63 layout type (2 = SWIZZLE_128B)
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor for kind::f16: BF16 A and B, FP32 D.
//   bits 4-5 D format (1 = F32); 7-9 A format (1 = BF16); 10-12 B format (1 = BF16)
//   bit 15 A major (0 = K-major, 1 = MN-major); bit 16 B major
//   bits 17-22 N >> 3; bits 24-28 M >> 4
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Number formats
// ---------------------------------------------------------------------------
// Exact decode of an OCP FP8-E4M3FN byte (every finite value fits in fp32).
__device__ __forceinline__ float e4m3_to_float(uint32_t byte) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(byte), __NV_E4M3);
  return __half2float(__half(h));
}

// fp32 -> E4M3FN, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t float_to_e4m3(float x) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// Pack two fp32 into a BF16x2 word (round to nearest even): lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t lop3_select(uint32_t a, uint32_t b, uint32_t m) {
  // (a & ~m) | (b & m)
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xCA;" : "=r"(d) : "r"(m), "r"(b), "r"(a));
  return d;
}

// A per-block 16-entry BF16 lookup table held in 8 registers as byte planes:
// lo[i] holds the low bytes of entries 4i..4i+3, hi[i] their high bytes.
struct Lut16 {
  uint32_t lo[4];
  uint32_t hi[4];
};

// Build the table of BF16(RN32(codebook[j] * scale)), j = 0..15.
__device__ __forceinline__ Lut16 make_lut16(const float (&cb)[16], float scale) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = pack_bf16x2(__fmul_rn(cb[2 * i], scale), __fmul_rn(cb[2 * i + 1], scale));
  Lut16 t;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t.lo[i] = prmt(p[2 * i], p[2 * i + 1], 0x6420);
    t.hi[i] = prmt(p[2 * i], p[2 * i + 1], 0x7531);
  }
  return t;
}

// Look up four 4-bit codes held in bits 0-15 of `sel` (code i in bits 4i..4i+3).
// Returns two BF16x2 words: out0 = (entry(c0), entry(c1)), out1 = (entry(c2), entry(c3)),
// the lower-indexed element in the low half.
__device__ __forceinline__ void lut16_lookup4(const Lut16 &t, uint32_t sel, uint32_t &out0, uint32_t &out1) {
  const uint32_t idx = sel & 0x7777u;
  // byte i of m = 0xFF when code i >= 8 (sign-replicate mode of prmt on bit 3 of each code)
  const uint32_t m = prmt(sel << 4, sel, 0xD9C8u);
  const uint32_t lo = lop3_select(prmt(t.lo[0], t.lo[1], idx), prmt(t.lo[2], t.lo[3], idx), m);
  const uint32_t hi = lop3_select(prmt(t.hi[0], t.hi[1], idx), prmt(t.hi[2], t.hi[3], idx), m);
  out0 = prmt(lo, hi, 0x5140u);
  out1 = prmt(lo, hi, 0x7362u);
}

// A codebook is "symmetric" when codebook[15 - i] == -codebook[i] bit for bit
// (eq. 2's NF4 levels are).  Then BF16(RN32(q[c] * s)) for c < 8 is the exact
// negation of the entry for 15 - c (negation and round-to-nearest-even commute),
// so eight magnitudes and a sign bit give all sixteen entries.
struct Lut8 {
  uint32_t lo[2];   // low bytes of |entry(8 + j)|, j = 0..7
  uint32_t hi[2];   // high bytes (sign bit clear)
};

__device__ __forceinline__ Lut8 make_lut8(const float (&cb)[16], float scale) {
  uint32_t p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = pack_bf16x2(__fmul_rn(cb[8 + 2 * i], scale), __fmul_rn(cb[9 + 2 * i], scale));
  Lut8 t;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    t.lo[i] = prmt(p[2 * i], p[2 * i + 1], 0x6420);
    t.hi[i] = prmt(p[2 * i], p[2 * i + 1], 0x7531);
  }
  return t;
}

// Magnitude indices of eight codes: c >= 8 -> c - 8, c < 8 -> 7 - c.
__device__ __forceinline__ uint32_t mag_index8(uint32_t w) {
  const uint32_t neg = ~(w >> 3) & 0x11111111u;   // 1 in each nibble whose code is < 8
  return (w ^ (neg * 7u)) & 0x77777777u;
}

// Four codes in bits 0-15 of `codes` (their magnitude indices in bits 0-15 of
// `mag`): out0 = (entry(c0), entry(c1)), out1 = (entry(c2), entry(c3)).
__device__ __forceinline__ void lut8_lookup4(const Lut8 &t, uint32_t codes, uint32_t mag, uint32_t &out0,
                                             uint32_t &out1) {
  const uint32_t lo = prmt(t.lo[0], t.lo[1], mag);
  uint32_t hi = prmt(t.hi[0], t.hi[1], mag);
  // byte i of m = 0xFF when code i >= 8 (sign-replicate mode of prmt on bit 3)
  const uint32_t m = prmt(codes << 4, codes, 0xD9C8u);
  hi |= ~m & 0x80808080u;   // negative entries for codes below 8
  out0 = prmt(lo, hi, 0x5140u);
  out1 = prmt(lo, hi, 0x7362u);
}

// Eight codes of `w` (code i in bits 4i..4i+3): o0 = (entry(c0), entry(c1)),
// o1 = (entry(c2), entry(c3)), o2 = (entry(c4), entry(c5)), o3 = (entry(c6), entry(c7)).
// The sign masks of both halves come from one shifted copy of the word: byte i
// of m_lo (m_hi) is 0xFF when code i (4 + i) is >= 8, by prmt's sign-replicate
// mode on the byte whose bit 7 holds that code's bit 3.
__device__ __forceinline__ void lut8_lookup8(const Lut8 &t, uint32_t w, uint32_t &o0, uint32_t &o1, uint32_t &o2,
                                             uint32_t &o3) {
  const uint32_t mag = mag_index8(w);
  const uint32_t magh = mag >> 16;
  const uint32_t w4 = w << 4;
  const uint32_t m_lo = prmt(w4, w, 0xD9C8u);
  const uint32_t m_hi = prmt(w4, w, 0xFBEAu);
  const uint32_t lo0 = prmt(t.lo[0], t.lo[1], mag);
  const uint32_t hi0 = prmt(t.hi[0], t.hi[1], mag) | (~m_lo & 0x80808080u);
  const uint32_t lo1 = prmt(t.lo[0], t.lo[1], magh);
  const uint32_t hi1 = prmt(t.hi[0], t.hi[1], magh) | (~m_hi & 0x80808080u);
  o0 = prmt(lo0, hi0, 0x5140u);
  o1 = prmt(lo0, hi0, 0x7362u);
  o2 = prmt(lo1, hi1, 0x5140u);
  o3 = prmt(lo1, hi1, 0x7362u);
}

// x >> 16 on the multiply pipe (the high word of x * 2^16)
__device__ __forceinline__ uint32_t shr16_mul(uint32_t x) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, 65536;" : "=r"(r) : "r"(x));
  return r;
}

// Magnitude indices of eight codes (c >= 8 -> c - 8, c < 8 -> 7 - c): the low
// three bits of each code, flipped where bit 3 is clear; the flip mask
// (7 in each such nibble) is (~w & 0x88888888) * 7 / 8, a multiply-high.
__device__ __forceinline__ uint32_t mag_index8_mul(uint32_t w) {
  uint32_t flip;
  asm("mul.hi.u32 %0, %1, 0xE0000000;" : "=r"(flip) : "r"(~w & 0x88888888u));
  return (w ^ flip) & 0x77777777u;
}

// Eight codes of `w` -> four BF16x2 words (entry(c0), entry(c1)), ..,
// (entry(c6), entry(c7)) from a sign-symmetric 8-magnitude table (as
// lut8_lookup8, with the two shifts on the multiply pipe).
__device__ __forceinline__ void sym_lookup8(const Lut8 &t, uint32_t w, uint32_t &o0, uint32_t &o1, uint32_t &o2,
                                            uint32_t &o3) {
  const uint32_t mag = mag_index8_mul(w);
  const uint32_t magh = shr16_mul(mag);
  const uint32_t w4 = w * 16u;
  const uint32_t m_lo = prmt(w4, w, 0xD9C8u);
  const uint32_t m_hi = prmt(w4, w, 0xFBEAu);
  const uint32_t lo0 = prmt(t.lo[0], t.lo[1], mag);
  const uint32_t hi0 = prmt(t.hi[0], t.hi[1], mag) | (~m_lo & 0x80808080u);
  const uint32_t lo1 = prmt(t.lo[0], t.lo[1], magh);
  const uint32_t hi1 = prmt(t.hi[0], t.hi[1], magh) | (~m_hi & 0x80808080u);
  o0 = prmt(lo0, hi0, 0x5140u);
  o1 = prmt(lo0, hi0, 0x7362u);
  o2 = prmt(lo1, hi1, 0x5140u);
  o3 = prmt(lo1, hi1, 0x7362u);
}

// One 64-weight block's lookup table: eight magnitudes and the sign bit for a
// sign-symmetric codebook, all sixteen entries otherwise.
template <bool SYM>
struct BlockLut;
template <>
struct BlockLut<true> {
  Lut8 t;
  __device__ __forceinline__ void make(const float (&cb)[16], float s) { t = make_lut8(cb, s); }
  __device__ __forceinline__ void lookup8(uint32_t w, uint32_t &o0, uint32_t &o1, uint32_t &o2, uint32_t &o3) const {
    sym_lookup8(t, w, o0, o1, o2, o3);
  }
};
template <>
struct BlockLut<false> {
  Lut16 t;
  __device__ __forceinline__ void make(const float (&cb)[16], float s) { t = make_lut16(cb, s); }
  __device__ __forceinline__ void lookup8(uint32_t w, uint32_t &o0, uint32_t &o1, uint32_t &o2, uint32_t &o3) const {
    lut16_lookup4(t, w, o0, o1);
    lut16_lookup4(t, shr16_mul(w), o2, o3);
  }
};

}  // namespace qlora
