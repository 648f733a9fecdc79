// gemm_common.cuh -- device helpers shared by the fused NF4 GEMM kernels:
// shared-memory stores, named barriers, the per-block code loads and the
// dequantization of one 64-weight block into one 128-byte swizzled row.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace gemm {

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// bar.red.or over `count` threads of named barrier `id`: every thread gets the OR.
__device__ __forceinline__ bool named_bar_any(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred P, Q;\n\t"
      "setp.ne.u32 P, %1, 0;\n\t"
      "bar.red.or.pred Q, %2, %3, P;\n\t"
      "selp.u32 %0, 1, 0, Q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// A work unit of a CTA pair: weight-side tile m_pair (256 rows of the MMA's
// M side) against tokens tok0 .. tok0 + ntok - 1 (ntok = 256, or 128 for a
// half tile).
struct Unit {
  int m_pair;
  int tok0;
  int ntok;
};

__device__ __forceinline__ Unit unit_of(const GemmParams &p, int u) {
  int tile = u, half = -1;
  if (u >= p.units_full) {
    const int h = u - p.units_full;
    tile = p.units_full + (h >> 1);
    half = h & 1;
  }
  Unit r;
  r.m_pair = tile % p.m_tiles;
  r.tok0 = (tile / p.m_tiles) * 256 + (half > 0 ? 128 : 0);
  r.ntok = half < 0 ? 256 : 128;
  return r;
}

// One 64-weight block's inputs for a dequantizing thread, as loaded: the
// scale s_b = RN32(fp8 * c2) is formed only when the block is dequantized, so
// that issuing the loads never waits for them.
struct BlockIn {
  uint4 c0, c1;     // 32 code bytes
  uint32_t fbyte;   // E4M3 scale byte (0 for a row outside the matrix)
  float c2;         // second-level scale (0 for a row outside the matrix)
};

__device__ __forceinline__ BlockIn load_block(const GemmParams &p, int64_t blk, bool valid) {
  BlockIn in;
  if (valid) {
    // cached loads: the second half of the 32-byte sector then hits L1, and the
    // codes, which every token tile re-reads, keep the normal L2 policy
    const uint4 *cp = reinterpret_cast<const uint4 *>(p.codes + blk * 32);
    in.c0 = __ldg(cp);
    in.c1 = __ldg(cp + 1);
    in.fbyte = __ldg(p.scales + blk);
    in.c2 = __ldg(p.c2 + (blk >> 8));
  } else {
    in.c0 = make_uint4(0, 0, 0, 0);
    in.c1 = in.c0;
    in.fbyte = 0u;
    in.c2 = 0.f;
  }
  return in;
}

// Dequantize one block into one 128-byte swizzled shared-memory row.
template <bool SYM>
__device__ __forceinline__ void dequant_row(const float (&cb)[16], const BlockIn &in, uint32_t row_addr,
                                            uint32_t phase) {
  BlockLut<SYM> lut;
  lut.make(cb, __fmul_rn(e4m3_to_float(in.fbyte), in.c2));
  const uint32_t w[8] = {in.c0.x, in.c0.y, in.c0.z, in.c0.w, in.c1.x, in.c1.y, in.c1.z, in.c1.w};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t o0, o1, o2, o3;
    lut.lookup8(w[c], o0, o1, o2, o3);
    st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ phase) << 4), o0, o1, o2, o3);
  }
}

// Copy up to 64 BF16 values (zero-padded) into one swizzled shared-memory row.
__device__ __forceinline__ void copy_row(const uint16_t *src, int n_valid, bool aligned16, uint32_t row_addr,
                                         uint32_t phase) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t v[4] = {0, 0, 0, 0};
    const int e0 = c * 8;
    if (aligned16 && e0 + 8 <= n_valid) {
      const uint4 q = *reinterpret_cast<const uint4 *>(src + e0);
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t h = (e0 + i < n_valid) ? static_cast<uint32_t>(src[e0 + i]) : 0u;
        v[i >> 1] |= h << ((i & 1) * 16);
      }
    }
    st_shared_v4(row_addr + ((static_cast<uint32_t>(c) ^ phase) << 4), v[0], v[1], v[2], v[3]);
  }
}

}  // namespace gemm
}  // namespace qlora
