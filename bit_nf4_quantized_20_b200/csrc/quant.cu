// quant.cu -- NF4 quantization with double quantization, and dequantization.
//
// Quantize ("QLoRA: Efficient Fine-Tuning", Step 1 eq. 1 and eq. 2, Step 2;
// "QLoRA & 4-bit Fine-Tuning", Innovation 2):
//   c1_b   = max |w| over block b of 64 consecutive weights (eq. 1, alpha = 1)
//   w_hat  = RN32(w / c1_b)                       (0 for an all-zero block)
//   code   = #{ j : w_hat >= t_j }                (nearest level, ties up)
//   c2_g   = RN32(max_{b in g} c1_b / 448)        (g = 256 consecutive blocks)
//   f_b    = E4M3_RNE_satfinite(RN32(c1_b / c2_g))  (0 when c2_g == 0)
// Dequantize:  W' = BF16_RNE(RN32(codebook[code] * RN32(fp8(f_b) * c2_g)))
//
// One CTA quantizes one double-quantization group (256 blocks = 16,384
// weights): 8 lanes share a block, each loading 8 BF16 weights with one
// 128-bit load; the block absmax is an integer max of |bits| reduced with
// three xor-shuffles; the group max is a CTA reduction.
//
// The code needs no division per weight.  For c1 > 0, RN32(w / c1) >= t_j
// exactly when w >= mid_j * c1 (or w > mid_j * c1, by the tie rule), where
// mid_j is the real midpoint between t_j and the fp32 value below it; mid_j
// has at most 25 significant bits and c1 8, so the product is exact in double.
// Each block turns its 15 thresholds into the smallest BF16 weights that reach
// them, B_j, and code = #{ j : w >= B_j } by the same 4-step search.
//
// Variant (snap_dq): the block is normalised by the scale it is dequantized
// with, s_b = RN32(fp8(f_b) * c2_g), instead of c1_b (w_hat = 0 where s_b = 0).
// s_b has at most 24 significant bits, so mid_j * s_b (<= 49 bits) is still
// exact in double and the same boundary construction applies.

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int QT = 256;

// Number of boundaries b_j <= x (b non-decreasing), by a branch-free binary
// search: the first two levels select between register-held boundaries, the
// last two read the block's table in shared memory.
__device__ __forceinline__ uint32_t snap_code(float x, float t3, float t7, float t11, const float *s_thr) {
  uint32_t c = (x >= t7) ? 8u : 0u;
  const float th = c ? t11 : t3;
  c += (x >= th) ? 4u : 0u;
  c += (x >= s_thr[c + 1]) ? 2u : 0u;
  c += (x >= s_thr[c]) ? 1u : 0u;
  return c;
}

// The smallest BF16 value w with w >= mid * c1 (incl) or w > mid * c1 (not
// incl), for c1 > 0; +Inf when no finite BF16 value qualifies.
__device__ __forceinline__ float snap_boundary(float c1, double mid, bool incl) {
  const double P = mid * static_cast<double>(c1);   // exact
  const float f = __double2float_ru(P);             // the smallest fp32 >= P
  uint32_t u = __float_as_uint(f);
  if ((u & 0xFFFFu) != 0u) u = (f > 0.f) ? ((u + 0x10000u) & 0xFFFF0000u) : (u & 0xFFFF0000u);
  float b = __uint_as_float(u);                     // the smallest BF16 >= f, hence >= P
  if (!incl && static_cast<double>(b) == P) {       // strictly above P: the next BF16 up
    if ((u & 0x7FFFFFFFu) == 0u) u = 0x00010000u;
    else u = (b > 0.f) ? u + 0x10000u : u - 0x10000u;
    b = __uint_as_float(u);
  }
  return b;
}

__global__ void __launch_bounds__(QT) quantize_kernel(const uint4 *__restrict__ w, int64_t n_blocks,
                                                      uint32_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                      float *__restrict__ c2, const SnapTable tab,
                                                      int snap_dq, uint32_t *status) {
  __shared__ float s_bnd[256 * 16];   // per block of the group: B_0 .. B_14
  __shared__ float s_wmax[QT / 32];

  const int64_t g = blockIdx.x;
  const int64_t b0 = g * 256;
  const int nb = static_cast<int>(min(static_cast<int64_t>(256), n_blocks - b0));
  const int tid = threadIdx.x;
  const int sub = tid & 7;    // which 8 weights of the block
  const int bw = tid >> 3;    // block within a slab of 32 blocks

  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bl = i * 32 + bw;
    if (bl < nb) {
      v[i] = __ldg(w + (b0 + bl) * 8 + sub);
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }

  // block absmax as an integer max over |bits| (BF16 order = magnitude order)
  float c1[8];
  uint32_t bad = 0;
  float tmax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = v[i].x & 0x7FFF7FFFu, b = v[i].y & 0x7FFF7FFFu, c = v[i].z & 0x7FFF7FFFu,
                   d = v[i].w & 0x7FFF7FFFu;
    uint32_t m = max(max(max(a & 0xFFFFu, a >> 16), max(b & 0xFFFFu, b >> 16)),
                     max(max(c & 0xFFFFu, c >> 16), max(d & 0xFFFFu, d >> 16)));
    bad |= (m >= 0x7F80u) ? 1u : 0u;
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
    c1[i] = __uint_as_float(m << 16);
    tmax = fmaxf(tmax, c1[i]);
  }
#pragma unroll
  for (int o = 8; o < 32; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
  if ((tid & 31) == 0) s_wmax[tid >> 5] = tmax;
  __syncthreads();
  float gmax = s_wmax[0];
#pragma unroll
  for (int i = 1; i < QT / 32; ++i) gmax = fmaxf(gmax, s_wmax[i]);

  const float c2v = __fdiv_rn(gmax, 448.0f);
  if (tid == 0) c2[g] = c2v;
  // each block's scale byte, and the divisor its codes are snapped against
  uint32_t fb[8];
  float dv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    fb[i] = c2v > 0.f ? float_to_e4m3(__fdiv_rn(c1[i], c2v)) : 0u;
    dv[i] = snap_dq ? __fmul_rn(e4m3_to_float(fb[i]), c2v) : c1[i];
  }

  // the block's boundaries: lane `sub` of its 8 lanes forms B_sub and B_{sub + 8}
  // (a block whose divisor is zero gets boundaries that give every weight the
  // code of 0)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bl = i * 32 + bw;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = sub + 8 * h;
      if (j < 15) {
        float bj;
        if (dv[i] > 0.f) bj = snap_boundary(dv[i], tab.mid[j], ((tab.incl >> j) & 1u) != 0u);
        else bj = j < static_cast<int>(tab.snap0) ? -INFINITY : INFINITY;
        s_bnd[bl * 16 + j] = bj;
      }
    }
  }
  __syncwarp();   // a block's 8 lanes are in one warp

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bl = i * 32 + bw;
    if (bl < nb) {
      if (sub == 0) scales[b0 + bl] = static_cast<uint8_t>(fb[i]);
      const uint32_t hw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      const float *bnd = s_bnd + bl * 16;
      const float b3 = bnd[3], b7 = bnd[7], b11 = bnd[11];
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t bits = (e & 1) ? (hw[e >> 1] & 0xFFFF0000u) : (hw[e >> 1] << 16);
        word |= snap_code(__uint_as_float(bits), b3, b7, b11, bnd) << (4 * e);
      }
      codes[(b0 + bl) * 8 + sub] = word;
    }
  }
  if (__any_sync(0xffffffffu, bad) && (tid & 31) == 0) set_status(status, DEV_NONFINITE);
}

__global__ void __launch_bounds__(256) dequant_kernel(const uint2 *__restrict__ codes,
                                                      const uint8_t *__restrict__ scales,
                                                      const float *__restrict__ c2, int64_t n_units,
                                                      const SnapTable tab, uint4 *__restrict__ out) {
  __shared__ float s_cb[16];
  if (threadIdx.x < 16) s_cb[threadIdx.x] = tab.codebook[threadIdx.x];
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_units; i += stride) {
    const uint2 c = __ldg(codes + i);       // 16 codes
    const int64_t blk = i >> 2;             // 4 units of 16 weights per block
    const float s = __fmul_rn(e4m3_to_float(__ldg(scales + blk)), __ldg(c2 + (blk >> 8)));
    const uint32_t words[2] = {c.x, c.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t o[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float lo = s_cb[(words[h] >> (8 * p)) & 15u];
        const float hi = s_cb[(words[h] >> (8 * p + 4)) & 15u];
        o[p] = pack_bf16x2(__fmul_rn(lo, s), __fmul_rn(hi, s));
      }
      out[2 * i + h] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Adapter merge for export ("QLoRA: Efficient Fine-Tuning", Step 3: eq. 3's two
// terms as one matrix W0 + s B A):
//   out[n, k] = BF16_RNE(fma(s, d, W'[n, k])),   d = sum_j B[n, j] A[j, k] in fp32,
// with W' formed exactly as dequant_kernel forms it (so the frozen part is the
// BF16 dequantized weight) and j ascending.  One thread per 16 consecutive
// weights of a row (a unit never crosses a row: K % 64 == 0).
__global__ void __launch_bounds__(256) merge_kernel(const uint2 *__restrict__ codes,
                                                    const uint8_t *__restrict__ scales,
                                                    const float *__restrict__ c2, int64_t n_units, int64_t K,
                                                    const SnapTable tab, const uint16_t *__restrict__ A,
                                                    const uint16_t *__restrict__ B, int r, float s,
                                                    uint4 *__restrict__ out) {
  __shared__ float s_cb[16];
  if (threadIdx.x < 16) s_cb[threadIdx.x] = tab.codebook[threadIdx.x];
  __syncthreads();
  const int64_t units_per_row = K / 16;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_units; i += stride) {
    const int64_t n = i / units_per_row, k0 = (i - n * units_per_row) * 16;
    const uint2 c = __ldg(codes + i);       // 16 codes
    const int64_t blk = i >> 2;             // 4 units of 16 weights per block
    const float sc = __fmul_rn(e4m3_to_float(__ldg(scales + blk)), __ldg(c2 + (blk >> 8)));
    float w[16], d[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t word = e < 8 ? c.x : c.y;
      const float q = s_cb[(word >> (4 * (e & 7))) & 15u];
      w[e] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(q, sc)));
      d[e] = 0.f;
    }
    const uint16_t *brow = B + n * r;
    for (int j = 0; j < r; ++j) {
      const float b = __uint_as_float(static_cast<uint32_t>(__ldg(brow + j)) << 16);
      const uint4 *ap = reinterpret_cast<const uint4 *>(A + static_cast<int64_t>(j) * K + k0);
      const uint4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
      const uint32_t aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint32_t bits = (e & 1) ? (aw[e >> 1] & 0xFFFF0000u) : (aw[e >> 1] << 16);
        d[e] = fmaf(b, __uint_as_float(bits), d[e]);
      }
    }
    uint32_t o[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) o[p] = pack_bf16x2(fmaf(s, d[2 * p], w[2 * p]), fmaf(s, d[2 * p + 1], w[2 * p + 1]));
    out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

cudaError_t launch_merge(const uint8_t *codes, const uint8_t *scales, const float *c2, int64_t N, int64_t K,
                         const float (&codebook)[16], const uint16_t *A, const uint16_t *B, int r, float s,
                         uint16_t *out, cudaStream_t st, int num_sms) {
  const int64_t n_units = N * K / 16;
  if (n_units <= 0) return cudaSuccess;
  SnapTable tab;
  for (int i = 0; i < 16; ++i) tab.codebook[i] = codebook[i];
  for (int i = 0; i < 15; ++i) tab.thr[i] = 0.f;
  int64_t blocks = (n_units + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(reinterpret_cast<const uint2 *>(codes), scales, c2,
                                                               n_units, K, tab, A, B, r, s,
                                                               reinterpret_cast<uint4 *>(out));
  return cudaGetLastError();
}

cudaError_t launch_quantize(const uint16_t *w, int64_t n_blocks, uint8_t *codes, uint8_t *scales, float *c2,
                            const SnapTable &tab, bool snap_dq, uint32_t *status, cudaStream_t st, int num_sms) {
  (void)num_sms;
  const int64_t groups = (n_blocks + 255) / 256;
  if (groups <= 0) return cudaSuccess;
  quantize_kernel<<<static_cast<unsigned>(groups), QT, 0, st>>>(reinterpret_cast<const uint4 *>(w), n_blocks,
                                                                 reinterpret_cast<uint32_t *>(codes), scales, c2,
                                                                 tab, snap_dq ? 1 : 0, status);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales, const float *c2, int64_t n_weights,
                              const float (&codebook)[16], uint16_t *out, cudaStream_t st, int num_sms) {
  const int64_t n_units = n_weights / 16;
  if (n_units <= 0) return cudaSuccess;
  SnapTable tab;
  for (int i = 0; i < 16; ++i) tab.codebook[i] = codebook[i];
  for (int i = 0; i < 15; ++i) tab.thr[i] = 0.f;
  int64_t blocks = (n_units + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  dequant_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(reinterpret_cast<const uint2 *>(codes), scales,
                                                                 c2, n_units, tab, reinterpret_cast<uint4 *>(out));
  return cudaGetLastError();
}

}  // namespace qlora
