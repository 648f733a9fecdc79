// optim.cu -- the adapters' optimizer step with its state in unified memory.
//
// "What is QLoRA?", "The three pieces" (paged optimizers: the optimizer state
// lives in CUDA unified memory, which the driver pages out to host memory when
// the GPU runs short and back when a kernel touches it) and "Worked example"
// (adapters in fp32 with Adam moments); "QLoRA & 4-bit Fine-Tuning",
// Innovation 3.  The step is Adam (Kingma & Ba, 2015) with decoupled weight
// decay (Loshchilov & Hutter, 2019):
//
//   p <- p (1 - lr wd)
//   m <- b1 m + (1 - b1) g;   v <- b2 v + (1 - b2) g^2
//   p <- p - lr (m / bc1) / (sqrt(v / bc2) + eps),   bc_i = 1 - b_i^step
//
// with p, m, v FP32 (in device or managed memory alike: the kernel only loads
// and stores them), g the BF16 gradient the backward wrote (dA or dB), and an
// optional BF16 copy of the new p for the next forward.  HBM-bound: 28 bytes
// per parameter (read p, m, v, g; write p, m, v, BF16 p).  One thread handles
// eight consecutive parameters with 16-byte loads and stores; a grid of a few
// CTAs per SM strides over the array.

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void adam_one(float &p, float &m, float &v, float g, const AdamArgs &a) {
  p = __fmul_rn(p, a.decay);
  m = fmaf(a.beta1, m, __fmul_rn(a.one_minus_beta1, g));
  v = fmaf(a.beta2, v, __fmul_rn(a.one_minus_beta2, __fmul_rn(g, g)));
  const float m_hat = __fdiv_rn(m, a.bc1);
  const float v_hat = __fdiv_rn(v, a.bc2);
  p = p - __fmul_rn(a.lr, __fdiv_rn(m_hat, __fadd_rn(__fsqrt_rn(v_hat), a.eps)));
}

__global__ void __launch_bounds__(256) adam_kernel(float *__restrict__ param, float *__restrict__ m,
                                                   float *__restrict__ v, const uint16_t *__restrict__ grad,
                                                   uint16_t *__restrict__ out_bf16, int64_t n, const AdamArgs a) {
  const int64_t n8 = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < n8; i += stride) {
    float4 *pp = reinterpret_cast<float4 *>(param) + 2 * i;
    float4 *mp = reinterpret_cast<float4 *>(m) + 2 * i;
    float4 *vp = reinterpret_cast<float4 *>(v) + 2 * i;
    const uint4 gw = __ldcs(reinterpret_cast<const uint4 *>(grad) + i);
    float4 p0 = __ldcs(pp), p1 = __ldcs(pp + 1), m0 = __ldcs(mp), m1 = __ldcs(mp + 1), v0 = __ldcs(vp),
           v1 = __ldcs(vp + 1);
    adam_one(p0.x, m0.x, v0.x, bf16_lo(gw.x), a);
    adam_one(p0.y, m0.y, v0.y, bf16_hi(gw.x), a);
    adam_one(p0.z, m0.z, v0.z, bf16_lo(gw.y), a);
    adam_one(p0.w, m0.w, v0.w, bf16_hi(gw.y), a);
    adam_one(p1.x, m1.x, v1.x, bf16_lo(gw.z), a);
    adam_one(p1.y, m1.y, v1.y, bf16_hi(gw.z), a);
    adam_one(p1.z, m1.z, v1.z, bf16_lo(gw.w), a);
    adam_one(p1.w, m1.w, v1.w, bf16_hi(gw.w), a);
    __stcs(pp, p0);
    __stcs(pp + 1, p1);
    __stcs(mp, m0);
    __stcs(mp + 1, m1);
    __stcs(vp, v0);
    __stcs(vp + 1, v1);
    if (out_bf16)
      __stcs(reinterpret_cast<uint4 *>(out_bf16) + i,
             make_uint4(pack_bf16x2(p0.x, p0.y), pack_bf16x2(p0.z, p0.w), pack_bf16x2(p1.x, p1.y),
                        pack_bf16x2(p1.z, p1.w)));
  }
  // the last n % 8 parameters, one per thread of the first CTA
  if (blockIdx.x == 0 && threadIdx.x < n - 8 * n8) {
    const int64_t j = 8 * n8 + threadIdx.x;
    float p = param[j], mm = m[j], vv = v[j];
    adam_one(p, mm, vv, __uint_as_float(static_cast<uint32_t>(grad[j]) << 16), a);
    param[j] = p;
    m[j] = mm;
    v[j] = vv;
    if (out_bf16) out_bf16[j] = __bfloat16_as_ushort(__float2bfloat16_rn(p));
  }
}

}  // namespace

cudaError_t launch_adam(float *param, float *m, float *v, const uint16_t *grad, uint16_t *out_bf16, int64_t n,
                        const AdamArgs &a, cudaStream_t st, int num_sms) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n / 8 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  adam_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(param, m, v, grad, out_bf16, n, a);
  return cudaGetLastError();
}

}  // namespace qlora
