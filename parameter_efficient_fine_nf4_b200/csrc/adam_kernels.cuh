// One Adam step on a trainable fp32 tensor (the adapter factors A and B).
//
// [P1] "The update LoRA is allowed to learn": only A and B carry optimiser
// state.  [P2] "Why full fine-tuning costs so much": mixed-precision Adam
// keeps a 16-bit forward copy, an fp32 master and fp32 moments m, v per
// parameter.  The update is bias-corrected Adam (Kingma and Ba 2015,
// Algorithm 1) with decoupled weight decay (Loshchilov and Hutter 2019):
//   m     = beta1 m + (1 - beta1) g
//   v     = beta2 v + (1 - beta2) g^2
//   theta = theta - lr (m c1 / (sqrt(v c2) + eps) + wd theta),
//   c1 = 1 / (1 - beta1^t), c2 = 1 / (1 - beta2^t)  (host, float64 -> fp32)
// and the bf16 forward copy is theta rounded to nearest.  All in fp32, one
// pass over 30 bytes per parameter (16 read, 14 written): HBM-bound.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace qlora {

struct AdamArgs {
  float lr, beta1, beta2, omb1, omb2, c1, c2, eps, wd;
};

__device__ __forceinline__ float adam_one(float& theta, float& m, float& v, float g, const AdamArgs& a) {
  m = __fmaf_rn(a.beta1, m, __fmul_rn(a.omb1, g));
  v = __fmaf_rn(a.beta2, v, __fmul_rn(a.omb2, __fmul_rn(g, g)));
  const float den = __fadd_rn(__fsqrt_rn(__fmul_rn(v, a.c2)), a.eps);
  const float upd = __fdiv_rn(__fmul_rn(m, a.c1), den);
  theta = __fmaf_rn(-a.lr, __fmaf_rn(a.wd, theta, upd), theta);
  return theta;
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Units of four parameters (16-byte loads and stores); the n % 4 tail is
// taken by the first threads one parameter each.
__global__ void __launch_bounds__(256) adam_step_kernel(float* __restrict__ master, uint16_t* __restrict__ w16,
                                                        float* __restrict__ m, float* __restrict__ v,
                                                        const float* __restrict__ grad, int64_t n,
                                                        const AdamArgs a) {
  const int64_t n4 = n / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < n4; u += stride) {
    float4 th = reinterpret_cast<const float4*>(master)[u];
    float4 mm = reinterpret_cast<const float4*>(m)[u];
    float4 vv = reinterpret_cast<const float4*>(v)[u];
    const float4 g = __ldcs(reinterpret_cast<const float4*>(grad) + u);
    adam_one(th.x, mm.x, vv.x, g.x, a);
    adam_one(th.y, mm.y, vv.y, g.y, a);
    adam_one(th.z, mm.z, vv.z, g.z, a);
    adam_one(th.w, mm.w, vv.w, g.w, a);
    reinterpret_cast<float4*>(master)[u] = th;
    reinterpret_cast<float4*>(m)[u] = mm;
    reinterpret_cast<float4*>(v)[u] = vv;
    reinterpret_cast<uint2*>(w16)[u] = make_uint2(bf16x2_bits(th.x, th.y), bf16x2_bits(th.z, th.w));
  }
  const int64_t tail = n - n4 * 4;
  const int64_t i = n4 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blockIdx.x == 0 && threadIdx.x < tail) {
    float th = master[i], mm = m[i], vv = v[i];
    adam_one(th, mm, vv, grad[i], a);
    master[i] = th;
    m[i] = mm;
    v[i] = vv;
    const __nv_bfloat16 b = __float2bfloat16_rn(th);
    w16[i] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace qlora
