// Fused AdamW step over fp32 parameters, gradients and moment states, for the trainable LoRA adapters.
//
// The paged optimizer of the PEFT page (zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA end to
// end"; QLoRA explainer, prism.theerrors.in, "The three innovations") keeps the optimizer states in unified
// memory, which the driver pages between GPU and host; this kernel is the step that reads and writes them,
// and it runs unchanged on device memory or on managed memory (resident, or paged back in by its own
// accesses). The update is the standard decoupled-weight-decay AdamW (Loshchilov & Hutter, 2019):
//   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
//   p <- p - [lr / (1 - b1^t)] m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// in fp32 (IEEE division and square root), the two bias-correction factors formed once on the host in
// fp64. Optionally the updated parameter is also written as bf16, the copy the linear layer consumes.
// One pass over HBM: 16 B read + 12 B written per parameter (+ 2 B with the bf16 copy).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace qnf4 {

struct AdamWArgs {
  float keep;          // 1 - lr * wd
  float beta1, one_minus_beta1;
  float beta2, one_minus_beta2;
  float step_size;     // lr / (1 - beta1^t)
  float inv_bc2_sqrt;  // 1 / sqrt(1 - beta2^t)
  float eps;
};

constexpr int kAdamThreads = 256;

__device__ __forceinline__ void adamw_one(float& p, float g, float& m, float& v, const AdamWArgs& a) {
  const float pd = p * a.keep;
  m = __fmaf_rn(a.beta1, m, a.one_minus_beta1 * g);
  v = __fmaf_rn(a.beta2, v, a.one_minus_beta2 * (g * g));
  const float denom = __fmaf_rn(__fsqrt_rn(v), a.inv_bc2_sqrt, a.eps);
  p = pd - a.step_size * __fdiv_rn(m, denom);
}

template <bool kBf16Copy>
__global__ void __launch_bounds__(kAdamThreads) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                            float* __restrict__ m, float* __restrict__ v,
                                                            __nv_bfloat16* __restrict__ p16, int64_t n,
                                                            AdamWArgs a) {
  const int64_t n4 = n / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 pv = reinterpret_cast<const float4*>(p)[i];
    const float4 gv = __ldcs(reinterpret_cast<const float4*>(g) + i);
    float4 mv = reinterpret_cast<const float4*>(m)[i];
    float4 vv = reinterpret_cast<const float4*>(v)[i];
    adamw_one(pv.x, gv.x, mv.x, vv.x, a);
    adamw_one(pv.y, gv.y, mv.y, vv.y, a);
    adamw_one(pv.z, gv.z, mv.z, vv.z, a);
    adamw_one(pv.w, gv.w, mv.w, vv.w, a);
    reinterpret_cast<float4*>(p)[i] = pv;
    reinterpret_cast<float4*>(m)[i] = mv;
    reinterpret_cast<float4*>(v)[i] = vv;
    if constexpr (kBf16Copy) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(pv.x, pv.y), hi = __floats2bfloat162_rn(pv.z, pv.w);
      uint2 o;
      o.x = *reinterpret_cast<uint32_t*>(&lo);
      o.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(p16)[i] = o;
    }
  }
  // the ragged tail (n % 4 elements), one thread each
  const int64_t t = 4 * n4 + threadIdx.x;
  if (blockIdx.x == 0 && t < n) {
    float pp = p[t], mm = m[t], vv = v[t];
    adamw_one(pp, g[t], mm, vv, a);
    p[t] = pp;
    m[t] = mm;
    v[t] = vv;
    if constexpr (kBf16Copy) p16[t] = __float2bfloat16_rn(pp);
  }
}

}  // namespace qnf4
