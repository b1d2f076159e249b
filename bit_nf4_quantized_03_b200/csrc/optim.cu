// Paged AdamW, 32-bit, for the LoRA adapters ("QLoRA Explained": Paged
// Optimizers and optim = "paged_adamw_32bit"; "QLoRA: Quantized Low-Rank
// Adaptation": "Paged optimizers (the storage unit)").
//
// The arithmetic is AdamW with decoupled weight decay (Loshchilov and
// Hutter) on fp32 master weights with fp32 first and second moments:
//   g = grad * grad_scale
//   m = b1 m + (1 - b1) g
//   v = b2 v + (1 - b2) g^2
//   p = p (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// One pass reads p, g, m, v and writes p, m, v and, optionally, the bf16
// copy of p that the GEMMs read: 30 bytes per parameter, HBM-bound.
//
// "Paged" is where the states live: unified (managed) memory that the driver
// may move to host RAM when device memory runs short, prefetched back to the
// device before the step. The step itself runs on any device-accessible
// pointers.
#include <cmath>

#include "qlora_kernels.h"

namespace qlora {

namespace {

struct AdamCoef {
  float b1, b2, one_m_b1, one_m_b2;
  float step_size;      // lr / (1 - b1^t)
  float inv_sqrt_bc2;   // 1 / sqrt(1 - b2^t)
  float eps, decay;     // decay = 1 - lr * wd
  float gscale;
};

__device__ __forceinline__ void adam1(float& p, float g, float& m, float& v, const AdamCoef& c) {
  g = g * c.gscale;
  m = __fmaf_rn(c.b1, m, c.one_m_b1 * g);
  v = __fmaf_rn(c.b2, v, c.one_m_b2 * (g * g));
  const float denom = __fmaf_rn(sqrtf(v), c.inv_sqrt_bc2, c.eps);
  p = __fmaf_rn(p, c.decay, -(c.step_size * m) / denom);
}

__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    uint16_t* __restrict__ p_bf16, int64_t count, AdamCoef c) {
  griddep_enter();
  const int64_t n4 = count / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 pp = reinterpret_cast<float4*>(p)[i];
    const float4 gg = __ldcs(reinterpret_cast<const float4*>(g) + i);
    float4 mm = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    adam1(pp.x, gg.x, mm.x, vv.x, c);
    adam1(pp.y, gg.y, mm.y, vv.y, c);
    adam1(pp.z, gg.z, mm.z, vv.z, c);
    adam1(pp.w, gg.w, mm.w, vv.w, c);
    reinterpret_cast<float4*>(p)[i] = pp;
    reinterpret_cast<float4*>(m)[i] = mm;
    reinterpret_cast<float4*>(v)[i] = vv;
    if (p_bf16 != nullptr)
      reinterpret_cast<uint2*>(p_bf16)[i] = make_uint2(pack_bf16x2(pp.x, pp.y), pack_bf16x2(pp.z, pp.w));
  }
  // the last count % 4 parameters
  const int64_t t = n4 * 4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < count && t < n4 * 4 + 4) {
    float pp = p[t], mm = m[t], vv = v[t];
    adam1(pp, g[t], mm, vv, c);
    p[t] = pp;
    m[t] = mm;
    v[t] = vv;
    if (p_bf16 != nullptr) p_bf16[t] = __bfloat16_as_ushort(__float2bfloat16_rn(pp));
  }
}

}  // namespace

cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, uint16_t* p_bf16, int64_t count, float lr,
                         float beta1, float beta2, float eps, float weight_decay, float grad_scale, int32_t step,
                         int num_sms, cudaStream_t st) {
  AdamCoef c;
  c.b1 = beta1;
  c.b2 = beta2;
  c.one_m_b1 = static_cast<float>(1.0 - static_cast<double>(beta1));
  c.one_m_b2 = static_cast<float>(1.0 - static_cast<double>(beta2));
  const double bc1 = 1.0 - std::pow(static_cast<double>(beta1), step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(beta2), step);
  c.step_size = static_cast<float>(static_cast<double>(lr) / bc1);
  c.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
  c.eps = eps;
  c.decay = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(weight_decay));
  c.gscale = grad_scale;
  int64_t blocks = (count / 4 + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  if (blocks < 1) blocks = 1;
  return launch_pdl(adamw_kernel, static_cast<int>(blocks), 256, 0, st, 1, p, g, m, v, p_bf16, count, c);
}

}  // namespace qlora
