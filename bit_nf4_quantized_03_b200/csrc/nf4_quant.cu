// NF4 quantization (first level), double quantization of the block scales
// (second level) and standalone dequantization to BF16.
//
// Format, as defined by "QLoRA: Quantized Low-Rank Adaptation"
// (completesystemdesign.dev), Piece 1 / Piece 2 and the section "NF4: a
// 4-bit format matched to weight statistics": blocks of 64 consecutive
// weights, one absmax scale per block, each weight snapped to the nearest of
// 16 levels and stored in 4 bits (element 2j in the low nibble of byte j).
// "Double quantization (the label-index-card trick)" stores the scales
// themselves as 8-bit floats (E4M3) in blocks of 256 with one fp32 scale per
// block and one fp32 mean offset per tensor.
#include "qlora_device.cuh"
#include "qlora_kernels.h"

namespace qlora {

__device__ int g_device_error = 0;

// ---------------------------------------------------------------------------
// Stage 1: absmax, codes, plain scales / fp32 absmax for double quant.
// Each half-warp owns one 64-block: 16 lanes x float4 (128-bit loads).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t nf4_code(float x, const Nf4Table& t) {
  // number of thresholds strictly below x (a value on a threshold rounds down)
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) c += (x > t.mid[i]) ? 1u : 0u;
  return c;
}

template <bool kDQ>
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const float* __restrict__ W, int64_t n_elem,
                                                           Nf4Table tab, uint8_t* __restrict__ codes,
                                                           uint16_t* __restrict__ scale_bf16,
                                                           float* __restrict__ absmax_out) {
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const int64_t nfull = n_elem / 64;                     // complete blocks
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float4* W4 = reinterpret_cast<const float4*>(W);

  constexpr int U = 4;   // block pairs in flight per warp
  for (int64_t base = warp * 2 * U; base < nfull; base += nwarps * 2 * U) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t b = base + 2 * u + (lane >> 4);
      v[u] = (b < nfull) ? __ldcs(W4 + b * 16 + hl) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t b = base + 2 * u + (lane >> 4);
      float m = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      uint32_t q;
      if (m < 1.17549435e-38f) {          // zero or subnormal absmax: exact-zero level
        q = 0x7777u;
      } else {
        const float inv = __frcp_rn(m);
        q = nf4_code(__fmul_rn(v[u].x, inv), tab) | (nf4_code(__fmul_rn(v[u].y, inv), tab) << 4) |
            (nf4_code(__fmul_rn(v[u].z, inv), tab) << 8) | (nf4_code(__fmul_rn(v[u].w, inv), tab) << 12);
      }
      if (b < nfull) {
        reinterpret_cast<uint16_t*>(codes)[b * 16 + hl] = static_cast<uint16_t>(q);
        if (hl == 0) {
          if (kDQ) absmax_out[b] = m;
          else scale_bf16[b] = __bfloat16_as_ushort(__float2bfloat16_rn(m));
        }
      }
    }
  }

  // ragged last block (n_elem % 64 != 0): one warp, scalar loads
  const int64_t tail = n_elem - nfull * 64;
  if (tail > 0 && blockIdx.x == 0 && threadIdx.x < 32) {
    const int64_t b = nfull;
    float w0 = (2 * lane < tail) ? W[b * 64 + 2 * lane] : 0.f;
    float w1 = (2 * lane + 1 < tail) ? W[b * 64 + 2 * lane + 1] : 0.f;
    float m = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    uint32_t c0 = 7, c1 = 7;
    if (m >= 1.17549435e-38f) {
      const float inv = __frcp_rn(m);
      c0 = nf4_code(__fmul_rn(w0, inv), tab);
      c1 = nf4_code(__fmul_rn(w1, inv), tab);
    }
    if (2 * lane + 1 >= tail) c1 = 0;    // odd tail: high nibble stays 0
    if (2 * lane < tail) codes[b * 32 + lane] = static_cast<uint8_t>(c0 | (c1 << 4));
    if (lane == 0) {
      if (kDQ) absmax_out[b] = m;
      else scale_bf16[b] = __bfloat16_as_ushort(__float2bfloat16_rn(m));
    }
  }
}

// ---------------------------------------------------------------------------
// Fixed-order fp64 sum of the absmax values: a pairwise tree over the array
// zero-padded to a power of two. Each pass reduces aligned chunks of 512 to
// one value with the same tree shape, so chaining passes gives exactly the
// tree over the padded array (adding exact zeros changes nothing).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) pairwise_sum_pass(const T* __restrict__ in, int64_t n_in,
                                                          double* __restrict__ out, int64_t count_for_mean,
                                                          float* __restrict__ mean_out) {
  __shared__ double s[256];
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * 512 + 2 * threadIdx.x;
  const double a = (i0 < n_in) ? static_cast<double>(in[i0]) : 0.0;
  const double b = (i0 + 1 < n_in) ? static_cast<double>(in[i0 + 1]) : 0.0;
  s[threadIdx.x] = a + b;
  __syncthreads();
  for (int stride = 1; stride < 256; stride <<= 1) {
    if ((threadIdx.x & (2 * stride - 1)) == 0) s[threadIdx.x] = s[threadIdx.x] + s[threadIdx.x + stride];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[blockIdx.x] = s[0];
    if (mean_out != nullptr) *mean_out = static_cast<float>(s[0] / static_cast<double>(count_for_mean));
  }
}

// ---------------------------------------------------------------------------
// Stage 2: per 256-block, d = a - mean, s2 = max|d| / 448, q = e4m3(d / s2).
// One CTA of 256 threads per second-level block.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_fp8_kernel(const float* __restrict__ absmax, int64_t nblk,
                                                      const float* __restrict__ mean_in,
                                                      uint8_t* __restrict__ q_out,
                                                      float* __restrict__ s2_out,
                                                      float* __restrict__ mean_out) {
  __shared__ float wmax[8];
  const float mean = *mean_in;
  const int64_t b = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const bool valid = b < nblk;
  const float d = valid ? __fsub_rn(absmax[b], mean) : 0.f;
  float m = fabsf(d);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, wmax[i]);
  const float s2 = (amax == 0.f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (valid) {
    q_out[b] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fdiv_rn(d, s2), __NV_SATFINITE, __NV_E4M3));
  }
  if (threadIdx.x == 0) {
    s2_out[blockIdx.x] = s2;
    if (blockIdx.x == 0) *mean_out = mean;
  }
}

// ---------------------------------------------------------------------------
// Standalone dequantization: one thread per 64-block, table lookups, 128-bit
// loads of codes and 128-bit stores of bf16.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) nf4_dequantize_kernel(const uint8_t* __restrict__ codes, ScaleSrc ss,
                                                             int64_t n_elem, Nf4Table tab,
                                                             uint16_t* __restrict__ out) {
  const int64_t nfull = n_elem / 64;
  const float mean = (ss.dq_mean != nullptr) ? __ldg(ss.dq_mean) : 0.f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nfull; b += stride) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + b * 32);
    const uint4 c0 = __ldcs(src);
    const uint4 c1 = __ldcs(src + 1);
    const Nf4Lut lut = nf4_build_lut(tab, block_scale(ss, b, mean));
    uint4* dst = reinterpret_cast<uint4*>(out + b * 64);
    __stcs(dst + 0, nf4_lookup8(lut, c0.x));
    __stcs(dst + 1, nf4_lookup8(lut, c0.y));
    __stcs(dst + 2, nf4_lookup8(lut, c0.z));
    __stcs(dst + 3, nf4_lookup8(lut, c0.w));
    __stcs(dst + 4, nf4_lookup8(lut, c1.x));
    __stcs(dst + 5, nf4_lookup8(lut, c1.y));
    __stcs(dst + 6, nf4_lookup8(lut, c1.z));
    __stcs(dst + 7, nf4_lookup8(lut, c1.w));
  }
  const int64_t tail = n_elem - nfull * 64;
  if (tail > 0 && blockIdx.x == 0 && threadIdx.x < tail) {
    const int64_t b = nfull;
    const int i = threadIdx.x;
    const uint8_t byte = codes[b * 32 + i / 2];
    const uint32_t code = (i & 1) ? (byte >> 4) : (byte & 15u);
    const Nf4Lut lut = nf4_build_lut(tab, block_scale(ss, b, mean));
    uint32_t v01, v23;
    nf4_lookup4(lut, code, v01, v23);
    out[b * 64 + i] = static_cast<uint16_t>(v01 & 0xFFFFu);
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static int grid_for(int64_t work_items, int per_cta, int max_ctas) {
  int64_t g = (work_items + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  if (g > max_ctas) g = max_ctas;
  return static_cast<int>(g);
}

cudaError_t launch_quantize(const float* W, int64_t n_elem, const Nf4Table& tab, uint8_t* codes,
                            uint16_t* scale_bf16, uint8_t* scale_fp8, float* dq_scale, float* dq_mean,
                            void* ws, int num_sms, cudaStream_t st) {
  const int64_t nblk = (n_elem + 63) / 64;
  const bool dq = (scale_fp8 != nullptr);
  // each warp covers 8 blocks per iteration; aim for several waves of 8 warps per SM
  const int grid = grid_for((nblk + 63) / 64, 1, num_sms * 8);
  float* absmax = reinterpret_cast<float*>(ws);
  if (dq) {
    nf4_quantize_kernel<true><<<grid, 256, 0, st>>>(W, n_elem, tab, codes, nullptr, absmax);
    count_launches(1);
  } else {
    nf4_quantize_kernel<false><<<grid, 256, 0, st>>>(W, n_elem, tab, codes, scale_bf16, nullptr);
    count_launches(1);
    return cudaGetLastError();
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // fixed-order fp64 sum -> mean (into the ws slot after the partial sums)
  const QuantWsLayout L = quant_ws_layout(n_elem);
  double* part_a = reinterpret_cast<double*>(static_cast<char*>(ws) + L.part_a_off);
  double* part_b = reinterpret_cast<double*>(static_cast<char*>(ws) + L.part_b_off);
  float* mean_tmp = reinterpret_cast<float*>(static_cast<char*>(ws) + L.mean_off);
  int64_t n = nblk;
  int64_t g = (n + 511) / 512;
  pairwise_sum_pass<float><<<static_cast<int>(g), 256, 0, st>>>(absmax, n, part_a, nblk,
                                                                 g == 1 ? mean_tmp : nullptr);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  double* src = part_a;
  double* dst = part_b;
  while (g > 1) {
    n = g;
    g = (n + 511) / 512;
    pairwise_sum_pass<double><<<static_cast<int>(g), 256, 0, st>>>(src, n, dst, nblk,
                                                                    g == 1 ? mean_tmp : nullptr);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    double* t = src;
    src = dst;
    dst = t;
  }
  const int64_t nb2 = (nblk + 255) / 256;
  dq_fp8_kernel<<<static_cast<int>(nb2), 256, 0, st>>>(absmax, nblk, mean_tmp, scale_fp8, dq_scale, dq_mean);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const ScaleSrc& ss, int64_t n_elem, const Nf4Table& tab,
                              uint16_t* out, int num_sms, cudaStream_t st) {
  const int64_t nblk = (n_elem + 63) / 64;
  const int grid = grid_for(nblk, 256, num_sms * 8);
  nf4_dequantize_kernel<<<grid, 256, 0, st>>>(codes, ss, n_elem, tab, out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
