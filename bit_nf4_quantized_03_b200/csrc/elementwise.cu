// Small memory-bound kernels around the tensor-core GEMMs: split reductions
// of the low-rank products, hi/lo bf16 splitting, gradient finalisation and
// the SiLU-gated glue between the MLP projections.
#include <cstring>
#include "qlora_kernels.h"

namespace qlora {

__device__ __forceinline__ uint16_t f2bf(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// sum over t < splits of src[t * stride], in the order t = 0, 1, ... (the same value as a
// plain loop), with eight loads in flight at a time instead of one
__device__ __forceinline__ float sum_splits(const float* __restrict__ src, int splits, int64_t stride) {
  float s = 0.f;
  for (int t0 = 0; t0 < splits; t0 += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = (t0 + u < splits) ? __ldcg(src + static_cast<int64_t>(t0 + u) * stride) : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t0 + u < splits) s += v[u];
  }
  return s;
}

static int blocks_for(int64_t n, int threads) {
  int64_t g = (n + threads - 1) / threads;
  if (g > 148 * 32) g = 148 * 32;
  return static_cast<int>(g < 1 ? 1 : g);
}

// U (or G) = sum over split partials [split][rows][r_pad], fixed order.
// Writes any of: fp32 [rows, r]; bf16(scale * U) [rows, r_pad]; hi/lo bf16 [rows, r_pad].
// With `extra_src`, the same pass also splits a second fp32 [rows, r] matrix into hi/lo
// bf16 [rows, r_pad] (the saved U next to G in the backward): one launch for both.
__global__ void lora_finalize_kernel(const float* __restrict__ part, int splits, int64_t part_stride, int64_t rows,
                                     int r, int r_pad, float scale, float* __restrict__ out_f32,
                                     uint16_t* __restrict__ out_scaled, uint16_t* __restrict__ out_hi,
                                     uint16_t* __restrict__ out_lo, float pre, const float* __restrict__ extra_src,
                                     uint16_t* __restrict__ extra_hi, uint16_t* __restrict__ extra_lo) {
  griddep_enter();
  const int64_t total = rows * r_pad;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = idx / r_pad;
    const int j = static_cast<int>(idx - row * r_pad);
    float s = (j < r) ? sum_splits(part + idx, splits, part_stride) : 0.f;
    s = __fmul_rn(pre, s);
    if (out_f32 != nullptr && j < r) out_f32[row * r + j] = s;
    if (out_scaled != nullptr) out_scaled[idx] = f2bf(__fmul_rn(scale, s));
    if (out_hi != nullptr) {
      const uint16_t h = f2bf(s);
      out_hi[idx] = h;
      out_lo[idx] = f2bf(__fsub_rn(s, bf2f(h)));
    }
    if (extra_src != nullptr) {
      const float e = (j < r) ? extra_src[row * r + j] : 0.f;
      const uint16_t h = f2bf(e);
      extra_hi[idx] = h;
      extra_lo[idx] = f2bf(__fsub_rn(e, bf2f(h)));
    }
  }
}

cudaError_t launch_lora_finalize(const float* part, int splits, int64_t part_stride, int64_t rows, int32_t r,
                                 int32_t r_pad, float scale, float* out_f32, uint16_t* out_scaled_bf16,
                                 uint16_t* out_hi, uint16_t* out_lo, cudaStream_t st, float pre,
                                 const float* extra_src, uint16_t* extra_hi, uint16_t* extra_lo) {
  const int64_t total = rows * r_pad;
  return launch_pdl(lora_finalize_kernel, blocks_for(total, 256), 256, 0, st, 1, part, splits, part_stride, rows,
                    static_cast<int>(r), static_cast<int>(r_pad), scale, out_f32, out_scaled_bf16, out_hi, out_lo,
                    pre, extra_src, extra_hi, extra_lo);
}

// dB[row, j] (+)= scale * sum_t part[t][row][j]
__global__ void grad_finalize_kernel(const float* __restrict__ part, int splits, int64_t part_stride, int64_t rows,
                                     int r, int ld_part, float scale, float* __restrict__ out, int accumulate) {
  griddep_enter();
  const int64_t total = rows * r;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = idx / r;
    const int64_t j = idx - row * r;
    const float s = __fmul_rn(scale, sum_splits(part + row * ld_part + j, splits, part_stride));
    out[idx] = accumulate ? (out[idx] + s) : s;
  }
}

// dA[j, row] (+)= scale * sum_t part[t][row][j]: 32 x 32 tiles through shared memory, so
// that both the partials (rows of ld_part) and dA (rows of `rows`) are read and written
// along their contiguous dimension. 256 threads: warp w sums rows w, w + 8, ... of the
// tile (lane = j), then writes j = w, w + 8, ... (lane = row).
__global__ void __launch_bounds__(256) grad_finalize_t_kernel(const float* __restrict__ part, int splits,
                                                              int64_t part_stride, int64_t rows, int r, int ld_part,
                                                              float scale, float* __restrict__ out, int accumulate) {
  griddep_enter();
  __shared__ float tile[32][33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tr = (rows + 31) / 32;
  const int64_t tj = (r + 31) / 32;
  for (int64_t t = blockIdx.x; t < tr * tj; t += gridDim.x) {
    const int64_t row0 = (t % tr) * 32;
    const int j0 = static_cast<int>(t / tr) * 32;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rl = warp + 8 * i;
      const int64_t row = row0 + rl;
      const int j = j0 + lane;
      tile[rl][lane] = (row < rows && j < r) ? sum_splits(part + row * ld_part + j, splits, part_stride) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int jl = warp + 8 * i;
      const int j = j0 + jl;
      const int64_t row = row0 + lane;
      if (j < r && row < rows) {
        const float s = __fmul_rn(scale, tile[lane][jl]);
        const int64_t o = static_cast<int64_t>(j) * rows + row;
        out[o] = accumulate ? (out[o] + s) : s;
      }
    }
    __syncthreads();
  }
}

cudaError_t launch_grad_finalize(const float* part, int splits, int64_t part_stride, int64_t rows, int32_t r,
                                 int32_t ld_part, float scale, float* out, int transpose, int accumulate,
                                 cudaStream_t st) {
  if (transpose) {
    const int64_t tiles = ((rows + 31) / 32) * ((r + 31) / 32);
    const int grid = static_cast<int>(tiles < 148 * 8 ? tiles : 148 * 8);
    return launch_pdl(grad_finalize_t_kernel, grid < 1 ? 1 : grid, 256, 0, st, 1, part, splits, part_stride, rows,
                      static_cast<int>(r), static_cast<int>(ld_part), scale, out, accumulate);
  }
  return launch_pdl(grad_finalize_kernel, blocks_for(rows * r, 256), 256, 0, st, 1, part, splits, part_stride, rows,
                    static_cast<int>(r), static_cast<int>(ld_part), scale, out, accumulate);
}

// out[row, col] (+)= sum_t part[t][row][col], 4 columns per thread.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, int64_t part_stride, int64_t rows,
                                     int64_t cols, int64_t ld_part, void* __restrict__ out, int out_bf16,
                                     int accumulate) {
  griddep_enter();
  // eight consecutive columns per thread (cols % 8 == 0): two 16-byte partial loads per
  // split and one 16-byte BF16 (or two fp32) accesses of the output
  const int64_t c8 = cols / 8;
  const int64_t total = rows * c8;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = idx / c8;
    const int64_t col = (idx - row * c8) * 8;
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // four splits' loads in flight at a time, added in split order
    for (int t0 = 0; t0 < splits; t0 += 4) {
      float4 a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + u < splits) {
          const float4* src = reinterpret_cast<const float4*>(part + (t0 + u) * part_stride + row * ld_part + col);
          a[u] = __ldcs(src);
          b[u] = __ldcs(src + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + u < splits) {
          s[0] += a[u].x; s[1] += a[u].y; s[2] += a[u].z; s[3] += a[u].w;
          s[4] += b[u].x; s[5] += b[u].y; s[6] += b[u].z; s[7] += b[u].w;
        }
      }
    }
    if (out_bf16) {
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + row * cols + col);
      if (accumulate) {
        const uint4 y = *o;
        const uint32_t w[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[2 * j] += __uint_as_float(w[j] << 16);
          s[2 * j + 1] += __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
      uint4 r;
      r.x = pack_bf16x2(s[0], s[1]);
      r.y = pack_bf16x2(s[2], s[3]);
      r.z = pack_bf16x2(s[4], s[5]);
      r.w = pack_bf16x2(s[6], s[7]);
      *o = r;
    } else {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + row * cols + col);
      if (accumulate) {
        const float4 y0 = o[0], y1 = o[1];
        s[0] += y0.x; s[1] += y0.y; s[2] += y0.z; s[3] += y0.w;
        s[4] += y1.x; s[5] += y1.y; s[6] += y1.z; s[7] += y1.w;
      }
      o[0] = make_float4(s[0], s[1], s[2], s[3]);
      o[1] = make_float4(s[4], s[5], s[6], s[7]);
    }
  }
}

cudaError_t launch_splitk_reduce(const float* part, int splits, int64_t part_stride, int64_t rows, int64_t cols,
                                 int64_t ld_part, void* out, int out_bf16, int accumulate, cudaStream_t st) {
  if (cols % 8 != 0 || ld_part % 8 != 0) return cudaErrorInvalidValue;
  return launch_pdl(splitk_reduce_kernel, blocks_for(rows * (cols / 8), 256), 256, 0, st, 1, part, splits,
                    part_stride, rows, cols, ld_part, out, out_bf16, accumulate);
}

// ---------------------------------------------------------------------------
// U = X A^T for a few tokens on CUDA cores (the tensor-core path would pad the
// 128-row tile with mostly empty rows), finished in the same launch. A cluster of
// eight CTAs per adapter row j splits K into eight slices: each thread takes 8
// consecutive K at a stride of 1024 within its slice for every token, a fixed-order
// block reduction gives the slice's partial, and the cluster's first CTA adds the
// eight partials in slice order through distributed shared memory. It writes U
// (fp32, optional) and bf16(scale * U) for the forward's K extension; rows j >= r
// of the padded operand get zeros. The fused GEMM that follows may be launched to
// start early and overlap this kernel (it waits before reading bf16(scale * U)).
// ---------------------------------------------------------------------------
constexpr int kSmallThreads = 128;
constexpr int kSmallSlices = 8;     // CTAs per cluster (portable cluster size)

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

template <int MMAX>
__global__ void __launch_bounds__(kSmallThreads) lora_down_small_kernel(const uint16_t* __restrict__ X, int m,
                                                                       int64_t k, const uint16_t* __restrict__ A,
                                                                       int r, int r_pad, float scale, float pre,
                                                                       float* __restrict__ out_f32,
                                                                       uint16_t* __restrict__ out_scaled) {
  __shared__ float red[kSmallThreads / 32][MMAX];
  __shared__ float slice_sum[MMAX];
  // the fused GEMM launched after this kernel may start streaming its weight once every
  // CTA is past this point; it waits for this grid before it reads bf16(scale * U)
  griddep_enter();
  const int j = blockIdx.x / kSmallSlices;
  const uint32_t slice = cluster_ctarank();
  const int64_t slice_len = ((k / 8 + kSmallSlices - 1) / kSmallSlices) * 8;
  const int64_t k0 = static_cast<int64_t>(slice) * slice_len;
  const int64_t k1 = (k0 + slice_len < k) ? k0 + slice_len : k;
  float acc[MMAX];
#pragma unroll
  for (int i = 0; i < MMAX; ++i) acc[i] = 0.f;
  if (j < r) {
    for (int64_t kk = k0 + static_cast<int64_t>(threadIdx.x) * 8; kk < k1; kk += kSmallThreads * 8) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * k + kk));
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
      float af[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        af[2 * t] = __uint_as_float(aw[t] << 16);
        af[2 * t + 1] = __uint_as_float(aw[t] & 0xFFFF0000u);
      }
#pragma unroll
      for (int i = 0; i < MMAX; ++i) {
        if (i < m) {
          const uint4 x = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(i) * k + kk));
          const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            acc[i] = fmaf(__uint_as_float(xw[t] << 16), af[2 * t], acc[i]);
            acc[i] = fmaf(__uint_as_float(xw[t] & 0xFFFF0000u), af[2 * t + 1], acc[i]);
          }
        }
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < MMAX; ++i) {
    float v = acc[i];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) red[warp][i] = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kSmallThreads / 32; ++w) v += red[w][i];
    slice_sum[i] = v;
  }
  cluster_sync();                          // every slice's partial is in its CTA's shared memory
  if (slice == 0) {
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
      float u = 0.f;
      for (uint32_t t = 0; t < kSmallSlices; ++t) u += ld_shared_cluster_f32(smem_cluster_addr(&slice_sum[i], t));
      u = __fmul_rn(pre, u);
      if (out_f32 != nullptr && j < r) out_f32[static_cast<int64_t>(i) * r + j] = u;
      out_scaled[static_cast<int64_t>(i) * r_pad + j] = f2bf(__fmul_rn(scale, u));
    }
  }
  cluster_sync();                          // no CTA leaves while the first one still reads its partial
}

cudaError_t launch_lora_down_small(const uint16_t* X, int64_t m, int64_t k, const uint16_t* A, int32_t r,
                                   int32_t r_pad, float scale, float* U32, uint16_t* sU, cudaStream_t st, float pre) {
  if (m > 64 || k % 8 != 0) return cudaErrorInvalidValue;
  const int mi = static_cast<int>(m);
  const int grid = static_cast<int>(r_pad) * kSmallSlices;
  if (m <= 16)
    return launch_pdl(lora_down_small_kernel<16>, grid, kSmallThreads, 0, st, kSmallSlices, X, mi, k, A,
                      static_cast<int>(r), static_cast<int>(r_pad), scale, pre, U32, sU);
  return launch_pdl(lora_down_small_kernel<64>, grid, kSmallThreads, 0, st, kSmallSlices, X, mi, k, A,
                    static_cast<int>(r), static_cast<int>(r_pad), scale, pre, U32, sU);
}

// ---------------------------------------------------------------------------
// Self-test of the failure path: one thread waits on an mbarrier that nothing
// ever arrives on, with a short limit; the wait gives up, records the device
// error word and the kernel returns normally.
// ---------------------------------------------------------------------------
__global__ void selftest_wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  const uint32_t a = smem_u32(&bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_suspend(a, 0, kSuspendHintNs)) {   // the same suspending wait the pipelines use
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicExch(&g_device_error, kErrWaitTimeout);
      return;
    }
  }
}

cudaError_t launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t st) {
  selftest_wait_timeout_kernel<<<1, 1, 0, st>>>(limit_ns);
  count_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Expansion rate: how many weights per SM-clock the NF4 expansion itself sustains
// when nothing else runs. Each thread repeatedly takes one 64-block's 32 bytes of
// codes from shared memory, builds that block's table from a fresh scale and
// looks up its 64 BF16 weights (nf4_build_lut + nf4_lookup8, the code the GEMM,
// dequantize and merge kernels run); the results are folded so that none is
// dead. Cycles are taken per CTA with clock64 around the loop.
// ---------------------------------------------------------------------------
constexpr int kExpandThreads = 512;
__device__ unsigned long long g_expand_cycles[1024];
__device__ uint32_t g_expand_sink;

__global__ void __launch_bounds__(kExpandThreads, 1) expand_rate_kernel(const __grid_constant__ Nf4Table tab,
                                                                        int iters) {
  __shared__ __align__(16) uint32_t codes[kExpandThreads * 8];
  for (int i = threadIdx.x; i < kExpandThreads * 8; i += blockDim.x)
    codes[i] = 0x9E3779B9u * static_cast<uint32_t>(i + 1 + blockIdx.x * 977);
  __syncthreads();
  const uint4* mine = reinterpret_cast<const uint4*>(codes) + 2 * threadIdx.x;
  float c = 0.01f + 1e-6f * static_cast<float>(threadIdx.x);
  uint32_t acc = 0;
  const unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    const uint4 w0 = mine[0], w1 = mine[1];
    const Nf4Lut lut = nf4_build_lut(tab, c);
    c = __fadd_rn(c, 1e-7f);
    const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 o = nf4_lookup8(lut, ws[q] ^ static_cast<uint32_t>(it));
      acc ^= o.x ^ o.y ^ o.z ^ o.w;
    }
  }
  const unsigned long long t1 = clock64();
  __syncthreads();
  if (threadIdx.x == 0) g_expand_cycles[blockIdx.x] = t1 - t0;
  if (acc == 0x5EEDF00Du) g_expand_sink = acc;
}

cudaError_t launch_expand_rate(const Nf4Table& tab, int iters, int grid, int* threads, cudaStream_t st) {
  if (grid < 1 || grid > 1024 || iters < 1) return cudaErrorInvalidValue;
  expand_rate_kernel<<<grid, kExpandThreads, 0, st>>>(tab, iters);
  count_launches(1);
  *threads = kExpandThreads;
  return cudaGetLastError();
}

cudaError_t read_expand_cycles(unsigned long long* out, int grid) {
  return cudaMemcpyFromSymbol(out, g_expand_cycles, sizeof(unsigned long long) * static_cast<size_t>(grid));
}

// ---------------------------------------------------------------------------
// SiLU-gated glue: h = silu(g) * u ; dg = dh*u*sig*(1 + g*(1-sig)), du = dh*g*sig
// ---------------------------------------------------------------------------
__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

__global__ void silu_gate_fwd_kernel(const uint16_t* __restrict__ g, const uint16_t* __restrict__ u,
                                     uint16_t* __restrict__ h, int64_t count) {
  griddep_enter();
  const int64_t n8 = count / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 gv = __ldcs(reinterpret_cast<const uint4*>(g) + i);
    const uint4 uv = __ldcs(reinterpret_cast<const uint4*>(u) + i);
    const uint32_t ga[4] = {gv.x, gv.y, gv.z, gv.w}, ua[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t o[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float g0 = __uint_as_float(ga[t] << 16), g1 = __uint_as_float(ga[t] & 0xFFFF0000u);
      const float u0 = __uint_as_float(ua[t] << 16), u1 = __uint_as_float(ua[t] & 0xFFFF0000u);
      o[t] = pack_bf16x2(g0 * sigmoidf_(g0) * u0, g1 * sigmoidf_(g1) * u1);
    }
    __stcs(reinterpret_cast<uint4*>(h) + i, make_uint4(o[0], o[1], o[2], o[3]));
  }
  for (int64_t i = n8 * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float gg = bf2f(g[i]);
    h[i] = f2bf(gg * sigmoidf_(gg) * bf2f(u[i]));
  }
}

__global__ void silu_gate_bwd_kernel(const uint16_t* __restrict__ dh, const uint16_t* __restrict__ g,
                                     const uint16_t* __restrict__ u, uint16_t* __restrict__ dg,
                                     uint16_t* __restrict__ du, int64_t count) {
  griddep_enter();
  const int64_t n8 = count / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 dv = __ldcs(reinterpret_cast<const uint4*>(dh) + i);
    const uint4 gv = __ldcs(reinterpret_cast<const uint4*>(g) + i);
    const uint4 uv = __ldcs(reinterpret_cast<const uint4*>(u) + i);
    const uint32_t da[4] = {dv.x, dv.y, dv.z, dv.w}, ga[4] = {gv.x, gv.y, gv.z, gv.w}, ua[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float d[2] = {__uint_as_float(da[t] << 16), __uint_as_float(da[t] & 0xFFFF0000u)};
      float gg[2] = {__uint_as_float(ga[t] << 16), __uint_as_float(ga[t] & 0xFFFF0000u)};
      float uu[2] = {__uint_as_float(ua[t] << 16), __uint_as_float(ua[t] & 0xFFFF0000u)};
      float rg[2], ru[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float s = sigmoidf_(gg[e]);
        ru[e] = d[e] * gg[e] * s;
        rg[e] = d[e] * uu[e] * s * (1.0f + gg[e] * (1.0f - s));
      }
      og[t] = pack_bf16x2(rg[0], rg[1]);
      ou[t] = pack_bf16x2(ru[0], ru[1]);
    }
    __stcs(reinterpret_cast<uint4*>(dg) + i, make_uint4(og[0], og[1], og[2], og[3]));
    __stcs(reinterpret_cast<uint4*>(du) + i, make_uint4(ou[0], ou[1], ou[2], ou[3]));
  }
  for (int64_t i = n8 * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float d = bf2f(dh[i]), gg = bf2f(g[i]), uu = bf2f(u[i]);
    const float s = sigmoidf_(gg);
    du[i] = f2bf(d * gg * s);
    dg[i] = f2bf(d * uu * s * (1.0f + gg * (1.0f - s)));
  }
}

cudaError_t launch_silu_gate_fwd(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t count,
                                 cudaStream_t st) {
  return launch_pdl(silu_gate_fwd_kernel, blocks_for((count + 7) / 8, 256), 256, 0, st, 1, g, u, h, count);
}

cudaError_t launch_silu_gate_bwd(const uint16_t* dh, const uint16_t* g, const uint16_t* u, uint16_t* dg,
                                 uint16_t* du, int64_t count, cudaStream_t st) {
  return launch_pdl(silu_gate_bwd_kernel, blocks_for((count + 7) / 8, 256), 256, 0, st, 1, dh, g, u, dg, du,
                    count);
}

}  // namespace qlora
