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
#include <cstring>

#include "qlora_device.cuh"
#include <utility>

#include "qlora_kernels.h"

namespace qlora {

__device__ int g_device_error = 0;
__device__ int g_bounds_site = 0;

// ---------------------------------------------------------------------------
// Stage 1: absmax, codes, plain scales / fp32 absmax for double quant.
//
// The weights stream through a 3-stage shared-memory ring filled by TMA: the
// tensor is viewed as rows of one 64-block (256 B), and each 32 KB chunk of
// 128 blocks arrives as two 128-row boxes of half-blocks, 128-byte swizzled,
// so lanes reading the same offset of different blocks hit different banks.
// Two lanes share one 64-block (32 weights each): one shuffle gives the
// block's absmax, each lane takes the IEEE reciprocal and searches the codes
// of its 32 weights (32 independent chains), and writes them as one 16-byte
// store. A ragged last block is read from global memory.
//
// The code of x = w * (1/absmax) is found with one comparison: x's bucket is
// j = round(16 x) (-16 .. 16), the buckets [j/16 - 1/32, j/16 + 1/32] widened
// by 1e-3; a widened bucket holds at most one decision threshold (neighbouring
// thresholds are >= 0.08 apart), so code = (thresholds below the bucket) +
// (x > the bucket's threshold), exactly the number of thresholds strictly
// below x. j comes out of one fused multiply-add, 1.5 * 2^23 + 16 x rounded to
// an integer (the sum's ulp is 1), whose low six bits, inserted at bit 3 of
// the 512-byte aligned table's address, address the 8-byte entry of j mod 64;
// the widening covers ties and the rounding.
//
// In double-quant mode each chunk's 128 absmax values are also reduced in
// fp64 with the fixed pairwise tree (the first levels of the tensor-wide sum
// that defines the mean): 16 blocks per warp by shuffles, then the chunk's 8
// warp sums.
// ---------------------------------------------------------------------------
constexpr int kQChunk = 128;     // 64-blocks per chunk: 32 KB of fp32 weights
constexpr int kQStages = 3;
constexpr int kQCtasPerSm = 2;    // resident CTAs per SM (shared memory: kQStages stages each)
constexpr int kQStage = kQChunk * 256;                // bytes per stage: two 16 KB boxes of half-blocks
constexpr int kQSmem = kQStages * kQStage + 1024;     // + alignment of the swizzled stages

__device__ __forceinline__ uint32_t nf4_code_bucket(float x, uint32_t tab_addr) {
  const float r = __fmaf_rn(x, 16.0f, 12582912.0f);     // 1.5 * 2^23 + round(16 x)
  uint32_t a;
  asm("bfi.b32 %0, %1, %2, 3, 6;" : "=r"(a) : "r"(__float_as_uint(r)), "r"(tab_addr));
  float thr;
  uint32_t base;
  asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(thr), "=r"(base) : "r"(a));
  return base + ((x > thr) ? 1u : 0u);
}

__device__ __forceinline__ uint32_t bfi4(uint32_t word, uint32_t code, uint32_t pos) {
  uint32_t d;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(d) : "r"(code), "r"(word), "r"(pos));
  return d;
}

// Codes of one lane's eight weights (x = w * inv); the first four (lo) go to
// nibbles 0..3 of the 16-bit result, the next four (hi) to nibbles 4..7.
__device__ __forceinline__ uint32_t nf4_codes8(const float4& lo, const float4& hi, float inv, uint32_t tab) {
  uint32_t w = 0;
  w = bfi4(w, nf4_code_bucket(__fmul_rn(lo.x, inv), tab), 0);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(lo.y, inv), tab), 4);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(lo.z, inv), tab), 8);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(lo.w, inv), tab), 12);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(hi.x, inv), tab), 16);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(hi.y, inv), tab), 20);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(hi.z, inv), tab), 24);
  w = bfi4(w, nf4_code_bucket(__fmul_rn(hi.w, inv), tab), 28);
  return w;
}

__device__ __forceinline__ float absmax8(const float4& a, const float4& b) {
  return fmaxf(fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))),
               fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
}

// Fixed pairwise tree (fp64) over part[0..n) zero-padded to a power of two,
// by one CTA (any multiple of 32 threads: the warps only share out the groups,
// the tree is the same), without writing global memory. Each warp reduces an
// aligned group of 512: lane l loads elements l, l + 32, ..., l + 480 of the
// group (coalesced); five xor-shuffle levels sum each aligned run of 32
// (neighbouring elements sit in neighbouring lanes, and a + b == b + a
// exactly, so each node is the same left + right), and four levels inside the
// lane pair up the 16 runs. The group sums go to shared memory and the next
// level runs on them, until one value is left. Zero padding at any level
// leaves the result unchanged (x + 0 == x), so this equals the tree over the
// whole power-of-two-padded array. `buf` holds 2 * kTreeBuf doubles.
constexpr int kTreeBuf = 2048;               // group sums per level: n <= 2048 * 512 on the first level

__device__ double tree_sum_cta(const double* __restrict__ part, int64_t n, double* buf) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double* src = part;
  bool global_src = true;
  int pp = 0;
  while (n > 1) {
    const int64_t groups = (n + 511) / 512;
    double* dst = buf + pp * kTreeBuf;
    for (int64_t g = warp; g < groups; g += (blockDim.x >> 5)) {
      double v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int64_t idx = g * 512 + j * 32 + lane;
        v[j] = (idx < n) ? (global_src ? __ldcg(src + idx) : src[idx]) : 0.0;
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1)
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = v[j] + __shfl_xor_sync(0xffffffffu, v[j], off);
#pragma unroll
      for (int w = 1; w < 16; w <<= 1)
#pragma unroll
        for (int j = 0; j < 16; j += 2 * w) v[j] = v[j] + v[j + w];
      if (lane == 0) dst[g] = v[0];
    }
    __syncthreads();
    src = dst;
    global_src = false;
    pp ^= 1;
    n = groups;
  }
  const double r = global_src ? __ldcg(src) : src[0];
  __syncthreads();
  return r;
}

template <bool kDQ>
__global__ void __launch_bounds__(256, kQCtasPerSm) nf4_quantize_kernel(const __grid_constant__ CUtensorMap wmap,
                                                              const float* __restrict__ W, int64_t n_elem,
                                                              Nf4Buckets bk, uint8_t* __restrict__ codes,
                                                              uint16_t* __restrict__ scale_bf16,
                                                              float* __restrict__ absmax_out,
                                                              double* __restrict__ part_out) {
  extern __shared__ __align__(16) uint8_t q_raw[];    // aligned to 1024 below, at run time (the runtime places it after the static arrays)
  uint8_t* q_stage = q_raw + ((1024u - (smem_u32(q_raw) & 1023u)) & 1023u);
  if ((smem_u32(q_stage) & 1023u) != 0u) {   // the swizzled TMA boxes need a 1024-byte aligned stage
    if (threadIdx.x == 0) atomicExch(&g_device_error, kErrBadLayout);
    return;
  }
  __shared__ __align__(512) float2 s_tab[64];       // entry j mod 64 for bucket j = round(16 x)
  __shared__ double s_part[2][8];             // per chunk: the eight warps' sums of 16 blocks (by chunk parity)
  __shared__ __align__(8) uint64_t full[kQStages];
  const int tid = threadIdx.x;
  const int h = tid & 1;                      // half of the block: elements 32h .. 32h + 31
  const int lb = tid >> 1;                    // block within the chunk
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t nfull = n_elem / 64;
  const int64_t tail = n_elem - nfull * 64;
  const int64_t nblk = nfull + (tail > 0 ? 1 : 0);
  const int64_t nchunks = (nblk + kQChunk - 1) / kQChunk;
  const int64_t my_n = (nchunks > blockIdx.x) ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if ((smem_u32(s_tab) & 511u) != 0u) {      // the bucket address is built by inserting bits 3..8
    if (tid == 0) atomicExch(&g_device_error, kErrBadLayout);
    return;
  }
  if (tid < 64) {
    // slot t holds bucket j = t (t < 32) or t - 64; only j = -16 .. 16 are ever indexed
    const int j = (tid < 32) ? tid : tid - 64;
    s_tab[tid] = (j >= -16 && j <= 16) ? make_float2(bk.thr[j + 16], __int_as_float(bk.base[j + 16]))
                                       : make_float2(__int_as_float(0x7f800000), __int_as_float(15));
  }
  if (tid == 0) {
    for (int st = 0; st < kQStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
    if (nfull > 0) tma_prefetch_desc(&wmap);
  }
  __syncthreads();
  // launched with programmatic dependence: W may still be being written by the kernel
  // before this one until this returns; the kernel after this one may be scheduled now
  griddep_wait();
  griddep_launch_dependents();
  auto issue = [&](int64_t i) {
    const int64_t b0 = (blockIdx.x + i * gridDim.x) * kQChunk;
    const int st = static_cast<int>(i % kQStages);
    if (b0 < nfull) {
      // rows past nfull arrive zero-filled and are counted in full
      uint8_t* dst = q_stage + st * kQStage;
      mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(kQStage));
      if (tma_start_ok(0, static_cast<int32_t>(b0), 4, 64, dst, 50) && qlora_check(b0 < nfull, 51))
        tma_load_2d(dst, &wmap, &full[st], 0, static_cast<int32_t>(b0));
      if (tma_start_ok(32, static_cast<int32_t>(b0), 4, 64, dst + kQStage / 2, 52))
        tma_load_2d(dst + kQStage / 2, &wmap, &full[st], 32, static_cast<int32_t>(b0));
    } else {
      mbar_arrive(&full[st]);                  // only the ragged last block: read from global memory
    }
  };
  if (tid == 0)
    for (int64_t i = 0; i < my_n && i < kQStages; ++i) issue(i);
  const uint32_t swz = static_cast<uint32_t>(lb & 7);       // 128-byte swizzle of this lane's row
  for (int64_t i = 0; i < my_n; ++i) {
    const int st = static_cast<int>(i % kQStages);
    if (!mbar_wait(&full[st], static_cast<uint32_t>((i / kQStages) & 1))) break;
    const int64_t b0 = (blockIdx.x + i * gridDim.x) * kQChunk;
    const int64_t b = b0 + lb;
    // block class: 0 = whole block in the stage, 1 = ragged last block, 2 = past the tensor
    const int cls = (b < nfull) ? 0 : ((b == nfull && tail > 0) ? 1 : 2);
    float4 v[8];
    if (cls == 0) {
      const uint32_t row = smem_u32(q_stage + st * kQStage + h * (kQStage / 2)) + static_cast<uint32_t>(lb) * 128u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(v[c].x), "=f"(v[c].y), "=f"(v[c].z), "=f"(v[c].w)
                     : "r"(row + ((static_cast<uint32_t>(c) ^ swz) << 4))
                     : "memory");
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float* f = reinterpret_cast<float*>(&v[c]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t el = 32 * h + 4 * c + e;
          f[e] = (cls == 1 && el < tail) ? W[b * 64 + el] : 0.f;
        }
      }
    }
    float m = fmaxf(fmaxf(absmax8(v[0], v[1]), absmax8(v[2], v[3])), fmaxf(absmax8(v[4], v[5]), absmax8(v[6], v[7])));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));     // the partner lane holds the other half
    uint4 word = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);  // zero or subnormal absmax
    if (cls != 2 && m >= 1.17549435e-38f) {
      const float inv = __frcp_rn(m);
      const uint32_t tab = smem_u32(s_tab);
      word.x = nf4_codes8(v[0], v[1], inv, tab);
      word.y = nf4_codes8(v[2], v[3], inv, tab);
      word.z = nf4_codes8(v[4], v[5], inv, tab);
      word.w = nf4_codes8(v[6], v[7], inv, tab);
    }
    if (cls == 0) {
      if (qlora_check((b + 1) * 64 <= n_elem, 53)) *reinterpret_cast<uint4*>(codes + b * 32 + h * 16) = word;
    } else if (cls == 1) {
      // only the bytes that hold present elements; an odd tail keeps its high nibble 0
      const uint32_t ww[4] = {word.x, word.y, word.z, word.w};
#pragma unroll
      for (int byte = 0; byte < 16; ++byte) {
        const int64_t e0 = 32 * h + 2 * byte;
        if (e0 < tail) {
          uint32_t c = (ww[byte >> 2] >> (8 * (byte & 3))) & 0xFFu;
          if (e0 + 1 >= tail) c &= 0x0Fu;
          codes[b * 32 + 16 * h + byte] = static_cast<uint8_t>(c);
        }
      }
    }
    if (h == 0 && b < nblk) {
      if (kDQ) absmax_out[b] = m;
      else scale_bf16[b] = __bfloat16_as_ushort(__float2bfloat16_rn(m));
    }
    if (kDQ) {
      // first four levels of the fixed pairwise tree over the warp's 16 adjacent blocks
      // (lane 2j + h holds block 16 * warp + j; both lanes of a block hold its absmax)
      double t = (b < nblk) ? static_cast<double>(m) : 0.0;
      t = t + __shfl_xor_sync(0xffffffffu, t, 2);
      t = t + __shfl_xor_sync(0xffffffffu, t, 4);
      t = t + __shfl_xor_sync(0xffffffffu, t, 8);
      t = t + __shfl_xor_sync(0xffffffffu, t, 16);
      if (lane == 0) s_part[i & 1][warp] = t;
    }
    fence_proxy_async_smem();                 // reads of the stage ordered before its refill
    __syncthreads();                          // stage consumed, tree nodes written
    if (tid == 0 && i + kQStages < my_n) issue(i + kQStages);
    if (kDQ && tid < 32) {
      // remaining three levels over the chunk's 8 warp sums, in index order (xor-shuffle pairs)
      double t = (tid < 8) ? s_part[i & 1][tid] : 0.0;
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) t = t + __shfl_xor_sync(0xffffffffu, t, off);
      if (tid == 0) part_out[blockIdx.x + i * gridDim.x] = t;
    }
  }
}

// ---------------------------------------------------------------------------
// Stage 2: the mean, by one CTA of 1024 threads over the per-chunk partials
// (the rest of the fixed tree), written to dq_mean.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) dq_mean_kernel(const double* __restrict__ part, int64_t nchunks,
                                                       int64_t nblk, float* __restrict__ mean_out) {
  __shared__ double tree_buf[2 * kTreeBuf];
  griddep_wait();                      // the partials of stage 1 are complete and visible
  griddep_launch_dependents();
  const double S = tree_sum_cta(part, nchunks, tree_buf);
  if (threadIdx.x == 0) *mean_out = static_cast<float>(S / static_cast<double>(nblk));
}

// ---------------------------------------------------------------------------
// Stage 3: per 256-block d = a - mean, s2 = max|d| / 448, q = e4m3(d / s2).
// Each CTA takes up to kFinishPer 256-blocks (one absmax per thread each),
// requested together, and reduces all of them in one barrier.
// ---------------------------------------------------------------------------
constexpr int kFinishPer = 8;                 // 256-blocks per CTA, loaded up front

__global__ void __launch_bounds__(256) dq_finish_kernel(const float* __restrict__ mean_in,
                                                         const float* __restrict__ absmax, int64_t nblk,
                                                         uint8_t* __restrict__ q_out, float* __restrict__ s2_out) {
  __shared__ float wmax[kFinishPer][8];
  griddep_wait();                      // the mean (and, before it, stage 1's absmax values) are visible
  griddep_launch_dependents();
  const int64_t nb2 = (nblk + 255) / 256;
  float a[kFinishPer];
#pragma unroll
  for (int j = 0; j < kFinishPer; ++j) {
    const int64_t b = (static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(j) * gridDim.x) * 256 + threadIdx.x;
    a[j] = (b < nblk) ? __ldcg(absmax + b) : 0.f;
  }
  const float mean = __ldcg(mean_in);
  float d[kFinishPer];
#pragma unroll
  for (int j = 0; j < kFinishPer; ++j) {
    const int64_t b = (static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(j) * gridDim.x) * 256 + threadIdx.x;
    d[j] = (b < nblk) ? __fsub_rn(a[j], mean) : 0.f;
    float m = fabsf(d[j]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) wmax[j][threadIdx.x >> 5] = m;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kFinishPer; ++j) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(j) * gridDim.x;
    if (c >= nb2) break;
    float amax = wmax[j][0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, wmax[j][i]);
    const float s2 = (amax == 0.f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    const int64_t b = c * 256 + threadIdx.x;
    if (b < nblk) q_out[b] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fdiv_rn(d[j], s2), __NV_SATFINITE, __NV_E4M3));
    if (threadIdx.x == 0) s2_out[c] = s2;
  }
}

// ---------------------------------------------------------------------------
// Standalone dequantization. The codes of 256 consecutive blocks (one
// second-level scale block, 8 KB) are streamed into a 3-stage shared-memory
// ring by bulk copies; each lane expands one 64-block through the per-block
// lookup table into a 128-byte row of a per-warp stage (16-byte chunks
// XOR-swizzled by the row, conflict-free), and the warp then writes its 32
// rows (4 KB of contiguous output) with fully coalesced 512-byte stores.
// ---------------------------------------------------------------------------
constexpr int kDChunk = 256;
constexpr int kDStages = 3;
constexpr int kDSmem = kDStages * kDChunk * 32 + 8 * 4096;

__global__ void __launch_bounds__(256, 3) nf4_dequantize_kernel(const uint8_t* __restrict__ codes, ScaleSrc ss,
                                                                int64_t n_elem, Nf4Table tab,
                                                                uint16_t* __restrict__ out) {
  extern __shared__ __align__(128) uint8_t d_smem[];
  __shared__ __align__(8) uint64_t full[kDStages];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int64_t nfull = n_elem / 64;
  const int64_t nchunks = (nfull + kDChunk - 1) / kDChunk;
  const int64_t my_n = (nchunks > blockIdx.x) ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  uint8_t* ring = d_smem;
  const uint32_t stage_out = smem_u32(d_smem + kDStages * kDChunk * 32 + warp * 4096);
  if (tid == 0) {
    for (int st = 0; st < kDStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // launched with programmatic dependence: the codes and scales may still be being written
  // by the kernel before this one until this returns
  griddep_wait();
  griddep_launch_dependents();
  auto issue = [&](int64_t i) {
    const int64_t b0 = (blockIdx.x + i * gridDim.x) * kDChunk;
    int64_t nb = nfull - b0;
    nb = nb > kDChunk ? kDChunk : nb;
    const int st = static_cast<int>(i % kDStages);
    mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(nb * 32));
    bulk_load(ring + st * (kDChunk * 32), codes + b0 * 32, static_cast<uint32_t>(nb * 32), &full[st]);
  };
  if (tid == 0)
    for (int64_t i = 0; i < my_n && i < kDStages; ++i) issue(i);
  const float mean = (ss.dq_mean != nullptr) ? __ldg(ss.dq_mean) : 0.f;
  const uint32_t x = (lane >> 2) & 1;           // read order that keeps the two 16-byte loads conflict-free
  // the scale of this lane's block in the next chunk is loaded one chunk ahead
  float c_next = 0.f;
  {
    const int64_t bn = static_cast<int64_t>(blockIdx.x) * kDChunk + warp * 32 + lane;
    if (my_n > 0 && bn < nfull) c_next = block_scale(ss, bn, mean);
  }
  for (int64_t i = 0; i < my_n; ++i) {
    const int st = static_cast<int>(i % kDStages);
    const int64_t b0 = (blockIdx.x + i * gridDim.x) * kDChunk + warp * 32;
    const int64_t b = b0 + lane;
    const float c = c_next;
    {
      const int64_t bn = b + static_cast<int64_t>(gridDim.x) * kDChunk;
      if (i + 1 < my_n && bn < nfull) c_next = block_scale(ss, bn, mean);
    }
    if (!mbar_wait(&full[st], static_cast<uint32_t>((i / kDStages) & 1))) break;
    if (b < nfull && qlora_check(b0 >= 0, 54)) {
      const uint32_t src = smem_u32(ring + st * (kDChunk * 32) + (warp * 32 + lane) * 32);
      uint4 h0, h1;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(h0.x), "=r"(h0.y), "=r"(h0.z), "=r"(h0.w) : "r"(src + 16 * x) : "memory");
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(h1.x), "=r"(h1.y), "=r"(h1.z), "=r"(h1.w) : "r"(src + 16 * (x ^ 1)) : "memory");
      const uint4 c0 = x ? h1 : h0;
      const uint4 c1 = x ? h0 : h1;
      const Nf4Lut lut = nf4_build_lut(tab, c);
      const uint32_t row = stage_out + lane * 128;
      const int sw = lane & 7;
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = nf4_lookup8(lut, words[j]);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((j ^ sw) << 4)), "r"(v.x), "r"(v.y),
                     "r"(v.z), "r"(v.w)
                     : "memory");
      }
    }
    __syncwarp();
    const int64_t nvalid = (nfull - b0 < 32) ? (nfull - b0) : 32;
    uint4* dst = reinterpret_cast<uint4*>(out + b0 * 64);
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int o = it * 512 + lane * 16;     // byte offset in the warp's 4 KB of output
      const int blk = o >> 7;
      const int chunk = (o >> 4) & 7;
      if (blk < nvalid && qlora_check((b0 + blk + 1) * 64 <= n_elem, 55)) {
        uint4 v;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(stage_out + blk * 128 + ((chunk ^ (blk & 7)) << 4))
                     : "memory");
        __stcs(dst + (o >> 4), v);
      }
    }
    fence_proxy_async_smem();                  // reads of the stage ordered before its bulk-copy refill
    __syncthreads();                           // code stage consumed by every warp
    if (tid == 0 && i + kDStages < my_n) issue(i + kDStages);
  }
  const int64_t tail = n_elem - nfull * 64;
  if (tail > 0 && blockIdx.x == 0 && tid < tail) {
    const int64_t b = nfull;
    const int e = tid;
    const uint8_t byte = codes[b * 32 + e / 2];
    const uint32_t code = (e & 1) ? (byte >> 4) : (byte & 15u);
    const Nf4Lut lut = nf4_build_lut(tab, block_scale(ss, b, mean));
    uint32_t v01, v23;
    nf4_lookup4(lut, code, v01, v23);
    out[b * 64 + e] = static_cast<uint16_t>(v01 & 0xFFFFu);
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

template <typename K>
static cudaError_t set_smem_once(K kernel, int bytes, bool* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

cudaError_t launch_quantize(const float* W, int64_t n_elem, const Nf4Table& tab, const Nf4Buckets& bk,
                            uint8_t* codes, uint16_t* scale_bf16, uint8_t* scale_fp8, float* dq_scale,
                            float* dq_mean, void* ws, int num_sms, cudaStream_t st) {
  (void)tab;
  static bool smem_set[2][64] = {};
  const int64_t nblk = (n_elem + 63) / 64;
  const bool dq = (scale_fp8 != nullptr);
  const int64_t nchunks = (nblk + kQChunk - 1) / kQChunk;
  const int64_t slots = static_cast<int64_t>(kQCtasPerSm) * num_sms;
  const int grid = static_cast<int>(nchunks < slots ? nchunks : slots);
  // W as rows of one 64-block; boxes of 128 rows x 32 floats (128 B, swizzled)
  CUtensorMap wmap;
  std::memset(&wmap, 0, sizeof(wmap));
  const int64_t nfull = n_elem / 64;
  if (nfull > 0 && !tmap_2d(&wmap, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 64, static_cast<uint64_t>(nfull), 256, 32,
                            kQChunk, 128))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (!dq) {
    e = set_smem_once(nf4_quantize_kernel<false>, kQSmem, smem_set[0]);
    if (e != cudaSuccess) return e;
    return launch_pdl(nf4_quantize_kernel<false>, grid, 256, kQSmem, st, 1, wmap, W, n_elem, bk, codes, scale_bf16,
                      static_cast<float*>(nullptr), static_cast<double*>(nullptr));
  }
  const QuantWsLayout L = quant_ws_layout(n_elem);
  float* absmax = reinterpret_cast<float*>(static_cast<char*>(ws) + L.absmax_off);
  double* part_a = reinterpret_cast<double*>(static_cast<char*>(ws) + L.part_a_off);
  // stage 1 also writes one fp64 tree sum per chunk (the first levels of the fixed-order sum)
  e = set_smem_once(nf4_quantize_kernel<true>, kQSmem, smem_set[1]);
  if (e != cudaSuccess) return e;
  e = launch_pdl(nf4_quantize_kernel<true>, grid, 256, kQSmem, st, 1, wmap, W, n_elem, bk, codes,
                 static_cast<uint16_t*>(nullptr), absmax, part_a);
  if (e != cudaSuccess) return e;
  // the rest of the tree and the mean (one CTA), then the E4M3 pass
  e = launch_pdl(dq_mean_kernel, 1, 1024, 0, st, 1, static_cast<const double*>(part_a), nchunks, nblk, dq_mean);
  if (e != cudaSuccess) return e;
  const int64_t nb2 = (nblk + 255) / 256;
  // enough CTAs that each takes at most kFinishPer 256-blocks, at least one per SM when there is work
  int64_t g2 = (nb2 + kFinishPer - 1) / kFinishPer;
  if (g2 < num_sms) g2 = nb2 < num_sms ? nb2 : num_sms;
  const int grid2 = static_cast<int>(g2);
  return launch_pdl(dq_finish_kernel, grid2, 256, 0, st, 1, static_cast<const float*>(dq_mean),
                    static_cast<const float*>(absmax), nblk, scale_fp8, dq_scale);
}

cudaError_t launch_dequantize(const uint8_t* codes, const ScaleSrc& ss, int64_t n_elem, const Nf4Table& tab,
                              uint16_t* out, int num_sms, cudaStream_t st) {
  static bool smem_set[64] = {};
  const cudaError_t e = set_smem_once(nf4_dequantize_kernel, kDSmem, smem_set);
  if (e != cudaSuccess) return e;
  const int64_t nfull = n_elem / 64;
  const int64_t nchunks = (nfull + kDChunk - 1) / kDChunk;
  int64_t grid = nchunks < 3LL * num_sms ? nchunks : 3LL * num_sms;
  if (grid < 1) grid = 1;
  return launch_pdl(nf4_dequantize_kernel, static_cast<int>(grid), 256, kDSmem, st, 1, codes, ss, n_elem, tab, out);
}

}  // namespace qlora
