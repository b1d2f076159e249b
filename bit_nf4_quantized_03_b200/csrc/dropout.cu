// LoRA dropout on the input of the low-rank branch ("QLoRA Explained",
// Step 3: LoraConfig lora_dropout = 0.05, and its hyperparameter quick
// reference). Inverted dropout as PEFT applies it: the branch sees M * X and
// its result is scaled by 1 / (1 - p) (folded into the low-rank finalize and
// the masked dX epilogue, so the masked activations stay exact in bf16).
//
// The keep mask comes from the counter-based generator Philox4x32-10
// (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2,
// 3", SC 2011): counter = (e / 8 as two 32-bit words, offset as two words),
// key = seed as two words. Element e of X (row-major) uses 16-bit lane e % 8
// of the four output words (word (e % 8) / 2, low half first) and is kept iff
// that value >= round(p * 65536). One generator call covers the eight
// elements of one 16-byte vector of X, so each thread handles eight elements
// per call and writes one mask byte (bit j = element 8g + j).
#include "qlora_kernels.h"

namespace qlora {

namespace {

struct Words4 {
  uint32_t w[4];
};

__device__ __forceinline__ Words4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                                uint32_t k1) {
#pragma unroll
  for (int rnd = 0; rnd < 10; ++rnd) {
    const uint32_t lo0 = 0xD2511F53u * c0;
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2);
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    if (rnd < 9) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
  }
  return Words4{{c0, c1, c2, c3}};
}

// zero the bf16 elements of a 16-byte vector whose mask bit is clear
__device__ __forceinline__ uint4 apply_bits(uint4 x, uint32_t bits) {
  uint32_t v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t keep_lo = ((bits >> (2 * j)) & 1u) ? 0x0000FFFFu : 0u;
    const uint32_t keep_hi = ((bits >> (2 * j + 1)) & 1u) ? 0xFFFF0000u : 0u;
    v[j] &= (keep_lo | keep_hi);
  }
  return make_uint4(v[0], v[1], v[2], v[3]);
}

__global__ void __launch_bounds__(256) dropout_mask_kernel(const uint4* __restrict__ X, int64_t groups, uint32_t thr,
                                                           uint64_t seed, uint64_t offset, uint4* __restrict__ Xd,
                                                           uint8_t* __restrict__ mask) {
  griddep_enter();
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const uint32_t c2 = static_cast<uint32_t>(offset), c3 = static_cast<uint32_t>(offset >> 32);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const Words4 r = philox4x32_10(static_cast<uint32_t>(g), static_cast<uint32_t>(static_cast<uint64_t>(g) >> 32),
                                   c2, c3, k0, k1);
    uint32_t bits = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t r16 = (r.w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
      bits |= (r16 >= thr ? 1u : 0u) << j;
    }
    Xd[g] = apply_bits(__ldcs(X + g), bits);
    mask[g] = static_cast<uint8_t>(bits);
  }
}

__global__ void __launch_bounds__(256) mask_apply_kernel(const uint4* __restrict__ X, int64_t groups,
                                                         const uint8_t* __restrict__ mask, uint4* __restrict__ Xd) {
  griddep_enter();
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x)
    Xd[g] = apply_bits(__ldcs(X + g), __ldg(mask + g));
}

int grid_for(int64_t groups) {
  int64_t g = (groups + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_dropout_mask(const uint16_t* X, int64_t count, uint32_t thr, uint64_t seed, uint64_t offset,
                                uint16_t* Xd, uint8_t* mask, cudaStream_t st) {
  const int64_t groups = count / 8;
  return launch_pdl(dropout_mask_kernel, grid_for(groups), 256, 0, st, 1, reinterpret_cast<const uint4*>(X), groups,
                    thr, seed, offset, reinterpret_cast<uint4*>(Xd), mask);
}

cudaError_t launch_mask_apply(const uint16_t* X, int64_t count, const uint8_t* mask, uint16_t* Xd, cudaStream_t st) {
  const int64_t groups = count / 8;
  return launch_pdl(mask_apply_kernel, grid_for(groups), 256, 0, st, 1, reinterpret_cast<const uint4*>(X), groups,
                    mask, reinterpret_cast<uint4*>(Xd));
}

}  // namespace qlora
