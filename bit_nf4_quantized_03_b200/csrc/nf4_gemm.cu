// Tensor-core GEMM for the low-rank branch of the layer (sm_100a): the
// skinny products U = X A^T, G = dY B and the adapter gradients dB = dY^T U,
// dA^T = X^T G. TMA-staged operand tiles in 128-byte-swizzled shared memory,
// tcgen05.mma (kind::f16, BF16 x BF16 -> FP32) accumulating in TMEM, and a
// persistent, warp-specialised schedule:
//
//   warp 0      TMA producer
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2-5   epilogue: TMEM -> registers -> global (one TMEM lane quarter each)
//
// Operands may be K-major or MN-major (the reduction over tokens reads X and
// dY transposed without a copy); the gradient variant multiplies one A tile
// by a hi and a lo bf16 B tile into the same accumulator, carrying an fp32
// operand at ~2^-17 relative precision. The reduction can be split across
// CTAs into fp32 partials (reduced later in a fixed order). The frozen NF4
// weight is handled by nf4_wgemm.cu.
#include <cudaTypedefs.h>

#include <mutex>

#include "qlora_kernels.h"

namespace qlora {

template <int kBN, int kStages, bool kAMn, int kBMode, bool kExt, bool kHiLo, int kEpiGroups = 1>
struct GemmCfg {
  static constexpr int BN = kBN;
  static constexpr int Stages = kStages;
  static constexpr bool AMn = kAMn;
  static constexpr int BMode = kBMode;
  static constexpr bool Ext = kExt;
  static constexpr bool HiLo = kHiLo;
  static constexpr bool BMn = (kBMode == kB_TmaMN);
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBTile = BN * 64 * 2;
  static constexpr int kBBytes = kBTile * (HiLo ? 2 : 1);
  // Epilogue warp groups: 1 = warps 2-5 drain both accumulator buffers in turn; 2 = warps
  // 2-5 drain buffer 0 and warps 6-9 buffer 1, so two units' output round trips overlap
  // (the masked dX pass, whose units are one K step each and bound by that round trip).
  static constexpr int EpiGroups = kEpiGroups;
  static constexpr int kThreads = (2 + 4 * kEpiGroups) * 32;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 256;
  static constexpr int kEpiStage = 4 * kEpiGroups * 32 * 32 * 4;   // one 32 x 32 fp32 chunk per epilogue warp
  static constexpr int kSmemBytes = Stages * (kABytes + kBBytes) + kEpiStage + 1024 + kBarBytes;
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM alloc size");
  static_assert(kEpiGroups == 1 || kEpiGroups == 2, "one epilogue group per accumulator buffer at most");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ void decode_unit(const GemmParams& p, int u, int& mb, int& nb, int& split,
                                            int& kt0, int& nmain, int& next) {
  split = u % p.splits;
  const int t = u / p.splits;
  nb = t % p.tiles_n;
  mb = t / p.tiles_n;
  kt0 = split * p.k_per_split;
  int kt1 = kt0 + p.k_per_split;
  if (kt1 > p.k_tiles) kt1 = p.k_tiles;
  nmain = kt1 - kt0;
  next = (split == 0) ? p.ext_tiles : 0;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Epilogue store of 32 consecutive accumulator columns of one row.
__device__ __forceinline__ void store_row32(const GemmParams& p, int split, int row, int col0,
                                            const uint32_t (&v)[32]) {
  if (row >= p.rows) return;
  if (p.out_mode == kOutPartial) {
    float* o = static_cast<float*>(p.out) + split * p.part_stride + static_cast<int64_t>(row) * p.ld_out + col0;
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(o + j) = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                      __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
    return;
  }
  const bool full = (col0 + 32 <= p.cols);
  if (p.out_mode == kOutF32) {
    float* o = static_cast<float*>(p.out) + static_cast<int64_t>(row) * p.ld_out + col0;
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 x = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                               __uint_as_float(v[j + 3]));
        if (p.accumulate) {
          const float4 y = *reinterpret_cast<const float4*>(o + j);
          x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
        }
        *reinterpret_cast<float4*>(o + j) = x;
      }
    } else {
      for (int j = 0; j < 32 && col0 + j < p.cols; ++j) {
        float x = __uint_as_float(v[j]);
        if (p.accumulate) x += o[j];
        o[j] = x;
      }
    }
    return;
  }
  // bf16
  uint16_t* o = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(row) * p.ld_out + col0;
  if (full) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      float x[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) x[t] = __uint_as_float(v[j + t]);
      if (p.accumulate) {
        const uint4 y = *reinterpret_cast<const uint4*>(o + j);
        const uint32_t yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          x[2 * t] += __uint_as_float(yy[t] << 16);
          x[2 * t + 1] += __uint_as_float(yy[t] & 0xFFFF0000u);
        }
      }
      uint4 w;
      w.x = pack_bf16x2(x[0], x[1]);
      w.y = pack_bf16x2(x[2], x[3]);
      w.z = pack_bf16x2(x[4], x[5]);
      w.w = pack_bf16x2(x[6], x[7]);
      *reinterpret_cast<uint4*>(o + j) = w;
    }
  } else {
    for (int j = 0; j < 32 && col0 + j < p.cols; ++j) {
      float x = __uint_as_float(v[j]);
      if (p.accumulate) x += __uint_as_float(static_cast<uint32_t>(o[j]) << 16);
      o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
    }
  }
}

// Masked accumulate (dropout dX) of one warp's 32 rows x NCH*32 columns of a unit:
// out += keep_scale * D where the mask bit of the element is set. Every output vector
// and mask byte of the unit is requested first (one memory round trip per unit); then
// each 32-column chunk of the accumulator goes through a 128B-swizzled fp32 staging tile
// so that four lanes share one output row and every access covers 8 rows x 64 bytes.
template <int NCH, bool f32>
__device__ __forceinline__ void masked_acc_unit(const GemmParams& p, uint32_t stage, int lane, int row0, int col0,
                                                uint32_t t_row) {
  const int sub = lane >> 2;            // row within a pass of 8 rows
  const int cc = (lane & 3) * 8;        // first of this lane's eight columns within a chunk
  uint4 y[NCH][4], y2[f32 ? NCH : 1][4];
  uint32_t bits[NCH][4];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int row = row0 + pass * 8 + sub;
      y[c][pass] = make_uint4(0u, 0u, 0u, 0u);
      if (f32) y2[f32 ? c : 0][pass] = make_uint4(0u, 0u, 0u, 0u);
      bits[c][pass] = 0u;
      // a group of eight columns lies wholly inside or wholly outside the row (cols % 64 == 0)
      if (row < p.rows && col0 + c * 32 + cc < p.cols) {
        const int64_t e0 = static_cast<int64_t>(row) * p.ld_out + col0 + c * 32 + cc;   // a multiple of 8
        bits[c][pass] = __ldg(p.mask + e0 / 8);
        if (f32) {
          const uint4* o = reinterpret_cast<const uint4*>(static_cast<const float*>(p.out) + e0);
          y[c][pass] = o[0];
          y2[f32 ? c : 0][pass] = o[1];
        } else {
          y[c][pass] = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.out) + e0);
        }
      }
    }
  const uint32_t mine = stage + lane * 128;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(t_row + c * 32, v);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_shared_v4(mine + ((j ^ (lane & 7)) << 4), make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
    __syncwarp();
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int rr = pass * 8 + sub;
      const int row = row0 + rr;
      if (row >= p.rows || col0 + c * 32 + cc >= p.cols) continue;
      const uint32_t src = stage + rr * 128;
      const uint4 a0 = ld_shared_v4(src + (((cc >> 2) ^ (rr & 7)) << 4));
      const uint4 a1 = ld_shared_v4(src + ((((cc >> 2) + 1) ^ (rr & 7)) << 4));
      const float d[8] = {__uint_as_float(a0.x), __uint_as_float(a0.y), __uint_as_float(a0.z), __uint_as_float(a0.w),
                          __uint_as_float(a1.x), __uint_as_float(a1.y), __uint_as_float(a1.z), __uint_as_float(a1.w)};
      float add[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) add[t] = ((bits[c][pass] >> t) & 1u) ? __fmul_rn(p.keep_scale, d[t]) : 0.f;
      const int64_t e0 = static_cast<int64_t>(row) * p.ld_out + col0 + c * 32 + cc;
      if (f32) {
        uint4* o = reinterpret_cast<uint4*>(static_cast<float*>(p.out) + e0);
        o[0] = make_uint4(__float_as_uint(__uint_as_float(y[c][pass].x) + add[0]),
                          __float_as_uint(__uint_as_float(y[c][pass].y) + add[1]),
                          __float_as_uint(__uint_as_float(y[c][pass].z) + add[2]),
                          __float_as_uint(__uint_as_float(y[c][pass].w) + add[3]));
        const uint4 z = y2[f32 ? c : 0][pass];
        o[1] = make_uint4(__float_as_uint(__uint_as_float(z.x) + add[4]), __float_as_uint(__uint_as_float(z.y) + add[5]),
                          __float_as_uint(__uint_as_float(z.z) + add[6]), __float_as_uint(__uint_as_float(z.w) + add[7]));
      } else {
        const uint32_t yy[4] = {y[c][pass].x, y[c][pass].y, y[c][pass].z, y[c][pass].w};
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
          w[t] = pack_bf16x2(__uint_as_float(yy[t] << 16) + add[2 * t],
                             __uint_as_float(yy[t] & 0xFFFF0000u) + add[2 * t + 1]);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + e0) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncwarp();                       // the staging tile is rewritten by the next chunk
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::Stages * C::kABytes;
  uint8_t* sEpi = sB + C::Stages * C::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + C::kEpiStage);
  uint64_t* tma_full = bars;
  uint64_t* empty = bars + C::Stages;
  uint64_t* acc_full = bars + 2 * C::Stages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.tiles_n * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::Stages; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    fence_mbar_init();
  }
  griddep_enter();
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.a);
      tma_prefetch_desc(&maps.b);
      if (C::Ext || C::HiLo) tma_prefetch_desc(&maps.b2);
      if (C::Ext) tma_prefetch_desc(&maps.a2);
      int stage = 0;
      uint32_t ph = 0;
      uint32_t pending = 0;      // stages with a load whose completion nobody has waited for yet
      uint32_t pend_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        decode_unit(p, u, mb, nb, split, kt0, nmain, next);
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { ok = false; break; }
          pending &= ~(1u << stage);
          uint8_t* a_dst = sA + stage * C::kABytes;
          uint8_t* b_dst = sB + stage * C::kBBytes;
          uint64_t* bar = &tma_full[stage];
          if (i < nmain) {
            const int kt = kt0 + i;
            mbar_arrive_expect_tx(bar, C::kABytes + C::kBBytes);
            const int64_t kext = static_cast<int64_t>(p.k_tiles) * 64;    // reduction length, rounded up
            if (C::AMn) {
              if (tma_start_ok(mb * 128, kt * 64, 2, p.rows, a_dst, 30))
                tma_load_2d(a_dst, &maps.a, bar, mb * 128, kt * 64);
              if (tma_start_ok(mb * 128 + 64, kt * 64, 2, p.rows + 64, a_dst + 8192, 31))
                tma_load_2d(a_dst + 8192, &maps.a, bar, mb * 128 + 64, kt * 64);
            } else if (tma_start_ok(kt * 64, mb * 128, 2, kext, a_dst, 32)) {
              tma_load_2d(a_dst, &maps.a, bar, kt * 64, mb * 128);
            }
            if (C::BMode == kB_TmaK) {
              if (tma_start_ok(kt * 64, nb * C::BN, 2, kext, b_dst, 33))
                tma_load_2d(b_dst, &maps.b, bar, kt * 64, nb * C::BN);
            } else {
#pragma unroll
              for (int j = 0; j < C::BN / 64; ++j) {
                if (tma_start_ok(nb * C::BN + 64 * j, kt * 64, 2, p.cols + 64 * j, b_dst + j * 8192, 34))
                  tma_load_2d(b_dst + j * 8192, &maps.b, bar, nb * C::BN + 64 * j, kt * 64);
                if (C::HiLo &&
                    tma_start_ok(nb * C::BN + 64 * j, kt * 64, 2, p.cols + 64 * j, b_dst + C::kBTile + j * 8192, 35))
                  tma_load_2d(b_dst + C::kBTile + j * 8192, &maps.b2, bar, nb * C::BN + 64 * j, kt * 64);
              }
            }
          } else {
            const int e = i - nmain;
            mbar_arrive_expect_tx(bar, C::kABytes + C::kBTile);
            if (tma_start_ok(e * 64, mb * 128, 2, p.ext_tiles * 64, a_dst, 36))
              tma_load_2d(a_dst, &maps.a2, bar, e * 64, mb * 128);
            if (!C::BMn) {
              if (tma_start_ok(e * 64, nb * C::BN, 2, p.ext_tiles * 64, b_dst, 37))
                tma_load_2d(b_dst, &maps.b2, bar, e * 64, nb * C::BN);
            } else {
#pragma unroll
              for (int j = 0; j < C::BN / 64; ++j)
                if (tma_start_ok(nb * C::BN + 64 * j, e * 64, 2, p.cols + 64 * j, b_dst + j * 8192, 38))
                  tma_load_2d(b_dst + j * 8192, &maps.b2, bar, nb * C::BN + 64 * j, e * 64);
            }
          }
          pending |= (1u << stage);
          pend_par = (pend_par & ~(1u << stage)) | (ph << stage);
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
      }
      if (ok) {
        // tail: re-acquire every stage once, so that the MMA's last releases
        // (asynchronous tcgen05.commit arrivals) have landed before exit
        for (int s = 0; s < C::Stages; ++s) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) break;
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
      } else {     // error path: let copies already in flight land before the CTA exits
        for (int s = 0; s < C::Stages; ++s)
          if (pending & (1u << s)) mbar_wait(&tma_full[s], (pend_par >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BN, C::AMn, C::BMn);
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        decode_unit(p, u, mb, nb, split, kt0, nmain, next);
        if (!mbar_wait(&acc_empty[acc], aph ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = C::AMn ? umma_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                       : umma_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = C::BMn ? umma_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                       : umma_desc_sw128(b_addr + kk * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
            if (C::HiLo) {
              const uint64_t bd2 = umma_desc_sw128(b_addr + C::kBTile + kk * 2048, 8192, 1024);
              umma_bf16(d_tmem, ad, bd2, idesc, 1u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
    }
    __syncwarp();
  } else if (warp < 2 + 4 * C::EpiGroups) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int eg = (warp - 2) >> 2;         // with two groups: the accumulator buffer this group drains
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      if (C::EpiGroups == 2 && acc != eg) {
        acc ^= 1;
        if (acc == 0) aph ^= 1;
        continue;
      }
      int mb, nb, split, kt0, nmain, next;
      decode_unit(p, u, mb, nb, split, kt0, nmain, next);
      if (!mbar_wait(&acc_full[acc], aph)) break;
      tc_fence_after();
      const int row = mb * 128 + q * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      if (p.out_mode == kOutMaskAccBF16 || p.out_mode == kOutMaskAccF32) {
        if (p.out_mode == kOutMaskAccF32) {   // fp32 dX: two round trips of half the columns (registers)
#pragma unroll 1
          for (int h = 0; h < 2; ++h)
            masked_acc_unit<C::BN / 64, true>(p, smem_u32(sEpi + (warp - 2) * 4096), lane, mb * 128 + q * 32,
                                              nb * C::BN + h * (C::BN / 2), t_row + h * (C::BN / 2));
        } else
          masked_acc_unit<C::BN / 32, false>(p, smem_u32(sEpi + (warp - 2) * 4096), lane, mb * 128 + q * 32,
                                             nb * C::BN, t_row);
      } else {
#pragma unroll 1
        for (int c = 0; c < C::BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
          store_row32(p, split, row, nb * C::BN + c * 32, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                        : swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                        : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <class C>
static cudaError_t launch_cfg(const GemmParams& p, const GemmMaps& maps, int grid, cudaStream_t st) {
  static bool attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(qlora_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  return launch_pdl(qlora_gemm_kernel<C>, grid, C::kThreads, C::kSmemBytes, st, 1, p, maps);
}

using CfgDownK = GemmCfg<64, 6, false, kB_TmaK, false, false>;
using CfgDownMN = GemmCfg<64, 6, false, kB_TmaMN, false, false>;
using CfgGrad = GemmCfg<64, 6, true, kB_TmaMN, false, true>;
using CfgDownK128 = GemmCfg<128, 5, false, kB_TmaK, false, false>;
using CfgDownMN128 = GemmCfg<128, 5, false, kB_TmaMN, false, false>;
using CfgGrad128 = GemmCfg<128, 4, true, kB_TmaMN, false, true>;
using CfgUpMasked = GemmCfg<128, 4, false, kB_TmaMN, false, false, 2>;

int gemm_bn(GemmKind kind) {
  switch (kind) {
    case kGemmLoraDownK128: case kGemmLoraDownMN128: case kGemmLoraGrad128: case kGemmLoraUpMasked: return 128;
    default: return 64;
  }
}

static cudaError_t launch_gemm_impl(GemmKind kind, const GemmParams& p, const GemmMaps& maps, int grid,
                                    cudaStream_t st) {
  switch (kind) {
    case kGemmLoraDownK: return launch_cfg<CfgDownK>(p, maps, grid, st);
    case kGemmLoraDownMN: return launch_cfg<CfgDownMN>(p, maps, grid, st);
    case kGemmLoraGrad: return launch_cfg<CfgGrad>(p, maps, grid, st);
    case kGemmLoraDownK128: return launch_cfg<CfgDownK128>(p, maps, grid, st);
    case kGemmLoraDownMN128: return launch_cfg<CfgDownMN128>(p, maps, grid, st);
    case kGemmLoraGrad128: return launch_cfg<CfgGrad128>(p, maps, grid, st);
    case kGemmLoraUpMasked: return launch_cfg<CfgUpMasked>(p, maps, grid, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm(GemmKind kind, const GemmParams& p, const GemmMaps& maps, int grid, cudaStream_t st) {
  return launch_gemm_impl(kind, p, maps, grid, st);
}

}  // namespace qlora
