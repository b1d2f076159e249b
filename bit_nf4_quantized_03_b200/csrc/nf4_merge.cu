// Adapter merge onto the dequantized weight (sm_100a):
//
//   W_merged[n, k] = W'[n, k] + s * (B[n, :r] . A[:r, k]),   s = alpha / r
//
// A trained adapter cannot be folded into the 4-bit codes themselves (no
// level lies between the 16 NF4 levels), so it is merged onto a dequantized
// copy ("QLoRA: Quantized Low-Rank Adaptation", Price 2: deployment
// friction; "QLoRA Explained", Step 5: Save and Merge Adapters). The result
// is written in BF16, or in FP32 when it is to be quantized again.
//
// The rank-r product is a dense contraction, so it runs on the tensor cores:
// each 128 x 256 output tile is one TMEM accumulator fed by tcgen05.mma over
// K = r (zero-padded to 64 by the TMA), with B as the K-major 128-row operand
// and A as the MN-major 256-column operand. The epilogue warps then add the
// dequantized weight, expanded from the packed codes with the same per-block
// lookup table as the fused GEMM, and store the merged rows. The kernel is
// bound by HBM: half a byte of codes plus the scales in, two (or four) bytes
// out per weight; A and B are re-read from L2.
//
// Every global access of the hot loop goes through the TMA engine: the code
// tiles arrive 128-byte swizzled in a shared-memory ring several tiles ahead
// of use, and each epilogue warp stages its 32 x 32 output chunk in swizzled
// shared memory and writes it with a tiled TMA store.
//
//   warp 0      TMA producer (adapter tiles, code tiles)
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2-9   epilogue: two warps per TMEM lane quarter, 128 columns each
#include <cudaTypedefs.h>

#include <mutex>

#include "qlora_kernels.h"

namespace qlora {

namespace {

constexpr int kMergeBN = 256;                        // output columns per tile (MMA N)
constexpr int kOpStages = 2;                         // adapter-operand stages (one 64-wide K step each)
constexpr int kCodeStages = 3;                       // code-tile stages (one tile each)
constexpr int kATile = 128 * 64 * 2;                 // B rows [128, 64] bf16, K-major
constexpr int kBTile = kMergeBN * 64 * 2;            // A rows [64, 256] bf16, MN-major (four 64-column chunks)
constexpr int kCodeTile = 128 * (kMergeBN / 2);      // packed codes [128 rows, 128 bytes]
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * kMergeBN;

template <bool kF32>
struct MergeSmem {
  static constexpr int kChunk = 32 * 32 * (kF32 ? 4 : 2);     // one warp's 32 x 32 output chunk
  static constexpr int kOps = kOpStages * (kATile + kBTile);
  static constexpr int kCodes = kCodeStages * kCodeTile;
  static constexpr int kOut = kEpiWarps * 2 * kChunk;         // double-buffered per warp
  static constexpr int kBytes = kOps + kCodes + kOut + 1024 + 256;
  static_assert(kBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void merge_decode(const MergeParams& p, int u, int& mb, int& nb) {
  // column tiles of one row band are adjacent, so B's 128-row tile stays hot
  mb = u / p.tiles_n;
  nb = u - mb * p.tiles_n;
}

// Merge 32 values of one row, fp32(w' + s * acc) with w' from the block's table,
// and write them to this lane's row of the warp's swizzled staging chunk.
template <bool kF32>
__device__ __forceinline__ void merge_stage32(uint32_t chunk, int lane, const Nf4Lut& lut, uint4 codes, float s,
                                              const uint32_t (&v)[32]) {
  const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
  float r[32];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint4 d = nf4_lookup8(lut, cw[g]);
    const uint32_t dd[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int e = 8 * g + 2 * t;
      r[e] = __fmaf_rn(s, __uint_as_float(v[e]), __uint_as_float(dd[t] << 16));
      r[e + 1] = __fmaf_rn(s, __uint_as_float(v[e + 1]), __uint_as_float(dd[t] & 0xFFFF0000u));
    }
  }
  if (kF32) {
    // 128-byte rows, 128B swizzle: 16-byte unit j of row l sits at unit j ^ (l & 7)
    const uint32_t row = chunk + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      sts128(row + ((j ^ (lane & 7)) << 4),
                   make_uint4(__float_as_uint(r[4 * j]), __float_as_uint(r[4 * j + 1]), __float_as_uint(r[4 * j + 2]),
                              __float_as_uint(r[4 * j + 3])));
  } else {
    // 64-byte rows, 64B swizzle: 16-byte unit j of row l sits at unit j ^ ((l >> 1) & 3)
    const uint32_t row = chunk + lane * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      sts128(row + ((j ^ ((lane >> 1) & 3)) << 4),
                   make_uint4(pack_bf16x2(r[8 * j], r[8 * j + 1]), pack_bf16x2(r[8 * j + 2], r[8 * j + 3]),
                              pack_bf16x2(r[8 * j + 4], r[8 * j + 5]), pack_bf16x2(r[8 * j + 6], r[8 * j + 7])));
  }
}

template <bool kF32>
__global__ void __launch_bounds__(kThreads, 1)
    qlora_merge_kernel(const __grid_constant__ MergeParams p, const __grid_constant__ CUtensorMap map_b,
                       const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_codes,
                       const __grid_constant__ CUtensorMap map_out) {
  using S = MergeSmem<kF32>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + kOpStages * kATile;
  uint8_t* sC = sB + kOpStages * kBTile;
  uint8_t* sOut = sC + kCodeStages * kCodeTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + S::kOut);
  uint64_t* op_full = bars;
  uint64_t* op_empty = op_full + kOpStages;
  uint64_t* code_full = op_empty + kOpStages;
  uint64_t* code_empty = code_full + kCodeStages;
  uint64_t* acc_full = code_empty + kCodeStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(&op_full[s], 1);
      mbar_init(&op_empty[s], 1);
    }
    for (int s = 0; s < kCodeStages; ++s) {
      mbar_init(&code_full[s], 1);
      mbar_init(&code_empty[s], kEpiWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiWarps);
    }
    fence_mbar_init();
  }
  griddep_enter();
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_b);
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_codes);
      int os = 0, cs = 0;
      uint32_t oph = 0, cph = 0;
      uint32_t opend = 0, opar = 0, cpend = 0, cpar = 0;   // loads nobody has waited for yet
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb;
        merge_decode(p, u, mb, nb);
        if (!mbar_wait(&code_empty[cs], cph ^ 1)) { ok = false; break; }
        cpend &= ~(1u << cs);
        mbar_arrive_expect_tx(&code_full[cs], kCodeTile);
        if (tma_start_ok(nb * (kMergeBN / 2), mb * 128, 1, p.k / 2, sC + cs * kCodeTile, 40))
          tma_load_2d(sC + cs * kCodeTile, &map_codes, &code_full[cs], nb * (kMergeBN / 2), mb * 128);
        cpend |= (1u << cs);
        cpar = (cpar & ~(1u << cs)) | (cph << cs);
        if (++cs == kCodeStages) { cs = 0; cph ^= 1; }
        for (int ks = 0; ks < p.k_steps; ++ks) {
          if (!mbar_wait(&op_empty[os], oph ^ 1)) { ok = false; break; }
          opend &= ~(1u << os);
          uint64_t* bar = &op_full[os];
          mbar_arrive_expect_tx(bar, kATile + kBTile);
          if (tma_start_ok(ks * 64, mb * 128, 2, p.k_steps * 64, sA + os * kATile, 41))
            tma_load_2d(sA + os * kATile, &map_b, bar, ks * 64, mb * 128);
#pragma unroll
          for (int j = 0; j < kMergeBN / 64; ++j)
            if (tma_start_ok(nb * kMergeBN + 64 * j, ks * 64, 2, p.k + 64 * j + 64, sB + os * kBTile + j * 8192, 42))
              tma_load_2d(sB + os * kBTile + j * 8192, &map_a, bar, nb * kMergeBN + 64 * j, ks * 64);
          opend |= (1u << os);
          opar = (opar & ~(1u << os)) | (oph << os);
          if (++os == kOpStages) { os = 0; oph ^= 1; }
        }
      }
      if (ok) {
        // re-acquire every stage once so the last asynchronous releases land before exit
        for (int s = 0; s < kOpStages; ++s) {
          if (!mbar_wait(&op_empty[os], oph ^ 1)) break;
          if (++os == kOpStages) { os = 0; oph ^= 1; }
        }
      } else {
        for (int s = 0; s < kOpStages; ++s)
          if (opend & (1u << s)) mbar_wait(&op_full[s], (opar >> s) & 1u);
        for (int s = 0; s < kCodeStages; ++s)
          if (cpend & (1u << s)) mbar_wait(&code_full[s], (cpar >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kMergeBN, false, true);
      int os = 0;
      uint32_t oph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        if (!mbar_wait(&acc_empty[acc], aph ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kMergeBN);
        for (int ks = 0; ks < p.k_steps; ++ks) {
          if (!mbar_wait(&op_full[os], oph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + os * kATile);
          const uint32_t b_addr = smem_u32(sB + os * kBTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = umma_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(b_addr + kk * 2048, 8192, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&op_empty[os]);
          if (++os == kOpStages) { os = 0; oph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;       // which 128 of the tile's 256 columns
    const int ew = warp - 2;
    const int tr = q * 32 + lane;           // row within the 128-row tile
    const float mean = (p.scales.dq_mean != nullptr) ? __ldg(p.scales.dq_mean) : 0.0f;
    const int64_t kblocks = p.k / 64;
    const uint32_t out_base = smem_u32(sOut + ew * 2 * S::kChunk);
    int acc = 0, cs = 0, sb = 0, issued = 0;
    uint32_t aph = 0, cph = 0;
    auto raw_scales = [&](int u, RawScale (&rs)[2]) {
      int mb, nb;
      merge_decode(p, u, mb, nb);
      const int64_t row = static_cast<int64_t>(mb) * 128 + tr;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int64_t col = static_cast<int64_t>(nb) * kMergeBN + half * 128 + 64 * b;
        rs[b] = (row < p.n && col < p.k) ? load_raw_scale(p.scales, row * kblocks + col / 64) : RawScale{0u, 0.f};
      }
    };
    RawScale cur[2], nxt[2];
    if (blockIdx.x < units) raw_scales(blockIdx.x, cur);
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      int mb, nb;
      merge_decode(p, u, mb, nb);
      if (u + static_cast<int>(gridDim.x) < units) raw_scales(u + gridDim.x, nxt);
      const int row0 = mb * 128 + q * 32;
      const int col0 = nb * kMergeBN + half * 128;
      // this row's 64 code bytes (128 columns) from the swizzled code tile
      if (!mbar_wait(&code_full[cs], cph)) break;
      const uint32_t crow = smem_u32(sC + cs * kCodeTile) + tr * 128;
      uint4 codes[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) codes[c] = lds128(crow + (((half * 4 + c) ^ (tr & 7)) << 4));
      const int cs_used = cs;
      if (++cs == kCodeStages) { cs = 0; cph ^= 1; }

      if (!mbar_wait(&acc_full[acc], aph)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kMergeBN + half * 128);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales, cur[b], mean));
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int c = 2 * b + c2;
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
          // the staging buffer is free once the store issued two chunks ago has read it
          if (issued >= 2 && lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          const uint32_t chunk = out_base + sb * S::kChunk;
          merge_stage32<kF32>(chunk, lane, lut, codes[c], p.scale, v);
          fence_proxy_async_smem();
          __syncwarp();
          const int col = col0 + 32 * c;
          if (lane == 0) {
            if (row0 < p.n && col < p.k &&
                tma_start_ok(col, row0, kF32 ? 4 : 2, p.k, sOut + ew * 2 * S::kChunk + sb * S::kChunk, 43))
              tma_store_2d(&map_out, sOut + ew * 2 * S::kChunk + sb * S::kChunk, col, row0);
            bulk_commit_group();
          }
          ++issued;
          sb ^= 1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[acc]);
        // the code slot is released only after its values were used and the proxy fence above
        // ordered the reads before the async-proxy refill
        mbar_arrive(&code_empty[cs_used]);
      }
      acc ^= 1;
      if (acc == 0) aph ^= 1;
      cur[0] = nxt[0];
      cur[1] = nxt[1];
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <bool kF32>
cudaError_t launch_merge_impl(const MergeParams& p, const MergeMaps& m, int grid, cudaStream_t st) {
  static bool attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(qlora_merge_kernel<kF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               MergeSmem<kF32>::kBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  return launch_pdl(qlora_merge_kernel<kF32>, grid, kThreads, MergeSmem<kF32>::kBytes, st, 1, p, m.b, m.a, m.codes,
                    m.out);
}

}  // namespace

int merge_tile_cols() { return kMergeBN; }

cudaError_t launch_merge(const MergeParams& p, const MergeMaps& maps, int grid, bool out_f32, cudaStream_t st) {
  return out_f32 ? launch_merge_impl<true>(p, maps, grid, st) : launch_merge_impl<false>(p, maps, grid, st);
}

}  // namespace qlora
