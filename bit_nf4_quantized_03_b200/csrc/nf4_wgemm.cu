// Fused NF4 GEMM with the frozen weight as the 128-row tensor-core operand.
//
//   forward   Y^T[n, m]  = W[n, :] . X[m, :]^T      + B[n, :] . (s U)[m, :]^T
//   backward dX^T[k, m]  = W[:, k]^T . dY[m, :]^T   + A[:, k]^T . (s G)[m, :]^T
//
// Each 128 x 64 block of W is dequantized once per K step ("right before the
// GPU multiplies", "QLoRA: Quantized Low-Rank Adaptation", Piece 2 and
// "Batched 4-bit matmuls") straight into the 128-byte-swizzled shared-memory
// tile that the tcgen05.mma descriptor reads, and is then reused by every
// token of the tile: one MMA covers up to 256 tokens (its N), and for long
// token counts two MMAs (two TMEM accumulators of 192 columns) share the same
// weight tile, so each dequantized weight serves 384 tokens. Putting W on the
// 128-row side is what makes this reuse possible, and at a handful of tokens
// (M = 16) it wastes no tensor-core rows on padding.
//
// Warp roles (448 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA: packed codes (32B/64B-swizzled so the reads below are
//               bank-conflict free), activation tiles, low-rank extension tiles
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue
//   warps 2-5   epilogue: TMEM -> registers -> global (row-major Y / dX)
//   warps 6-13  dequantizers: two lanes per weight row (32 codes each) expand
//               every K step of the 128-row tile
#include <cudaTypedefs.h>

#include <mutex>

#include "qlora_kernels.h"

namespace qlora {

template <int kBN, int kNAcc, int kStages, bool kBwd, int kGroups = 2>
struct WCfg {
  static constexpr int BN = kBN;            // tokens per MMA (N)
  static constexpr int NAcc = kNAcc;        // MMAs (token sub-tiles) sharing one dequantized weight tile
  static constexpr int TOK = BN * NAcc;     // tokens per tile
  static constexpr int Stages = kStages;
  static constexpr bool Bwd = kBwd;         // A = W^T (MN-major) for dX, A = W (K-major) for Y
  // Dequantizer layout: 2 = two groups of four warps, group g expands the stages with
  // index parity g (one lane per 64-block); 1 = all eight warps on every stage (two
  // lanes per 64-block).
  static constexpr int Groups = kGroups;
  static constexpr int kDeqArrivals = (kGroups == 2) ? 4 : 8;
  static constexpr int kATile = 128 * 64 * 2;
  static constexpr int kBTile = TOK * 64 * 2;
  static constexpr int kRBytes = 4096;      // packed codes of one 128 x 64 weight tile
  static constexpr int kThreads = 14 * 32;
  static constexpr int kAccBufs = (2 * TOK <= 512) ? 2 : 1;   // double-buffer the accumulators when TMEM allows
  static constexpr int kTmemCols = (kAccBufs * TOK <= 32) ? 32 : (kAccBufs * TOK <= 64) ? 64 : (kAccBufs * TOK <= 128) ? 128
                                   : (kAccBufs * TOK <= 256) ? 256 : 512;
  static constexpr int kSmemBytes = Stages * (kATile + kBTile + kRBytes) + 1024 + 256;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(BN % 32 == 0 || BN == 16, "epilogue reads 32 columns at a time");
  static_assert(kAccBufs * TOK <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kGroups == 1 || (kGroups == 2 && kStages % 2 == 0), "stage parity picks the group");
};

constexpr int kRasterGroup = 4;   // token tiles per raster group (L2 reuse of both operands)

__device__ __forceinline__ void wdecode(const GemmParams& p, int u, int& mb, int& nb, int& split, int& kt0,
                                        int& nmain, int& next) {
  split = u % p.splits;
  const int t = u / p.splits;
  const int per_group = kRasterGroup * p.tiles_m;
  const int g = t / per_group;
  const int within = t - g * per_group;
  int gsize = p.tiles_n - g * kRasterGroup;
  if (gsize > kRasterGroup) gsize = kRasterGroup;
  mb = within / gsize;
  nb = g * kRasterGroup + (within - mb * gsize);
  kt0 = split * p.k_per_split;
  int kt1 = kt0 + p.k_per_split;
  if (kt1 > p.k_tiles) kt1 = p.k_tiles;
  nmain = kt1 - kt0;
  next = (split == 0) ? p.ext_tiles : 0;
}

__device__ __forceinline__ void st_shared_v4_w(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4_w(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Raw scale of one block, loaded ahead of use; turned into the fp32 scale later.
// Epilogue: 32 (or 16) consecutive tokens of one output feature.
template <int kCount>
__device__ __forceinline__ void wstore(const GemmParams& p, int split, int feat, int tok0, const uint32_t (&v)[32]) {
  if (feat >= p.rows) return;
  const int64_t ld = p.ld_out;
#pragma unroll
  for (int j = 0; j < kCount; ++j) {
    const int m = tok0 + j;
    if (m >= p.cols) break;
    const float x = __uint_as_float(v[j]);
    const int64_t off = static_cast<int64_t>(m) * ld + feat;
    if (p.out_mode == kOutPartial) {
      static_cast<float*>(p.out)[split * p.part_stride + off] = x;
    } else if (p.out_mode == kOutF32) {
      float* o = static_cast<float*>(p.out) + off;
      *o = p.accumulate ? (*o + x) : x;
    } else {
      uint16_t* o = static_cast<uint16_t*>(p.out) + off;
      const float y = p.accumulate ? (x + __uint_as_float(static_cast<uint32_t>(*o) << 16)) : x;
      *o = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    qlora_wgemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ WMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::Stages * C::kATile;
  uint8_t* sR = sB + C::Stages * C::kBTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + C::Stages * C::kRBytes);
  uint64_t* tma_full = bars;
  uint64_t* deq_full = bars + C::Stages;
  uint64_t* empty = bars + 2 * C::Stages;
  uint64_t* acc_full = bars + 3 * C::Stages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.tiles_n * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::Stages; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&deq_full[s], C::kDeqArrivals);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    fence_mbar_init();
  }
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
      tma_prefetch_desc(&maps.act);
      tma_prefetch_desc(&maps.codes);
      tma_prefetch_desc(&maps.a2);
      tma_prefetch_desc(&maps.b2);
      int stage = 0;
      uint32_t ph = 0;
      uint32_t pending = 0, pend_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { ok = false; break; }
          uint64_t* bar = &tma_full[stage];
          uint8_t* a_dst = sA + stage * C::kATile;
          uint8_t* b_dst = sB + stage * C::kBTile;
          if (i < nmain) {
            const int kt = kt0 + i;
            mbar_arrive_expect_tx(bar, C::kRBytes + C::kBTile);
            if (C::Bwd) tma_load_2d(sR + stage * C::kRBytes, &maps.codes, bar, mb * 64, kt * 64);
            else tma_load_2d(sR + stage * C::kRBytes, &maps.codes, bar, kt * 32, mb * 128);
#pragma unroll
            for (int t = 0; t < C::NAcc; ++t)
              tma_load_2d(b_dst + t * (C::BN * 128), &maps.act, bar, kt * 64, nb * C::TOK + t * C::BN);
          } else {
            const int e = i - nmain;
            mbar_arrive_expect_tx(bar, C::kATile + C::kBTile);
            if (C::Bwd) {
              tma_load_2d(a_dst, &maps.a2, bar, mb * 128, e * 64);
              tma_load_2d(a_dst + 8192, &maps.a2, bar, mb * 128 + 64, e * 64);
            } else {
              tma_load_2d(a_dst, &maps.a2, bar, e * 64, mb * 128);
            }
#pragma unroll
            for (int t = 0; t < C::NAcc; ++t)
              tma_load_2d(b_dst + t * (C::BN * 128), &maps.b2, bar, e * 64, nb * C::TOK + t * C::BN);
          }
          pending |= (1u << stage);
          pend_par = (pend_par & ~(1u << stage)) | (ph << stage);
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
      }
      if (ok) {
        for (int s = 0; s < C::Stages; ++s) {   // tail: every stage released once more
          if (!mbar_wait(&empty[stage], ph ^ 1)) break;
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
      } else {
        for (int s = 0; s < C::Stages; ++s)
          if (pending & (1u << s)) mbar_wait(&tma_full[s], (pend_par >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BN, C::Bwd, false);
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        if (!mbar_wait(&acc_empty[acc], aph ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::TOK);
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          if (!mbar_wait(&deq_full[stage], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::kATile);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = C::Bwd ? umma_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                       : umma_desc_sw128(a_addr + kk * 32, 16, 1024);
#pragma unroll
            for (int t = 0; t < C::NAcc; ++t) {
              const uint64_t bd = umma_desc_sw128(b_addr + t * (C::BN * 128) + kk * 32, 16, 1024);
              umma_bf16(d_tmem + t * C::BN, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == C::kAccBufs) { acc = 0; aph ^= 1; }
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      if (!mbar_wait(&acc_full[acc], aph)) break;
      tc_fence_after();
      const int feat = mb * 128 + q * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::TOK);
      if (C::BN == 16) {
        uint32_t v[32];
        tmem_ld_32x32b_x16(t_row, v);
        tmem_ld_wait();
        wstore<16>(p, split, feat, nb * C::TOK, v);
      } else {
#pragma unroll 1
        for (int c = 0; c < C::TOK / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
          wstore<32>(p, split, feat, nb * C::TOK + c * 32, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == C::kAccBufs) { acc = 0; aph ^= 1; }
    }
  } else if (C::Groups == 2) {
    // ------------------------------------------------------------ dequantizers (two groups)
    // Group g (four warps) expands the stages with index parity g, so two K steps are in
    // flight at once. Forward: thread = W row of the 128-row tile, one 64-block per K step.
    // Backward: thread = (W row i of the 64-row K step, 64-column block c of the tile).
    const int grp = (warp - 6) >> 2;
    const int gt = threadIdx.x - 192 - 128 * grp;    // 0..127
    const float mean = (p.scales.dq_mean != nullptr) ? __ldg(p.scales.dq_mean) : 0.f;
    const int i_mn = gt & 63;
    const int c_mn = gt >> 6;
    uint32_t r_off0, r_off1, a_off;
    int sw;
    if (!C::Bwd) {
      const uint32_t x = (gt >> 2) & 1;                         // 32B swizzle of the code tile
      r_off0 = gt * 32 + 16 * x;
      r_off1 = gt * 32 + 16 * (x ^ 1);
      a_off = (gt >> 3) * 1024 + (gt & 7) * 128;
      sw = gt & 7;
    } else {
      const uint32_t x = (i_mn >> 1) & 3;                       // 64B swizzle of the code tile
      r_off0 = i_mn * 64 + 16 * ((2 * c_mn) ^ x);
      r_off1 = i_mn * 64 + 16 * ((2 * c_mn + 1) ^ x);
      a_off = c_mn * 8192 + (i_mn >> 3) * 1024 + (i_mn & 7) * 128;
      sw = i_mn & 7;
    }
    int stage = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      const int first = ((stage & 1) == grp) ? 0 : 1;
      auto block_of = [&](int i, bool& valid) -> int64_t {
        const int kt = kt0 + i;
        int64_t wrow, kb;
        if (!C::Bwd) { wrow = static_cast<int64_t>(mb) * 128 + gt; kb = kt; }
        else { wrow = static_cast<int64_t>(kt) * 64 + i_mn; kb = static_cast<int64_t>(mb) * 2 + c_mn; }
        valid = (wrow < p.w_rows) && (kb < p.w_kblocks);
        return wrow * p.w_kblocks + kb;
      };
      // scale prefetch: own K steps are every other step; keep four of them in flight
      RawScale r0{0u, 0.f}, r1{0u, 0.f}, r2{0u, 0.f}, r3{0u, 0.f};
      {
        bool v;
        int64_t bb = block_of(first, v);
        if (first < nmain && v) r0 = load_raw_scale(p.scales, bb);
        bb = block_of(first + 2, v);
        if (first + 2 < nmain && v) r1 = load_raw_scale(p.scales, bb);
        bb = block_of(first + 4, v);
        if (first + 4 < nmain && v) r2 = load_raw_scale(p.scales, bb);
        bb = block_of(first + 6, v);
        if (first + 6 < nmain && v) r3 = load_raw_scale(p.scales, bb);
      }
      for (int i = 0; i < nmain + next; ++i) {
        if ((stage & 1) == grp) {
          if (i < nmain) {
            bool valid, v4;
            block_of(i, valid);
            const int64_t b4 = block_of(i + 8, v4);
            RawScale r4{0u, 0.f};
            if (i + 8 < nmain && v4) r4 = load_raw_scale(p.scales, b4);
            if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
            const uint32_t adst = smem_u32(sA + stage * C::kATile) + a_off;
            if (valid) {
              const uint32_t rsrc = smem_u32(sR + stage * C::kRBytes);
              const uint4 w0 = ld_shared_v4_w(rsrc + r_off0);
              const uint4 w1 = ld_shared_v4_w(rsrc + r_off1);
              const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales, r0, mean));
              st_shared_v4_w(adst + ((0 ^ sw) << 4), nf4_lookup8(lut, w0.x));
              st_shared_v4_w(adst + ((1 ^ sw) << 4), nf4_lookup8(lut, w0.y));
              st_shared_v4_w(adst + ((2 ^ sw) << 4), nf4_lookup8(lut, w0.z));
              st_shared_v4_w(adst + ((3 ^ sw) << 4), nf4_lookup8(lut, w0.w));
              st_shared_v4_w(adst + ((4 ^ sw) << 4), nf4_lookup8(lut, w1.x));
              st_shared_v4_w(adst + ((5 ^ sw) << 4), nf4_lookup8(lut, w1.y));
              st_shared_v4_w(adst + ((6 ^ sw) << 4), nf4_lookup8(lut, w1.z));
              st_shared_v4_w(adst + ((7 ^ sw) << 4), nf4_lookup8(lut, w1.w));
            } else {
              const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
              for (int j = 0; j < 8; ++j) st_shared_v4_w(adst + (j << 4), z);
            }
            fence_proxy_async_smem();
            r0 = r1;
            r1 = r2;
            r2 = r3;
            r3 = r4;
          } else {
            if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&deq_full[stage]);
        }
        if (++stage == C::Stages) { stage = 0; ph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ dequantizers (all warps)
    // 256 threads per K step. Forward: thread = (W row r of the 128-row tile, half h of
    // its 64-block). Backward: thread = (W row i of the 64-row K step, 64-column block c
    // of the 128-column tile, half h).
    const int gt = threadIdx.x - 192;                 // 0..255
    const float mean = (p.scales.dq_mean != nullptr) ? __ldg(p.scales.dq_mean) : 0.f;
    int row_f = 0, i_mn = 0, c_mn = 0, h;
    uint32_t r_off, a_off;
    int sw;
    if (!C::Bwd) {
      row_f = gt >> 1;
      h = gt & 1;
      const uint32_t x = (row_f >> 2) & 1;                  // 32B swizzle of the code tile
      r_off = row_f * 32 + 16 * (h ^ x);
      a_off = (row_f >> 3) * 1024 + (row_f & 7) * 128;
      sw = row_f & 7;
    } else {
      i_mn = gt & 63;
      c_mn = (gt >> 6) & 1;
      h = gt >> 7;
      const uint32_t x = (i_mn >> 1) & 3;                   // 64B swizzle of the code tile
      r_off = i_mn * 64 + 16 * ((2 * c_mn + h) ^ x);
      a_off = c_mn * 8192 + (i_mn >> 3) * 1024 + (i_mn & 7) * 128;
      sw = i_mn & 7;
    }
    int stage = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      auto block_of = [&](int i, bool& valid) -> int64_t {
        const int kt = kt0 + i;
        int64_t wrow, kb;
        if (!C::Bwd) { wrow = static_cast<int64_t>(mb) * 128 + row_f; kb = kt; }
        else { wrow = static_cast<int64_t>(kt) * 64 + i_mn; kb = static_cast<int64_t>(mb) * 2 + c_mn; }
        valid = (wrow < p.w_rows) && (kb < p.w_kblocks);
        return wrow * p.w_kblocks + kb;
      };
      // scale prefetch: two K steps ahead
      RawScale r0{0u, 0.f}, r1{0u, 0.f};
      {
        bool v0, v1;
        const int64_t b0 = block_of(0, v0);
        const int64_t b1 = block_of(1, v1);
        if (0 < nmain && v0) r0 = load_raw_scale(p.scales, b0);
        if (1 < nmain && v1) r1 = load_raw_scale(p.scales, b1);
      }
      for (int i = 0; i < nmain + next; ++i) {
        if (i < nmain) {
          bool valid, v2;
          block_of(i, valid);
          const int64_t b2 = block_of(i + 2, v2);
          RawScale r2{0u, 0.f};
          if (i + 2 < nmain && v2) r2 = load_raw_scale(p.scales, b2);
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          const uint32_t adst = smem_u32(sA + stage * C::kATile) + a_off;
          if (valid) {
            const uint4 w = ld_shared_v4_w(smem_u32(sR + stage * C::kRBytes) + r_off);
            const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales, r0, mean));
            const int j0 = 4 * h;
            st_shared_v4_w(adst + (((j0 + 0) ^ sw) << 4), nf4_lookup8(lut, w.x));
            st_shared_v4_w(adst + (((j0 + 1) ^ sw) << 4), nf4_lookup8(lut, w.y));
            st_shared_v4_w(adst + (((j0 + 2) ^ sw) << 4), nf4_lookup8(lut, w.z));
            st_shared_v4_w(adst + (((j0 + 3) ^ sw) << 4), nf4_lookup8(lut, w.w));
          } else {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int j = 0; j < 4; ++j) st_shared_v4_w(adst + ((4 * h + j) << 4), z);
          }
          fence_proxy_async_smem();
          r0 = r1;
          r1 = r2;
        } else {
          // extension step: the producer loads the A tile; keep the phases in step
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&deq_full[stage]);
        if (++stage == C::Stages) { stage = 0; ph ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <class C>
static cudaError_t launch_wcfg(const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st) {
  static bool attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(qlora_wgemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  qlora_wgemm_kernel<C><<<grid, C::kThreads, C::kSmemBytes, st>>>(p, maps);
  return cudaGetLastError();
}

int wgemm_box_rows(int bn) { return bn == 384 ? 192 : bn; }

int wgemm_bn(int64_t tokens) {
  if (tokens <= 16) return 16;
  if (tokens <= 64) return 64;
  if (tokens <= 128) return 128;
  return 256;
}

cudaError_t launch_wgemm(bool bwd, int bn, const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st,
                         double algo_flops) {
  const bool timed = timing_active();
  if (timed) timing_record(st, true, algo_flops);
  cudaError_t e = cudaErrorInvalidValue;
  if (!bwd) {
    switch (bn) {
      case 16: e = launch_wcfg<WCfg<16, 1, 8, false>>(p, maps, grid, st); break;
      case 64: e = launch_wcfg<WCfg<64, 1, 8, false>>(p, maps, grid, st); break;
      case 128: e = launch_wcfg<WCfg<128, 1, 6, false>>(p, maps, grid, st); break;
      case 256: e = launch_wcfg<WCfg<256, 1, 4, false>>(p, maps, grid, st); break;
    }
  } else {
    switch (bn) {
      case 16: e = launch_wcfg<WCfg<16, 1, 8, true>>(p, maps, grid, st); break;
      case 64: e = launch_wcfg<WCfg<64, 1, 8, true>>(p, maps, grid, st); break;
      case 128: e = launch_wcfg<WCfg<128, 1, 6, true>>(p, maps, grid, st); break;
      case 256: e = launch_wcfg<WCfg<256, 1, 4, true>>(p, maps, grid, st); break;
    }
  }
  if (timed) timing_record(st, false, algo_flops);
  count_launches(1);
  return e;
}

}  // namespace qlora
