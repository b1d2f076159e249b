// Fused NF4 GEMM with the frozen weight as the 128-row tensor-core operand.
//
//   forward   Y^T[n, m]  = W[n, :] . X[m, :]^T      + B[n, :] . (s U)[m, :]^T
//   backward dX^T[k, m]  = W[:, k]^T . dY[m, :]^T   + A[:, k]^T . (s G)[m, :]^T
//
// Each 128 x 64 block of W is dequantized once per K step ("right before the
// GPU multiplies", "QLoRA: Quantized Low-Rank Adaptation", Piece 2 and
// "Batched 4-bit matmuls") straight into the 128-byte-swizzled shared-memory
// tile that the tcgen05.mma descriptor reads, and is then reused by every
// token of the tile: one MMA covers up to 256 tokens (its N). Putting W on
// the 128-row side is what makes this reuse possible, and at a handful of
// tokens (M = 16) it wastes no tensor-core rows on padding.
//
// Three independent shared-memory rings keep the expansion off the critical
// path of the activation loads:
//   codes  packed 4-bit codes of one K step (4 KB), prefetched many steps
//          ahead and released by the dequantizers once the step is expanded;
//   A      the dequantized weight tile of one K step (16 KB), written by the
//          dequantizers, released by the MMA's completion;
//   X      the activation tile of one K step, loaded by TMA, released by
//          the MMA's completion.
// The low-rank branch is appended as extra K steps: its A-side tile (B or A
// of the adapter) enters the A ring by TMA, its token-side tile (s U or s G)
// the X ring.
//
// Warp roles (480 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA: activation / low-rank token tiles (X ring)
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue
//   warps 2-5   epilogue: TMEM -> registers -> global (row-major Y / dX)
//   warps 6-13  dequantizers, two groups of four warps that take alternate
//               K steps; one thread expands one 64-block per step
//   warp 14     TMA: packed codes (codes ring)
#include <cudaTypedefs.h>

#include <mutex>

#include "qlora_kernels.h"

namespace qlora {

template <int kBN, int kAStages, int kXStages, int kRStages, bool kBwd>
struct WCfg {
  static constexpr int BN = kBN;            // tokens per tile (MMA N)
  static constexpr int AStages = kAStages;  // dequantized weight tiles in flight
  static constexpr int XStages = kXStages;  // activation tiles in flight
  static constexpr int RStages = kRStages;  // code tiles in flight
  static constexpr bool Bwd = kBwd;         // A = W^T (MN-major) for dX, A = W (K-major) for Y
  static constexpr int kATile = 128 * 64 * 2;
  static constexpr int kXTile = BN * 64 * 2;
  static constexpr int kRBytes = 4096;      // packed codes of one 128 x 64 weight tile
  static constexpr int kGroupWarps = 4;     // warps per dequantizer group (one A-tile arrival each)
  static constexpr int kThreads = 15 * 32;
  static constexpr int kAccBufs = (2 * BN <= 512) ? 2 : 1;   // double-buffer the accumulators when TMEM allows
  static constexpr int kTmemCols = (kAccBufs * BN <= 32) ? 32 : (kAccBufs * BN <= 64) ? 64 : (kAccBufs * BN <= 128) ? 128
                                   : (kAccBufs * BN <= 256) ? 256 : 512;
  static constexpr int kBarBytes = 8 * (2 * (kAStages + kXStages + kRStages) + 4) + 16;
  static constexpr int kSmemBytes = AStages * kATile + XStages * kXTile + RStages * kRBytes + 1024 + kBarBytes;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(BN % 32 == 0 || BN == 16, "epilogue reads 32 columns at a time");
  static_assert(AStages % 2 == 0, "the two dequantizer groups alternate A slots");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
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
  uint8_t* sX = sA + C::AStages * C::kATile;
  uint8_t* sR = sX + C::XStages * C::kXTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + C::RStages * C::kRBytes);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + C::AStages;
  uint64_t* x_full = a_empty + C::AStages;
  uint64_t* x_empty = x_full + C::XStages;
  uint64_t* r_full = x_empty + C::XStages;
  uint64_t* r_empty = r_full + C::RStages;
  uint64_t* acc_full = r_empty + C::RStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.tiles_n * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::AStages; ++s) {
      mbar_init(&a_full[s], C::kGroupWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < C::XStages; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    for (int s = 0; s < C::RStages; ++s) {
      mbar_init(&r_full[s], 1);
      mbar_init(&r_empty[s], C::kGroupWarps);
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
    // ------------------------------------------------ producer: activation tiles (X ring)
    if (lane == 0) {
      tma_prefetch_desc(&maps.act);
      tma_prefetch_desc(&maps.b2);
      uint32_t gs = 0;
      uint32_t pending = 0, pend_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        for (int i = 0; i < nmain + next; ++i, ++gs) {
          const int xs = static_cast<int>(gs % C::XStages);
          const uint32_t xph = (gs / C::XStages) & 1u;
          if (!mbar_wait(&x_empty[xs], xph ^ 1)) { ok = false; break; }
          pending &= ~(1u << xs);
          uint64_t* bar = &x_full[xs];
          mbar_arrive_expect_tx(bar, C::kXTile);
          if (i < nmain) tma_load_2d(sX + xs * C::kXTile, &maps.act, bar, (kt0 + i) * 64, nb * C::BN);
          else tma_load_2d(sX + xs * C::kXTile, &maps.b2, bar, (i - nmain) * 64, nb * C::BN);
          pending |= (1u << xs);
          pend_par = (pend_par & ~(1u << xs)) | (xph << xs);
        }
      }
      if (ok) {
        // every X slot released once more: the MMA's last asynchronous releases have landed
        for (int s = 0; s < C::XStages; ++s, ++gs)
          if (!mbar_wait(&x_empty[gs % C::XStages], ((gs / C::XStages) & 1u) ^ 1)) break;
      } else {
        for (int s = 0; s < C::XStages; ++s)
          if (pending & (1u << s)) mbar_wait(&x_full[s], (pend_par >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 14) {
    // ------------------------------------------------ producer: packed codes (codes ring)
    if (lane == 0) {
      tma_prefetch_desc(&maps.codes);
      uint32_t rs = 0;
      uint32_t pending = 0, pend_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        for (int i = 0; i < nmain; ++i, ++rs) {
          const int rsl = static_cast<int>(rs % C::RStages);
          const uint32_t rph = (rs / C::RStages) & 1u;
          if (!mbar_wait(&r_empty[rsl], rph ^ 1)) { ok = false; break; }
          pending &= ~(1u << rsl);
          uint64_t* bar = &r_full[rsl];
          mbar_arrive_expect_tx(bar, C::kRBytes);
          const int kt = kt0 + i;
          if (C::Bwd) tma_load_2d(sR + rsl * C::kRBytes, &maps.codes, bar, mb * 64, kt * 64);
          else tma_load_2d(sR + rsl * C::kRBytes, &maps.codes, bar, kt * 32, mb * 128);
          pending |= (1u << rsl);
          pend_par = (pend_par & ~(1u << rsl)) | (rph << rsl);
        }
      }
      if (!ok) {
        for (int s = 0; s < C::RStages; ++s)
          if (pending & (1u << s)) mbar_wait(&r_full[s], (pend_par >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BN, C::Bwd, false);
      uint32_t gs = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        if (!mbar_wait(&acc_empty[acc], aph ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int i = 0; i < nmain + next; ++i, ++gs) {
          const int as = static_cast<int>(gs % C::AStages);
          const int xs = static_cast<int>(gs % C::XStages);
          if (!mbar_wait(&a_full[as], (gs / C::AStages) & 1u)) { ok = false; break; }
          if (!mbar_wait(&x_full[xs], (gs / C::XStages) & 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + as * C::kATile);
          const uint32_t x_addr = smem_u32(sX + xs * C::kXTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = C::Bwd ? umma_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                       : umma_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(x_addr + kk * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&a_empty[as]);
          umma_commit(&x_empty[xs]);
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == C::kAccBufs) { acc = 0; aph ^= 1; }
      }
      if (ok) {
        // the last releases of the A ring are asynchronous arrivals: see them land before exit
        for (int j = 1; j <= C::AStages && static_cast<uint32_t>(j) <= gs; ++j) {
          const uint32_t g = gs - j;
          if (!mbar_wait(&a_empty[g % C::AStages], (g / C::AStages) & 1u)) break;
        }
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      if (!mbar_wait(&acc_full[acc], aph)) break;
      tc_fence_after();
      const int feat = mb * 128 + q * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      if (C::BN == 16) {
        uint32_t v[32];
        tmem_ld_32x32b_x16(t_row, v);
        tmem_ld_wait();
        wstore<16>(p, split, feat, nb * C::BN, v);
      } else {
#pragma unroll 1
        for (int c = 0; c < C::BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
          wstore<32>(p, split, feat, nb * C::BN + c * 32, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == C::kAccBufs) { acc = 0; aph ^= 1; }
    }
  } else if (warp < 14) {
    // ------------------------------------------------ dequantizers (two groups)
    // Group g (four warps) expands the K steps whose running index has parity g, so two
    // steps are expanded at once. Forward: thread = W row of the 128-row tile, one 64-block
    // per step. Backward: thread = (W row i of the 64-row K step, 64-column block c).
    const int grp = (warp - 6) >> 2;
    const int gw = (warp - 6) & 3;
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
    uint32_t gs = 0, rs = 0;
    bool ok = true;
    bool ext_pending = false;
    int ext_slot = 0;
    uint32_t ext_par = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      const int first = ((gs & 1u) == static_cast<uint32_t>(grp)) ? 0 : 1;
      auto block_of = [&](int i, bool& valid) -> int64_t {
        const int kt = kt0 + i;
        int64_t wrow, kb;
        if (!C::Bwd) { wrow = static_cast<int64_t>(mb) * 128 + gt; kb = kt; }
        else { wrow = static_cast<int64_t>(kt) * 64 + i_mn; kb = static_cast<int64_t>(mb) * 2 + c_mn; }
        valid = (wrow < p.w_rows) && (kb < p.w_kblocks);
        return wrow * p.w_kblocks + kb;
      };
      // scale prefetch: own steps are every other step; keep four of them in flight
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
      for (int i = 0; i < nmain + next; ++i, ++gs) {
        const bool mine = (gs & 1u) == static_cast<uint32_t>(grp);
        const int as = static_cast<int>(gs % C::AStages);
        if (i < nmain) {
          if (mine) {
            bool valid, v4;
            block_of(i, valid);
            const int64_t b4 = block_of(i + 8, v4);
            RawScale r4{0u, 0.f};
            if (i + 8 < nmain && v4) r4 = load_raw_scale(p.scales, b4);
            const int rsl = static_cast<int>(rs % C::RStages);
            if (!mbar_wait(&r_full[rsl], (rs / C::RStages) & 1u)) { ok = false; break; }
            const uint32_t rsrc = smem_u32(sR + rsl * C::kRBytes);
            const uint4 w0 = ld_shared_v4_w(rsrc + r_off0);
            const uint4 w1 = ld_shared_v4_w(rsrc + r_off1);
            const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales, r0, mean));
            if (!mbar_wait(&a_empty[as], ((gs / C::AStages) & 1u) ^ 1)) { ok = false; break; }
            const uint32_t adst = smem_u32(sA + as * C::kATile) + a_off;
            if (valid) {
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
            // the fence orders this thread's reads of the code slot and writes of the A slot before
            // the async-proxy accesses that follow the releases (the MMA read, the next TMA refill)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&a_full[as]);
              mbar_arrive(&r_empty[rsl]);
            }
            r0 = r1;
            r1 = r2;
            r2 = r3;
            r3 = r4;
          }
          ++rs;      // every main step advances the codes ring, whichever group expands it
        } else if (mine) {
          // low-rank extension step: the group's first warp loads the A-side tile into the A slot
          if (!mbar_wait(&a_empty[as], ((gs / C::AStages) & 1u) ^ 1)) { ok = false; break; }
          if (gw == 0 && lane == 0) {
            uint64_t* bar = &a_full[as];
            uint8_t* dst = sA + as * C::kATile;
            const int e = i - nmain;
            mbar_arrive_expect_tx(bar, C::kATile);
            if (C::Bwd) {
              tma_load_2d(dst, &maps.a2, bar, mb * 128, e * 64);
              tma_load_2d(dst + 8192, &maps.a2, bar, mb * 128 + 64, e * 64);
            } else {
              tma_load_2d(dst, &maps.a2, bar, e * 64, mb * 128);
            }
            ext_pending = true;
            ext_slot = as;
            ext_par = (gs / C::AStages) & 1u;
          } else if (lane == 0) {
            mbar_arrive(&a_full[as]);
          }
          __syncwarp();
        }
      }
    }
    // error path: a low-rank tile this thread requested must land before the CTA exits
    if (!ok && ext_pending) mbar_wait(&a_full[ext_slot], ext_par);
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

int wgemm_box_rows(int bn) { return bn; }

int wgemm_bn(int64_t tokens) {
  if (tokens <= 16) return 16;
  if (tokens <= 64) return 64;
  if (tokens <= 128) return 128;
  return 256;
}

// Ring depths per token-tile width (dequantized tiles, activation tiles, code tiles).
template <bool kBwd> using WCfg16 = WCfg<16, 2, 8, 16, kBwd>;
template <bool kBwd> using WCfg64 = WCfg<64, 6, 8, 12, kBwd>;
template <bool kBwd> using WCfg128 = WCfg<128, 4, 6, 12, kBwd>;
template <bool kBwd> using WCfg256 = WCfg<256, 4, 4, 8, kBwd>;

cudaError_t launch_wgemm(bool bwd, int bn, const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st,
                         double algo_flops) {
  const bool timed = timing_active();
  if (timed) timing_record(st, true, algo_flops);
  cudaError_t e = cudaErrorInvalidValue;
  if (!bwd) {
    switch (bn) {
      case 16: e = launch_wcfg<WCfg16<false>>(p, maps, grid, st); break;
      case 64: e = launch_wcfg<WCfg64<false>>(p, maps, grid, st); break;
      case 128: e = launch_wcfg<WCfg128<false>>(p, maps, grid, st); break;
      case 256: e = launch_wcfg<WCfg256<false>>(p, maps, grid, st); break;
    }
  } else {
    switch (bn) {
      case 16: e = launch_wcfg<WCfg16<true>>(p, maps, grid, st); break;
      case 64: e = launch_wcfg<WCfg64<true>>(p, maps, grid, st); break;
      case 128: e = launch_wcfg<WCfg128<true>>(p, maps, grid, st); break;
      case 256: e = launch_wcfg<WCfg256<true>>(p, maps, grid, st); break;
    }
  }
  if (timed) timing_record(st, false, algo_flops);
  count_launches(1);
  return e;
}

}  // namespace qlora
