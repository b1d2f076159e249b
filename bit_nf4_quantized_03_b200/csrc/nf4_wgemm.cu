// Fused NF4 GEMM with the frozen weight as the tensor-core M operand.
//
//   forward   Y^T[n, m]  = W[n, :] . X[m, :]^T      + B[n, :] . (s U)[m, :]^T
//   backward dX^T[k, m]  = W[:, k]^T . dY[m, :]^T   + A[:, k]^T . (s G)[m, :]^T
//
// Each 128 x 64 block of W is dequantized once per K step ("right before the
// GPU multiplies", "QLoRA: Quantized Low-Rank Adaptation", Piece 2 and
// "Batched 4-bit matmuls") straight into the 128-byte-swizzled shared-memory
// tile that the tcgen05.mma descriptor reads, and is then reused by every
// token of the tile. Putting W on the M side is what makes this reuse
// possible, and at a handful of tokens (M = 16) it wastes no tensor-core rows
// on padding. Two kernels:
//   qlora_wgemm_kernel       one CTA per 128-row weight tile, 16 to 128 tokens
//                            per tile (MMA N), split K at few tokens
//   qlora_wgemm_pair_kernel  above 128 tokens: two CTAs (a cluster on two SMs)
//                            share a 256-row tile through tcgen05 cta_group::2;
//                            above 1024 tokens each expanded weight tile feeds
//                            two 256-token MMAs (512 tokens per unit), which
//                            halves the expansion work per flop
//
// Warp roles (one CTA per SM, persistent over tiles):
//   warp 0      TMA: packed codes (32B/64B-swizzled so the reads below are
//               bank-conflict free), activation tiles, low-rank extension tiles
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue
//   warps 2-5   epilogue: TMEM -> registers -> global (row-major Y / dX)
//   warps 6-    dequantizers: groups of four warps take turns on the K steps
//               (three groups in the single-CTA kernel, two in the pair);
//               one thread expands one row's 64-block per step
//   last warp   (single-CTA kernel at 16 tokens) a second tcgen05.mma issuer:
//               every other K step, into an accumulator of its own
#include <cudaTypedefs.h>

#include <cstring>
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
  // Dequantizer layout: G >= 2 = G groups of four warps, group g expands the stages
  // whose index is g modulo G (one lane per 64-block); 1 = all eight warps on every
  // stage (two lanes per 64-block).
  static constexpr int Groups = kGroups;
  static constexpr int kDeqArrivals = (kGroups >= 2) ? 4 : 8;
  static constexpr int kATile = 128 * 64 * 2;
  static constexpr int kBTile = TOK * 64 * 2;
  static constexpr int kRBytes = 4096;      // packed codes of one 128 x 64 weight tile
  // MMA-issuing threads: at 16 tokens the issue of the four small MMAs of every K step sets the
  // pace, so a second warp issues every other K step into an accumulator of its own (the two
  // are added in the epilogue); it is the warp after the dequantizers
  static constexpr int kIssuers = (TOK == 16) ? 2 : 1;
  static constexpr int kIssuer2Warp = 6 + 4 * (kGroups >= 2 ? kGroups : 2);
  static constexpr int kThreads = (kIssuer2Warp + (kIssuers - 1)) * 32;
  static constexpr int kAccBufs = (2 * TOK <= 512) ? 2 : 1;   // double-buffer the accumulators when TMEM allows
  static constexpr int kAccCols = kAccBufs * kIssuers * TOK;
  static constexpr int kTmemCols = (kAccCols <= 32) ? 32 : (kAccCols <= 64) ? 64 : (kAccCols <= 128) ? 128
                                   : (kAccCols <= 256) ? 256 : 512;
  static constexpr int kSmemBytes = Stages * (kATile + kBTile + kRBytes) + 1024 + 256;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(BN % 32 == 0 || BN == 16, "epilogue reads 32 columns at a time");
  static_assert(kAccCols <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kGroups == 1 || (kGroups >= 2 && kStages % kGroups == 0), "the stage index modulo G picks the group");
};

// Token tiles per raster group (L2 reuse of both operands): p.raster when set, else 4.
constexpr int kRasterGroup = 4;
constexpr int64_t kPair512From = 1024;   // above this many tokens a CTA pair takes 512 per unit


__device__ __forceinline__ void wdecode(const GemmParams& p, int u, int& mb, int& nb, int& split, int& kt0,
                                        int& nmain, int& next) {
  split = u % p.splits;
  const int t = u / p.splits;
  const int rg = (p.raster > 0) ? p.raster : kRasterGroup;
  const int per_group = rg * p.tiles_m;
  const int g = t / per_group;
  const int within = t - g * per_group;
  int gsize = p.tiles_n - g * rg;
  if (gsize > rg) gsize = rg;
  mb = within / gsize;
  nb = g * rg + (within - mb * gsize);
  kt0 = split * p.k_per_split;
  int kt1 = kt0 + p.k_per_split;
  if (kt1 > p.k_tiles) kt1 = p.k_tiles;
  nmain = kt1 - kt0;
  next = (split == 0) ? p.ext_tiles * (p.groups > 1 ? p.groups : 1) : 0;   // every layer's extension
}

// Layer of main K step kt in a grouped GEMM (0 for one layer).
__device__ __forceinline__ int wlayer(const GemmParams& p, int kt) {
  return (p.groups > 1) ? (kt >= p.k_begin[1] ? 1 : 0) + ((p.groups > 2 && kt >= p.k_begin[2]) ? 1 : 0) : 0;
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

// Epilogue: 32 (or 16) consecutive tokens of one output feature. When accumulating,
// every old value of the chunk is read before any is written back, so the chunk
// costs one memory round trip (a load after each store could not be reordered: the
// compiler cannot prove the addresses distinct).
template <int kCount>
__device__ __forceinline__ void wstore(const GemmParams& p, int split, int feat, int tok0, const uint32_t (&v)[32]) {
  if (feat >= p.rows) return;
  if (!qlora_check(feat < p.ld_out && tok0 >= 0 && (p.out_mode != kOutPartial || split < p.splits), 17)) return;
  const int64_t ld = p.ld_out;
  const int nvalid = p.cols - tok0;     // tokens of the chunk inside the output (may be < kCount or <= 0)
  if (p.accumulate && p.out_mode != kOutPartial) {
    constexpr int kBatch = (kCount == 32) ? 32 : 8;   // smaller batches keep the 16-token kernel unspilled
#pragma unroll
    for (int j0 = 0; j0 < kCount; j0 += kBatch) {
      float old[kBatch];
#pragma unroll
      for (int jj = 0; jj < kBatch; ++jj) {
        const int j = j0 + jj;
        old[jj] = 0.f;
        if (j < nvalid) {
          const int64_t off = static_cast<int64_t>(tok0 + j) * ld + feat;
          if (p.out_mode == kOutF32) old[jj] = static_cast<const float*>(p.out)[off];
          else old[jj] = __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p.out)[off]) << 16);
        }
      }
#pragma unroll
      for (int jj = 0; jj < kBatch; ++jj) {
        const int j = j0 + jj;
        if (j < nvalid) {
          const int64_t off = static_cast<int64_t>(tok0 + j) * ld + feat;
          const float y = __uint_as_float(v[j]) + old[jj];
          if (p.out_mode == kOutF32) static_cast<float*>(p.out)[off] = y;
          else static_cast<uint16_t*>(p.out)[off] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
        }
      }
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < kCount; ++j) {
    const int m = tok0 + j;
    if (m >= p.cols) break;
    const float x = __uint_as_float(v[j]);
    const int64_t off = static_cast<int64_t>(m) * ld + feat;
    if (p.out_mode == kOutPartial) {
      static_cast<float*>(p.out)[split * p.part_stride + off] = x;
    } else if (p.out_mode == kOutF32) {
      static_cast<float*>(p.out)[off] = x;
    } else {
      static_cast<uint16_t*>(p.out)[off] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
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
      mbar_init(&acc_full[a], C::kIssuers);      // one commit per issuing thread and unit
      mbar_init(&acc_empty[a], 4);
    }
    fence_mbar_init();
  }
  // an early launch streams the weight before the grid before it has finished (the
  // producer waits before the extension); otherwise nothing is touched before it has
  if (!p.early) griddep_enter();
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
      tma_prefetch_desc(&maps.act[0]);
      tma_prefetch_desc(&maps.codes[0]);
      tma_prefetch_desc(&maps.a2[0]);
      tma_prefetch_desc(&maps.b2[0]);
      int stage = 0;
      uint32_t ph = 0;
      uint32_t pending = 0, pend_par = 0;
      bool ok = true;
      bool ext_ready = false;   // the low-rank operand (s*U or s*G) of the previous launch is visible
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { ok = false; break; }
          uint64_t* bar = &tma_full[stage];
          uint8_t* a_dst = sA + stage * C::kATile;
          uint8_t* b_dst = sB + stage * C::kBTile;
          if (i >= nmain && !ext_ready) {
            // a launch that may start early (programmatic dependent launch) streams the weight
            // while the kernel that writes the low-rank operand finishes; wait here, before the
            // first load of that operand (a no-op for an ordinary launch)
            griddep_wait();
            ext_ready = true;
          }
          if (i < nmain) {
            const int kt = kt0 + i;
            mbar_arrive_expect_tx(bar, C::kRBytes + C::kBTile);
            if (C::Bwd) {
              if (tma_start_ok(mb * 64, kt * 64, 1, p.w_kblocks * 32, sR + stage * C::kRBytes, 10))
                tma_load_2d(sR + stage * C::kRBytes, &maps.codes[0], bar, mb * 64, kt * 64);
            } else if (tma_start_ok(kt * 32, mb * 128, 1, p.w_kblocks * 32, sR + stage * C::kRBytes, 11)) {
              tma_load_2d(sR + stage * C::kRBytes, &maps.codes[0], bar, kt * 32, mb * 128);
            }
#pragma unroll
            for (int t = 0; t < C::NAcc; ++t)
              if (tma_start_ok(kt * 64, nb * C::TOK + t * C::BN, 2, C::Bwd ? p.w_rows[0] : p.w_kblocks * 64,
                               b_dst + t * (C::BN * 128), 12))
                tma_load_2d(b_dst + t * (C::BN * 128), &maps.act[0], bar, kt * 64, nb * C::TOK + t * C::BN);
          } else {
            const int e = i - nmain;
            mbar_arrive_expect_tx(bar, C::kATile + C::kBTile);
            if (C::Bwd) {
              if (tma_start_ok(mb * 128, e * 64, 2, p.w_kblocks * 64, a_dst, 13))
                tma_load_2d(a_dst, &maps.a2[0], bar, mb * 128, e * 64);
              if (tma_start_ok(mb * 128 + 64, e * 64, 2, p.w_kblocks * 64, a_dst + 8192, 14))
                tma_load_2d(a_dst + 8192, &maps.a2[0], bar, mb * 128 + 64, e * 64);
            } else if (tma_start_ok(e * 64, mb * 128, 2, p.ext_tiles * 64, a_dst, 15)) {
              tma_load_2d(a_dst, &maps.a2[0], bar, e * 64, mb * 128);
            }
#pragma unroll
            for (int t = 0; t < C::NAcc; ++t)
              if (tma_start_ok(e * 64, nb * C::TOK + t * C::BN, 2, p.ext_tiles * 64, b_dst + t * (C::BN * 128), 16))
                tma_load_2d(b_dst + t * (C::BN * 128), &maps.b2[0], bar, e * 64, nb * C::TOK + t * C::BN);
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
  } else if (warp == 1 || (C::kIssuers == 2 && warp == C::kIssuer2Warp)) {
    // ------------------------------------------------------------ MMA issuer(s)
    // issuer e takes the unit's K steps i with i % kIssuers == e, into its own accumulator
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BN, C::Bwd, false);
      const int e = (warp == 1) ? 0 : 1;
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
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((acc * C::kIssuers + e) * C::TOK);
        for (int i = 0; i < nmain + next; ++i) {
          if (i % C::kIssuers != e) {
            if (++stage == C::Stages) { stage = 0; ph ^= 1; }
            continue;
          }
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          if (!mbar_wait(&deq_full[stage], ph)) { ok = false; break; }
          // operands reach the MMA through the barriers alone (TMA completion; the
          // dequantizers' fence.proxy.async before their arrival): no tcgen05 fence here
          const uint32_t a_addr = smem_u32(sA + stage * C::kATile);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBTile);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = C::Bwd ? umma_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                       : umma_desc_sw128(a_addr + kk * 32, 16, 1024);
#pragma unroll
            for (int t = 0; t < C::NAcc; ++t) {
              const uint64_t bd = umma_desc_sw128(b_addr + t * (C::BN * 128) + kk * 32, 16, 1024);
              umma_bf16(d_tmem + t * C::BN, ad, bd, idesc, (i > e || kk > 0) ? 1u : 0u);
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
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * C::kIssuers * C::TOK);
      if (C::BN == 16) {
        uint32_t v[32];
        tmem_ld_32x32b_x16(t_row, v);
        if (C::kIssuers == 2 && nmain + next > 1) {
          // the second issuer's accumulator (written only when the unit has a second K step)
          uint32_t w[32];
          tmem_ld_32x32b_x16(t_row + C::TOK, w);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__fadd_rn(__uint_as_float(v[j]), __uint_as_float(w[j])));
        } else {
          tmem_ld_wait();
        }
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
  } else if (C::Groups >= 2) {
    // ------------------------------------------------------------ dequantizers (G groups)
    // Group g (four warps) expands the stages whose index is g modulo G, so G K steps are
    // in flight at once. Forward: thread = W row of the 128-row tile, one 64-block per K step.
    // Backward: thread = (W row i of the 64-row K step, 64-column block c of the tile).
    const int grp = (warp - 6) >> 2;
    const int gt = threadIdx.x - 192 - 128 * grp;    // 0..127
    const float mean = (p.scales[0].dq_mean != nullptr) ? __ldg(p.scales[0].dq_mean) : 0.f;
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
      constexpr int G = C::Groups;
      const int first = (grp - stage % G + G) % G;     // this group's first K step of the unit
      auto block_of = [&](int i, bool& valid) -> int64_t {
        const int kt = kt0 + i;
        int64_t wrow, kb;
        if (!C::Bwd) { wrow = static_cast<int64_t>(mb) * 128 + gt; kb = kt; }
        else { wrow = static_cast<int64_t>(kt) * 64 + i_mn; kb = static_cast<int64_t>(mb) * 2 + c_mn; }
        valid = (wrow < p.w_rows[0]) && (kb < p.w_kblocks);
        return wrow * p.w_kblocks + kb;
      };
      // scale prefetch: own K steps are every G-th step; keep four of them in flight
      RawScale r0{0u, 0.f}, r1{0u, 0.f}, r2{0u, 0.f}, r3{0u, 0.f};
      {
        bool v;
        int64_t bb = block_of(first, v);
        if (first < nmain && v) r0 = load_raw_scale(p.scales[0], bb);
        bb = block_of(first + G, v);
        if (first + G < nmain && v) r1 = load_raw_scale(p.scales[0], bb);
        bb = block_of(first + 2 * G, v);
        if (first + 2 * G < nmain && v) r2 = load_raw_scale(p.scales[0], bb);
        bb = block_of(first + 3 * G, v);
        if (first + 3 * G < nmain && v) r3 = load_raw_scale(p.scales[0], bb);
      }
      for (int i = 0; i < nmain + next; ++i) {
        if (stage % G == grp) {
          if (i < nmain) {
            bool valid, v4;
            block_of(i, valid);
            const int64_t b4 = block_of(i + 4 * G, v4);
            RawScale r4{0u, 0.f};
            if (i + 4 * G < nmain && v4) r4 = load_raw_scale(p.scales[0], b4);
            if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
            const uint32_t adst = smem_u32(sA + stage * C::kATile) + a_off;
            if (valid) {
              const uint32_t rsrc = smem_u32(sR + stage * C::kRBytes);
              const uint4 w0 = ld_shared_v4_w(rsrc + r_off0);
              const uint4 w1 = ld_shared_v4_w(rsrc + r_off1);
              const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales[0], r0, mean));
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
    const float mean = (p.scales[0].dq_mean != nullptr) ? __ldg(p.scales[0].dq_mean) : 0.f;
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
        valid = (wrow < p.w_rows[0]) && (kb < p.w_kblocks);
        return wrow * p.w_kblocks + kb;
      };
      // scale prefetch: two K steps ahead
      RawScale r0{0u, 0.f}, r1{0u, 0.f};
      {
        bool v0, v1;
        const int64_t b0 = block_of(0, v0);
        const int64_t b1 = block_of(1, v1);
        if (0 < nmain && v0) r0 = load_raw_scale(p.scales[0], b0);
        if (1 < nmain && v1) r1 = load_raw_scale(p.scales[0], b1);
      }
      for (int i = 0; i < nmain + next; ++i) {
        if (i < nmain) {
          bool valid, v2;
          block_of(i, valid);
          const int64_t b2 = block_of(i + 2, v2);
          RawScale r2{0u, 0.f};
          if (i + 2 < nmain && v2) r2 = load_raw_scale(p.scales[0], b2);
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          const uint32_t adst = smem_u32(sA + stage * C::kATile) + a_off;
          if (valid) {
            const uint4 w = ld_shared_v4_w(smem_u32(sR + stage * C::kRBytes) + r_off);
            const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales[0], r0, mean));
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

// ---------------------------------------------------------------------------
// CTA-pair version for 256-token tiles (tcgen05 cta_group::2).
//
// The two CTAs of a cluster share one tile of 256 weight rows x 256 tokens.
// CTA r expands weight rows r*128.. of the tile into its own shared memory and
// loads tokens r*128.. of the activation tile; one M = 256, N = 256 MMA issued
// by the even CTA reads both halves of both operands, and each CTA's TMEM
// receives the accumulator of its own 128 weight rows over all 256 tokens.
// Per SM and K step this streams half the activation bytes of the single-CTA
// kernel (16 KB instead of 32 KB), the L2-to-SM traffic that bounds that
// kernel at 256 tokens, and halves the activation reads from shared memory.
//
// Barriers (E = the even CTA):
//   tma_full[s]   in E: E's producer expects both CTAs' activation (and
//                 extension) bytes; both CTAs' TMA loads complete on it
//   codes_full[s] in each CTA: that CTA's code tile landed (local TMA); on an
//                 extension step a plain arrival, so it has a phase per stage use
//   deq_full[d]   in E: one arrival per dequantizer warp of both CTAs (8) per
//                 main K step; its ring index d counts main steps only
//   empty[s]      in each CTA: E's MMA completion, multicast (stage reusable)
//   acc_full[a]   in each CTA: E's MMA completion, multicast (accumulator a)
//   acc_empty[a]  in E: one arrival per epilogue warp of both CTAs (8)
// ---------------------------------------------------------------------------
template <int kStages, bool kBwd, int kGroups, int kNT>
struct PCfg {
  static constexpr int BN = 256;             // tokens per MMA (N), HALF of them in each CTA
  static constexpr int HALF = 128;
  // Token tiles of BN per unit: with 2, each expanded weight tile feeds two MMAs (512
  // tokens), halving the expansion work per flop; the two accumulators then fill TMEM,
  // so the epilogue of a unit is not overlapped with the next unit's MMAs.
  static constexpr int NT = kNT;
  static constexpr int TOK = BN * NT;
  static constexpr int kAccSets = (kNT == 1) ? 2 : 1;
  static constexpr int Stages = kStages;
  static constexpr bool Bwd = kBwd;
  static constexpr int kATile = 128 * 64 * 2;
  static constexpr int kBTile = HALF * 64 * 2;
  static constexpr int kRBytes = 4096;
  // Dequantizer groups of four warps: group g expands the main K steps whose ring
  // index is g modulo kGroups, so kGroups steps are in expansion at once.
  static constexpr int Groups = kGroups;
  // Epilogue warps: four (one per TMEM lane quarter) draining every column, or eight,
  // two per quarter each draining half the columns (the second four after the dequantizers).
  static constexpr int EpiWarps = (kNT == 2) ? 8 : 4;
  static constexpr int kDeqWarp0 = 6;
  static constexpr int kEpi2Warp0 = 6 + 4 * kGroups;
  static constexpr int kThreads = (6 + 4 * kGroups + (EpiWarps - 4)) * 32;
  static constexpr int kTmemCols = 512;      // two accumulators of 256 columns
  static constexpr int kBStage = NT * kBTile;  // activation bytes of one stage in one CTA
  static constexpr int kSmemBytes = Stages * (kATile + kBStage + kRBytes) + 1024 + 256;
  static_assert(kStages % kGroups == 0, "the ring index modulo kGroups picks the dequantizer group");
  static_assert(kNT == 1 || kNT == 2, "one or two token tiles per unit");
  static_assert(kAccSets * TOK <= kTmemCols, "TMEM columns");
  static_assert(4 * kStages + 4 <= 31, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    qlora_wgemm_pair_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ WMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);   // same offsets in both CTAs
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::Stages * C::kATile;
  uint8_t* sR = sB + C::Stages * C::kBStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + C::Stages * C::kRBytes);
  uint64_t* tma_full = bars;
  uint64_t* codes_full = tma_full + C::Stages;
  uint64_t* deq_full = codes_full + C::Stages;
  uint64_t* empty = deq_full + C::Stages;
  uint64_t* acc_full = empty + C::Stages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool even = (rank == 0);
  const int pair = static_cast<int>(cluster_id_x());
  const int pairs = static_cast<int>(cluster_count_x());
  const int units = p.tiles_m * p.tiles_n * p.splits;     // tiles_m counts 256-row tiles

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::Stages; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&codes_full[s], 1);
      mbar_init(&deq_full[s], 8);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * C::EpiWarps);    // every epilogue warp of both CTAs
    }
    fence_mbar_init();
  }
  griddep_enter();
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();      // both CTAs' barriers exist before any remote arrival or load lands on them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const int ng = (p.groups > 1) ? p.groups : 1;
      for (int l = 0; l < ng; ++l) {
        tma_prefetch_desc(&maps.act[l]);
        tma_prefetch_desc(&maps.codes[l]);
        tma_prefetch_desc(&maps.a2[l]);
        tma_prefetch_desc(&maps.b2[l]);
      }
      int stage = 0;
      uint32_t ph = 0;
      uint32_t pend_codes = 0, pend_full = 0, pend_par = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += pairs) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        const int mh = 2 * mb + rank;                      // this CTA's 128-row tile
        const int tok0 = nb * C::TOK + rank * C::HALF;     // + t * BN for token tile t
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { ok = false; break; }
          pend_codes &= ~(1u << stage);
          pend_full &= ~(1u << stage);
          const uint32_t full_e = smem_cluster_addr(&tma_full[stage], 0);
          uint8_t* a_dst = sA + stage * C::kATile;
          uint8_t* b_dst = sB + stage * C::kBStage;
          if (i < nmain) {
            const int l = wlayer(p, kt0 + i);
            const int kt = kt0 + i - p.k_begin[l];          // K step within layer l
            mbar_arrive_expect_tx(&codes_full[stage], C::kRBytes);
            if (C::Bwd) {
              if (tma_start_ok(mh * 64, kt * 64, 1, p.w_kblocks * 32, sR + stage * C::kRBytes, 20))
                tma_load_2d(sR + stage * C::kRBytes, &maps.codes[l], &codes_full[stage], mh * 64, kt * 64);
            } else if (tma_start_ok(kt * 32, mh * 128, 1, p.w_kblocks * 32, sR + stage * C::kRBytes, 21)) {
              tma_load_2d(sR + stage * C::kRBytes, &maps.codes[l], &codes_full[stage], kt * 32, mh * 128);
            }
            pend_codes |= (1u << stage);
            if (even) mbar_arrive_expect_tx(&tma_full[stage], 2 * C::kBStage);
#pragma unroll
            for (int t = 0; t < C::NT; ++t)
              if (tma_start_ok(kt * 64, tok0 + t * C::BN, 2, C::Bwd ? p.w_rows[l] : p.w_kblocks * 64,
                               b_dst + t * C::kBTile, 22))
                tma_load_2d_pair(b_dst + t * C::kBTile, &maps.act[l], full_e, kt * 64, tok0 + t * C::BN);
          } else {
            const int l = (i - nmain) / p.ext_tiles;       // layer of this extension step
            const int e = i - nmain - l * p.ext_tiles;
            // no codes for an extension step: complete codes_full's phase anyway, so that its
            // phases count every use of the stage as the dequantizers' ring phase does
            mbar_arrive(&codes_full[stage]);
            if (even) mbar_arrive_expect_tx(&tma_full[stage], 2 * (C::kATile + C::kBStage));
            if (C::Bwd) {
              if (tma_start_ok(mh * 128, e * 64, 2, p.w_kblocks * 64, a_dst, 23))
                tma_load_2d_pair(a_dst, &maps.a2[l], full_e, mh * 128, e * 64);
              if (tma_start_ok(mh * 128 + 64, e * 64, 2, p.w_kblocks * 64, a_dst + 8192, 24))
                tma_load_2d_pair(a_dst + 8192, &maps.a2[l], full_e, mh * 128 + 64, e * 64);
            } else if (tma_start_ok(e * 64, mh * 128, 2, p.ext_tiles * 64, a_dst, 25)) {
              tma_load_2d_pair(a_dst, &maps.a2[l], full_e, e * 64, mh * 128);
            }
#pragma unroll
            for (int t = 0; t < C::NT; ++t)
              if (tma_start_ok(e * 64, tok0 + t * C::BN, 2, p.ext_tiles * 64, b_dst + t * C::kBTile, 26))
                tma_load_2d_pair(b_dst + t * C::kBTile, &maps.b2[l], full_e, e * 64, tok0 + t * C::BN);
          }
          pend_full |= (1u << stage);
          pend_par = (pend_par & ~(1u << stage)) | (ph << stage);
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
      }
      if (ok) {
        for (int s = 0; s < C::Stages; ++s) {   // every stage released once more: no load still lands
          if (!mbar_wait(&empty[stage], ph ^ 1)) break;
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
      } else {
        for (int s = 0; s < C::Stages; ++s) {
          if (pend_codes & (1u << s)) mbar_wait(&codes_full[s], (pend_par >> s) & 1u);
          if (even && (pend_full & (1u << s))) mbar_wait(&tma_full[s], (pend_par >> s) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (even && lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(C::BN, C::Bwd, false, 256);
      // Descriptors: fixed fields once; per stage only the start address (16-byte units)
      // changes, and a K step of 16 moves it by 32 bytes (K-major) or 2048 bytes (MN-major).
      const uint64_t a_desc0 = C::Bwd ? umma_desc_sw128(smem_u32(sA), 8192, 1024) : umma_desc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = umma_desc_sw128(smem_u32(sB), 16, 1024);
      constexpr uint64_t kAStep = C::Bwd ? (2048 >> 4) : (32 >> 4);
      constexpr uint64_t kBStep = 32 >> 4;
      int stage = 0, dstage = 0, acc = 0;
      uint32_t ph = 0, dph = 0, aph = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += pairs) {
        int mb, nb, split, kt0, nmain, next;
        wdecode(p, u, mb, nb, split, kt0, nmain, next);
        if (!mbar_wait(&acc_empty[acc], aph ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::TOK);
        for (int i = 0; i < nmain + next; ++i) {
          if (!mbar_wait(&tma_full[stage], ph)) { ok = false; break; }
          if (i < nmain) {
            if (!mbar_wait(&deq_full[dstage], dph)) { ok = false; break; }
            if (++dstage == C::Stages) { dstage = 0; dph ^= 1; }
          }
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(stage) * (C::kATile >> 4);
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(stage) * (C::kBStage >> 4);
#pragma unroll
          for (int t = 0; t < C::NT; ++t) {
            const uint32_t dt = d_tmem + static_cast<uint32_t>(t * C::BN);
            const uint64_t bt = bd + static_cast<uint64_t>(t) * (C::kBTile >> 4);
            umma_bf16_pair(dt, ad, bt, idesc, i > 0 ? 1u : 0u);
            umma_bf16_pair(dt, ad + kAStep, bt + kBStep, idesc, 1u);
            umma_bf16_pair(dt, ad + 2 * kAStep, bt + 2 * kBStep, idesc, 1u);
            umma_bf16_pair(dt, ad + 3 * kAStep, bt + 3 * kBStep, idesc, 1u);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == C::Stages) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[acc], 0x3);
        if (++acc == C::kAccSets) { acc = 0; aph ^= 1; }
      }
    }
    __syncwarp();
  } else if (warp < C::kDeqWarp0 || warp >= C::kEpi2Warp0) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;                                           // TMEM lane quarter
    constexpr int kCols = C::TOK / (C::EpiWarps / 4);                 // columns per warp
    const int col0 = (warp >= C::kEpi2Warp0) ? kCols : 0;
    const uint32_t acc_empty_e0 = smem_cluster_addr(&acc_empty[0], 0);
    const uint32_t acc_empty_e1 = smem_cluster_addr(&acc_empty[1], 0);
    int acc = 0;
    uint32_t aph = 0;
    for (int u = pair; u < units; u += pairs) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      if (!mbar_wait(&acc_full[acc], aph)) break;
      tc_fence_after();
      const int feat = (2 * mb + rank) * 128 + q * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::TOK);
#pragma unroll 1
      for (int c = col0; c < col0 + kCols; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_row + c, v);
        tmem_ld_wait();
        wstore<32>(p, split, feat, nb * C::TOK + c, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc ? acc_empty_e1 : acc_empty_e0);
      if (++acc == C::kAccSets) { acc = 0; aph ^= 1; }
    }
  } else {
    // ------------------------------------------------------------ dequantizers (both CTAs)
    // As in the single-CTA kernel, on this CTA's 128-row tile, with C::Groups groups taking
    // main K steps in turn; each warp reports its finished tile to the even CTA's deq_full.
    const int grp = (warp - C::kDeqWarp0) >> 2;
    const int gt = threadIdx.x - 32 * C::kDeqWarp0 - 128 * grp;    // 0..127
    // each layer's double-quant mean (a grouped GEMM has up to kWGroupMax weights)
    const int ng = (p.groups > 1) ? p.groups : 1;
    const float mean0 = (p.scales[0].dq_mean != nullptr) ? __ldg(p.scales[0].dq_mean) : 0.f;
    const float mean1 = (ng > 1 && p.scales[1].dq_mean != nullptr) ? __ldg(p.scales[1].dq_mean) : 0.f;
    const float mean2 = (ng > 2 && p.scales[2].dq_mean != nullptr) ? __ldg(p.scales[2].dq_mean) : 0.f;
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
    const uint32_t deq_e = smem_cluster_addr(deq_full, 0);    // deq_full[d] of the even CTA: deq_e + 8 d
    int stage = 0, dstage = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int u = pair; u < units && ok; u += pairs) {
      int mb, nb, split, kt0, nmain, next;
      wdecode(p, u, mb, nb, split, kt0, nmain, next);
      const int mh = 2 * mb + rank;
      const int first = (grp - dstage % C::Groups + C::Groups) % C::Groups;   // first own main step
      constexpr int G = C::Groups;
      // block index of main step i in its layer's scales (layer returned in l)
      auto block_of = [&](int i, bool& valid, int& l) -> int64_t {
        l = wlayer(p, kt0 + i);
        const int kt = kt0 + i - p.k_begin[l];
        int64_t wrow, kb;
        if (!C::Bwd) { wrow = static_cast<int64_t>(mh) * 128 + gt; kb = kt; }
        else { wrow = static_cast<int64_t>(kt) * 64 + i_mn; kb = static_cast<int64_t>(mh) * 2 + c_mn; }
        valid = (wrow < p.w_rows[l]) && (kb < p.w_kblocks);
        return wrow * p.w_kblocks + kb;
      };
      RawScale r0{0u, 0.f}, r1{0u, 0.f}, r2{0u, 0.f}, r3{0u, 0.f};
      {
        bool v;
        int l;
        int64_t bb = block_of(first, v, l);
        if (first < nmain && v) r0 = load_raw_scale(p.scales[l], bb);
        bb = block_of(first + G, v, l);
        if (first + G < nmain && v) r1 = load_raw_scale(p.scales[l], bb);
        bb = block_of(first + 2 * G, v, l);
        if (first + 2 * G < nmain && v) r2 = load_raw_scale(p.scales[l], bb);
        bb = block_of(first + 3 * G, v, l);
        if (first + 3 * G < nmain && v) r3 = load_raw_scale(p.scales[l], bb);
      }
      for (int i = 0; i < nmain + next; ++i) {
        if (i < nmain) {
          if (dstage % G == grp) {
            bool valid, v4;
            int l, l4;
            block_of(i, valid, l);
            const int64_t b4 = block_of(i + 4 * G, v4, l4);
            RawScale r4{0u, 0.f};
            if (i + 4 * G < nmain && v4) r4 = load_raw_scale(p.scales[l4], b4);
            if (!mbar_wait(&codes_full[stage], ph)) { ok = false; break; }
            const uint32_t adst = smem_u32(sA + stage * C::kATile) + a_off;
            if (valid) {
              const uint32_t rsrc = smem_u32(sR + stage * C::kRBytes);
              const uint4 w0 = ld_shared_v4_w(rsrc + r_off0);
              const uint4 w1 = ld_shared_v4_w(rsrc + r_off1);
              const float mean = (l == 0) ? mean0 : (l == 1) ? mean1 : mean2;
              const Nf4Lut lut = nf4_build_lut(p.tab, raw_to_scale(p.scales[l], r0, mean));
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
            // expanded tile visible to the async proxy (either SM's tensor core reads it);
            // code reads ordered before the slot's async refill
            fence_proxy_async_smem();
            r0 = r1;
            r1 = r2;
            r2 = r3;
            r3 = r4;
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(deq_e + static_cast<uint32_t>(dstage) * 8u);
          }
          if (++dstage == C::Stages) dstage = 0;
        }
        if (++stage == C::Stages) { stage = 0; ph ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();      // no CTA leaves while the other may still arrive on its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

template <class C>
static cudaError_t launch_pcfg(const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st) {
  static bool attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(qlora_wgemm_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::kSmemBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  if (grid < 2 || (grid & 1)) return cudaErrorInvalidValue;
  return launch_pdl(qlora_wgemm_pair_kernel<C>, grid, C::kThreads, C::kSmemBytes, st, 2, p, maps);
}

// CTA pairs of the 256-token kernel that fit on the device at once (one CTA per SM).
int wgemm_pair_slots() {
  static int cached[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 74;   // no device: a B200's 148 SMs
  std::lock_guard<std::mutex> g(mu);
  if (cached[dev] > 0) return cached[dev];
  using C = PCfg<6, false, 2, 1>;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  int slots = sms / 2;
  if (cudaFuncSetAttribute(qlora_wgemm_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, qlora_wgemm_pair_kernel<C>, &cfg) == cudaSuccess && n > 0 && n < slots)
      slots = n;
  }
  cudaGetLastError();
  cached[dev] = slots > 0 ? slots : 1;
  return cached[dev];
}

template <class C>
static cudaError_t launch_wcfg(const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st, bool early) {
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
  GemmParams q = p;
  q.early = early ? 1 : 0;
  return launch_pdl(qlora_wgemm_kernel<C>, grid, C::kThreads, C::kSmemBytes, st, 1, q, maps);
}

int wgemm_box_rows(int bn) { return bn >= 256 ? 128 : bn; }   // a CTA pair loads half of each 256-token tile

int wgemm_tile_rows(int bn) { return bn >= 256 ? 256 : 128; }  // weight rows per tile (two CTAs from 256 tokens)

int wgemm_grid(const GemmParams& p, int bn, int sms) {
  const int64_t units = static_cast<int64_t>(p.tiles_m) * p.tiles_n * p.splits;
  if (bn >= 256) return static_cast<int>(2 * std::min<int64_t>(units, wgemm_pair_slots()));
  return static_cast<int>(std::min<int64_t>(units, sms));
}

int wgemm_bn(int64_t tokens) {
  if (tokens <= 16) return 16;
  if (tokens <= 64) return 64;
  if (tokens <= 128) return 128;
  if (tokens <= kPair512From) return 256;
  return 512;
}

cudaError_t launch_wgemm(bool bwd, int bn, const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st,
                         double algo_flops, bool early) {
  // the tile counts must be those of the kernel this width selects
  if (p.tiles_n != (static_cast<int64_t>(p.cols) + bn - 1) / bn ||
      p.tiles_m != (static_cast<int64_t>(p.rows) + wgemm_tile_rows(bn) - 1) / wgemm_tile_rows(bn))
    return cudaErrorInvalidValue;
  const bool timed = timing_active();
  if (timed) timing_record(st, true, algo_flops);
  cudaError_t e = cudaErrorInvalidValue;
  if (!bwd) {
    switch (bn) {
      case 16: e = launch_wcfg<WCfg<16, 1, 9, false, 3>>(p, maps, grid, st, early); break;
      case 64: e = launch_wcfg<WCfg<64, 1, 6, false, 3>>(p, maps, grid, st, early); break;
      case 128: e = launch_wcfg<WCfg<128, 1, 6, false, 3>>(p, maps, grid, st, early); break;
      case 256: e = launch_pcfg<PCfg<6, false, 2, 1>>(p, maps, grid, st); break;   // CTA pair
      case 512: e = launch_pcfg<PCfg<4, false, 2, 2>>(p, maps, grid, st); break;   // CTA pair, two token tiles
    }
  } else {
    switch (bn) {
      case 16: e = launch_wcfg<WCfg<16, 1, 9, true, 3>>(p, maps, grid, st, early); break;
      case 64: e = launch_wcfg<WCfg<64, 1, 6, true, 3>>(p, maps, grid, st, early); break;
      case 128: e = launch_wcfg<WCfg<128, 1, 6, true, 3>>(p, maps, grid, st, early); break;
      case 256: e = launch_pcfg<PCfg<6, true, 2, 1>>(p, maps, grid, st); break;    // CTA pair
      case 512: e = launch_pcfg<PCfg<4, true, 2, 2>>(p, maps, grid, st); break;    // CTA pair, two token tiles
    }
  }
  if (timed) timing_record(st, false, algo_flops);
  return e;
}

}  // namespace qlora
