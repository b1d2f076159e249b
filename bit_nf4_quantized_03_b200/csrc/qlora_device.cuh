// Device-side building blocks shared by the kernels of libqlora (sm_100a only):
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM alloc, UMMA
// descriptors, MMA issue/commit, TMEM loads), and the NF4 per-block lookup
// table that turns packed 4-bit codes into BF16 with byte permutes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

// Level table handed to every kernel by value (lives in the parameter bank).
// lv: the 16 NF4 levels (fp32, ascending); mid: the 15 fp32 decision
// thresholds fp32(fp32(lv[i] + lv[i+1]) * 0.5).
struct Nf4Table {
  float lv[16];
  float mid[16];
};

// Exact one-comparison code search for the quantizer: 33 buckets of width
// 1/16 centred on j/16, j = -16 .. 16 (entry j + 16): bucket j is the x with
// round(16 x) = j, [j/16 - 1/32, j/16 + 1/32], widened by 1e-3 on each side;
// thr is the single decision threshold inside the widened bucket (+inf if
// none) and base the number of thresholds below it. code(x) = base + (x > thr).
constexpr int kNf4Buckets = 33;
struct Nf4Buckets {
  float thr[kNf4Buckets];
  int32_t base[kNf4Buckets];
};

// Device error word: kernels write a non-zero code here when a bounded wait
// gives up, so the host can read the failure instead of the GPU hanging.
enum : int { kErrNone = 0, kErrWaitTimeout = 1, kErrBadLayout = 2, kErrBounds = 3 };   // values of g_device_error
extern __device__ int g_device_error;
extern __device__ int g_bounds_site;       // first failed bounds check (bounds-check build)

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// bf16x2 from two fp32 values, round to nearest even: low half = lo.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Bounds checks. In a build with -DQLORA_BOUNDS_CHECK (build.py --bounds-check)
// qlora_check records a failed condition -- kErrBounds in the error word and the
// site number in g_bounds_site, first failure kept -- and returns false, so the
// caller skips the access it guards (a skipped TMA load then leaves its barrier
// incomplete, and the bounded waits end the kernel). No assert, no trap. In the
// normal build both helpers are constant true and cost nothing.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool qlora_check(bool ok, int site) {
#ifdef QLORA_BOUNDS_CHECK
  if (!ok) {
    atomicCAS(&g_bounds_site, 0, site);
    atomicExch(&g_device_error, kErrBounds);
  }
  return ok;
#else
  (void)ok;
  (void)site;
  return true;
#endif
}

// Start of a 2D TMA tile: x (innermost, in elements of elem_bytes) on a 16-byte
// boundary, x and y not negative, shared-memory address 16-byte aligned, and x
// less than one tile (256 elements) past the tensor's inner extent. A tile may
// start past the edge by design on ragged shapes -- the load reads the fill
// value there -- but a start further out means a wrong plan.
__device__ __forceinline__ bool tma_start_ok(int32_t x, int32_t y, int elem_bytes, int64_t inner, const void* smem,
                                             int site) {
#ifdef QLORA_BOUNDS_CHECK
  return qlora_check(x >= 0 && y >= 0 && (static_cast<int64_t>(x) * elem_bytes) % 16 == 0 && x < inner + 256 &&
                         (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 15u) == 0,
                     site);
#else
  (void)x;
  (void)y;
  (void)elem_bytes;
  (void)inner;
  (void)smem;
  (void)site;
  return true;
#endif
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended (up to `hint_ns`) until the
// phase completes instead of returning at once, so a waiting warp does not
// take issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up after
// roughly `kWaitLimitNs` of wall time, records kErrWaitTimeout and returns
// false; every caller then abandons its loop so the whole CTA can exit.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr uint32_t kSuspendHintNs = 20000;         // longest suspension per try (20 us)

__device__ __forceinline__ bool mbar_wait(uint64_t* bar_ptr, uint32_t parity) {
  const uint32_t bar = smem_u32(bar_ptr);
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t tries = 0;
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, kSuspendHintNs)) return true;
    if ((++tries & 15u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicCAS(&g_device_error, kErrNone, kErrWaitTimeout);   // an earlier error (its cause) is kept
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------
// Programmatic dependent launch. griddep_wait: block until the grids this one was
// launched after have completed and their writes are visible (returns at once when
// the launch did not allow an early start). griddep_launch_dependents: from this CTA's
// side, a grid launched after this one with that allowance may start now.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
// Programmatic dependent launch, at a kernel's start: wait until the grid before this one
// on the stream has completed and its writes are visible, then allow the grid after this
// one to be scheduled (it waits in turn before it touches memory). A no-op for a launch
// without the programmatic attribute.
__device__ __forceinline__ void griddep_enter() {
  griddep_wait();
  griddep_launch_dependents();
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Contiguous bulk copy global -> shared (TMA engine, no tensor map, no
// multicast). Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  if (!qlora_check(bytes > 0 && (bytes & 15u) == 0 && (reinterpret_cast<uintptr_t>(gsrc) & 15u) == 0 &&
                       (static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst)) & 15u) == 0,
                   90))
    return;
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Tiled store shared -> global through the TMA engine (bulk-group completion).
// Elements outside the tensor are not written. x must be 16-byte aligned.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed bulk groups are still in flight (writes complete).
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA descriptors, MMA, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile.
// lbo/sbo in bytes. K-major: rows of 128 B, 8-row groups `sbo` apart (lbo
// unused). MN-major: 64-element MN chunks `lbo` apart, 8-row K groups `sbo`
// apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;                      // descriptor version for sm_100
  d |= 2ull << 61;                      // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::f16 with BF16 A/B, FP32 accumulate, M = 128.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int n, bool a_mn_major, bool b_mn_major, int m = 128) {
  return (1u << 4)                                  // D format: f32
         | (1u << 7)                                // A format: bf16
         | (1u << 10)                               // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16 (256 for a CTA pair)
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs on neighbouring SMs) for tcgen05 cta_group::2:
// one M = 256 MMA issued by the even CTA reads each CTA's half of A and B from
// that CTA's shared memory and writes each CTA's half of D into its own TMEM.
// Every tcgen05 instruction of a kernel that pairs uses cta_group::2.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t smem_cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Both CTAs of the cluster reach this point (hardware barrier, release/acquire).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier of any CTA of the cluster (address from smem_cluster_addr).
// Default (CTA-scope) release: a cluster-scope release would first wait for every
// memory access of the thread still in flight, scale prefetches included. Each
// arrival that hands over a shared-memory tile follows fence.proxy.async by the
// writing threads, and each CTA's tensor core reads its own CTA's half.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 2D TMA load into this CTA's shared memory whose completion (bytes) is counted
// on an mbarrier of the pair's even CTA (`bar_cluster` from smem_cluster_addr).
// No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
// Both CTAs' warp with the same index allocate together; the same column base
// is returned in each CTA.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A . B^T over the pair: M = 256 (128 rows of A per CTA), N columns
// (N / 2 rows of B per CTA); issued by one thread of the even CTA.
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive, on the barrier at this offset in each CTA of `cta_mask`, once every
// pair MMA issued so far is done (multicast completion signal, not a load).
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp gets TMEM lane
// (warp's lane quarter base + i), columns col..col+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// NF4 dequantization of one 64-block through a per-block lookup table.
//
// For a block with scale c the 16 possible outputs are T[j] = bf16(fp32(lv[j]
// * c)) -- exactly the values the format defines, computed once per block
// instead of once per weight. The table is held as byte planes (lo[g] holds
// the low bytes of T[4g..4g+3], hi[g] the high bytes) so that PRMT can index
// it with 3-bit selectors; bit 3 of each code chooses between the two
// 8-entry halves.
// ---------------------------------------------------------------------------
struct Nf4Lut {
  uint32_t lo[4];
  uint32_t hi[4];
};

__device__ __forceinline__ Nf4Lut nf4_build_lut(const Nf4Table& t, float c) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = pack_bf16x2(__fmul_rn(t.lv[2 * i], c), __fmul_rn(t.lv[2 * i + 1], c));
  Nf4Lut l;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    l.lo[g] = prmt(p[2 * g], p[2 * g + 1], 0x6420);
    l.hi[g] = prmt(p[2 * g], p[2 * g + 1], 0x7531);
  }
  return l;
}

// Four codes in the low 16 bits of `s` (code i in bits 4i..4i+3) -> four
// bf16 values as two bf16x2 words (element order preserved).
__device__ __forceinline__ void nf4_lookup4(const Nf4Lut& l, uint32_t s, uint32_t& out01,
                                            uint32_t& out23) {
  const uint32_t idx = s & 0x7777u;
  const uint32_t sel = ((s >> 1) & 0x4444u) | 0x3210u;
  const uint32_t la = prmt(l.lo[0], l.lo[1], idx);
  const uint32_t lb = prmt(l.lo[2], l.lo[3], idx);
  const uint32_t ha = prmt(l.hi[0], l.hi[1], idx);
  const uint32_t hb = prmt(l.hi[2], l.hi[3], idx);
  const uint32_t lo = prmt(la, lb, sel);
  const uint32_t hi = prmt(ha, hb, sel);
  out01 = prmt(lo, hi, 0x5140);
  out23 = prmt(lo, hi, 0x7362);
}

// Eight codes (one 32-bit word of packed nibbles) -> 8 bf16 as a uint4.
__device__ __forceinline__ uint4 nf4_lookup8(const Nf4Lut& l, uint32_t w) {
  uint4 o;
  nf4_lookup4(l, w, o.x, o.y);
  nf4_lookup4(l, w >> 16, o.z, o.w);
  return o;
}

// Scale of block `b`: BF16 mode widens the stored bf16; double-quant mode
// rebuilds fp32(fp32(e4m3(q) * s2[b / 256]) + mean).
__device__ __forceinline__ float e4m3_to_float(uint8_t q) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q), __NV_E4M3);
  return __half2float(__half(h));
}

struct ScaleSrc {
  const uint16_t* bf16;      // BF16 mode (else null)
  const uint8_t* fp8;        // double-quant mode
  const float* dq_scale;
  const float* dq_mean;
};

__device__ __forceinline__ float block_scale(const ScaleSrc& s, int64_t b, float mean) {
  if (s.bf16 != nullptr) {
    const uint32_t bits = static_cast<uint32_t>(__ldg(s.bf16 + b)) << 16;
    return __uint_as_float(bits);
  }
  const float q = e4m3_to_float(__ldg(s.fp8 + b));
  return __fadd_rn(__fmul_rn(q, __ldg(s.dq_scale + (b >> 8))), mean);
}

// Raw scale bytes of one block, loaded ahead of use; raw_to_scale gives the
// same fp32 value as block_scale.
struct RawScale {
  uint32_t q;
  float s2;
};

__device__ __forceinline__ RawScale load_raw_scale(const ScaleSrc& s, int64_t b) {
  RawScale r;
  if (s.bf16 != nullptr) {
    r.q = __ldg(s.bf16 + b);
    r.s2 = 0.f;
  } else {
    r.q = __ldg(s.fp8 + b);
    r.s2 = __ldg(s.dq_scale + (b >> 8));
  }
  return r;
}

__device__ __forceinline__ float raw_to_scale(const ScaleSrc& s, const RawScale& r, float mean) {
  if (s.bf16 != nullptr) return __uint_as_float(r.q << 16);
  return __fadd_rn(__fmul_rn(e4m3_to_float(static_cast<uint8_t>(r.q)), r.s2), mean);
}

}  // namespace qlora
