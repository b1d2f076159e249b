// Internal launch interface between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "qlora_device.cuh"

namespace qlora {

// ----------------------------------------------------------------- quantize
struct QuantWsLayout {
  size_t absmax_off, part_a_off, part_b_off, mean_off, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline QuantWsLayout quant_ws_layout(int64_t n_elem) {
  const int64_t nblk = (n_elem + 63) / 64;
  const int64_t pa = (nblk + 127) / 128;          // one fp64 partial per 128 blocks
  const int64_t pb = (pa + 511) / 512 + 1;
  QuantWsLayout L;
  L.absmax_off = 0;
  L.part_a_off = align_up(static_cast<size_t>(nblk) * 4, 256);
  L.part_b_off = L.part_a_off + align_up(static_cast<size_t>(pa) * 8, 256);
  L.mean_off = L.part_b_off + align_up(static_cast<size_t>(pb) * 8, 256);
  L.total = L.mean_off + 256;
  return L;
}

// Largest tensor the double-quant mean supports: the fixed tree keeps at most 2048
// first-level group sums (groups of 512 chunk partials of 128 blocks of 64 weights).
constexpr int64_t kMaxDqElems = int64_t(2048) * 512 * 128 * 64;

cudaError_t launch_quantize(const float* W, int64_t n_elem, const Nf4Table& tab, const Nf4Buckets& bk,
                            uint8_t* codes, uint16_t* scale_bf16, uint8_t* scale_fp8, float* dq_scale,
                            float* dq_mean, void* ws, int num_sms, cudaStream_t st);
// Bucket table of the quantizer's code search, built from the 15 midpoints (qlora_abi.cu).
Nf4Buckets nf4_buckets_from_midpoints(const float* mid);
// The level table and bucket table every entry point uses, and the SM count of the
// current device (qlora_abi.cu; built once, cached).
const Nf4Table& host_table();
const Nf4Buckets& host_buckets();
int host_num_sms();
// Unique id of the calling thread's current CUDA context, 0 when none is current
// (qlora_noalloc.cu; ids are never reused within a process).
unsigned long long context_id();
cudaError_t launch_dequantize(const uint8_t* codes, const ScaleSrc& ss, int64_t n_elem, const Nf4Table& tab,
                              uint16_t* out, int num_sms, cudaStream_t st);

// --------------------------------------------------------------------- GEMM
// Operand sources of the low-rank tensor-core GEMM D[rows, cols] = sum_k A[row, k] B[col, k].
enum BMode : int {
  kB_TmaK = 0,    // bf16 [cols, K] row-major via TMA (K-major)
  kB_TmaMN = 1,   // bf16 [K, cols] row-major via TMA (MN-major)
};

enum OutMode : int {
  kOutBF16 = 0,     // bf16 [rows, cols] with leading dimension ld_out
  kOutF32 = 1,      // fp32 [rows, cols]
  kOutPartial = 2,  // fp32 split-K partial: out + split * part_stride, [rows, ld_out]
  kOutMaskAccBF16 = 3,  // bf16 out += keep_scale * D where the bit mask keeps the element (dropout dX)
  kOutMaskAccF32 = 4,   // fp32 out, same
};

// Layers at most in one grouped weight GEMM (the backward of projections that share an
// input: q, k and v; or gate and up).
constexpr int kWGroupMax = 3;

struct GemmParams {
  int32_t rows, cols;          // problem size of D
  int32_t tiles_m, tiles_n;    // 128-row and BN-col tiles
  int32_t k_tiles;             // main-loop 64-wide K steps
  int32_t ext_tiles;           // extra K steps from the second operand pair (low-rank branch)
  int32_t splits, k_per_split; // split of the main K steps
  // NF4 operand (weight-operand GEMM only). A grouped GEMM (CTA-pair kernel, backward)
  // runs its reduction over the layers in turn: layer l owns main K steps
  // [k_begin[l], k_begin[l + 1]) and extension steps [l * ext_tiles, (l + 1) * ext_tiles)
  // after every main step; one layer: groups = 1, k_begin = {0, k_tiles}.
  int32_t groups;
  int32_t k_begin[kWGroupMax + 1];
  ScaleSrc scales[kWGroupMax];
  int64_t w_kblocks;           // 64-blocks per row of W (the same for every layer of a group)
  int32_t w_rows[kWGroupMax];  // rows of each layer's W
  // output
  void* out;
  int64_t ld_out;
  int64_t part_stride;         // elements between split partials
  int32_t out_mode;
  int32_t accumulate;          // kOutBF16/kOutF32: out += D
  Nf4Table tab;
  // masked modes: bit (row * ld_out + col) of `mask` (bit e % 8 of byte e / 8) keeps the element
  const uint8_t* mask;
  float keep_scale;
  // weight GEMM: token tiles per raster group (0 = the kernel's default)
  int32_t raster;
  // single-CTA weight GEMM only (set by launch_wgemm): 1 = started before the grid that
  // writes the low-rank operand has finished; only the producer waits, before its first
  // extension load
  int32_t early;
};

struct GemmMaps {
  CUtensorMap a, b, a2, b2;    // b2 = lo half of B in the hi/lo mode (a2 unused)
};

// Host helpers (nf4_gemm.cu). swizzle: 0 none, 32, 64 or 128 (bytes).
bool tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle);

// Launch variants of the low-rank GEMM
enum GemmKind : int {
  kGemmLoraDownK = 2,  // A K-major, B K-major, BN = 64 (U = X A^T)
  kGemmLoraDownMN = 3, // A K-major, B MN-major, BN = 64 (G = dY B)
  kGemmLoraGrad = 4,   // A MN-major, B MN-major hi+lo, BN = 64 (dB, dA^T)
  kGemmLoraDownK128 = 5,
  kGemmLoraDownMN128 = 6,
  kGemmLoraGrad128 = 7,
  kGemmLoraUpMasked = 8,   // as kGemmLoraDownMN128 (K = rank), two epilogue groups: dropout's masked dX term
};

int gemm_bn(GemmKind kind);
cudaError_t launch_gemm(GemmKind kind, const GemmParams& p, const GemmMaps& maps, int grid, cudaStream_t st);

// Launch accounting (qlora_abi.cu): every kernel launch is counted; fused NF4
// GEMM launches can additionally be bracketed by timing events.
void count_launches(int n);
bool timing_active();
void timing_record(cudaStream_t st, bool start, double flops);

// Launch with programmatic dependent launch allowed: the grid may be scheduled while the
// grid before it on the stream finishes. Every kernel of the library starts with
// griddep_enter() (or, where stated, waits later), so it reads and writes nothing before
// the grid before it has completed, and the grid after it is scheduled only once all of
// this grid's CTAs are past that wait. `cluster_x` > 1 adds a cluster dimension.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                              int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(block), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int na = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    na = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  count_launches(1);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ------------------------------------------------------- weight-operand GEMM
// (nf4_wgemm.cu) D^T[features, tokens] with the dequantized weight as the
// 128-row MMA operand. GemmParams: rows = features (n forward, k backward),
// cols = tokens, tiles_m = features / 128, tiles_n = tokens / BN; the output is
// row-major [tokens, ld_out] (Y or dX), split partials the same way.
struct WMaps {          // one entry per layer of a group ([0] alone for one layer)
  CUtensorMap act[kWGroupMax];     // activations [tokens, reduction] bf16, box [64, BN], 128B swizzle
  CUtensorMap codes[kWGroupMax];   // packed codes [n, k/2] u8; forward box [32, 128] (32B swizzle), backward [64, 64] (64B)
  CUtensorMap a2[kWGroupMax];      // low-rank A-side tile: B_lora [n, r] (forward) or A_lora [r, k] (backward)
  CUtensorMap b2[kWGroupMax];      // low-rank B-side tile: s*U or s*G [tokens, r_pad]
};
int wgemm_bn(int64_t tokens);          // tokens per tile
int wgemm_box_rows(int bn);              // token rows per TMA box (each CTA of a pair loads half)
int wgemm_tile_rows(int bn);             // weight rows per tile: 256 when a CTA pair shares it
int wgemm_pair_slots();                  // CTA pairs resident at once
int wgemm_grid(const GemmParams& p, int bn, int sms);   // CTAs to launch (even for CTA pairs)
// early: the single-CTA kernel (bn <= 128) may start before the preceding kernel on the
// stream has finished (programmatic dependent launch); it waits for that kernel only
// before its first load of the low-rank operand, which that kernel must write and
// nothing else it reads or writes. Ignored by the CTA-pair kernel.
cudaError_t launch_wgemm(bool bwd, int bn, const GemmParams& p, const WMaps& maps, int grid, cudaStream_t st,
                         double algo_flops, bool early = false);

// ---------------------------------------------------------- adapter merge
// (nf4_merge.cu) out[n, k] = dequant(W) + scale * B . A, tiles of 128 rows x
// merge_tile_cols() columns; k_steps = 64-wide steps of the zero-padded rank.
struct MergeParams {
  int32_t tiles_m, tiles_n, k_steps;
  int64_t n, k;
  const uint8_t* codes;
  ScaleSrc scales;
  float scale;
  void* out;
  Nf4Table tab;
};
struct MergeMaps {
  CUtensorMap b;       // B [n, r] bf16, box [64, 128], 128B swizzle
  CUtensorMap a;       // A [r, k] bf16, box [64, 64], 128B swizzle
  CUtensorMap codes;   // packed codes [n, k/2] u8, box [128, 128], 128B swizzle
  CUtensorMap out;     // W_out [n, k]: bf16 box [32, 32] 64B swizzle, or fp32 box [32, 32] 128B swizzle
};
int merge_tile_cols();
cudaError_t launch_merge(const MergeParams& p, const MergeMaps& maps, int grid, bool out_f32, cudaStream_t st);

// ------------------------------------------------------------- elementwise
// U = pre * (sum of the split partials); writes fp32 U, bf16(scale * U), hi/lo bf16 of U (each nullable).
// extra_src (nullable): a second fp32 [rows, r] matrix split into hi/lo bf16 [rows, r_pad] in the same launch.
cudaError_t launch_lora_finalize(const float* part, int splits, int64_t part_stride, int64_t rows,
                                 int32_t r, int32_t r_pad, float scale, float* out_f32,
                                 uint16_t* out_scaled_bf16, uint16_t* out_hi, uint16_t* out_lo,
                                 cudaStream_t st, float pre = 1.0f, const float* extra_src = nullptr,
                                 uint16_t* extra_hi = nullptr, uint16_t* extra_lo = nullptr);
cudaError_t launch_grad_finalize(const float* part, int splits, int64_t part_stride, int64_t rows,
                                 int32_t r, int32_t ld_part, float scale, float* out, int transpose,
                                 int accumulate, cudaStream_t st);
cudaError_t launch_splitk_reduce(const float* part, int splits, int64_t part_stride, int64_t rows,
                                 int64_t cols, int64_t ld_part, void* out, int out_bf16, int accumulate,
                                 cudaStream_t st);
// U = X A^T on CUDA cores for a few tokens (m <= 64, k % 8 == 0), one launch, no
// workspace: fp32 pre * U [m, r] (nullable) and bf16(scale * pre * U) [m, r_pad]
// (padding columns zeroed).
cudaError_t launch_lora_down_small(const uint16_t* X, int64_t m, int64_t k, const uint16_t* A, int32_t r,
                                   int32_t r_pad, float scale, float* U32, uint16_t* sU, cudaStream_t st,
                                   float pre = 1.0f);
// LoRA dropout (dropout.cu): keep mask from Philox4x32-10, masked copy of X, packed mask bits.
cudaError_t launch_dropout_mask(const uint16_t* X, int64_t count, uint32_t thr, uint64_t seed, uint64_t offset,
                                uint16_t* Xd, uint8_t* mask, cudaStream_t st);
cudaError_t launch_mask_apply(const uint16_t* X, int64_t count, const uint8_t* mask, uint16_t* Xd, cudaStream_t st);
// AdamW step on fp32 masters (optim.cu); p_bf16 (nullable) receives bf16(p).
cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, uint16_t* p_bf16, int64_t count, float lr,
                         float beta1, float beta2, float eps, float weight_decay, float grad_scale, int32_t step,
                         int num_sms, cudaStream_t st);
cudaError_t launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t st);
// Expansion-rate measurement (elementwise.cu): `grid` CTAs of *threads threads each
// expand iters 64-blocks per thread; read_expand_cycles copies the per-CTA cycles.
cudaError_t launch_expand_rate(const Nf4Table& tab, int iters, int grid, int* threads, cudaStream_t st);
cudaError_t read_expand_cycles(unsigned long long* out, int grid);
cudaError_t launch_silu_gate_fwd(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t count,
                                 cudaStream_t st);
cudaError_t launch_silu_gate_bwd(const uint16_t* dh, const uint16_t* g, const uint16_t* u, uint16_t* dg,
                                 uint16_t* du, int64_t count, cudaStream_t st);

}  // namespace qlora
