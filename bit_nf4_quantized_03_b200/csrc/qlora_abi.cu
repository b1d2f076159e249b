// C ABI of libqlora: argument checks, the NF4 level table, workspace planning
// and the launch sequence of each entry point. See include/qlora.h.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/qlora.h"
#include "qlora_kernels.h"

using namespace qlora;

// ---------------------------------------------------------------------------
// Launch accounting and the optional device-time hook for the fused GEMMs.
// ---------------------------------------------------------------------------
namespace qlora {
namespace {
std::atomic<int64_t> g_launches{0};
std::atomic<bool> g_timing_on{false};
std::mutex g_timing_mu;
std::vector<cudaEvent_t> g_events;     // pairs: start, stop
std::vector<double> g_event_flops;
size_t g_events_used = 0;
std::vector<double> g_last_ms, g_last_flops;   // per launch, from the last qlora_timing_end
}  // namespace

void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

Nf4Buckets nf4_buckets_from_midpoints(const float* mid) {
  // Widened buckets [j/16 - 1/32 - eps, j/16 + 1/32 + eps], j = b - 16: neighbouring
  // thresholds are >= 0.08 apart, wider than a widened bucket, so each holds at most one.
  const double eps = 1e-3;
  Nf4Buckets bk;
  for (int b = 0; b < kNf4Buckets; ++b) {
    const double j = b - 16;
    const double lo = j / 16.0 - 1.0 / 32.0 - eps, hi = j / 16.0 + 1.0 / 32.0 + eps;
    int below = 0;
    float thr = INFINITY;
    for (int i = 0; i < 15; ++i) {
      if (static_cast<double>(mid[i]) < lo) ++below;
      else if (static_cast<double>(mid[i]) <= hi) thr = mid[i];
    }
    bk.base[b] = below;
    bk.thr[b] = thr;
  }
  return bk;
}
bool timing_active() { return g_timing_on.load(std::memory_order_relaxed); }

void timing_record(cudaStream_t st, bool start, double flops) {
  std::lock_guard<std::mutex> g(g_timing_mu);
  if (!g_timing_on) return;
  if (start) {
    if (g_events_used + 2 > g_events.size()) return;
    cudaEventRecord(g_events[g_events_used], st);
    g_event_flops[g_events_used / 2] = flops;
  } else {
    if (g_events_used + 2 > g_events.size()) return;
    cudaEventRecord(g_events[g_events_used + 1], st);
    g_events_used += 2;
  }
}
}  // namespace qlora

namespace {

// ---------------------------------------------------------------------------
// NF4 levels: 16 quantiles of the standard normal distribution with an exact
// zero, normalised to [-1, 1] ("QLoRA Explained", "4-Bit NormalFloat (NF4)
// Quantization"; "QLoRA: Quantized Low-Rank Adaptation", "NF4: a 4-bit format
// matched to weight statistics"). Construction: 8 positive quantiles at
// probabilities equally spaced from delta to 1/2 (1/2 itself dropped), 7
// negative quantiles the same way on 8 points, and 0; divided by the largest.
// delta = ((1 - 1/30) + (1 - 1/32)) / 2 keeps the outermost quantile finite.
// The inverse CDF is found here by Newton's method on erfc.
// ---------------------------------------------------------------------------
double normal_quantile(double p) {
  const double inv_sqrt2 = 0.70710678118654752440;
  const double inv_sqrt2pi = 0.39894228040143267794;
  double x = 0.0;
  for (int it = 0; it < 100; ++it) {
    const double cdf = 0.5 * std::erfc(-x * inv_sqrt2);
    const double pdf = inv_sqrt2pi * std::exp(-0.5 * x * x);
    const double dx = (cdf - p) / pdf;
    x -= dx;
    if (std::fabs(dx) < 1e-17 * (1.0 + std::fabs(x))) break;
  }
  return x;
}

Nf4Table build_table() {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  double v[16];
  int n = 0;
  const double step9 = (0.5 - delta) / 8.0;   // 9 points delta..0.5
  const double step8 = (0.5 - delta) / 7.0;   // 8 points delta..0.5
  double pos[8], neg[7];
  for (int i = 0; i < 8; ++i) pos[i] = normal_quantile(i * step9 + delta);
  for (int i = 0; i < 7; ++i) neg[i] = -normal_quantile(i * step8 + delta);
  for (int i = 0; i < 7; ++i) v[n++] = neg[i];       // ascending: most negative first
  v[n++] = 0.0;
  for (int i = 7; i >= 0; --i) v[n++] = pos[i];
  const double vmax = pos[0];
  Nf4Table t;
  for (int i = 0; i < 16; ++i) t.lv[i] = static_cast<float>(v[i] / vmax);
  for (int i = 0; i < 15; ++i) t.mid[i] = (t.lv[i] + t.lv[i + 1]) * 0.5f;
  t.mid[15] = 2.0f;
  return t;
}

const Nf4Table& table() {
  static const Nf4Table t = build_table();
  return t;
}

const Nf4Buckets& buckets() {
  static const Nf4Buckets b = qlora::nf4_buckets_from_midpoints(table().mid);
  return b;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
}  // namespace

namespace qlora {
const Nf4Table& host_table() { return table(); }
const Nf4Buckets& host_buckets() { return buckets(); }
int host_num_sms() { return num_sms(); }
}  // namespace qlora

namespace {

bool weight_ok(const qlora_nf4_weight* w) {
  if (w == nullptr || w->n < 1 || w->k < 1) return false;
  if (w->blocksize != QLORA_BLOCKSIZE || w->dq_blocksize != QLORA_DQ_BLOCKSIZE) return false;
  if (w->codes == nullptr || !aligned16(w->codes)) return false;
  if (w->mode == QLORA_SCALE_BF16) return w->scale_bf16 != nullptr && aligned16(w->scale_bf16);
  if (w->mode == QLORA_SCALE_DQ_FP8)
    return w->scale_fp8 != nullptr && w->dq_scale != nullptr && w->dq_mean != nullptr && aligned16(w->scale_fp8) &&
           aligned16(w->dq_scale);
  return false;
}

ScaleSrc scale_src(const qlora_nf4_weight* w) {
  ScaleSrc s{};
  if (w->mode == QLORA_SCALE_BF16) {
    s.bf16 = w->scale_bf16;
  } else {
    s.fp8 = w->scale_fp8;
    s.dq_scale = w->dq_scale;
    s.dq_mean = w->dq_mean;
  }
  return s;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// ---------------------------------------------------------------------------
// Linear-layer plan: split counts and workspace carve-up. Deterministic in
// (m, n, k, r, SM count) so the size query and the call always agree.
// ---------------------------------------------------------------------------
struct Split {
  int splits = 1, kps = 1;
};

// Split of a low-rank GEMM's reduction (U, G, dB, dA) over a persistent grid of
// `sms` CTAs. These stream one 128 x 64 bf16 tile of the large operand per K step,
// so the makespan in K steps is the number of waves times the steps per unit; each
// split adds one fp32 partial of the [out_elems] result, written once and read
// once, mostly from L2 (charged at half the weight of HBM traffic). Few tiles over
// many SMs need a split to fill the grid; tiles just above the SM count need one
// to even out the last wave.
Split choose_lsplit(int64_t tiles, int64_t k_tiles, int sms, int64_t out_elems) {
  const double bytes_per_wave_step = static_cast<double>(sms) * 16384.0;
  Split best;
  best.kps = static_cast<int>(std::max<int64_t>(k_tiles, 1));
  best.splits = 1;
  double best_cost = 1e300;
  for (int64_t want = 1; want <= std::min<int64_t>(64, std::max<int64_t>(k_tiles, 1)); ++want) {
    const int64_t kps = cdiv(std::max<int64_t>(k_tiles, 1), want);
    const int64_t splits = cdiv(std::max<int64_t>(k_tiles, 1), kps);
    const int64_t waves = cdiv(std::max<int64_t>(tiles, 1) * splits, sms);
    double cost = static_cast<double>(waves) * (static_cast<double>(kps) + 1.0);
    if (splits > 1) cost += static_cast<double>(splits) * static_cast<double>(out_elems) * 4.0 / bytes_per_wave_step;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.kps = static_cast<int>(kps);
      best.splits = static_cast<int>(splits);
    }
  }
  return best;
}

// Split of the fused GEMM's reduction over a persistent grid of `sms` CTAs:
// the split count that minimises the makespan, measured in K steps of one
// 128-row weight tile (each unit also pays about one step to fill and drain
// its pipeline), plus the fp32 partial traffic a split adds (written once and
// read once by the reduction; bytes_per_step converts bytes to K steps).
Split choose_wsplit(int64_t tiles, int64_t k_tiles, int sms, int64_t out_elems) {
  const double bytes_per_step = 3.0e6;     // ~0.5 us of one expanded 128 x 64 tile against ~6 TB/s
  Split best;
  best.kps = static_cast<int>(std::max<int64_t>(k_tiles, 1));
  best.splits = 1;
  double best_cost = 1e300;
  for (int64_t want = 1; want <= std::min<int64_t>(64, std::max<int64_t>(k_tiles, 1)); ++want) {
    const int64_t kps = cdiv(std::max<int64_t>(k_tiles, 1), want);
    const int64_t splits = cdiv(std::max<int64_t>(k_tiles, 1), kps);
    const int64_t waves = cdiv(tiles * splits, sms);
    double cost = static_cast<double>(waves) * (static_cast<double>(kps) + 1.0);
    if (splits > 1) cost += 2.0 * static_cast<double>(splits) * static_cast<double>(out_elems) * 4.0 / bytes_per_step;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.kps = static_cast<int>(kps);
      best.splits = static_cast<int>(splits);
    }
  }
  return best;
}

struct Plan {
  int r_pad = 64;
  GemmKind down_k = kGemmLoraDownK, down_mn = kGemmLoraDownMN, grad = kGemmLoraGrad;
  Split u, g, db, da, fwd, bwd;
  int bn = 256;
  size_t off_u32 = 0, off_scaled = 0, off_hi_a = 0, off_lo_a = 0, off_hi_b = 0, off_lo_b = 0, off_part = 0,
         total = 0;
};

Plan make_plan(int64_t m, int64_t n, int64_t k, int32_t r) {
  Plan P;
  const int sms = num_sms();
  P.r_pad = (r <= 64) ? 64 : 128;
  if (P.r_pad == 128) {
    P.down_k = kGemmLoraDownK128;
    P.down_mn = kGemmLoraDownMN128;
    P.grad = kGemmLoraGrad128;
  }
  const int64_t tm = cdiv(m, 128);
  const int64_t rp64 = P.r_pad;
  P.u = choose_lsplit(tm, k / 64, sms, m * rp64);
  P.g = choose_lsplit(tm, cdiv(n, 64), sms, m * rp64);
  P.db = choose_lsplit(cdiv(n, 128), cdiv(m, 64), sms, n * rp64);
  P.da = choose_lsplit(cdiv(k, 128), cdiv(m, 64), sms, k * rp64);
  P.bn = wgemm_bn(m);
  const int64_t tok_tiles = cdiv(m, P.bn);
  const int64_t wrows = wgemm_tile_rows(P.bn);
  const int wslots = (wrows == 256) ? wgemm_pair_slots() : sms;   // a CTA pair works one 256-row tile
  const int64_t fwd_tiles = cdiv(n, wrows) * tok_tiles;
  P.fwd = choose_wsplit(fwd_tiles, k / 64, wslots, m * n);
  const int64_t bwd_tiles = cdiv(k, wrows) * tok_tiles;
  P.bwd = choose_wsplit(bwd_tiles, cdiv(n, 64), wslots, m * k);
  const size_t rp = static_cast<size_t>(P.r_pad);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  P.off_u32 = take(static_cast<size_t>(m) * r * 4);
  P.off_scaled = take(static_cast<size_t>(m) * rp * 2);
  P.off_hi_a = take(static_cast<size_t>(m) * rp * 2);
  P.off_lo_a = take(static_cast<size_t>(m) * rp * 2);
  P.off_hi_b = take(static_cast<size_t>(m) * rp * 2);
  P.off_lo_b = take(static_cast<size_t>(m) * rp * 2);
  size_t part = 0;
  part = std::max(part, static_cast<size_t>(P.u.splits) * m * rp);
  part = std::max(part, static_cast<size_t>(P.g.splits) * m * rp);
  part = std::max(part, static_cast<size_t>(P.db.splits) * n * rp);
  part = std::max(part, static_cast<size_t>(P.da.splits) * k * rp);
  if (P.fwd.splits > 1) part = std::max(part, static_cast<size_t>(P.fwd.splits) * m * n);
  // dX through fp32 partials: for split K, and for an accumulating dX on the CTA-pair path
  if (P.bwd.splits > 1 || wrows == 256)
    part = std::max(part, static_cast<size_t>(std::max(P.bwd.splits, 1)) * m * k);
  P.off_part = take(part * 4);
  P.total = off;
  return P;
}

bool linear_args_ok(const qlora_nf4_weight* w, const void* X, int64_t m, const void* A, const void* B) {
  if (!weight_ok(w) || X == nullptr || A == nullptr || B == nullptr) return false;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B)) return false;
  if (m < 1 || m > (int64_t(1) << 31) - 1) return false;
  if (w->n > (int64_t(1) << 31) - 1 || w->k > (int64_t(1) << 31) - 1) return false;
  return true;
}

int linear_shape_status(const qlora_nf4_weight* w, int32_t r) {
  if (w->k % 64 != 0 || w->n % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (!(r == 8 || r == 16 || r == 32 || r == 64 || r == 128)) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

GemmParams base_params(int64_t rows, int64_t cols, int bn, int64_t k_tiles, Split sp) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.rows = static_cast<int32_t>(rows);
  p.cols = static_cast<int32_t>(cols);
  p.tiles_m = static_cast<int32_t>(cdiv(rows, 128));
  p.tiles_n = static_cast<int32_t>(cdiv(cols, bn));
  p.k_tiles = static_cast<int32_t>(k_tiles);
  // one split covers the whole reduction
  p.splits = sp.splits > 1 ? sp.splits : 1;
  p.k_per_split = sp.splits > 1 ? sp.kps : static_cast<int32_t>(k_tiles);
  p.groups = 1;
  for (int l = 1; l <= kWGroupMax; ++l) p.k_begin[l] = static_cast<int32_t>(k_tiles);
  p.tab = table();
  return p;
}

// Persistent grid of a low-rank GEMM: one CTA per unit, at most one per SM, or `cap`.
int grid_of(const GemmParams& p, int cap = 0) {
  const int64_t units = static_cast<int64_t>(p.tiles_m) * p.tiles_n * p.splits;
  return static_cast<int>(std::min<int64_t>(units, cap > 0 ? cap : num_sms()));
}

const CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
const CUtensorMapDataType kU8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;

// bf16 matrix [rows, cols] row-major, 128-B swizzled boxes of [64 cols, box_rows].
bool map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  return tmap_2d(m, base, kBF16, static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                 static_cast<uint64_t>(cols) * 2, 64, box_rows, 128);
}

// Low-rank product U (or G): partial GEMM over the reduction, then finalize.
int run_lora_down(const Plan& P, bool b_mn, const uint16_t* act, int64_t m, int64_t red, const uint16_t* adapter,
                  int32_t r, float scale, char* ws, float* out_f32, uint16_t* out_scaled, uint16_t* out_hi,
                  uint16_t* out_lo, cudaStream_t st, float pre = 1.0f, const float* extra_src = nullptr,
                  uint16_t* extra_hi = nullptr, uint16_t* extra_lo = nullptr) {
  const Split sp = b_mn ? P.g : P.u;
  GemmParams p = base_params(m, P.r_pad, P.r_pad, b_mn ? cdiv(red, 64) : red / 64, sp);
  p.out = ws + P.off_part;
  p.ld_out = P.r_pad;
  p.part_stride = m * P.r_pad;
  p.out_mode = kOutPartial;
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  bool ok = map_bf16(&maps.a, act, m, red, 128);
  if (!b_mn) {  // adapter A [r, red] is K-major
    ok = ok && tmap_2d(&maps.b, adapter, kBF16, red, r, red * 2, 64, P.r_pad, 128);
  } else {      // adapter B [red, r] is MN-major (r contiguous)
    ok = ok && tmap_2d(&maps.b, adapter, kBF16, r, red, r * 2, 64, 64, 128);
  }
  if (!ok) return QLORA_ERR_CUDA;
  cudaError_t e = launch_gemm(b_mn ? P.down_mn : P.down_k, p, maps, grid_of(p), st);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  e = launch_lora_finalize(static_cast<const float*>(p.out), sp.splits, p.part_stride, m, r, P.r_pad, scale,
                           out_f32, out_scaled, out_hi, out_lo, st, pre, extra_src, extra_hi, extra_lo);
  return cuda_status(e);
}

// Dropout settings resolved on the host: 16-bit threshold and keep scale c.
struct Drop {
  bool on = false;
  uint32_t thr = 0;
  float keep = 1.0f;
  uint64_t seed = 0, offset = 0;
  uint8_t* mask = nullptr;
};

// QLORA_OK, or QLORA_ERR_INVALID for a rate outside [0, 1) or a missing/misaligned mask.
int resolve_drop(const qlora_dropout* d, Drop* out) {
  *out = Drop{};
  if (d == nullptr || d->p == 0.0f) return QLORA_OK;
  if (!(d->p > 0.0f && d->p < 1.0f)) return QLORA_ERR_INVALID;
  const double t = std::nearbyint(static_cast<double>(d->p) * 65536.0);
  if (t >= 65536.0) return QLORA_ERR_INVALID;
  if (d->mask == nullptr || !aligned16(d->mask)) return QLORA_ERR_INVALID;
  out->thr = static_cast<uint32_t>(t);
  if (out->thr == 0) return QLORA_OK;                     // rounds to no dropout
  out->on = true;
  out->keep = static_cast<float>(65536.0 / (65536.0 - t));
  out->seed = d->seed;
  out->offset = d->offset;
  out->mask = d->mask;
  return QLORA_OK;
}

size_t drop_ws_bytes(int64_t m, int64_t k) { return align_up(static_cast<size_t>(m) * k * 2, 256); }

// dX += keep * M * ((sG) A): the low-rank term of dX under dropout, one tcgen05 GEMM over the
// rank with the mask applied in the epilogue.
int run_lora_up_masked(const Plan& P, const uint16_t* sG, int64_t m, int64_t k, const uint16_t* A, int32_t r,
                       const Drop& D, void* dX, bool dx_f32, cudaStream_t st) {
  Split sp;
  sp.splits = 1;
  sp.kps = P.r_pad / 64;
  // 128-column tiles: each epilogue warp fetches 32 rows x 128 columns of dX in one round trip, and two
  // epilogue groups keep two units' round trips in flight
  GemmParams p = base_params(m, k, gemm_bn(kGemmLoraUpMasked), P.r_pad / 64, sp);
  p.out = dX;
  p.ld_out = k;
  p.out_mode = dx_f32 ? kOutMaskAccF32 : kOutMaskAccBF16;
  p.mask = D.mask;
  p.keep_scale = D.keep;
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  bool ok = map_bf16(&maps.a, sG, m, P.r_pad, 128);                              // [m, r_pad], K-major
  ok = ok && tmap_2d(&maps.b, A, kBF16, k, r, k * 2, 64, 64, 128);                 // A [r, k]: MN-major
  if (!ok) return QLORA_ERR_CUDA;
  return cuda_status(launch_gemm(kGemmLoraUpMasked, p, maps, grid_of(p), st));
}

// dB (rows = n, act = dY) or dA^T (rows = k, act = X): sum over tokens of act^T . [hi + lo].
int run_lora_grad(const Plan& P, const Split& sp, const uint16_t* act, int64_t m, int64_t rows, const uint16_t* hi,
                  const uint16_t* lo, int32_t r, float scale, float* out, int transpose, int accumulate, char* ws,
                  cudaStream_t st, int grid_cap = 0) {
  GemmParams p = base_params(rows, P.r_pad, P.r_pad, cdiv(m, 64), sp);
  p.out = ws + P.off_part;
  p.ld_out = P.r_pad;
  p.part_stride = rows * P.r_pad;
  p.out_mode = kOutPartial;
  GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  bool ok = tmap_2d(&maps.a, act, kBF16, rows, m, rows * 2, 64, 64, 128);          // [m, rows], MN-major A
  ok = ok && tmap_2d(&maps.b, hi, kBF16, P.r_pad, m, P.r_pad * 2, 64, 64, 128);    // [m, r_pad], MN-major B
  ok = ok && tmap_2d(&maps.b2, lo, kBF16, P.r_pad, m, P.r_pad * 2, 64, 64, 128);
  if (!ok) return QLORA_ERR_CUDA;
  cudaError_t e = launch_gemm(P.grad, p, maps, grid_of(p, grid_cap), st);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  e = launch_grad_finalize(static_cast<const float*>(p.out), sp.splits, p.part_stride, rows, r, P.r_pad, scale, out,
                           transpose, accumulate, st);
  return cuda_status(e);
}

// One layer's share of a dX GEMM.
struct DxLayer {
  const qlora_nf4_weight* w;
  const uint16_t* dY;       // [m, n_l]
  const uint16_t* A;        // A_l [r, k]
  const uint16_t* sG;       // bf16(s G_l) [m, r_pad]
};

// dX^T = sum_l (W_l^T . dY_l^T + A_l^T . (s G_l)^T), each W_l dequantized into the MN-major
// operand layout: one weight GEMM whose reduction runs over the layers in turn (layers that
// share the input X; the CTA-pair kernel alone takes more than one). `ext`: the low-rank
// terms ride as extension K steps. Split K, and an accumulating dX on the CTA-pair path, go
// through fp32 partials and the reduce pass: in the GEMM's epilogue the old dX values (rows
// ld apart) were read at a small fraction of the memory's speed and stalled the tensor cores.
int run_dx(const Plan& P, const DxLayer* L, int count, int64_t m, int64_t k, int32_t r, bool ext, void* dX,
           int32_t dx_dtype, bool acc_dx, char* wsb, cudaStream_t st) {
  const int bn = P.bn;
  if (count < 1 || count > kWGroupMax || (count > 1 && wgemm_tile_rows(bn) != 256)) return QLORA_ERR_INVALID;
  const Split& sp = P.bwd;
  const bool via_part = sp.splits > 1 || (acc_dx && wgemm_tile_rows(bn) == 256);
  int64_t k_tiles = 0;
  int32_t k_begin[kWGroupMax + 1] = {};
  for (int l = 0; l < count; ++l) {
    k_begin[l] = static_cast<int32_t>(k_tiles);
    k_tiles += cdiv(L[l].w->n, 64);
  }
  GemmParams p = base_params(k, m, bn, k_tiles, sp);
  p.tiles_m = static_cast<int32_t>(cdiv(k, wgemm_tile_rows(bn)));
  p.ext_tiles = ext ? P.r_pad / 64 : 0;
  p.groups = count;
  // a grouped reduction is long (every layer's K steps): units that run together share
  // each activation slice for longer, and two token tiles per raster group kept fewer of
  // them in flight (3.8 against 4.3 GB of DRAM traffic for the 65B gate/up pair, and
  // slightly faster, against four)
  p.raster = (count > 1) ? 2 : 0;
  for (int l = 0; l <= kWGroupMax; ++l) p.k_begin[l] = (l < count) ? k_begin[l] : static_cast<int32_t>(k_tiles);
  p.w_kblocks = k / 64;
  for (int l = 0; l < count; ++l) {
    p.scales[l] = scale_src(L[l].w);
    p.w_rows[l] = static_cast<int32_t>(L[l].w->n);
  }
  p.ld_out = k;
  if (via_part) {
    p.out = wsb + P.off_part;
    p.part_stride = m * k;
    p.out_mode = kOutPartial;
  } else {
    p.out = dX;
    p.out_mode = (dx_dtype == QLORA_DTYPE_FP32) ? kOutF32 : kOutBF16;
    p.accumulate = acc_dx ? 1 : 0;
  }
  WMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  bool ok = true;
  double flops = 0.0;
  for (int l = 0; l < count; ++l) {
    const int64_t n = L[l].w->n;
    ok = ok && map_bf16(&maps.act[l], L[l].dY, m, n, static_cast<uint32_t>(wgemm_box_rows(bn)));
    ok = ok && tmap_2d(&maps.codes[l], L[l].w->codes, kU8, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n),
                       static_cast<uint64_t>(k / 2), 64, 64, 64);
    ok = ok && tmap_2d(&maps.a2[l], L[l].A, kBF16, k, r, k * 2, 64, 64, 128);
    ok = ok && map_bf16(&maps.b2[l], L[l].sG, m, P.r_pad, static_cast<uint32_t>(wgemm_box_rows(bn)));
    flops += 2.0 * double(m) * double(k) * double(n + (ext ? r : 0));
  }
  if (!ok) return QLORA_ERR_CUDA;
  if (launch_wgemm(true, bn, p, maps, wgemm_grid(p, bn, num_sms()), st, flops) != cudaSuccess) return QLORA_ERR_CUDA;
  if (via_part &&
      launch_splitk_reduce(static_cast<const float*>(p.out), p.splits, p.part_stride, m, k, k, dX,
                           dx_dtype == QLORA_DTYPE_BF16, acc_dx ? 1 : 0, st) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// SMs that a one-layer dX GEMM leaves idle and that can take the adapter gradients beside it
// (0: run them after it). Only a dX GEMM with one split and no accumulation qualifies: it
// writes dX directly and no fp32 partial. The gradients need enough SMs to end within the dX
// GEMM's time: a low-rank K step streams 32 KB from memory, a weight K step runs a 256 x 512
// x 64 MMA; the first is taken as about a third of the second.
int dx_idle_sms(const Plan& P, int64_t m, int64_t n, int64_t k, bool acc_dx) {
  constexpr int kMinIdle = 16;
  if (acc_dx || P.bwd.splits != 1) return 0;
  const int sms = num_sms();
  const bool pair = wgemm_tile_rows(P.bn) == 256;
  const int64_t units = cdiv(k, wgemm_tile_rows(P.bn)) * cdiv(m, P.bn);
  const int64_t slots = pair ? wgemm_pair_slots() : sms;
  const int64_t grid = (pair ? 2 : 1) * std::min<int64_t>(units, slots);
  const int idle = static_cast<int>(sms - grid);
  if (idle < kMinIdle) return 0;
  const int64_t dx_steps = cdiv(units, slots) * (cdiv(n, 64) + P.r_pad / 64);
  auto grad_steps = [&](const Split& sp, int64_t rows) {
    return cdiv(cdiv(rows, 128) * sp.splits, idle) * (sp.kps + 1);
  };
  const int64_t side_steps = grad_steps(P.db, n) + grad_steps(P.da, k);
  return (side_steps <= 3 * dx_steps) ? idle : 0;
}

// An internal stream (and a fork and a join event) per thread and CUDA context, on which a
// backward runs work beside its dX GEMM. Created on the first call outside a stream capture;
// a call under capture before that runs everything on the caller's stream.
struct SideStream {
  unsigned long long ctx = 0;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

SideStream* side_stream(cudaStream_t st) {
  thread_local std::vector<SideStream> cache;
  const unsigned long long ctx = context_id();
  if (ctx == 0) return nullptr;
  for (SideStream& c : cache)
    if (c.ctx == ctx) return &c;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (cs != cudaStreamCaptureStatusNone) return nullptr;
  SideStream c;
  c.ctx = ctx;
  if (cudaStreamCreateWithFlags(&c.s, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&c.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming) != cudaSuccess) {
    (void)cudaGetLastError();
    if (c.join != nullptr) cudaEventDestroy(c.join);
    if (c.fork != nullptr) cudaEventDestroy(c.fork);
    if (c.s != nullptr) cudaStreamDestroy(c.s);
    return nullptr;
  }
  cache.push_back(c);
  return &cache.back();
}

// Workspace of a grouped backward: every layer's bf16(s G_l) (read together by the fused dX
// GEMM), then one scratch area that the layers use in turn and the dX GEMM after them.
struct GroupPlan {
  size_t off_sg[kWGroupMax] = {};
  size_t off_scratch = 0, total = 0;
};

GroupPlan make_group_plan(int32_t count, int64_t m, const int64_t* n, int64_t k, int32_t r) {
  GroupPlan G;
  const int r_pad = (r <= 64) ? 64 : 128;
  size_t off = 0;
  int64_t n_total = 0;
  size_t scratch = 0;
  for (int l = 0; l < count; ++l) {
    G.off_sg[l] = off;
    off += align_up(static_cast<size_t>(m) * r_pad * 2, 256);
    n_total += n[l];
    scratch = std::max(scratch, make_plan(m, n[l], k, r).total);
  }
  scratch = std::max(scratch, make_plan(m, n_total, k, r).total);
  G.off_scratch = off;
  G.total = off + scratch;
  return G;
}

}  // namespace

extern "C" {

const char* qlora_status_string(int s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_DEVICE: return "a kernel gave up on a bounded wait";
    case QLORA_ERR_BOUNDS: return "a bounds check failed (bounds-checking build)";
    default: return "unknown status";
  }
}

const char* qlora_version(void) { return "qlora-nf4-b200 0.1 (sm_100a)"; }

int qlora_nf4_levels(float levels[16], float mid[15]) {
  const Nf4Table& t = table();
  if (levels != nullptr) std::memcpy(levels, t.lv, sizeof(float) * 16);
  if (mid != nullptr) std::memcpy(mid, t.mid, sizeof(float) * 15);
  return QLORA_OK;
}

size_t qlora_nf4_quantize_workspace_bytes(int64_t n, int64_t k, int32_t mode) {
  if (mode != QLORA_SCALE_DQ_FP8 || n < 1 || k < 1) return 0;
  return quant_ws_layout(n * k).total;
}

int qlora_nf4_quantize(const float* W, qlora_nf4_weight* w, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (W == nullptr || !aligned16(W) || !weight_ok(w)) return QLORA_ERR_INVALID;
  const int64_t n_elem = w->n * w->k;
  const bool dq = (w->mode == QLORA_SCALE_DQ_FP8);
  if (dq) {
    if (n_elem > kMaxDqElems) return QLORA_ERR_UNSUPPORTED;
    if (ws == nullptr || !aligned16(ws) || ws_bytes < quant_ws_layout(n_elem).total) return QLORA_ERR_WORKSPACE;
  }
  const cudaError_t e =
      launch_quantize(W, n_elem, table(), buckets(), w->codes, dq ? nullptr : w->scale_bf16, dq ? w->scale_fp8 : nullptr,
                      dq ? w->dq_scale : nullptr, dq ? w->dq_mean : nullptr, ws, num_sms(),
                      reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

int qlora_nf4_dequantize(const qlora_nf4_weight* w, uint16_t* out_bf16, qlora_stream_t stream) {
  if (!weight_ok(w) || out_bf16 == nullptr || !aligned16(out_bf16)) return QLORA_ERR_INVALID;
  const cudaError_t e = launch_dequantize(w->codes, scale_src(w), w->n * w->k, table(), out_bf16, num_sms(),
                                          reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

size_t qlora_linear_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t r) {
  if (m < 1 || n < 1 || k < 1 || r < 1 || r > 128) return 0;
  return make_plan(m, n, k, r).total;
}

size_t qlora_linear_workspace_bytes_ex(int64_t m, int64_t n, int64_t k, int32_t r, const qlora_dropout* drop) {
  const size_t base = qlora_linear_workspace_bytes(m, n, k, r);
  Drop D;
  if (base == 0 || resolve_drop(drop, &D) != QLORA_OK) return 0;
  return base + (D.on ? drop_ws_bytes(m, k) : 0);
}

int qlora_lora_merge(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int32_t r, float alpha,
                     void* W_out, int32_t out_dtype, qlora_stream_t stream) {
  if (!weight_ok(w) || A == nullptr || B == nullptr || W_out == nullptr) return QLORA_ERR_INVALID;
  if (!aligned16(A) || !aligned16(B) || !aligned16(W_out)) return QLORA_ERR_INVALID;
  if (out_dtype != QLORA_DTYPE_BF16 && out_dtype != QLORA_DTYPE_FP32) return QLORA_ERR_INVALID;
  if (w->k % 64 != 0 || !(r == 8 || r == 16 || r == 32 || r == 64 || r == 128)) return QLORA_ERR_UNSUPPORTED;
  const int64_t n = w->n, k = w->k;
  const int64_t tiles_m = cdiv(n, 128), tiles_n = cdiv(k, merge_tile_cols());
  if (tiles_m * tiles_n > INT32_MAX) return QLORA_ERR_UNSUPPORTED;
  MergeParams p;
  std::memset(&p, 0, sizeof(p));
  p.tiles_m = static_cast<int32_t>(tiles_m);
  p.tiles_n = static_cast<int32_t>(tiles_n);
  p.k_steps = static_cast<int32_t>(cdiv(r, 64));
  p.n = n;
  p.k = k;
  p.codes = w->codes;
  p.scales = scale_src(w);
  p.scale = alpha / static_cast<float>(r);
  p.out = W_out;
  p.tab = table();
  const bool f32 = (out_dtype == QLORA_DTYPE_FP32);
  MergeMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  bool ok = tmap_2d(&maps.b, B, kBF16, r, n, r * 2, 64, 128, 128);
  ok = ok && tmap_2d(&maps.a, A, kBF16, k, r, k * 2, 64, 64, 128);
  ok = ok && tmap_2d(&maps.codes, w->codes, kU8, k / 2, n, k / 2, 128, 128, 128);
  ok = ok && (f32 ? tmap_2d(&maps.out, W_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, k, n, k * 4, 32, 32, 128)
                  : tmap_2d(&maps.out, W_out, kBF16, k, n, k * 2, 32, 32, 64));
  if (!ok) return QLORA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>(tiles_m * tiles_n, num_sms()));
  return cuda_status(launch_merge(p, maps, grid, f32, reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_linear_fwd(const qlora_nf4_weight* w, const uint16_t* X, int64_t m, const uint16_t* A, const uint16_t* B,
                     int32_t r, float alpha, void* Y, int32_t y_dtype, float* U_save, void* ws, size_t ws_bytes,
                     qlora_stream_t stream) {
  return qlora_linear_fwd_ex(w, X, m, A, B, r, alpha, Y, y_dtype, U_save, nullptr, ws, ws_bytes, stream);
}

int qlora_linear_fwd_ex(const qlora_nf4_weight* w, const uint16_t* X, int64_t m, const uint16_t* A,
                        const uint16_t* B, int32_t r, float alpha, void* Y, int32_t y_dtype, float* U_save,
                        const qlora_dropout* drop, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!linear_args_ok(w, X, m, A, B) || Y == nullptr || !aligned16(Y)) return QLORA_ERR_INVALID;
  if (y_dtype != QLORA_DTYPE_BF16 && y_dtype != QLORA_DTYPE_FP32) return QLORA_ERR_INVALID;
  if (U_save != nullptr && !aligned16(U_save)) return QLORA_ERR_INVALID;
  const int sst = linear_shape_status(w, r);
  if (sst != QLORA_OK) return sst;
  Drop D;
  if (resolve_drop(drop, &D) != QLORA_OK) return QLORA_ERR_INVALID;
  const int64_t n = w->n, k = w->k;
  const Plan P = make_plan(m, n, k, r);
  const size_t need = P.total + (D.on ? drop_ws_bytes(m, k) : 0);
  if (ws == nullptr || !aligned16(ws) || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* wsb = static_cast<char*>(ws);
  const float s = alpha / static_cast<float>(r);
  uint16_t* sU = reinterpret_cast<uint16_t*>(wsb + P.off_scaled);

  // LoRA dropout: the low-rank branch reads M * X (exact in bf16); c is applied to U
  const uint16_t* Xl = X;
  if (D.on) {
    uint16_t* Xd = reinterpret_cast<uint16_t*>(wsb + P.total);
    if (launch_dropout_mask(X, m * k, D.thr, D.seed, D.offset, Xd, D.mask, st) != cudaSuccess) return QLORA_ERR_CUDA;
    Xl = Xd;
  }

  // U = c (M * X) A^T (fp32, optionally saved) and bf16(s * U) for the K extension
  if (m <= 64) {
    if (launch_lora_down_small(Xl, m, k, A, r, P.r_pad, s, U_save, sU, st, D.keep) != cudaSuccess)
      return QLORA_ERR_CUDA;
  } else {
    const int rc = run_lora_down(P, false, Xl, m, k, A, r, s, wsb, U_save, sU, nullptr, nullptr, st, D.keep);
    if (rc != QLORA_OK) return rc;
  }

  // Y^T = W . X^T + B . (sU)^T with W dequantized on the fly (weight as the 128-row operand)
  GemmParams p = base_params(n, m, P.bn, k / 64, P.fwd);
  p.tiles_m = static_cast<int32_t>(cdiv(n, wgemm_tile_rows(P.bn)));
  p.ext_tiles = P.r_pad / 64;
  p.scales[0] = scale_src(w);
  p.w_kblocks = k / 64;
  p.w_rows[0] = static_cast<int32_t>(n);
  p.ld_out = n;
  if (P.fwd.splits > 1) {
    p.out = wsb + P.off_part;
    p.part_stride = m * n;
    p.out_mode = kOutPartial;
  } else {
    p.out = Y;
    p.out_mode = (y_dtype == QLORA_DTYPE_FP32) ? kOutF32 : kOutBF16;
  }
  WMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  bool ok = map_bf16(&maps.act[0], X, m, k, static_cast<uint32_t>(wgemm_box_rows(P.bn)));
  ok = ok && tmap_2d(&maps.codes[0], w->codes, kU8, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n),
                     static_cast<uint64_t>(k / 2), 32, 128, 32);
  ok = ok && tmap_2d(&maps.a2[0], B, kBF16, r, n, r * 2, 64, 128, 128);
  ok = ok && map_bf16(&maps.b2[0], sU, m, P.r_pad, static_cast<uint32_t>(wgemm_box_rows(P.bn)));
  if (!ok) return QLORA_ERR_CUDA;
  const double fwd_flops = 2.0 * double(m) * double(n) * double(k + r);
  // at few tokens U comes from lora_down_small_kernel right before: the GEMM may start streaming
  // the weight while that kernel runs, and waits for it before its K extension
  cudaError_t e = launch_wgemm(false, P.bn, p, maps, wgemm_grid(p, P.bn, num_sms()), st, fwd_flops, m <= 64);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  if (P.fwd.splits > 1) {
    e = launch_splitk_reduce(static_cast<const float*>(p.out), P.fwd.splits, p.part_stride, m, n, n, Y,
                             y_dtype == QLORA_DTYPE_BF16, 0, st);
    if (e != cudaSuccess) return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

int qlora_linear_bwd(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* dY, int64_t m, const uint16_t* A,
                     const uint16_t* B, int32_t r, float alpha, const float* U_saved, void* dX, int32_t dx_dtype,
                     float* dA, float* dB, int32_t flags, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  return qlora_linear_bwd_ex(w, X, dY, m, A, B, r, alpha, U_saved, dX, dx_dtype, dA, dB, flags, nullptr, ws,
                             ws_bytes, stream);
}

int qlora_linear_bwd_ex(const qlora_nf4_weight* w, const uint16_t* X, const uint16_t* dY, int64_t m,
                        const uint16_t* A, const uint16_t* B, int32_t r, float alpha, const float* U_saved,
                        void* dX, int32_t dx_dtype, float* dA, float* dB, int32_t flags, const qlora_dropout* drop,
                        void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!linear_args_ok(w, X, m, A, B) || dY == nullptr || !aligned16(dY)) return QLORA_ERR_INVALID;
  if (dA == nullptr || dB == nullptr || !aligned16(dA) || !aligned16(dB)) return QLORA_ERR_INVALID;
  if (dX != nullptr && (!aligned16(dX) || (dx_dtype != QLORA_DTYPE_BF16 && dx_dtype != QLORA_DTYPE_FP32)))
    return QLORA_ERR_INVALID;
  if (U_saved != nullptr && !aligned16(U_saved)) return QLORA_ERR_INVALID;
  if ((flags & ~(QLORA_BWD_ACCUMULATE_GRADS | QLORA_BWD_ACCUMULATE_DX)) != 0) return QLORA_ERR_INVALID;
  const int sst = linear_shape_status(w, r);
  if (sst != QLORA_OK) return sst;
  Drop D;
  if (resolve_drop(drop, &D) != QLORA_OK) return QLORA_ERR_INVALID;
  const int64_t n = w->n, k = w->k;
  const Plan P = make_plan(m, n, k, r);
  const size_t need = P.total + (D.on ? drop_ws_bytes(m, k) : 0);
  if (ws == nullptr || !aligned16(ws) || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* wsb = static_cast<char*>(ws);
  const float s = alpha / static_cast<float>(r);
  uint16_t* sG = reinterpret_cast<uint16_t*>(wsb + P.off_scaled);
  // LoRA dropout: M * X rebuilt from the forward's mask (dA and, without U_saved, U read it)
  const uint16_t* Xl = X;
  if (D.on) {
    uint16_t* Xd = reinterpret_cast<uint16_t*>(wsb + P.total);
    if (launch_mask_apply(X, m * k, D.mask, Xd, st) != cudaSuccess) return QLORA_ERR_CUDA;
    Xl = Xd;
  }
  uint16_t* g_hi = reinterpret_cast<uint16_t*>(wsb + P.off_hi_b);
  uint16_t* g_lo = reinterpret_cast<uint16_t*>(wsb + P.off_lo_b);
  uint16_t* u_hi = reinterpret_cast<uint16_t*>(wsb + P.off_hi_a);
  uint16_t* u_lo = reinterpret_cast<uint16_t*>(wsb + P.off_lo_a);
  const int acc_grads = (flags & QLORA_BWD_ACCUMULATE_GRADS) ? 1 : 0;

  // G = dY B: bf16(s G) for the dX extension, hi/lo bf16 for dA; the saved U's hi/lo bf16
  // split for dB comes out of the same finalize launch
  int rc = run_lora_down(P, true, dY, m, n, B, r, s, wsb, nullptr, sG, g_hi, g_lo, st, 1.0f, U_saved,
                         U_saved != nullptr ? u_hi : nullptr, U_saved != nullptr ? u_lo : nullptr);
  if (rc != QLORA_OK) return rc;
  // U = X A^T as hi/lo bf16 for dB, recomputed when not saved
  if (U_saved == nullptr) {
    rc = run_lora_down(P, false, Xl, m, k, A, r, s, wsb, nullptr, nullptr, u_hi, u_lo, st, D.keep);
    if (rc != QLORA_OK) return rc;
  }

  const float s_da = D.on ? s * D.keep : s;
  const bool acc_dx = (flags & QLORA_BWD_ACCUMULATE_DX) != 0;
  const int idle = (dX != nullptr && !D.on) ? dx_idle_sms(P, m, n, k, acc_dx) : 0;
  SideStream* side = (idle > 0) ? side_stream(st) : nullptr;
  if (side != nullptr) {
    // dB and dA do not depend on dX: they run beside the dX GEMM on the SMs its grid leaves
    // idle, with the same splits (the same partials, added in the same order). dX writes no
    // fp32 partial here (one split, not accumulating), so the two share no workspace.
    if (cudaEventRecord(side->fork, st) != cudaSuccess || cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
    const DxLayer L{w, dY, A, sG};
    int rc_dx = run_dx(P, &L, 1, m, k, r, true, dX, dx_dtype, false, wsb, st);
    int rc_g = run_lora_grad(P, P.db, dY, m, n, u_hi, u_lo, r, s, dB, 0, acc_grads, wsb, side->s, idle);
    if (rc_g == QLORA_OK) rc_g = run_lora_grad(P, P.da, Xl, m, k, g_hi, g_lo, r, s_da, dA, 1, acc_grads, wsb, side->s, idle);
    // join even after a failed launch, so that the caller's stream (and a capture on it) ends
    // after everything this call queued
    if (cudaEventRecord(side->join, side->s) != cudaSuccess || cudaStreamWaitEvent(st, side->join, 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return (rc_dx != QLORA_OK) ? rc_dx : rc_g;
  }

  if (dX != nullptr) {
    const DxLayer L{w, dY, A, sG};
    rc = run_dx(P, &L, 1, m, k, r, !D.on, dX, dx_dtype, acc_dx, wsb, st);
    if (rc != QLORA_OK) return rc;
    if (D.on) {
      rc = run_lora_up_masked(P, sG, m, k, A, r, D, dX, dx_dtype == QLORA_DTYPE_FP32, st);
      if (rc != QLORA_OK) return rc;
    }
  }
  rc = run_lora_grad(P, P.db, dY, m, n, u_hi, u_lo, r, s, dB, 0, acc_grads, wsb, st);
  if (rc != QLORA_OK) return rc;
  return run_lora_grad(P, P.da, Xl, m, k, g_hi, g_lo, r, s_da, dA, 1, acc_grads, wsb, st);
}

size_t qlora_linear_group_workspace_bytes(int32_t count, int64_t m, const int64_t* n, int64_t k, int32_t r) {
  if (count < 1 || count > kWGroupMax || n == nullptr || m < 1 || k < 1 || r < 1 || r > 128) return 0;
  for (int l = 0; l < count; ++l)
    if (n[l] < 1) return 0;
  return make_group_plan(count, m, n, k, r).total;
}

int qlora_linear_bwd_group(int32_t count, const qlora_nf4_weight* const* w, const uint16_t* X,
                           const uint16_t* const* dY, int64_t m, const uint16_t* const* A, const uint16_t* const* B,
                           int32_t r, float alpha, const float* const* U_saved, void* dX, int32_t dx_dtype,
                           float* const* dA, float* const* dB, int32_t flags, void* ws, size_t ws_bytes,
                           qlora_stream_t stream) {
  if (count < 1 || count > kWGroupMax || w == nullptr || dY == nullptr || A == nullptr || B == nullptr ||
      dA == nullptr || dB == nullptr)
    return QLORA_ERR_INVALID;
  if ((flags & ~(QLORA_BWD_ACCUMULATE_GRADS | QLORA_BWD_ACCUMULATE_DX)) != 0) return QLORA_ERR_INVALID;
  if (dX != nullptr && (!aligned16(dX) || (dx_dtype != QLORA_DTYPE_BF16 && dx_dtype != QLORA_DTYPE_FP32)))
    return QLORA_ERR_INVALID;
  int64_t n[kWGroupMax] = {};
  for (int l = 0; l < count; ++l) {
    if (!linear_args_ok(w[l], X, m, A[l], B[l]) || dY[l] == nullptr || !aligned16(dY[l])) return QLORA_ERR_INVALID;
    if (dA[l] == nullptr || dB[l] == nullptr || !aligned16(dA[l]) || !aligned16(dB[l])) return QLORA_ERR_INVALID;
    if (U_saved != nullptr && U_saved[l] != nullptr && !aligned16(U_saved[l])) return QLORA_ERR_INVALID;
    if (w[l]->k != w[0]->k) return QLORA_ERR_INVALID;
    const int sst = linear_shape_status(w[l], r);
    if (sst != QLORA_OK) return sst;
    n[l] = w[l]->n;
  }
  const int64_t k = w[0]->k;
  const GroupPlan G = make_group_plan(count, m, n, k, r);
  if (ws == nullptr || !aligned16(ws) || ws_bytes < G.total) return QLORA_ERR_WORKSPACE;
  char* wsb = static_cast<char*>(ws);
  char* scratch = wsb + G.off_scratch;
  const size_t scratch_bytes = G.total - G.off_scratch;
  int64_t n_total = 0;
  for (int l = 0; l < count; ++l) n_total += n[l];
  const Plan Pg = make_plan(m, n_total, k, r);
  const int acc_dx = flags & QLORA_BWD_ACCUMULATE_DX;
  const int acc_grads = flags & QLORA_BWD_ACCUMULATE_GRADS;

  if (count == 1 || dX == nullptr || wgemm_tile_rows(Pg.bn) != 256) {
    // one layer, no dX, or few tokens (the single-CTA weight GEMM takes one layer): the layers
    // one after the other, each adding its dX term to the previous ones
    for (int l = 0; l < count; ++l) {
      const int32_t fl = acc_grads | ((l > 0 || acc_dx) ? QLORA_BWD_ACCUMULATE_DX : 0);
      const int rc = qlora_linear_bwd_ex(w[l], X, dY[l], m, A[l], B[l], r, alpha,
                                         U_saved != nullptr ? U_saved[l] : nullptr, dX, dx_dtype, dA[l], dB[l], fl,
                                         nullptr, scratch, scratch_bytes, stream);
      if (rc != QLORA_OK) return rc;
    }
    return QLORA_OK;
  }

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float s = alpha / static_cast<float>(r);
  DxLayer L[kWGroupMax];
  for (int l = 0; l < count; ++l) {
    // G_l = dY_l B_l: bf16(s G_l) kept for the dX GEMM, hi/lo bf16 for dA_l; the saved U_l's
    // hi/lo split for dB_l in the same finalize launch (or U_l recomputed)
    const Plan P = make_plan(m, n[l], k, r);
    uint16_t* sG = reinterpret_cast<uint16_t*>(wsb + G.off_sg[l]);
    uint16_t* g_hi = reinterpret_cast<uint16_t*>(scratch + P.off_hi_b);
    uint16_t* g_lo = reinterpret_cast<uint16_t*>(scratch + P.off_lo_b);
    uint16_t* u_hi = reinterpret_cast<uint16_t*>(scratch + P.off_hi_a);
    uint16_t* u_lo = reinterpret_cast<uint16_t*>(scratch + P.off_lo_a);
    const float* Us = (U_saved != nullptr) ? U_saved[l] : nullptr;
    int rc = run_lora_down(P, true, dY[l], m, n[l], B[l], r, s, scratch, nullptr, sG, g_hi, g_lo, st, 1.0f, Us,
                           Us != nullptr ? u_hi : nullptr, Us != nullptr ? u_lo : nullptr);
    if (rc != QLORA_OK) return rc;
    if (Us == nullptr) {
      rc = run_lora_down(P, false, X, m, k, A[l], r, s, scratch, nullptr, nullptr, u_hi, u_lo, st);
      if (rc != QLORA_OK) return rc;
    }
    rc = run_lora_grad(P, P.db, dY[l], m, n[l], u_hi, u_lo, r, s, dB[l], 0, acc_grads, scratch, st);
    if (rc != QLORA_OK) return rc;
    rc = run_lora_grad(P, P.da, X, m, k, g_hi, g_lo, r, s, dA[l], 1, acc_grads, scratch, st);
    if (rc != QLORA_OK) return rc;
    L[l] = DxLayer{w[l], dY[l], A[l], sG};
  }
  // dX = sum_l (dY_l W_l + s G_l A_l): one weight GEMM over the layers' reductions in turn
  return run_dx(Pg, L, count, m, k, r, true, dX, dx_dtype, acc_dx != 0, scratch, st);
}

int qlora_adamw_step(float* param, const float* grad, float* m, float* v, uint16_t* param_bf16, int64_t count,
                     const qlora_adamw_config* cfg, qlora_stream_t stream) {
  if (cfg == nullptr || count < 0) return QLORA_ERR_INVALID;
  if (count == 0) return QLORA_OK;
  if (param == nullptr || grad == nullptr || m == nullptr || v == nullptr) return QLORA_ERR_INVALID;
  if (!aligned16(param) || !aligned16(grad) || !aligned16(m) || !aligned16(v)) return QLORA_ERR_INVALID;
  if (param_bf16 != nullptr && (reinterpret_cast<uintptr_t>(param_bf16) & 7u) != 0) return QLORA_ERR_INVALID;
  if (cfg->step < 1 || !(cfg->beta1 > 0.f && cfg->beta1 < 1.f) || !(cfg->beta2 > 0.f && cfg->beta2 < 1.f) ||
      !(cfg->eps > 0.f) || !std::isfinite(cfg->lr) || !std::isfinite(cfg->weight_decay) ||
      !std::isfinite(cfg->grad_scale))
    return QLORA_ERR_INVALID;
  return cuda_status(launch_adamw(param, grad, m, v, param_bf16, count, cfg->lr, cfg->beta1, cfg->beta2, cfg->eps,
                                  cfg->weight_decay, cfg->grad_scale, cfg->step, num_sms(),
                                  reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_paged_alloc(size_t bytes, void** out) {
  if (out == nullptr || bytes == 0) return QLORA_ERR_INVALID;
  *out = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  void* ptr = nullptr;
  if (cudaMallocManaged(&ptr, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
  // home on the current device; the driver may still migrate pages to host RAM under pressure
  cudaMemLocation loc;
  loc.type = cudaMemLocationTypeDevice;
  loc.id = dev;
  (void)cudaMemAdvise(ptr, bytes, cudaMemAdviseSetPreferredLocation, loc);
  (void)cudaGetLastError();      // the advice is a hint: a device without it still works
  *out = ptr;
  return QLORA_OK;
}

int qlora_paged_free(void* ptr) {
  if (ptr == nullptr) return QLORA_OK;
  return cuda_status(cudaFree(ptr));
}

int qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_host, qlora_stream_t stream) {
  if (ptr == nullptr || bytes == 0) return QLORA_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  cudaMemLocation loc;
  loc.type = to_host ? cudaMemLocationTypeHost : cudaMemLocationTypeDevice;
  loc.id = to_host ? 0 : dev;
  return cuda_status(cudaMemPrefetchAsync(ptr, bytes, loc, 0, reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_silu_gate_fwd(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t count, qlora_stream_t stream) {
  if (count < 0) return QLORA_ERR_INVALID;
  if (count == 0) return QLORA_OK;
  if (g == nullptr || u == nullptr || h == nullptr || !aligned16(g) || !aligned16(u) || !aligned16(h))
    return QLORA_ERR_INVALID;
  return cuda_status(launch_silu_gate_fwd(g, u, h, count, reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_silu_gate_bwd(const uint16_t* dh, const uint16_t* g, const uint16_t* u, uint16_t* dg, uint16_t* du,
                        int64_t count, qlora_stream_t stream) {
  if (count < 0) return QLORA_ERR_INVALID;
  if (count == 0) return QLORA_OK;
  if (dh == nullptr || g == nullptr || u == nullptr || dg == nullptr || du == nullptr) return QLORA_ERR_INVALID;
  if (!aligned16(dh) || !aligned16(g) || !aligned16(u) || !aligned16(dg) || !aligned16(du)) return QLORA_ERR_INVALID;
  return cuda_status(launch_silu_gate_bwd(dh, g, u, dg, du, count, reinterpret_cast<cudaStream_t>(stream)));
}

int64_t qlora_launch_count(void) { return qlora::g_launches.load(); }

int qlora_timing_begin(int32_t max_launches) {
  if (max_launches < 1) return QLORA_ERR_INVALID;
  std::lock_guard<std::mutex> g(qlora::g_timing_mu);
  for (cudaEvent_t ev : qlora::g_events) cudaEventDestroy(ev);
  qlora::g_events.assign(static_cast<size_t>(max_launches) * 2, nullptr);
  qlora::g_event_flops.assign(static_cast<size_t>(max_launches), 0.0);
  for (auto& ev : qlora::g_events)
    if (cudaEventCreate(&ev) != cudaSuccess) return QLORA_ERR_CUDA;
  qlora::g_events_used = 0;
  qlora::g_timing_on = true;
  return QLORA_OK;
}

int qlora_timing_end(double* total_ms, int32_t* launches, double* flops) {
  std::lock_guard<std::mutex> g(qlora::g_timing_mu);
  qlora::g_timing_on = false;
  double ms = 0.0, fl = 0.0;
  int rc = QLORA_OK;
  qlora::g_last_ms.clear();
  qlora::g_last_flops.clear();
  for (size_t i = 0; i + 1 < qlora::g_events_used; i += 2) {
    float t = 0.f;
    if (cudaEventSynchronize(qlora::g_events[i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, qlora::g_events[i], qlora::g_events[i + 1]) != cudaSuccess) {
      rc = QLORA_ERR_CUDA;
      break;
    }
    ms += t;
    fl += qlora::g_event_flops[i / 2];
    qlora::g_last_ms.push_back(t);
    qlora::g_last_flops.push_back(qlora::g_event_flops[i / 2]);
  }
  if (total_ms) *total_ms = ms;
  if (launches) *launches = static_cast<int32_t>(qlora::g_events_used / 2);
  if (flops) *flops = fl;
  for (cudaEvent_t ev : qlora::g_events) cudaEventDestroy(ev);
  qlora::g_events.clear();
  qlora::g_event_flops.clear();
  qlora::g_events_used = 0;
  return rc;
}

int qlora_timing_launch(int32_t index, double* ms, double* flops) {
  std::lock_guard<std::mutex> g(qlora::g_timing_mu);
  if (index < 0 || static_cast<size_t>(index) >= qlora::g_last_ms.size() || ms == nullptr || flops == nullptr)
    return QLORA_ERR_INVALID;
  *ms = qlora::g_last_ms[static_cast<size_t>(index)];
  *flops = qlora::g_last_flops[static_cast<size_t>(index)];
  return QLORA_OK;
}

int qlora_selftest_wait_timeout(int32_t limit_ms, qlora_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return QLORA_ERR_INVALID;
  return cuda_status(launch_selftest_wait_timeout(static_cast<uint64_t>(limit_ms) * 1000000ull,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_expand_rate(int32_t iters, double* weights_per_sm_clock, double* weights_per_second) {
  if (iters < 1 || iters > (1 << 20) || weights_per_sm_clock == nullptr || weights_per_second == nullptr)
    return QLORA_ERR_INVALID;
  const int grid = std::min(num_sms(), 1024);
  cudaStream_t st = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return QLORA_ERR_CUDA;
  int threads = 0;
  int rc = QLORA_OK;
  if (cudaEventRecord(e0, st) != cudaSuccess || launch_expand_rate(table(), iters, grid, &threads, st) != cudaSuccess ||
      cudaEventRecord(e1, st) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess)
    rc = QLORA_ERR_CUDA;
  float ms = 0.f;
  std::vector<unsigned long long> cyc(static_cast<size_t>(grid), 0ull);
  if (rc == QLORA_OK &&
      (cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess || read_expand_cycles(cyc.data(), grid) != cudaSuccess))
    rc = QLORA_ERR_CUDA;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (rc != QLORA_OK) return rc;
  unsigned long long most = 1;
  for (unsigned long long c : cyc) most = std::max(most, c);
  const double per_cta = static_cast<double>(threads) * iters * 64.0;
  *weights_per_sm_clock = per_cta / static_cast<double>(most);
  *weights_per_second = per_cta * grid / (static_cast<double>(ms) * 1e-3);
  return QLORA_OK;
}

int qlora_check_device_error(qlora_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, qlora::g_device_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(qlora::g_device_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    return v == qlora::kErrBounds ? QLORA_ERR_BOUNDS : QLORA_ERR_DEVICE;
  }
  return QLORA_OK;
}

int qlora_bounds_site(void) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, qlora::g_bounds_site, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(qlora::g_bounds_site, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // extern "C"
