/*
 * qlora.h -- C ABI of libqlora: the frozen-base linear layer of QLoRA on one
 * NVIDIA B200 (sm_100a).
 *
 * What it computes (sources are web pages on QLoRA, cited by title/section):
 *
 *  - Storage: each weight of the frozen base is snapped to the nearest of 16
 *    NormalFloat levels and kept in 4 bits, with one absmax scale per block of
 *    64 weights ("QLoRA: Quantized Low-Rank Adaptation", Piece 1 and the
 *    section "NF4: a 4-bit format matched to weight statistics"; "QLoRA
 *    Explained: Fine-Tune 70B+ LLMs on a Single GPU", section "4-Bit
 *    NormalFloat (NF4) Quantization").
 *  - Double quantization: the block scales themselves are stored as 8-bit
 *    floats (OCP E4M3) in blocks of 256 with one fp32 scale per block and one
 *    fp32 mean offset per tensor ("QLoRA: Quantized Low-Rank Adaptation",
 *    section "Double quantization (the label-index-card trick)"; "QLoRA
 *    Explained", section "Double Quantization").
 *  - Compute: right before the multiply each block is dequantized to BF16
 *    ("QLoRA: Quantized Low-Rank Adaptation", Piece 2; "Batched 4-bit
 *    matmuls") and used in
 *        Y = X W'^T + (alpha/r) (X A^T) B^T ,
 *    the backward pass computes dX = dY W' + (alpha/r)(dY B) A and the
 *    adapter gradients dA = (alpha/r)(dY B)^T X, dB = (alpha/r) dY^T (X A^T);
 *    the quantized base gets no gradient (same page, Piece 3; "What is
 *    QLoRA?", Key Characteristics: "Backpropagation through quantized
 *    weights").
 *
 * Bit-level format (fixed by this library where the pages are silent):
 *  - levels L[0..15]: the asymmetric normal-quantile construction with an
 *    exact zero at L[7] and L[0] = -1, L[15] = +1 (qlora_nf4_levels returns
 *    them); code(x) = number of fp32 midpoints fp32((L[i]+L[i+1])*0.5) that
 *    are strictly below x = fp32(w * fp32(1/absmax)); a block whose absmax
 *    is zero or subnormal is all code 7;
 *  - packing: byte j of `codes` holds element 2j in bits 0..3 and element
 *    2j+1 in bits 4..7 (row-major order of W, blocks never reordered);
 *  - BF16 mode: scale_bf16[b] = bf16_rn(absmax_b);
 *  - double-quant mode: mean = fp32(S / nblk), S the fp64 sum of all absmax
 *    values by a pairwise tree over the array zero-padded to a power of two;
 *    per 256-block j: d = fp32(absmax - mean), dq_scale[j] = fp32(max|d| /
 *    448) (1 when max|d| = 0), scale_fp8[b] = e4m3_rn_satfinite(fp32(d /
 *    dq_scale[j]));
 *  - dequantized weight: bf16_rn(fp32(L[code] * c)) with c = bf16 scale, or
 *    c = fp32(fp32(e4m3(q) * dq_scale[b/256]) + mean).
 *
 * Conventions for every function:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates device memory, never synchronizes, and keeps no state
 *    between calls other than a read-only level table, a device error word and
 *    the backward's internal stream and two events (per thread and context).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default), or
 *    ordered with it through events (qlora_linear_bwd).
 *  - Argument errors are detected on the host before anything is enqueued
 *    and return QLORA_ERR_INVALID / QLORA_ERR_UNSUPPORTED / QLORA_ERR_WORKSPACE;
 *    a failed launch returns QLORA_ERR_CUDA.
 *  - Matrices are row-major and contiguous. bf16 tensors are passed as
 *    uint16_t bit patterns. Every pointer must be 16-byte aligned.
 *  - Inputs must be finite; non-finite weights give unspecified codes.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qlora_stream_t; /* same type as cudaStream_t */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID = 1,     /* null pointer, bad size, misaligned pointer */
  QLORA_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels cover */
  QLORA_ERR_CUDA = 3,        /* a CUDA launch or query failed */
  QLORA_ERR_WORKSPACE = 4,   /* workspace pointer null or too small */
  QLORA_ERR_DEVICE = 5,      /* a kernel gave up on a bounded wait */
  QLORA_ERR_BOUNDS = 6       /* a bounds check failed (bounds-checking build only) */
} qlora_status;

typedef enum {
  QLORA_SCALE_BF16 = 0,  /* one bf16 absmax per 64 weights */
  QLORA_SCALE_DQ_FP8 = 1 /* double quantization (bnb_4bit_use_double_quant) */
} qlora_scale_mode;

typedef enum { QLORA_DTYPE_BF16 = 0, QLORA_DTYPE_FP32 = 1 } qlora_dtype;

enum { QLORA_BLOCKSIZE = 64, QLORA_DQ_BLOCKSIZE = 256 };

/* qlora_linear_bwd flags */
enum {
  QLORA_BWD_ACCUMULATE_GRADS = 1, /* dA += ..., dB += ... (gradient accumulation) */
  QLORA_BWD_ACCUMULATE_DX = 2     /* dX += ... (e.g. two projections reading the same X) */
};

/*
 * An NF4 weight W of shape [n, k] (out_features x in_features). Buffers:
 *   codes       ceil(n*k/2) bytes
 *   scale_bf16  nblk uint16     (BF16 mode; NULL otherwise)
 *   scale_fp8   nblk bytes      (double-quant mode)
 *   dq_scale    nblk2 floats    (double-quant mode)
 *   dq_mean     1 float         (double-quant mode)
 * with nblk = ceil(n*k/64), nblk2 = ceil(nblk/256). blocksize must be 64 and
 * dq_blocksize 256.
 */
typedef struct {
  int64_t n;
  int64_t k;
  int32_t blocksize;
  int32_t dq_blocksize;
  int32_t mode; /* qlora_scale_mode */
  int32_t reserved;
  uint8_t *codes;
  uint16_t *scale_bf16;
  uint8_t *scale_fp8;
  float *dq_scale;
  float *dq_mean;
} qlora_nf4_weight;

/* Human-readable name of a status code (static string). */
const char *qlora_status_string(int status);

/* Library version string. */
const char *qlora_version(void);

/* Host: writes the 16 fp32 NF4 levels (ascending) the kernels use and the 15
 * fp32 decision midpoints (mid may be NULL). Always QLORA_OK. */
int qlora_nf4_levels(float levels[16], float mid[15]);

/* Bytes of device workspace qlora_nf4_quantize needs (0 in BF16 mode). */
size_t qlora_nf4_quantize_workspace_bytes(int64_t n, int64_t k, int32_t mode);

/*
 * Quantize W (fp32 [n, k], device) into `w` (buffers and shape set by the
 * caller). Any n*k >= 1 (the last block may be partial). The double-quant
 * mode needs `ws` of at least qlora_nf4_quantize_workspace_bytes bytes and
 * n*k <= 2^33 (QLORA_ERR_UNSUPPORTED above that, nothing enqueued).
 * Deterministic: the same input gives the same bytes on every call.
 */
int qlora_nf4_quantize(const float *W, qlora_nf4_weight *w, void *ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * qlora_nf4_quantize without a workspace: this entry point allocates nothing.
 * It is for callers that cannot allocate device memory -- a plugin that a
 * host framework hands only input and output pointers while the framework
 * owns all device memory, or a latency-critical path that must not call
 * cudaMalloc (which can synchronize the device). No passage of the pages has
 * a counterpart; it is an interface convenience of this library.
 *  - The double-quant scratch is a fixed 16 MiB array inside the library,
 *    held by every GPU that loads the library until the process exits. It
 *    covers n*k <= 267,382,784 weights (e.g. 22016 x 8192 needs 11 MiB);
 *    larger requests return QLORA_ERR_UNSUPPORTED with nothing enqueued.
 *  - The first call on a device looks up the scratch's device address with
 *    that device current; make that first call before any stream capture.
 *    The address is kept per device and context: the first call after the
 *    device's context was destroyed and created again (cudaDeviceReset)
 *    looks it up again, so that call, too, belongs before any capture.
 *  - All calls share the one array, which keeps the last call's contents
 *    (each call writes every scratch word before reading it). Calls whose
 *    work overlaps on the GPU -- on different streams, or from different host
 *    threads -- race on it; serialize them.
 *  - Results are bit-identical to qlora_nf4_quantize.
 */
int qlora_nf4_quantize_noalloc(const float *W, qlora_nf4_weight *w, qlora_stream_t stream);

/* Dequantize `w` into out_bf16 ([n, k] bf16, device), bit-exact per the format above. */
int qlora_nf4_dequantize(const qlora_nf4_weight *w, uint16_t *out_bf16, qlora_stream_t stream);

/*
 * Merge a trained adapter onto the dequantized weight:
 *   W_out[n, k] = W'[n, k] + (alpha / r) * (B . A)[n, k]
 * where W' is the BF16 dequantization of `w` (the format above), A is [r, k]
 * and B is [n, r] (bf16, row-major, device). A 4-bit matrix cannot absorb
 * the adapter, so deployment merges it onto a dequantized copy ("QLoRA:
 * Quantized Low-Rank Adaptation", Price 2: deployment friction; "QLoRA
 * Explained", Step 5: Save and Merge Adapters). out_dtype QLORA_DTYPE_BF16
 * stores the BF16 copy; QLORA_DTYPE_FP32 stores fp32 values, ready to be
 * quantized again with qlora_nf4_quantize for deployment ("QLoRA vs LoRA",
 * FAQ on converting back to full precision).
 *  - Each element is fp32(w' + s * acc) with acc the fp32 tensor-core sum of
 *    the r products, then rounded once more to BF16 for QLORA_DTYPE_BF16.
 *  - W_out is [n, k] row-major, caller-owned, 16-byte aligned. Requires
 *    k % 64 == 0 and r in {8, 16, 32, 64, 128}; otherwise
 *    QLORA_ERR_UNSUPPORTED. Null or misaligned pointers: QLORA_ERR_INVALID.
 *    Nothing is enqueued on an error. No workspace; nothing is allocated.
 */
int qlora_lora_merge(const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                     void *W_out, int32_t out_dtype, qlora_stream_t stream);

/* Bytes of device workspace qlora_linear_fwd / qlora_linear_bwd need for m
 * tokens, an [n, k] weight and rank r. Above 128 tokens this includes an fp32
 * [m, k] buffer: a backward that accumulates into dX writes the GEMM's result
 * there and adds it to dX in one coalesced pass. */
size_t qlora_linear_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t r);

/*
 * Forward: Y[m, n] = X W'^T + (alpha/r) (X A^T) B^T.
 *   X  [m, k] bf16;  A [r, k] bf16;  B [n, r] bf16;
 *   Y  [m, n] in y_dtype (qlora_dtype);
 *   U_save: optional fp32 [m, r] output of U = X A^T (saved for backward).
 * Requires k % 64 == 0, n % 8 == 0, m >= 1, r in {8, 16, 32, 64, 128}.
 */
int qlora_linear_fwd(const qlora_nf4_weight *w, const uint16_t *X, int64_t m, const uint16_t *A,
                     const uint16_t *B, int32_t r, float alpha, void *Y, int32_t y_dtype, float *U_save,
                     void *ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * Backward through the frozen NF4 base:
 *   dX[m, k] (+)= dY W' + (alpha/r) (dY B) A      (skipped when dX is NULL)
 *   dA[r, k] (+)= (alpha/r) (dY B)^T X            fp32
 *   dB[n, r] (+)= (alpha/r) dY^T U, U = X A^T     fp32
 * U_saved: optional fp32 [m, r] from the forward pass (NULL: recomputed).
 * flags: QLORA_BWD_ACCUMULATE_GRADS and/or QLORA_BWD_ACCUMULATE_DX.
 * Same shape rules as qlora_linear_fwd.
 *
 * Token-sharded data parallelism ("QLoRA Explained", Hardware Requirements by
 * Model Size; the FAQ on one model over several GPUs): every rank holds the
 * same weight and adapters and calls qlora_linear_fwd / qlora_linear_bwd on
 * its own contiguous slice of the tokens (m = that slice). Y, U and dX of a
 * slice need nothing from other ranks. dA and dB are sums over tokens, so a
 * rank's call yields the partial sum over its slice; the full-batch gradient
 * is the fp32 sum of the ranks' dA and dB (one all-reduce, done by the
 * caller: the library holds no communicator). QLORA_BWD_ACCUMULATE_GRADS adds
 * into dA, dB instead, so several slices on one rank (gradient accumulation)
 * sum the same way before the exchange.
 *
 * Streams: when the dX GEMM leaves SMs idle (one split, dX not accumulated, no
 * dropout), dA and dB are computed beside it on an internal stream of the
 * library (one per host thread and CUDA context, created on that thread's first
 * such call outside a stream capture). That stream waits on an event recorded
 * on `stream`, and `stream` waits on one recorded after its work, so everything
 * the call enqueues is ordered as if it ran on `stream` alone, under a CUDA
 * graph capture too. The results are bit-identical either way.
 */
int qlora_linear_bwd(const qlora_nf4_weight *w, const uint16_t *X, const uint16_t *dY, int64_t m,
                     const uint16_t *A, const uint16_t *B, int32_t r, float alpha, const float *U_saved,
                     void *dX, int32_t dx_dtype, float *dA, float *dB, int32_t flags, void *ws,
                     size_t ws_bytes, qlora_stream_t stream);

/*
 * LoRA dropout on the input of the low-rank branch ("QLoRA Explained", Step 3:
 * LoraConfig lora_dropout = 0.05; hyperparameter quick reference). The pages
 * give only the rate; this library applies inverted dropout the way PEFT
 * does: the branch sees M * X, with keep mask M, and its output is scaled by
 * c = 1 / (1 - p). So U = c (M * X) A^T, dA = (alpha/r) c (dY B)^T (M * X),
 * and dX gets (alpha/r) c ((dY B) A) * M.
 *  - M comes from Philox4x32-10 (Salmon et al., SC 2011):
 *      counter = (e / 8 as two 32-bit words, offset as two words),
 *      key = seed as two words.
 *    Element e of X (row-major) reads the 16-bit lane e % 8 of the four
 *    output words (word (e % 8) / 2, low half first). It is kept iff that
 *    value >= round(p * 65536). The effective rate is round(p * 65536) / 65536,
 *    and c = 65536 / (65536 - round(p * 65536)).
 *  - p in [0, 1); p = 0 disables dropout.
 *  - mask: caller-owned device buffer of m * k / 8 bytes; element e is bit
 *    e % 8 of byte e / 8. The forward writes it. The backward reads it and
 *    does not draw again, so pass the same buffer (or the same bytes) to both.
 *  - Vary seed or offset per step to get a fresh mask.
 */
typedef struct {
  float p;
  int32_t reserved;
  uint64_t seed;
  uint64_t offset;
  uint8_t *mask;
} qlora_dropout;

/* Workspace for qlora_linear_fwd_ex / qlora_linear_bwd_ex. With dropout on,
 * it holds a masked copy of X as well (m * k * 2 more bytes). */
size_t qlora_linear_workspace_bytes_ex(int64_t m, int64_t n, int64_t k, int32_t r, const qlora_dropout *drop);

/* qlora_linear_fwd with optional LoRA dropout (drop NULL or p == 0: identical to
 * qlora_linear_fwd). U_save then holds U = c (M * X) A^T. Invalid p, or a NULL
 * or misaligned mask with p > 0: QLORA_ERR_INVALID. */
int qlora_linear_fwd_ex(const qlora_nf4_weight *w, const uint16_t *X, int64_t m, const uint16_t *A,
                        const uint16_t *B, int32_t r, float alpha, void *Y, int32_t y_dtype, float *U_save,
                        const qlora_dropout *drop, void *ws, size_t ws_bytes, qlora_stream_t stream);

/* qlora_linear_bwd with optional LoRA dropout; drop->mask must hold the forward's mask. */
int qlora_linear_bwd_ex(const qlora_nf4_weight *w, const uint16_t *X, const uint16_t *dY, int64_t m,
                        const uint16_t *A, const uint16_t *B, int32_t r, float alpha, const float *U_saved,
                        void *dX, int32_t dx_dtype, float *dA, float *dB, int32_t flags,
                        const qlora_dropout *drop, void *ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * Backward of up to three layers that read the same input X: the q, k and v
 * projections of an attention block, or the gate and up projections of a SiLU
 * MLP (the pages put LoRA on every linear layer: "QLoRA Explained", Step 3,
 * target_modules = "all-linear"). For layer l = 0 .. count - 1, with weight
 * w[l] ([n_l, k]; k the same for all), dY[l] [m, n_l], adapters A[l] [r, k]
 * and B[l] [n_l, r], and the same r and alpha:
 *   dX[m, k] (+)= sum_l (dY_l W'_l + (alpha/r) (dY_l B_l) A_l)
 *   dA[l], dB[l] (+)= as qlora_linear_bwd gives them for layer l
 * The value is that of qlora_linear_bwd called per layer with
 * QLORA_BWD_ACCUMULATE_DX from the second layer on; the sum is formed in one
 * fused GEMM whose reduction runs over the layers in turn (above 128 tokens),
 * so no layer's term passes through an fp32 partial. At most 128 tokens, or
 * with dX NULL, the layers run one after the other.
 *  - w, dY, A, B, dA, dB: arrays of count pointers, each as in
 *    qlora_linear_bwd; U_saved: NULL or an array of count pointers, each NULL
 *    (U_l recomputed) or fp32 [m, r] from that layer's forward.
 *  - flags: QLORA_BWD_ACCUMULATE_GRADS (every layer's dA, dB) and/or
 *    QLORA_BWD_ACCUMULATE_DX.
 *  - No LoRA dropout here (qlora_linear_bwd_ex per layer has it).
 *  - ws: qlora_linear_group_workspace_bytes(count, m, n, k, r) bytes, 16-byte
 *    aligned, device memory; the call reads and writes it and nothing else
 *    keeps it.
 *  - count outside 1..3, differing k, or an argument qlora_linear_bwd would
 *    reject: the same status as there, with nothing enqueued.
 */
int qlora_linear_bwd_group(int32_t count, const qlora_nf4_weight *const *w, const uint16_t *X,
                           const uint16_t *const *dY, int64_t m, const uint16_t *const *A,
                           const uint16_t *const *B, int32_t r, float alpha, const float *const *U_saved,
                           void *dX, int32_t dx_dtype, float *const *dA, float *const *dB, int32_t flags,
                           void *ws, size_t ws_bytes, qlora_stream_t stream);

/* Workspace of qlora_linear_bwd_group for count layers with n[l] output
 * features each (array of count), k input features, m tokens and rank r;
 * 0 for arguments it would reject. */
size_t qlora_linear_group_workspace_bytes(int32_t count, int64_t m, const int64_t *n, int64_t k, int32_t r);

/*
 * Paged AdamW, 32-bit, for the adapters ("QLoRA Explained": Paged Optimizers
 * and optim = "paged_adamw_32bit"; "QLoRA: Quantized Low-Rank Adaptation":
 * "Paged optimizers (the storage unit)"). AdamW with decoupled weight decay
 * on fp32 masters and fp32 moments, one fused pass per parameter array:
 *   g = grad * grad_scale;  m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2
 *   p = p (1 - lr wd) - (lr / (1 - b1^step)) m / (sqrt(v) / sqrt(1 - b2^step) + eps)
 * and, when param_bf16 is not NULL, param_bf16 = bf16(p) (the copy the GEMMs
 * read). All arrays hold `count` elements, are 16-byte aligned and device
 * accessible: device memory or qlora_paged_alloc memory. step >= 1;
 * 0 < b1, b2 < 1; eps > 0; else QLORA_ERR_INVALID with nothing enqueued.
 */
typedef struct {
  float lr;
  float beta1;
  float beta2;
  float eps;
  float weight_decay;
  float grad_scale;
  int32_t step;
  int32_t reserved;
} qlora_adamw_config;

int qlora_adamw_step(float *param, const float *grad, float *m, float *v, uint16_t *param_bf16, int64_t count,
                     const qlora_adamw_config *cfg, qlora_stream_t stream);

/* Paged memory for optimizer states: unified (managed) memory with the
 * current device as its preferred home. The driver may move it to host RAM
 * when device memory runs short; qlora_paged_prefetch moves it explicitly
 * (to_host = 0: to the current device, before the step; 1: to host RAM,
 * freeing device memory during a spike). The allocation is the caller's and
 * must be released with qlora_paged_free. These calls, unlike the compute
 * entry points, allocate. */
int qlora_paged_alloc(size_t bytes, void **out);
int qlora_paged_free(void *ptr);
int qlora_paged_prefetch(const void *ptr, size_t bytes, int32_t to_host, qlora_stream_t stream);

/* SiLU-gated MLP glue (bf16 in/out, fp32 math): h = silu(g) * u. */
int qlora_silu_gate_fwd(const uint16_t *g, const uint16_t *u, uint16_t *h, int64_t count, qlora_stream_t stream);

/* Backward of h = silu(g) * u: dg = dh*u*s*(1 + g*(1-s)), du = dh*g*s, s = sigmoid(g). */
int qlora_silu_gate_bwd(const uint16_t *dh, const uint16_t *g, const uint16_t *u, uint16_t *dg, uint16_t *du,
                        int64_t count, qlora_stream_t stream);

/* Number of kernels this library has launched in this process (all calls,
 * all devices). */
int64_t qlora_launch_count(void);

/* Device-time measurement of the fused NF4 tensor-core GEMMs (forward Y and
 * backward dX). Between qlora_timing_begin and qlora_timing_end the library
 * records a CUDA event pair on the launch stream around each such launch (at
 * most max_launches; the events are created here, no device memory is
 * allocated). qlora_timing_end waits for those events and returns the summed
 * device time in ms, the number of launches timed and their algorithmic
 * flops, 2 * rows * cols * (reduction + r). Process-wide, not thread-safe. */
int qlora_timing_begin(int32_t max_launches);
int qlora_timing_end(double *total_ms, int32_t *launches, double *flops);

/* Device time (ms) and algorithmic flops of launch `index` (0-based, launch
 * order) of the last qlora_timing_end. QLORA_ERR_INVALID for an index outside
 * [0, launches) or a null pointer. Process-wide, not thread-safe. */
int qlora_timing_launch(int32_t index, double *ms, double *flops);

/* Exercises the failure path without faulting the GPU: launches one thread
 * that waits on a barrier nobody arrives on and gives up after limit_ms
 * (1..2000), recording the device error word exactly as a stuck pipeline
 * would. The kernel then returns normally; qlora_check_device_error reports
 * QLORA_ERR_DEVICE once and the context stays usable. */
int qlora_selftest_wait_timeout(int32_t limit_ms, qlora_stream_t stream);

/* Measures how fast this library's NF4 expansion runs with nothing else on the
 * SMs: one CTA per SM, each thread repeatedly building a 64-block's table
 * bf16(fp32(L[j] * c)) and looking up its 64 BF16 weights from codes in
 * shared memory, `iters` blocks per thread (1..2^20). Writes the weights
 * expanded per SM-clock (the per-CTA clock64 count of the slowest CTA) and per
 * second (CUDA events around the launch). This is the ceiling on the weight
 * rate of any kernel that turns every weight into BF16 by this table, which
 * bounds the few-token forward when memory does not. Runs on the legacy
 * default stream of the current device and synchronizes it. The pages have no
 * counterpart; it is a measuring tool. */
int qlora_expand_rate(int32_t iters, double* weights_per_sm_clock, double* weights_per_second);

/* Reads and clears the device error word (set when a kernel gave up on a
 * bounded wait, or, in the bounds-checking build, when a check failed).
 * Synchronizes `stream`. Returns QLORA_OK, QLORA_ERR_DEVICE or QLORA_ERR_BOUNDS. */
int qlora_check_device_error(qlora_stream_t stream);

/* Bounds-checking build (compiled with -DQLORA_BOUNDS_CHECK): the kernels check
 * each TMA tile start (innermost coordinate on a 16-byte boundary and inside
 * the tensor, shared-memory address aligned), each bulk copy (16-byte aligned
 * addresses and size) and the main global stores against the sizes the host
 * planned; a failed check skips the access and records QLORA_ERR_BOUNDS and
 * the site number. This returns the first failing site since the last call
 * and clears it (0: none; always 0 in the normal build; -1: CUDA error). It
 * stands in for an external memory checker where none can run. */
int qlora_bounds_site(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
