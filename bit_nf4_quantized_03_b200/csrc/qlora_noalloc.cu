// Allocation-free NF4 quantization with double quantization.
//
// qlora_nf4_quantize needs a caller-supplied device workspace for the
// double-quant pass (the fp32 absmax of every 64-block, the fixed-order
// partial sums of the mean, the mean itself). Some callers cannot provide
// one: a plugin that a host framework hands only input and output pointers
// while the framework owns every byte of device memory, or a latency-critical
// path that must not call cudaMalloc (which can synchronize the whole
// device). This file serves them from a fixed scratch array compiled into the
// library, so the entry point below allocates nothing.
//
// The scratch is a file-scope __device__ array of kScratchBytes. Every GPU
// that loads the library holds it until the process exits. In host code the
// array's name is only a host-side stand-in for the device symbol, so its
// device address is looked up once per device (cudaGetSymbolAddress, with
// that device current) and passed to the kernels as a plain pointer. The
// address belongs to the device's current context: after a context is
// destroyed and created again (cudaDeviceReset, a released primary context)
// the module loads again, possibly elsewhere, so the cached address is keyed
// on the context and looked up again when the context changes.
#include <mutex>

#include "../../include/qlora.h"
#include "qlora_kernels.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;   // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Unique id of the calling thread's current context (0 when none is current yet),
// through the driver's cuCtxGetCurrent and cuCtxGetId reached via the runtime. Ids are
// never reused within a process, unlike context handles.
unsigned long long current_context_id() {
  using GetCur = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCur get_cur = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<GetCur>(ptr);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(ptr);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

}  // namespace

namespace qlora {
unsigned long long context_id() { return current_context_id(); }
}  // namespace qlora

namespace {

// Device address of the scratch array on the current device, looked up on the first
// call per device and again whenever that device's context has changed since.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = current_context_id();
  if (id == 0 || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != id) {
    // (the lookup also makes the device's context current when none was yet)
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    id = current_context_id();
    if (id == 0) return QLORA_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = id;
  }
  *out = g_scratch_addr[dev];
  return QLORA_OK;
}

bool aligned_16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool weight_buffers_ok(const qlora_nf4_weight* w) {
  if (w == nullptr || w->n < 1 || w->k < 1) return false;
  if (w->blocksize != QLORA_BLOCKSIZE || w->dq_blocksize != QLORA_DQ_BLOCKSIZE) return false;
  if (w->codes == nullptr || !aligned_16(w->codes)) return false;
  if (w->mode == QLORA_SCALE_BF16) return w->scale_bf16 != nullptr && aligned_16(w->scale_bf16);
  if (w->mode == QLORA_SCALE_DQ_FP8)
    return w->scale_fp8 != nullptr && w->dq_scale != nullptr && w->dq_mean != nullptr &&
           aligned_16(w->scale_fp8) && aligned_16(w->dq_scale);
  return false;
}

}  // namespace

extern "C" int qlora_nf4_quantize_noalloc(const float* W, qlora_nf4_weight* w, qlora_stream_t stream) {
  if (W == nullptr || !aligned_16(W) || !weight_buffers_ok(w)) return QLORA_ERR_INVALID;
  const int64_t n_elem = w->n * w->k;
  const bool dq = (w->mode == QLORA_SCALE_DQ_FP8);
  // Every scratch word a call reads is written earlier in the same call, so
  // nothing needs clearing between calls.
  if (dq && qlora::quant_ws_layout(n_elem).total > kScratchBytes) return QLORA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != QLORA_OK) return rc;
  // the same tables and SM count qlora_nf4_quantize uses, so the bytes are the same by construction
  const cudaError_t e = qlora::launch_quantize(W, n_elem, qlora::host_table(), qlora::host_buckets(), w->codes,
                                               dq ? nullptr : w->scale_bf16, dq ? w->scale_fp8 : nullptr,
                                               dq ? w->dq_scale : nullptr, dq ? w->dq_mean : nullptr, scratch,
                                               qlora::host_num_sms(), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
