// moe_layer_decode_noalloc: the fused decode step with its scratch memory in
// a file-scope device array, for callers that cannot allocate device memory.
//
// Some hosts hand a kernel library only its inputs and outputs and own every
// allocation themselves (a plugin slot in another runtime, a process under a
// fixed device-memory budget): such a caller has no way to provide the
// workspace that moe_layer needs. This entry point needs none. It runs the
// same kernel as moe_layer's decode path; only the scratch pointers differ.
//
// The scratch is kNoAllocBytes of device memory held by every GPU that loads
// this library until the process exits. Every call shares it, so calls that
// may overlap on the GPU (different streams, different host threads) race
// and must be serialised by the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "call_range.h"
#include "moe.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace {

// Header (256 B) + the launch's counters + logits, biased and unbiased
// (8 T E bytes) + the shared expert's gates (4 T bytes) + the intermediate
// activations (65 expert slots x T x I values, fp32 and fp16): enough for
// T I <= 4096 at E <= 1024 (the decode shapes: one token at I <= 2048, up to
// four at I <= 1024); a call whose scratch would not fit returns
// MOE_ERR_UNSUPPORTED.
constexpr size_t kNoAllocBytes = 2048u * 1024u;
constexpr int kNoAllocMaxT = 4, kNoAllocMaxE = 1024, kNoAllocMaxK = 16, kNoAllocMaxHI = 2048;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Driver calls reached through the runtime's entry-point table, so the
// library needs no link against libcuda (it loads on machines without a GPU).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Process-unique id of the current context (0 if there is none or the
// driver cannot tell).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa{}, qb{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || a == nullptr)
      return 0;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess || b == nullptr)
      return 0;
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct ScratchEntry {
  unsigned long long ctx_id;  // CUDA context the address belongs to (0 = none yet)
  void* ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

// Device address of the scratch array in the current device's current
// context. Host code may not use the symbol itself as a device pointer:
// cudaGetSymbolAddress gives the address, once per device, with that device
// current. The cached address is tied to the context it was taken in (its
// process-unique id): after cudaDeviceReset, or with another context
// current, the module is loaded anew and the address is looked up again.
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  unsigned long long id = current_context_id();
  if (id == 0 || g_scratch[dev].ctx_id != id || g_scratch[dev].ptr == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the primary context current if none was
    if (e != cudaSuccess) return e;
    if (id == 0) id = current_context_id();
    if (id == 0) return cudaErrorDeviceUninitialized;
    g_scratch[dev] = ScratchEntry{id, p};
  }
  *out = g_scratch[dev].ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_layer_decode_noalloc(const uint16_t* x, int32_t T, int32_t H, int32_t I, int32_t E,
                                               int32_t k, const float* w_router, const float* bias,
                                               int64_t bias_row_stride, const moe_expert* experts_dev,
                                               const moe_expert* shared_dev, int32_t* topk_idx, float* topk_w,
                                               float* logits_out, uint16_t* out, const moe_options* opts,
                                               void* stream) {
  const moe::CallRange range("moe_layer_decode_noalloc");
  if (T < 1 || H <= 0 || I <= 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T > kNoAllocMaxT || E > kNoAllocMaxE || k > kNoAllocMaxK || H > kNoAllocMaxHI || I > kNoAllocMaxHI)
    return MOE_ERR_UNSUPPORTED;
  if (!moe::decode_fused_eligible(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (bias_row_stride < 0 || (bias_row_stride > 0 && bias_row_stride < E)) return MOE_ERR_INVALID_ARG;
  if (!x || !w_router || !experts_dev || !topk_idx || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  const uintptr_t misalign = (reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_router) |
                              reinterpret_cast<uintptr_t>(out)) & 15u;
  if (misalign || (reinterpret_cast<uintptr_t>(experts_dev) & 7u)) return MOE_ERR_INVALID_ARG;

  const uint32_t flags = opts ? opts->flags : 0u;
  const float* gate = opts ? opts->shared_gate : nullptr;
  if ((flags & ~uint32_t(MOE_BIAS_SELECTION_ONLY)) || (reinterpret_cast<uintptr_t>(gate) & 15u))
    return MOE_ERR_INVALID_ARG;
  const size_t off_counters = 256;
  const size_t off_logits = moe::align256(off_counters + moe::kDecodeCounterBytes);
  const size_t off_logits_u = moe::align256(off_logits + 4u * size_t(T) * E);
  const size_t off_sgate = moe::align256(off_logits_u + 4u * size_t(T) * E);
  const size_t off_h = moe::align256(off_sgate + 4u * size_t(T));
  const size_t total = off_h + moe::decode_fused_ws_bytes(T, I);
  if (total > kNoAllocBytes) return MOE_ERR_UNSUPPORTED;

  void* base = nullptr;
  if (scratch_for_current_device(&base) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The previous call's status word and counters stay in the array: clear them.
  if (cudaMemsetAsync(base, 0, moe::kWsResetBytes, st) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = moe::launch_decode_fused(
      x, T, H, I, E, k, w_router, bias, bias_row_stride, experts_dev, shared_dev, topk_idx, topk_w, logits_out, out,
      moe::ws_at<float>(base, off_logits), moe::ws_at<float>(base, off_h), moe::ws_at<uint32_t>(base, off_counters),
      moe::ws_at<moe::WsHeader>(base, 0), moe::wait_cycles(), flags, gate, moe::ws_at<float>(base, off_logits_u),
      moe::ws_at<float>(base, off_sgate), opts ? opts->heat : nullptr, nullptr, nullptr, nullptr, nullptr, st);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
