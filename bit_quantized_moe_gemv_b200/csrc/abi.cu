// C ABI entry points: host-side argument checks, workspace carving and launch
// sequencing. No allocation, no host synchronisation (except moe_get_status).
#include <cuda_runtime.h>

#include <atomic>

#include "call_range.h"
#include "moe.h"
#include "moe_common.cuh"
#include "moe_internal.h"

using namespace moe;

namespace moe {
static std::atomic<uint64_t> g_launches{0};
static std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};
void count_launches(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }
long long wait_cycles() { return g_wait_cycles.load(std::memory_order_relaxed); }
}  // namespace moe

namespace {

constexpr int kDecodeMaxT = 4;  // larger batches take the tensor-core prefill path

bool shape_ok(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  if (T < 0 || H <= 0 || I <= 0 || E < 1 || E > kMaxE || k < 1 || k > E || k > kMaxK) return false;
  if (H % 64 || I % 64) return false;
  if (T * k > 0x7fffffffLL || T * H > (1LL << 40)) return false;
  return true;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

moe_status ws_check(void* ws, size_t ws_bytes, int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  if (ws == nullptr || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(T, H, I, E, k).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Router variants asked for by `opts` (NULL = none); unknown flags are refused.
bool read_opts(const moe_options* opts, uint32_t* flags, const float** gate) {
  *flags = opts ? opts->flags : 0u;
  *gate = opts ? opts->shared_gate : nullptr;
  if (*flags & ~uint32_t(MOE_BIAS_SELECTION_ONLY)) return false;
  return *gate == nullptr || aligned(*gate, 16);
}

}  // namespace

extern "C" {

size_t moe_workspace_size(int32_t T, int32_t H, int32_t I, int32_t E, int32_t k) {
  if (!shape_ok(T, H, I, E, k)) return 0;
  return ws_layout(T, H, I, E, k).total;
}

moe_status moe_route(const uint16_t* x, int32_t T, int32_t H, const float* w_router, int32_t E, const float* bias,
                     int64_t bias_row_stride, int32_t k, int32_t* topk_idx, float* topk_w, float* logits_out,
                     const moe_options* opts, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range("moe_route");
  uint32_t flags = 0;
  const float* gate = nullptr;
  if (!read_opts(opts, &flags, &gate)) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, H, 64, E, k)) return MOE_ERR_INVALID_ARG;
  if (bias_row_stride < 0 || (bias_row_stride > 0 && bias_row_stride < E)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_router, 16)) return MOE_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(T, H, 64, E, k);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  float* logits = logits_out ? logits_out : ws_at<float>(ws, L.logits);
  cudaError_t e = launch_route(x, T, H, w_router, E, bias, bias_row_stride, k, topk_idx, topk_w, logits,
                               ws_at<void>(ws, L.router), ws_at<WsHeader>(ws, 0), static_cast<cudaStream_t>(stream),
                               (flags & MOE_BIAS_SELECTION_ONLY) != 0);
  if (e == cudaSuccess && opts && opts->heat)
    e = launch_heat(topk_idx, (long long)T * k, E, opts->heat, static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

moe_status moe_dispatch(const int32_t* topk_idx, int32_t T, int32_t k, int32_t E, int32_t* counts, int32_t* offsets,
                        int32_t* perm_src, int32_t* inv_perm, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range("moe_dispatch");
  if (!shape_ok(T, 64, 64, E, k)) return MOE_ERR_INVALID_ARG;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !perm_src || !inv_perm)) return MOE_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(T, 64, 64, E, k);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(launch_dispatch(topk_idx, T, k, E, counts, offsets, perm_src, inv_perm, ws_at<int>(ws, L.hist),
                                     ws_at<WsHeader>(ws, 0), static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const uint16_t* x, int32_t T, int32_t H, int32_t I, int32_t k, int32_t E,
                          const int32_t* perm_src, const int32_t* offsets, const int32_t* counts,
                          const moe_expert* experts_dev, uint16_t* y_perm, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range("moe_expert_ffn");
  if (!shape_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !perm_src || !offsets || !counts || !experts_dev || !y_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y_perm, 16) || !aligned(experts_dev, 8)) return MOE_ERR_INVALID_ARG;
  moe_status s = ws_check(ws, ws_bytes, T, H, I, E, k);
  if (s != MOE_OK) return s;
  const WsLayout L = ws_layout(T, H, I, E, k);
  if (T > kDecodeMaxT && grouped_eligible(H, I, E, false))
    return cuda_status(launch_grouped_ffn(x, T, H, I, k, E, perm_src, offsets, counts, experts_dev, nullptr, nullptr,
                                          y_perm, nullptr, ws_at<void>(ws, L.gemm), ws_at<WsHeader>(ws, 0),
                                          static_cast<cudaStream_t>(stream)));
  // decode sizes: the fused decode kernel's expert phases on the given routing
  if (decode_fused_eligible(T, H, I, E, k))
    return cuda_status(launch_decode_fused(x, T, H, I, E, k, nullptr, nullptr, 0, experts_dev, nullptr, nullptr,
                                           nullptr, nullptr, nullptr, ws_at<float>(ws, L.logits),
                                           ws_at<float>(ws, L.dh), ws_at<uint32_t>(ws, L.dcnt),
                                           ws_at<WsHeader>(ws, 0), wait_cycles(), 0u, nullptr,
                                           ws_at<float>(ws, L.logits_u), ws_at<float>(ws, L.sgate), nullptr, perm_src,
                                           offsets, counts, y_perm, static_cast<cudaStream_t>(stream)));
  return cuda_status(launch_expert_ffn(x, T, H, I, k, E, perm_src, offsets, counts, experts_dev, false,
                                       ws_at<float>(ws, L.h), ws_at<int>(ws, L.active), y_perm, nullptr,
                                       ws_at<WsHeader>(ws, 0), static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const uint16_t* y_perm, const int32_t* inv_perm, const float* topk_w, int32_t T, int32_t H,
                       int32_t I, int32_t k, const uint16_t* x, const moe_expert* shared_dev, uint16_t* out,
                       const moe_options* opts, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range("moe_combine");
  uint32_t flags = 0;
  const float* gate = nullptr;
  if (!read_opts(opts, &flags, &gate)) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, H, I, k, k)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y_perm || !inv_perm || !topk_w || !out || (shared_dev && !x)) return MOE_ERR_INVALID_ARG;
  if (!aligned(y_perm, 16) || !aligned(out, 16) || (x && !aligned(x, 16))) return MOE_ERR_INVALID_ARG;
  moe_status s = ws_check(ws, ws_bytes, T, H, I, k, k);
  if (s != MOE_OK) return s;
  const WsLayout L = ws_layout(T, H, I, k, k);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* shared_y = nullptr;
  float* shared_scale = nullptr;
  if (shared_dev) {
    shared_y = ws_at<float>(ws, L.shared_y);
    cudaError_t e = cudaSuccess;
    if (gate) {
      shared_scale = ws_at<float>(ws, L.sgate);
      e = launch_shared_gate(x, T, H, gate, shared_scale, st);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (T > kDecodeMaxT && grouped_eligible(H, I, 0, true))
      e = launch_grouped_ffn(x, T, H, I, k, 0, nullptr, nullptr, nullptr, nullptr, shared_dev, nullptr, nullptr,
                             shared_y, ws_at<void>(ws, L.gemm), ws_at<WsHeader>(ws, 0), st);
    else
      e = launch_expert_ffn(x, T, H, I, k, 1, nullptr, nullptr, nullptr, shared_dev, true, ws_at<float>(ws, L.h),
                            nullptr, nullptr, shared_y, ws_at<WsHeader>(ws, 0), st);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  return cuda_status(launch_combine(y_perm, nullptr, inv_perm, topk_w, T, H, k, shared_y, shared_scale, out, st));
}

moe_status moe_layer(const uint16_t* x, int32_t T, int32_t H, int32_t I, int32_t E, int32_t k, const float* w_router,
                     const float* bias, int64_t bias_row_stride, const moe_expert* experts_dev,
                     const moe_expert* shared_dev, int32_t* topk_idx, float* topk_w, float* logits_out,
                     uint16_t* out, const moe_options* opts, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range("moe_layer");
  uint32_t flags = 0;
  const float* gate = nullptr;
  if (!read_opts(opts, &flags, &gate)) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, H, I, E, k)) return MOE_ERR_INVALID_ARG;
  if (bias_row_stride < 0 || (bias_row_stride > 0 && bias_row_stride < E)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !experts_dev || !topk_idx || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(out, 16) || !aligned(experts_dev, 8))
    return MOE_ERR_INVALID_ARG;
  moe_status s = ws_check(ws, ws_bytes, T, H, I, E, k);
  if (s != MOE_OK) return s;
  const WsLayout L = ws_layout(T, H, I, E, k);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WsHeader* hdr = ws_at<WsHeader>(ws, 0);
  if (decode_fused_eligible(T, H, I, E, k))
    return cuda_status(launch_decode_fused(x, T, H, I, E, k, w_router, bias, bias_row_stride, experts_dev, shared_dev,
                                           topk_idx, topk_w, logits_out, out, ws_at<float>(ws, L.logits),
                                           ws_at<float>(ws, L.dh), ws_at<uint32_t>(ws, L.dcnt), hdr,
                                           wait_cycles(), flags, gate, ws_at<float>(ws, L.logits_u),
                                           ws_at<float>(ws, L.sgate), opts ? opts->heat : nullptr, nullptr, nullptr,
                                           nullptr, nullptr, st));
  int* counts = ws_at<int>(ws, L.counts);
  int* offsets = ws_at<int>(ws, L.offsets);
  int* perm = ws_at<int>(ws, L.perm);
  int* inv = ws_at<int>(ws, L.inv);
  float* y_perm = ws_at<float>(ws, L.y_perm);  // fp32: out is rounded only once
  cudaError_t e = launch_route(x, T, H, w_router, E, bias, bias_row_stride, k, topk_idx, topk_w,
                               logits_out ? logits_out : ws_at<float>(ws, L.logits), ws_at<void>(ws, L.router),
                               hdr, st, (flags & MOE_BIAS_SELECTION_ONLY) != 0);
  if (e == cudaSuccess && opts && opts->heat) e = launch_heat(topk_idx, (long long)T * k, E, opts->heat, st);
  float* shared_scale = nullptr;
  if (e == cudaSuccess && shared_dev && gate) {
    shared_scale = ws_at<float>(ws, L.sgate);
    e = launch_shared_gate(x, T, H, gate, shared_scale, st);
  }
  if (e == cudaSuccess) e = launch_dispatch(topk_idx, T, k, E, counts, offsets, perm, inv, ws_at<int>(ws, L.hist), hdr, st);
  float* shared_y = nullptr;
  if (T > kDecodeMaxT && grouped_eligible(H, I, E, shared_dev != nullptr)) {
    if (shared_dev) shared_y = ws_at<float>(ws, L.shared_y);
    if (e == cudaSuccess)
      e = launch_grouped_ffn(x, T, H, I, k, E, perm, offsets, counts, experts_dev, shared_dev, y_perm, nullptr,
                             shared_y, ws_at<void>(ws, L.gemm), hdr, st);
    if (e == cudaSuccess) e = launch_combine(nullptr, y_perm, inv, topk_w, T, H, k, shared_y, shared_scale, out, st);
    return cuda_status(e);
  }
  if (e == cudaSuccess)
    e = launch_expert_ffn(x, T, H, I, k, E, perm, offsets, counts, experts_dev, false, ws_at<float>(ws, L.h),
                          ws_at<int>(ws, L.active), nullptr, y_perm, hdr, st);
  if (e == cudaSuccess && shared_dev) {
    shared_y = ws_at<float>(ws, L.shared_y);
    e = launch_expert_ffn(x, T, H, I, k, 1, nullptr, nullptr, nullptr, shared_dev, true,
                          ws_at<float>(ws, L.h) + size_t(T) * k * I, nullptr, nullptr, shared_y, hdr, st);
  }
  if (e == cudaSuccess) e = launch_combine(nullptr, y_perm, inv, topk_w, T, H, k, shared_y, shared_scale, out, st);
  return cuda_status(e);
}

moe_status moe_reset_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, kWsResetBytes, static_cast<cudaStream_t>(stream)));
}

moe_status moe_get_status(void* ws, void* stream, int32_t* device_status) {
  if (ws == nullptr || device_status == nullptr || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *device_status = v;
  return MOE_OK;
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int64_t moe_set_wait_cycles(int64_t cycles) {
  const long long v = cycles < 0 ? kDefaultWaitCycles : cycles;
  return g_wait_cycles.exchange(v, std::memory_order_relaxed);
}

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null pointer, misalignment or shape outside the limits)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or quantisation type";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than moe_workspace_size()";
    case MOE_ERR_CUDA: return "CUDA launch or copy failed";
    case MOE_ERR_DEVICE_FAULT: return "device-side check failed (expert id out of range or bad expert descriptor)";
    case MOE_ERR_TIMEOUT: return "bounded device wait expired";
    default: return "unknown status";
  }
}

}  // extern "C"
