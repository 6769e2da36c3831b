// Internal launcher declarations shared by the ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_common.cuh"

namespace moe {

// Host-side count of kernel launches (diagnostic).
void count_launches(int n);

enum TicketSlot { kTicketRoute = 0, kTicketDecodeRoute = 1, kTicketDecodeGateUp = 2 };

// tc_scratch: workspace for the tensor-core router (router_tc_ws_bytes), used
// for T > 4 when E is a multiple of 128.
// bias_selection_only: the bias picks the experts, the gates come from the
// unbiased logits.
cudaError_t launch_route(const uint16_t* x, int T, int H, const float* W, int E, const float* bias,
                         long long bstride, int k, int* topk_idx, float* topk_w, float* logits, void* tc_scratch,
                         WsHeader* hdr, cudaStream_t st, bool bias_selection_only);

bool router_tc_eligible(int T, int H, int E);
size_t router_tc_ws_bytes(long long T, int H, int E);
cudaError_t launch_router_tc(const uint16_t* x, int T, int H, const float* W, int E, const float* bias,
                             long long bstride, float* logits, void* scratch, WsHeader* hdr, cudaStream_t st);

// heat[e] += picks of expert e among the n ids (routing heat statistics).
cudaError_t launch_heat(const int* topk_idx, long long n, int E, uint32_t* heat, cudaStream_t st);

// Blocks the multi-block dispatch uses for n = T*k pairs (1 = single-CTA path).
int dispatch_blocks(long long n);

cudaError_t launch_dispatch(const int* topk_idx, int T, int k, int E, int* counts, int* offsets, int* perm_src,
                            int* inv_perm, int* hist, WsHeader* hdr, cudaStream_t st);

// Routed experts over dispatched rows (identity = false) or one expert over
// the T tokens in order (identity = true; used for the shared expert).
// Writes y as bf16 rows (y_bf16 != nullptr) or fp32 rows (y_f32 != nullptr).
cudaError_t launch_expert_ffn(const uint16_t* x, int T, int H, int I, int k, int E, const int* perm_src,
                              const int* offsets, const int* counts, const moe_expert* experts, bool identity,
                              float* h_ws, int* active_ws, uint16_t* y_bf16, float* y_f32, WsHeader* hdr,
                              cudaStream_t st);

// Decode step (T <= 4) as one cooperative launch whose warps stream weights
// into registers; see decode_fused.cu. logits_ws: fp32 [T][E]; h_ws:
// decode_fused_ws_bytes; counters: kDecodeCounterBytes, zero at launch.
// wait_cycles bounds every wait of the launch.
bool decode_fused_eligible(int T, int H, int I, int E, int k);
// flags: MOE_BIAS_SELECTION_ONLY (then logits_u_ws [T][E] holds the unbiased
// logits); shared_gate: fp32 [H] or NULL (then sgate_ws [T] holds g . x).
// perm_src/offsets/counts/y_perm non-null: experts only (moe_expert_ffn):
// the dispatched experts run on every row and write bf16 y_perm rows;
// w_router, shared, topk_idx, topk_w, out are then unused (may be null).
cudaError_t launch_decode_fused(const uint16_t* x, int T, int H, int I, int E, int k, const float* w_router,
                                const float* bias, long long bstride, const moe_expert* experts,
                                const moe_expert* shared, int* topk_idx, float* topk_w, float* logits_out,
                                uint16_t* out, float* logits_ws, float* h_ws, uint32_t* counters, WsHeader* hdr,
                                long long wait_cycles, uint32_t flags, const float* shared_gate, float* logits_u_ws,
                                float* sgate_ws, uint32_t* heat, const int32_t* perm_src, const int32_t* offsets,
                                const int32_t* counts, uint16_t* y_perm, cudaStream_t st);
constexpr long long kDefaultWaitCycles = 2000000000LL;  // about 1 s at the B200's clock
// The budget (SM clock cycles) every bounded wait of the fused decode launch
// gets: kDefaultWaitCycles unless moe_set_wait_cycles changed it.
long long wait_cycles();

// Prefill experts on tcgen05 (expert_gemm_sm100.cu): plan, gather, gate/up
// GEMM with SwiGLU epilogue, down GEMM. Routed rows go to y_f32 or y_bf16
// (dispatched order), the shared expert's rows (if any) to ys_f32 [T][H].
bool grouped_eligible(int H, int I, int E, bool with_shared);
size_t grouped_ws_bytes(long long T, int H, int I, int k, int E, bool with_shared);
cudaError_t launch_grouped_ffn(const uint16_t* x, int T, int H, int I, int k, int E, const int* perm_src,
                               const int* offsets, const int* counts, const moe_expert* experts,
                               const moe_expert* shared, float* y_f32, uint16_t* y_bf16, float* ys_f32,
                               void* scratch, WsHeader* hdr, cudaStream_t st);

// Combine routed rows given as bf16 (y_bf16) or fp32 (y_f32; the other NULL);
// shared_scale (nullable, [T]) weighs the shared expert's rows per token.
cudaError_t launch_combine(const uint16_t* y_bf16, const float* y_f32, const int* inv_perm, const float* topk_w,
                           int T, int H, int k, const float* shared_y, const float* shared_scale, uint16_t* out,
                           cudaStream_t st);

// scale[t] = sigmoid(gate_w . x_t): the sigmoid-gated shared expert's weight.
cudaError_t launch_shared_gate(const uint16_t* x, int T, int H, const float* gate_w, float* scale, cudaStream_t st);

}  // namespace moe
