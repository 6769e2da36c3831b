/*
 * moe.h - C ABI of the B200 (sm_100a) routed mixture-of-experts FFN step.
 *
 * The step is one MoE block of a Qwen3.8-Flash-Next-style layer. The telli.sh
 * page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
 * "稀疏架构创造了机会", gives its structure: each of the 48 layers holds 512
 * routed experts, and every token activates 10 of them plus one shared expert.
 * The cycleuser.org page "本地部署Qwen3.8-Flash-Next模型的两条路线…", sections
 * "硬件形态决定了各自的走法" and "精度和内存占用", stores the experts in 2-4 bit
 * block-quantised form and keeps the router and the shared expert beside them.
 * The same telli.sh page, section "GPU、RAM 和 SSD 各司其职", separates the
 * batched prefill kernels from the latency-bound decode kernels.
 *
 * The pages fix no router function, activation or bit layout. This library
 * reads them as: softmax over all E biased logits, top-k in (logit desc,
 * index asc) order, gates renormalised over the k picks; SwiGLU experts
 * h = silu(W_g x) * (W_u x), y = W_d h; an ungated shared expert added with
 * weight 1; the packed formats below.
 *
 * Conventions (all entry points):
 *  - Tensor arguments are DEVICE pointers owned by the caller. The library
 *    allocates nothing in these calls; scratch comes from the caller-owned
 *    workspace `ws` of `ws_bytes` bytes (>= moe_workspace_size(...)),
 *    256-byte aligned, which must not be shared by calls that may overlap.
 *  - bf16 and fp16 values are passed as their uint16 bit patterns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are
 *    asynchronous on it and do not synchronise the host.
 *  - Every call returns a moe_status. Host-side argument checks return
 *    MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE_TOO_SMALL
 *    before anything is launched. Launch failures return MOE_ERR_CUDA.
 *    Problems only the device can see (an expert id >= E, a malformed expert
 *    descriptor, an expired bounded wait) set a status word inside the
 *    workspace instead; read it with moe_get_status. No C++ exception crosses
 *    this boundary and no kernel traps.
 *  - Shape limits: 1 <= k <= E <= 1024, k <= 64; H and I multiples of 64;
 *    T >= 0 (T = 0 is a no-op).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t moe_status;

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1         /* null pointer, bad shape, k > E, ... */
#define MOE_ERR_UNSUPPORTED 2         /* shape/qtype combination not built */
#define MOE_ERR_WORKSPACE_TOO_SMALL 3 /* ws_bytes < moe_workspace_size(...) */
#define MOE_ERR_CUDA 4                /* a CUDA launch or copy failed */
#define MOE_ERR_DEVICE_FAULT 5        /* device-side check failed (bad id, descriptor) */
#define MOE_ERR_TIMEOUT 6             /* a bounded device wait expired */

/*
 * Packed weight formats. W is [rows = N outputs, cols = K inputs]; codes are
 * row-major [N, K*bits/8]; quantisation groups run along K.
 *  MOE_Q_INT4_SYM_G32     element 2i in the low nibble of byte i, 2i+1 in the
 *                         high nibble; q = c - 8 in [-8, 7];
 *                         w = q * scale[n, k/32]; scales fp16 [N, K/32].
 *  MOE_Q_INT2_ASYM_G16    element 4i+m in bits 2m..2m+1 of byte i; c in 0..3;
 *                         w = c * scale[n, k/16] + min[n, k/16];
 *                         scales and mins fp16 [N, K/16].
 *  MOE_Q_INT8_PER_CHANNEL two's-complement q; w = q * scale[n]; scales fp16 [N].
 */
#define MOE_Q_INT4_SYM_G32 1
#define MOE_Q_INT2_ASYM_G16 2
#define MOE_Q_INT8_PER_CHANNEL 3

/* One packed matrix. `codes`, `scales` and `mins` must be 16-byte aligned;
 * `mins` is NULL except for MOE_Q_INT2_ASYM_G16. `group` is 32, 16 or 0
 * (per channel) and must agree with `qtype`. */
typedef struct moe_qmatrix {
  int32_t qtype;
  int32_t rows;
  int32_t cols;
  int32_t group;
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* mins;
} moe_qmatrix;

/* One SwiGLU expert: gate and up are [I, H], down is [H, I]. The qtype may
 * differ between experts (mixed per-expert precision). */
typedef struct moe_expert {
  moe_qmatrix gate;
  moe_qmatrix up;
  moe_qmatrix down;
} moe_expert;

/*
 * Router variants, off by default (opts = NULL in every call that takes
 * them). The pages name a router and a shared expert without their
 * functions (telli.sh page, section "稀疏架构创造了机会"); these two common
 * alternatives are readings of that gap:
 *  MOE_BIAS_SELECTION_ONLY  the bias picks the experts but the gates are the
 *                           softmax of the unbiased logits W_r x, renormalised
 *                           over the picks (logits_out keeps the biased ones);
 *  shared_gate              DEVICE fp32 [H] g, or NULL: the shared expert's
 *                           output is scaled by sigmoid(g . x) per token.
 * and one statistic:
 *  heat                     DEVICE uint32 [E], or NULL: routing heat, the
 *                           number of times each expert was picked; every
 *                           call that routes (moe_route, moe_layer, the
 *                           no-alloc call) adds its T k picks, so counts
 *                           accumulate over calls until the caller clears
 *                           them (the on-GPU counterpart of the heat ranking
 *                           the cycleuser.org page, section
 *                           "硬件形态决定了各自的走法", keeps for its expert
 *                           cache).
 * The struct itself is read on the host during the call.
 */
#define MOE_BIAS_SELECTION_ONLY 1u
typedef struct moe_options {
  uint32_t flags;
  const float* shared_gate;
  uint32_t* heat;
} moe_options;

/* Bytes of workspace the calls below need for a problem of this size (the
 * same value serves every call). Returns 0 for shapes outside the limits.
 * Call moe_reset_status once on a new workspace before its first use. */
size_t moe_workspace_size(int32_t T, int32_t H, int32_t I, int32_t E, int32_t k);

/*
 * moe_route - router, softmax, top-k and renormalised gates.
 * Passage: telli.sh page, section "稀疏架构创造了机会" (k of E routed experts
 * per token per layer); cycleuser.org page, section "硬件形态决定了各自的走法"
 * (the router is a resident dense component).
 *   x         bf16 [T, H] row-major
 *   w_router  fp32 [E, H] row-major
 *   bias      fp32 [E] (bias_row_stride = 0) or [T, E] (bias_row_stride = E
 *             or more); may be NULL (no bias)
 *   topk_idx  int32 [T, k] out: expert ids in (logit desc, index asc) order
 *   topk_w    fp32 [T, k] out: softmax probabilities of the picks, renormalised
 *             to sum to 1
 *   logits_out fp32 [T, E] out, optional (NULL = not exported): the biased
 *             fp32 logits the selection was made on
 *   opts      NULL or router variants (flags: MOE_BIAS_SELECTION_ONLY)
 * Logits are accumulated in fp32 (fp32-exact products on the tensor-core path
 * for large T); gates use expf.
 */
moe_status moe_route(const uint16_t* x, int32_t T, int32_t H, const float* w_router, int32_t E,
                     const float* bias, int64_t bias_row_stride, int32_t k, int32_t* topk_idx,
                     float* topk_w, float* logits_out, const moe_options* opts, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * moe_dispatch - per-expert histogram, prefix sum and stable permutation.
 * Passage: telli.sh page, section "GPU、RAM 和 SSD 各司其职" (experts execute one
 * by one over the tokens that picked them, batched at prefill).
 *   topk_idx  int32 [T, k] expert ids in [0, E)
 *   counts    int32 [E] out: number of (t, j) pairs per expert
 *   offsets   int32 [E+1] out: exclusive prefix sum of counts
 *   perm_src  int32 [T*k] out: perm_src[r] = t*k + j of the pair placed at
 *             row r; rows of one expert are contiguous and in ascending t*k+j
 *   inv_perm  int32 [T*k] out: inv_perm[t*k + j] = r (-1 for an invalid id)
 * Bit-exact and deterministic (no order-dependent atomics). An id outside
 * [0, E) is left out of every expert and flags MOE_ERR_DEVICE_FAULT.
 */
moe_status moe_dispatch(const int32_t* topk_idx, int32_t T, int32_t k, int32_t E, int32_t* counts,
                        int32_t* offsets, int32_t* perm_src, int32_t* inv_perm, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * moe_expert_ffn - dequant-fused SwiGLU experts over the dispatched rows.
 * Passage: telli.sh page, section "稀疏架构创造了机会" (routed experts);
 * cycleuser.org page, sections "硬件形态决定了各自的走法" and "精度和内存占用"
 * (low-bit block-quantised expert weights).
 *   x           bf16 [T, H]
 *   perm_src, offsets, counts  as written by moe_dispatch
 *   experts_dev DEVICE array of E moe_expert descriptors (device memory)
 *   y_perm      bf16 [T*k, H] out: row r = expert(r) applied to token
 *               perm_src[r] / k, accumulated in fp32, rounded once to bf16
 * Malformed descriptors of a used expert flag MOE_ERR_DEVICE_FAULT and
 * their rows are left unwritten. Decode sizes (1 <= T <= 4, H and I
 * multiples of 256 up to 2048) run as one cooperative launch of the decode
 * kernel's expert phases: there a malformed descriptor or counts that do not
 * fit T tokens leave every row unwritten, and an expired bounded wait leaves
 * MOE_ERR_TIMEOUT (reset the workspace with moe_reset_status after either).
 */
moe_status moe_expert_ffn(const uint16_t* x, int32_t T, int32_t H, int32_t I, int32_t k, int32_t E,
                          const int32_t* perm_src, const int32_t* offsets, const int32_t* counts,
                          const moe_expert* experts_dev, uint16_t* y_perm, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * moe_combine - gate-weighted sum of the routed expert rows plus the shared
 * expert.
 * Passage: telli.sh page, section "稀疏架构创造了机会" (10 routed experts plus one
 * shared expert per token); cycleuser.org page, section "硬件形态决定了各自的走法"
 * (the shared expert is resident beside the router).
 *   y_perm      bf16 [T*k, H] from moe_expert_ffn
 *   inv_perm    int32 [T*k] from moe_dispatch
 *   topk_w      fp32 [T, k] from moe_route
 *   x           bf16 [T, H] (input of the shared expert)
 *   shared_dev  DEVICE pointer to one moe_expert, or NULL for no shared expert
 *   out         bf16 [T, H] out: sum over j = 0..k-1 in order, in fp32, plus
 *               the shared expert's fp32 output, rounded once (nearest-even)
 *   opts        NULL or router variants (shared_gate: the shared expert's
 *               output is scaled by sigmoid(shared_gate . x) per token)
 */
moe_status moe_combine(const uint16_t* y_perm, const int32_t* inv_perm, const float* topk_w, int32_t T,
                       int32_t H, int32_t I, int32_t k, const uint16_t* x, const moe_expert* shared_dev,
                       uint16_t* out, const moe_options* opts, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_layer - the whole step (route, dispatch, experts, combine) in one call.
 * Same arguments and layouts as the four calls above; dispatch arrays and
 * intermediate rows live in the workspace and stay fp32, so `out` is rounded
 * once. `logits_out` (fp32 [T, E], NULL = not exported) receives the biased
 * fp32 logits the selection was made on, as in moe_route; `opts` selects the
 * router variants (both fields used). Decode batches (1 <= T <= 4, H and I <= 2048) run as ONE cooperative
 * persistent kernel whose grid barriers are bounded: if one expires the call
 * leaves MOE_ERR_TIMEOUT in the status word, and the workspace must be reset
 * with moe_reset_status before it is used again.
 */
moe_status moe_layer(const uint16_t* x, int32_t T, int32_t H, int32_t I, int32_t E, int32_t k,
                     const float* w_router, const float* bias, int64_t bias_row_stride,
                     const moe_expert* experts_dev, const moe_expert* shared_dev, int32_t* topk_idx,
                     float* topk_w, float* logits_out, uint16_t* out, const moe_options* opts, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * moe_layer_decode_noalloc - moe_layer's fused decode step for callers that
 * cannot allocate device memory.
 * No counterpart on the pages: this is an interface variant, not a step of
 * the method. Some hosts give a kernel library only its inputs and outputs
 * and own every device allocation themselves (for example a plugin slot in
 * another runtime, or a process held to a fixed device-memory budget); they
 * cannot provide the workspace moe_layer needs. This call takes the same
 * arguments as moe_layer without `ws`/`ws_bytes`, allocates nothing (no
 * cudaMalloc, no allocating library routine) and keeps its scratch in a
 * 2 MiB device array inside the library, which every GPU that loads the
 * library holds until the process exits.
 *   Limits: 1 <= T <= 4, E <= 1024, k <= 16, 256 <= H, I <= 2048 (multiples
 *   of 256), within the fused decode kernel's own shape limits (the shapes
 *   moe_layer runs as one launch), and a scratch of at most 2 MiB
 *   (256 B + the counters + 8 T E bytes of logits + 65 T I activations in
 *   fp32 and fp16: T I <= 4096 at E <= 1024); anything else returns
 *   MOE_ERR_UNSUPPORTED.
 *   The first call on a device looks up the array's device address (once per
 *   device and CUDA context, with that device current); make that first call
 *   before any stream capture.
 *   All calls share the array: calls that may overlap on the GPU (other
 *   streams, other host threads) race and must be serialised by the caller.
 *   Device-side checks still skip bad experts, but their status word lives
 *   in the shared array and is cleared by the next call; use moe_layer when
 *   that status is needed.
 */
moe_status moe_layer_decode_noalloc(const uint16_t* x, int32_t T, int32_t H, int32_t I, int32_t E, int32_t k,
                                    const float* w_router, const float* bias, int64_t bias_row_stride,
                                    const moe_expert* experts_dev, const moe_expert* shared_dev,
                                    int32_t* topk_idx, float* topk_w, float* logits_out, uint16_t* out,
                                    const moe_options* opts, void* stream);

/* Clear the device status word of a workspace (asynchronous on `stream`).
 * Call once on a fresh workspace before its first use. */
moe_status moe_reset_status(void* ws, void* stream);

/* Synchronise `stream`, then read the device status word of `ws` into
 * *device_status (MOE_OK if no device-side check has failed since the last
 * reset). */
moe_status moe_get_status(void* ws, void* stream, int32_t* device_status);

/* Diagnostic: number of kernels this library has launched in this process
 * (host-side count of launch calls; thread-safe). */
uint64_t moe_launch_count(void);

/* Diagnostic for testing the failure path: the budget, in SM clock cycles,
 * of every bounded device-side wait (grid counter, expert readiness) of the
 * fused decode launches made after this call (moe_layer with T <= 4 and
 * moe_layer_decode_noalloc). A wait that is not met when its budget runs out
 * gives up: the launch ends early, its outputs are undefined and the status
 * word reads MOE_ERR_TIMEOUT (reset the workspace before reusing it). With
 * 0, a wait not met at its first check gives up at once. A negative value
 * restores the default (2e9 cycles, about one second). Process-wide and
 * thread-safe; returns the previous budget. Not meant for production use. */
int64_t moe_set_wait_cycles(int64_t cycles);

/* Static, NUL-terminated description of a status code. */
const char* moe_status_string(moe_status st);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
