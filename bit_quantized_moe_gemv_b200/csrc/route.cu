// Router: logits = x W_r^T + b (fp32), then softmax / top-k / renormalised gates.
//
// The telli.sh page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型",
// section "稀疏架构创造了机会", fixes the selection size (10 of 512 routed experts
// per token per layer). The softmax + renormalised top-k reading, and the
// (logit desc, index asc) order of the picks, are this library's reading of it.
//
// Decode (T <= 8): a GEMV over the fp32 router (4 MiB at E=512, H=2048) spread
// over many CTAs; the last CTA to finish (atomic ticket, no spinning) runs the
// top-k, so the step costs one launch.
// Prefill: a tiled fp32 GEMM writes the logits, then one warp per token runs
// the top-k.
#include <cuda_fp16.h>
#include <math_constants.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// ---------------------------------------------------------------- top-k
// Order-preserving 32-bit key of a float (NaN as -inf): a larger key is a
// larger value; 0 is never the key of a value.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) f = -CUDART_INF_F;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// Warp-level top-k over one row of E <= 32 NPER logits. Lane l holds the
// keys of experts l, l+32, ... in registers (0 = no expert or already
// picked). Each round takes every lane's best (a strict '>' keeps the lower
// index among equal keys), the largest key by a warp reduction and, among
// the lanes holding it, the lowest expert index by a second one; the
// winning lane clears that key. gbias, when not NULL, is the bias row of
// this token and the gates are taken on the unbiased logits (logit - bias)
// of the picks: the bias moves the selection only.
template <int NPER>
__device__ void warp_topk_row_n(const float* row, int E, int k, int* idx_out, float* w_out, float* s_val,
                                int* s_idx, const float* gbias) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NPER];
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? order_key(__ldcg(row + e)) : 0u;
  }
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < NPER; ++i)
      if (key[i] > bk) {
        bk = key[i];
        bi = i;
      }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t mine = bk == wk ? uint32_t(lane + 32 * bi) : 0xffffffffu;
    const uint32_t we = __reduce_min_sync(0xffffffffu, mine);
    if (mine == we) {
#pragma unroll
      for (int i = 0; i < NPER; ++i)
        if (i == bi) key[i] = 0u;
    }
    if (lane == 0) {
      s_val[j] = key_value(wk);
      s_idx[j] = int(we);
    }
  }
  __syncwarp();
  // Renormalised softmax over the picks: the full-softmax denominator cancels.
  if (gbias) {
    for (int j = lane; j < k; j += 32) s_val[j] -= gbias[s_idx[j]];
    __syncwarp();
  }
  float m = -CUDART_INF_F;
  for (int j = lane; j < k; j += 32) m = fmaxf(m, s_val[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float part = 0.f;
  for (int j = lane; j < k; j += 32) part += expf(s_val[j] - m);
  const float denom = warp_sum(part);
  for (int j = lane; j < k; j += 32) {
    idx_out[j] = s_idx[j];
    w_out[j] = expf(s_val[j] - m) / denom;
  }
  __syncwarp();
}
__device__ void warp_topk_row(const float* row, int E, int k, int* idx_out, float* w_out, float* s_val,
                              int* s_idx, const float* gbias) {
  if (E <= 512) warp_topk_row_n<16>(row, E, k, idx_out, w_out, s_val, s_idx, gbias);
  else warp_topk_row_n<32>(row, E, k, idx_out, w_out, s_val, s_idx, gbias);
}

// ---------------------------------------------------------------- decode GEMV
constexpr int kGemvWarps = 8;
constexpr int kGemvTmax = 8;

// One warp per expert row per iteration; x of all T tokens staged in smem as
// fp32. The last CTA to retire computes top-k for every token.
__global__ void __launch_bounds__(kGemvWarps * 32)
router_gemv_topk_kernel(const uint16_t* __restrict__ x, int T, int H, const float* __restrict__ W, int E,
                        const float* __restrict__ bias, long long bstride, int k, float* __restrict__ logits,
                        int* __restrict__ topk_idx, float* __restrict__ topk_w, WsHeader* hdr, int ticket_slot,
                        bool bias_selection_only) {
  extern __shared__ float smem[];
  float* xs = smem;  // [T][H]
  __shared__ float s_val[kGemvWarps][kMaxK];
  __shared__ int s_idx[kGemvWarps][kMaxK];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < T * H; i += blockDim.x) xs[i] = bf16_to_f32(x[i]);
  __syncthreads();

  for (int e = blockIdx.x * kGemvWarps + warp; e < E; e += gridDim.x * kGemvWarps) {
    const float4* wr = reinterpret_cast<const float4*>(W + size_t(e) * H);
    float acc[kGemvTmax];
#pragma unroll
    for (int t = 0; t < kGemvTmax; ++t) acc[t] = 0.f;
    for (int c = lane; c < H / 4; c += 32) {
      const float4 w4 = __ldg(wr + c);
#pragma unroll
      for (int t = 0; t < kGemvTmax; ++t) {
        if (t < T) {
          const float4 x4 = *reinterpret_cast<const float4*>(xs + t * H + 4 * c);
          acc[t] = fmaf(w4.x, x4.x, acc[t]);
          acc[t] = fmaf(w4.y, x4.y, acc[t]);
          acc[t] = fmaf(w4.z, x4.z, acc[t]);
          acc[t] = fmaf(w4.w, x4.w, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kGemvTmax; ++t) {
      if (t < T) {
        const float s = warp_sum(acc[t]);
        if (lane == 0) logits[size_t(t) * E + e] = s + (bias ? bias[t * bstride + e] : 0.f);
      }
    }
  }
  // Last-CTA top-k: no CTA waits on another.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&hdr->tickets[ticket_slot], 1u);
    s_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = warp; t < T; t += kGemvWarps)
    warp_topk_row(logits + size_t(t) * E, E, k, topk_idx + t * k, topk_w + t * k, s_val[warp], s_idx[warp],
                  bias_selection_only && bias ? bias + t * bstride : nullptr);
  if (threadIdx.x == 0) hdr->tickets[ticket_slot] = 0;
}

// ---------------------------------------------------------------- prefill GEMM
// logits[T,E] = x[T,H] W[E,H]^T + b. 64x64 CTA tile, 16-deep K slices,
// 256 threads with a 4x4 register tile each. fp32 FMA accumulation.
constexpr int kRB = 64, kRK = 16;

__global__ void __launch_bounds__(256)
router_gemm_kernel(const uint16_t* __restrict__ x, int T, int H, const float* __restrict__ W, int E,
                   const float* __restrict__ bias, long long bstride, float* __restrict__ logits) {
  __shared__ float xs[kRK][kRB + 4];
  __shared__ float ws[kRK][kRB + 4];
  const int t0 = blockIdx.y * kRB, e0 = blockIdx.x * kRB;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int kk = 0; kk < H; kk += kRK) {
    for (int i = threadIdx.x; i < kRB * kRK; i += 256) {
      const int r = i / kRK, c = i % kRK;
      const int t = t0 + r, e = e0 + r;
      xs[c][r] = t < T ? bf16_to_f32(x[size_t(t) * H + kk + c]) : 0.f;
      ws[c][r] = e < E ? W[size_t(e) * H + kk + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kRK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[c][ty * 4 + i];
        b[i] = ws[c][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) logits[size_t(t) * E + e] = acc[i][j] + (bias ? bias[t * bstride + e] : 0.f);
    }
  }
}

__global__ void __launch_bounds__(256)
topk_rows_kernel(const float* __restrict__ logits, int T, int E, int k, int* __restrict__ topk_idx,
                 float* __restrict__ topk_w, const float* __restrict__ gbias, long long gstride) {
  __shared__ float s_val[8][kMaxK];
  __shared__ int s_idx[8][kMaxK];
  const int warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  warp_topk_row(logits + size_t(t) * E, E, k, topk_idx + size_t(t) * k, topk_w + size_t(t) * k, s_val[warp],
                s_idx[warp], gbias ? gbias + t * gstride : nullptr);
}

// ---------------------------------------------------------------- launcher
cudaError_t launch_route(const uint16_t* x, int T, int H, const float* W, int E, const float* bias,
                         long long bstride, int k, int* topk_idx, float* topk_w, float* logits, void* tc_scratch,
                         WsHeader* hdr, cudaStream_t st, bool bias_selection_only) {
  if (T == 0) return cudaSuccess;
  if (T <= kGemvTmax) {
    const size_t smem = size_t(T) * H * sizeof(float);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(router_gemv_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem));
      if (e != cudaSuccess) return e;
    }
    const int grid = (E + kGemvWarps - 1) / kGemvWarps;
    router_gemv_topk_kernel<<<grid, kGemvWarps * 32, smem, st>>>(x, T, H, W, E, bias, bstride, k, logits, topk_idx,
                                                                 topk_w, hdr, kTicketRoute, bias_selection_only);
    count_launches(1);
    return cudaGetLastError();
  }
  if (tc_scratch && router_tc_eligible(T, H, E)) {
    cudaError_t e = launch_router_tc(x, T, H, W, E, bias, bstride, logits, tc_scratch, hdr, st);
    if (e != cudaSuccess) return e;
  } else {
    dim3 g((E + kRB - 1) / kRB, (T + kRB - 1) / kRB);
    router_gemm_kernel<<<g, 256, 0, st>>>(x, T, H, W, E, bias, bstride, logits);
    count_launches(1);
  }
  topk_rows_kernel<<<(T + 7) / 8, 256, 0, st>>>(logits, T, E, k, topk_idx, topk_w,
                                                bias_selection_only ? bias : nullptr, bstride);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
