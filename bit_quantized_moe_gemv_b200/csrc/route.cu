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
// Warp-level top-k over one row of E <= 1024 logits. Lane l holds experts
// l, l+32, ... in registers. NaN logits are treated as -inf. gbias, when not
// NULL, is the bias row of this token and the gates are taken on the
// unbiased logits (logit - bias) of the picks: the bias moves the selection
// only.
__device__ void warp_topk_row(const float* row, int E, int k, int* idx_out, float* w_out, float* s_val,
                              int* s_idx, const float* gbias) {
  const int lane = threadIdx.x & 31;
  float v[32];
  const int nper = (E + 31) / 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    float t = -CUDART_INF_F;
    if (i < nper && e < E) {
      t = __ldcg(row + e);
      if (t != t) t = -CUDART_INF_F;
    }
    v[i] = t;
  }
  uint32_t avail = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (i < nper && lane + 32 * i < E) avail |= 1u << i;

  for (int j = 0; j < k; ++j) {
    // Local best among available: larger value, ties to the lower index
    // (i ascending means index ascending, so a strict '>' keeps the first).
    float bv = -CUDART_INF_F;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((avail >> i) & 1u) {
        const int e = lane + 32 * i;
        if (be == 0x7fffffff || v[i] > bv) {
          bv = v[i];
          be = e;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const bool better = (oe != 0x7fffffff) && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be));
      if (better) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) avail &= ~(1u << (be >> 5));
    if (lane == 0) {
      s_val[j] = bv;
      s_idx[j] = be;
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
