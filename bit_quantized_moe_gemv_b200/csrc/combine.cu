// Combine: out[t] = sum_{j=0..k-1} w[t,j] * y_perm[inv_perm[t*k+j]] + shared(x_t),
// summed in j order in fp32 and rounded once to bf16 (nearest even).
//
// Each token uses its k routed experts plus the one shared expert: the telli.sh
// page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
// "稀疏架构创造了机会". The gate-weighted sum with an ungated shared expert is
// this library's reading of that sentence. A per-token weight on the shared
// expert (its sigmoid gate, when the caller asks for the gated variant) is
// applied here as well.
//
// Gather form (no atomics): one thread owns 8 consecutive outputs of a token
// and reads the k expert rows with 16-byte loads, so the result does not depend
// on scheduling.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// Eight consecutive values of row r of y (bf16 or fp32 rows) as fp32.
__device__ __forceinline__ void load8(const uint16_t* y, size_t off, float* v) {
  const uint4 q = *reinterpret_cast<const uint4*>(y + off);
  const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(u[i] << 16);
    v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8(const float* y, size_t off, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(y + off), b = *reinterpret_cast<const float4*>(y + off + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename YT>
__global__ void __launch_bounds__(256)
combine_kernel(const YT* __restrict__ y_perm, const int* __restrict__ inv_perm, const float* __restrict__ topk_w,
               int T, int H, int k, const float* __restrict__ shared_y, const float* __restrict__ shared_scale,
               uint16_t* __restrict__ out) {
  const int per_tok = H / 8;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (long long)T * per_tok) return;
  const int t = int(tid / per_tok), c = int(tid % per_tok);
  float acc[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.f;
  const long long nrows = (long long)T * k;
  for (int j = 0; j < k; ++j) {
    const int r = inv_perm[(long long)t * k + j];
    if (r < 0 || r >= nrows) continue;  // invalid expert id upstream (flagged there)
    const float w = topk_w[(long long)t * k + j];
    float v[8];
    load8(y_perm, (size_t)r * H + 8 * c, v);
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = fmaf(w, v[q], acc[q]);
  }
  if (shared_y) {
    const float4* s = reinterpret_cast<const float4*>(shared_y + (size_t)t * H + 8 * c);
    const float4 a = s[0], b = s[1];
    const float g = shared_scale ? shared_scale[t] : 1.f;
    acc[0] = fmaf(g, a.x, acc[0]); acc[1] = fmaf(g, a.y, acc[1]); acc[2] = fmaf(g, a.z, acc[2]);
    acc[3] = fmaf(g, a.w, acc[3]); acc[4] = fmaf(g, b.x, acc[4]); acc[5] = fmaf(g, b.y, acc[5]);
    acc[6] = fmaf(g, b.z, acc[6]); acc[7] = fmaf(g, b.w, acc[7]);
  }
  uint4 o;
  o.x = uint32_t(f32_to_bf16_rn(acc[0])) | (uint32_t(f32_to_bf16_rn(acc[1])) << 16);
  o.y = uint32_t(f32_to_bf16_rn(acc[2])) | (uint32_t(f32_to_bf16_rn(acc[3])) << 16);
  o.z = uint32_t(f32_to_bf16_rn(acc[4])) | (uint32_t(f32_to_bf16_rn(acc[5])) << 16);
  o.w = uint32_t(f32_to_bf16_rn(acc[6])) | (uint32_t(f32_to_bf16_rn(acc[7])) << 16);
  *reinterpret_cast<uint4*>(out + (size_t)t * H + 8 * c) = o;
}

cudaError_t launch_combine(const uint16_t* y_bf16, const float* y_f32, const int* inv_perm, const float* topk_w,
                           int T, int H, int k, const float* shared_y, const float* shared_scale, uint16_t* out,
                           cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const long long n = (long long)T * (H / 8);
  const unsigned grid = unsigned((n + 255) / 256);
  if (y_f32)
    combine_kernel<float><<<grid, 256, 0, st>>>(y_f32, inv_perm, topk_w, T, H, k, shared_y, shared_scale, out);
  else
    combine_kernel<uint16_t><<<grid, 256, 0, st>>>(y_bf16, inv_perm, topk_w, T, H, k, shared_y, shared_scale, out);
  count_launches(1);
  return cudaGetLastError();
}

// Sigmoid gate of the shared expert: scale[t] = 1 / (1 + exp(-(g . x_t))),
// one warp per token, fp32 dot product over the bf16 activations.
__global__ void __launch_bounds__(256)
shared_gate_kernel(const uint16_t* __restrict__ x, int T, int H, const float* __restrict__ g,
                   float* __restrict__ scale) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;
  float a = 0.f;
  for (int i = lane; i < H; i += 32) a = fmaf(g[i], bf16_to_f32(x[(size_t)t * H + i]), a);
  a = warp_sum(a);
  if (lane == 0) scale[t] = 1.f / (1.f + expf(-a));
}

cudaError_t launch_shared_gate(const uint16_t* x, int T, int H, const float* gate_w, float* scale, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  shared_gate_kernel<<<unsigned((T + 7) / 8), 256, 0, st>>>(x, T, H, gate_w, scale);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace moe
