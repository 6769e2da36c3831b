// Dispatch: per-expert histogram, exclusive prefix sum and a STABLE counting
// sort of the T*k (token, slot) pairs into expert-major order.
//
// The telli.sh page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型",
// section "GPU、RAM 和 SSD 各司其职", runs each expert over the tokens that picked
// it (batched at prefill); grouping the pairs by expert is what makes that a
// contiguous per-expert batch.
//
// Determinism: histograms are order-independent sums; ranks inside a block
// are computed warp by warp in index order (match_any + prefix over warps),
// and blocks own contiguous index ranges, so the permutation is identical on
// every run and equals a stable sort by expert id.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kDW = 8;  // warps per dispatch block

// Exclusive scan of a[0..n) in shared memory (n <= 1024) by a 256-thread block.
// Returns the total. Uses `tmp` (>= 8 ints of shared memory).
__device__ int block_exclusive_scan(int* a, int n, int* tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + 255) / 256;  // <= 4
  int loc[4];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = tid * per + i;
    loc[i] = (i < per && j < n) ? a[j] : 0;
    sum += loc[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < kDW; ++w) {
    if (w < warp) wbase += tmp[w];
    total += tmp[w];
  }
  int run = wbase + incl - sum;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = tid * per + i;
    if (i < per && j < n) a[j] = run;
    run += loc[i];
  }
  __syncthreads();
  return total;
}

__device__ __forceinline__ int load_id(const int* ids, long long p, int E, WsHeader* hdr, int* inv_perm) {
  const int e = ids[p];
  if (e < 0 || e >= E) {
    flag_error(hdr, MOE_ERR_DEVICE_FAULT, e);
    inv_perm[p] = -1;
    return -1;
  }
  return e;
}

__global__ void __launch_bounds__(kDW * 32)
dispatch_hist_kernel(const int* __restrict__ ids, long long n, int E, int* __restrict__ hist, WsHeader* hdr,
                     int* inv_perm) {
  __shared__ int h[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const long long chunk = (n + gridDim.x - 1) / gridDim.x;
  const long long lo = blockIdx.x * chunk, hi = min(n, lo + chunk);
  for (long long p = lo + threadIdx.x; p < hi; p += blockDim.x) {
    const int e = load_id(ids, p, E, hdr, inv_perm);
    if (e >= 0) atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[size_t(blockIdx.x) * E + e] = h[e];
}

// One block: per-expert running sums over the block rows -> counts, offsets,
// and per-(block, expert) global bases written back into hist.
__global__ void __launch_bounds__(256)
dispatch_scan_kernel(int nblocks, int E, int* __restrict__ hist, int* __restrict__ counts,
                     int* __restrict__ offsets) {
  __shared__ int c[kMaxE];
  __shared__ int tmp[kDW];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    int b = 0;
    for (; b + 8 <= nblocks; b += 8) {  // eight loads in flight, then the running sum
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = hist[size_t(b + i) * E + e];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        hist[size_t(b + i) * E + e] = run;
        run += v[i];
      }
    }
    for (; b < nblocks; ++b) {
      const int v = hist[size_t(b) * E + e];
      hist[size_t(b) * E + e] = run;
      run += v;
    }
    c[e] = run;
    counts[e] = run;
  }
  __syncthreads();
  const int total = block_exclusive_scan(c, E, tmp);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    offsets[e] = c[e];
    for (int b = 0; b < nblocks; ++b) hist[size_t(b) * E + e] += c[e];
  }
  if (threadIdx.x == 0) offsets[E] = total;
}

// Ranks this block's contiguous range warp by warp. With single = true the
// block is the only one: it also produces counts and offsets itself.
template <bool kSingle>
__global__ void __launch_bounds__(kDW * 32)
dispatch_scatter_kernel(const int* __restrict__ ids, long long n, int E, const int* __restrict__ hist,
                        int* __restrict__ counts, int* __restrict__ offsets, int* __restrict__ perm_src,
                        int* __restrict__ inv_perm, WsHeader* hdr) {
  __shared__ int wh[kDW][kMaxE];
  __shared__ int tot[kMaxE];
  __shared__ int tmp[kDW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kDW * E; i += blockDim.x) wh[i / E][i % E] = 0;
  __syncthreads();
  const long long chunk = (n + gridDim.x - 1) / gridDim.x;
  const long long lo = blockIdx.x * chunk, hi = min(n, lo + chunk);
  const long long sub = (hi - lo + kDW - 1) / kDW;
  const long long wlo = min(hi, lo + warp * sub), whi = min(hi, wlo + sub);
  // Pass 1: per-warp histogram of the warp's sub-range.
  for (long long p0 = wlo; p0 < whi; p0 += 32) {
    const long long p = p0 + lane;
    int e = -2;
    if (p < whi) {
      e = ids[p];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) wh[warp][e] += __popc(peers);
  }
  __syncthreads();
  // Per-expert bases: block base (global or in-block scan), then warps in order.
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int w = 0; w < kDW; ++w) s += wh[w][e];
    tot[e] = s;
  }
  __syncthreads();
  if (kSingle) {
    const int total = block_exclusive_scan(tot, E, tmp);  // tot[e] -> offset of e
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      offsets[e] = tot[e];
      int s = 0;
      for (int w = 0; w < kDW; ++w) s += wh[w][e];
      counts[e] = s;
    }
    if (threadIdx.x == 0) offsets[E] = total;
  } else {
    for (int e = threadIdx.x; e < E; e += blockDim.x) tot[e] = hist[size_t(blockIdx.x) * E + e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = tot[e];
    for (int w = 0; w < kDW; ++w) {
      const int v = wh[w][e];
      wh[w][e] = run;
      run += v;
    }
  }
  __syncthreads();
  // Pass 2: stable ranks; a warp's own cursor row is touched by that warp only.
  for (long long p0 = wlo; p0 < whi; p0 += 32) {
    const long long p = p0 + lane;
    int e = -2;
    if (p < whi) e = load_id(ids, p, E, hdr, inv_perm);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int pos = 0;
    if (e >= 0) pos = wh[warp][e] + __popc(peers & ((1u << lane) - 1u));
    __syncwarp();
    if (e >= 0) {
      perm_src[pos] = int(p);
      inv_perm[p] = pos;
      if (lane == __ffs(peers) - 1) wh[warp][e] += __popc(peers);
    }
    __syncwarp();
  }
}

int dispatch_blocks(long long n) {
  if (n <= 4096) return 1;
  long long b = (n + 2047) / 2048;
  return int(b > kDispatchMaxBlocks ? kDispatchMaxBlocks : b);
}

// Routing heat: heat[e] += number of picks of expert e (integer atomics, so
// the counts are exact and independent of order).
__global__ void __launch_bounds__(256) heat_kernel(const int* __restrict__ ids, long long n, int E,
                                                   uint32_t* __restrict__ heat) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(heat + e, 1u);
  }
}

cudaError_t launch_heat(const int* topk_idx, long long n, int E, uint32_t* heat, cudaStream_t st) {
  if (n == 0 || heat == nullptr) return cudaSuccess;
  const long long blocks = (n + 255) / 256;
  heat_kernel<<<unsigned(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(topk_idx, n, E, heat);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const int* topk_idx, int T, int k, int E, int* counts, int* offsets, int* perm_src,
                            int* inv_perm, int* hist, WsHeader* hdr, cudaStream_t st) {
  const long long n = (long long)T * k;
  const int B = dispatch_blocks(n);
  if (B == 1) {
    dispatch_scatter_kernel<true><<<1, kDW * 32, 0, st>>>(topk_idx, n, E, nullptr, counts, offsets, perm_src,
                                                          inv_perm, hdr);
    count_launches(1);
    return cudaGetLastError();
  }
  dispatch_hist_kernel<<<B, kDW * 32, 0, st>>>(topk_idx, n, E, hist, hdr, inv_perm);
  dispatch_scan_kernel<<<1, 256, 0, st>>>(B, E, hist, counts, offsets);
  dispatch_scatter_kernel<false><<<B, kDW * 32, 0, st>>>(topk_idx, n, E, hist, counts, offsets, perm_src, inv_perm,
                                                         hdr);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace moe
