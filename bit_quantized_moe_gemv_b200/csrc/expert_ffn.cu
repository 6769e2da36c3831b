// Dequant-fused SwiGLU experts over dispatched rows (general SIMT path).
//
// Each routed expert is an FFN over the tokens that picked it: the telli.sh
// page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
// "稀疏架构创造了机会". Its weights are block-quantised to 2-4 bits: the
// cycleuser.org page "本地部署Qwen3.8-Flash-Next模型的两条路线…", sections
// "硬件形态决定了各自的走法" and "精度和内存占用".
//
//   gate/up:  h[r, i] = silu(sum_k Wg[i,k] x[k]) * (sum_k Wu[i,k] x[k])
//   down:     y[r, n] = sum_i Wd[n,i] h[r, i]
//
// A work item is (expert, batch of up to kTB of its rows, block of output
// rows); a warp streams one weight row with 16-byte loads, dequantises in
// registers (fp32, exact) and reuses it for every token of the batch.
#include <cuda_fp16.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kTB = 8;        // tokens sharing one pass over a weight row
constexpr int kFW = 8;        // warps per CTA
constexpr int kRowsPerWarp = 4;
constexpr int kRB = kFW * kRowsPerWarp;  // weight rows per work item

// active[0] = number of non-empty experts, active[1] = total batches,
// active[2 .. 2+E) = their ids (ascending), active[2+E .. 2+2E+1) = batch prefix.
__global__ void __launch_bounds__(256) active_list_kernel(const int* __restrict__ counts, int E, int* active) {
  __shared__ int flag[kMaxE], nb[kMaxE];
  for (int e = threadIdx.x; e < kMaxE; e += blockDim.x) {
    const int c = e < E ? counts[e] : 0;
    flag[e] = c > 0;
    nb[e] = (c + kTB - 1) / kTB;
  }
  __syncthreads();
  // Scan flags and batch counts (E <= 1024, 256 threads x 4 elements).
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int lf[4], lb[4], sf = 0, sb = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lf[i] = flag[tid * 4 + i];
    lb[i] = nb[tid * 4 + i];
    sf += lf[i];
    sb += lb[i];
  }
  int pf = sf, pb = sb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, pf, o), b = __shfl_up_sync(0xffffffffu, pb, o);
    if (lane >= o) {
      pf += a;
      pb += b;
    }
  }
  __shared__ int wf[8], wb[8];
  if (lane == 31) {
    wf[warp] = pf;
    wb[warp] = pb;
  }
  __syncthreads();
  int bf = 0, bb = 0, tf = 0, tb = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) {
      bf += wf[w];
      bb += wb[w];
    }
    tf += wf[w];
    tb += wb[w];
  }
  int rf = bf + pf - sf, rb = bb + pb - sb;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid * 4 + i;
    if (lf[i]) {
      active[2 + rf] = e;
      active[2 + E + rf] = rb;
    }
    rf += lf[i];
    rb += lb[i];
  }
  if (tid == 0) {
    active[0] = tf;
    active[1] = tb;
    active[2 + E + tf] = tb;
  }
}

struct ItemMap {
  int expert;      // index into experts[]
  int row0, nrows; // dispatched rows [row0, row0 + nrows)
  int rb;          // block of weight rows
};

// Decode flattened item index -> (expert, batch rows, row block).
__device__ __forceinline__ ItemMap map_item(long long item, int nrb, bool identity, int T, const int* active, int E,
                                            const int* offsets, const int* counts) {
  ItemMap m;
  const long long gb = item / nrb;
  m.rb = int(item % nrb);
  if (identity) {
    m.expert = 0;
    m.row0 = int(gb) * kTB;
    m.nrows = min(kTB, T - m.row0);
    return m;
  }
  const int na = active[0];
  const int* pre = active + 2 + E;
  int lo = 0, hi = na - 1;  // last a with pre[a] <= gb
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= gb) lo = mid;
    else hi = mid - 1;
  }
  const int e = active[2 + lo];
  const int b = int(gb - pre[lo]);
  m.expert = e;
  m.row0 = offsets[e] + b * kTB;
  m.nrows = min(kTB, counts[e] - b * kTB);
  return m;
}

__device__ __forceinline__ int row_token(int r, bool identity, const int* perm_src, int k) {
  return identity ? r : perm_src[r] / k;
}

__global__ void __launch_bounds__(kFW * 32)
ffn_gate_up_kernel(const uint16_t* __restrict__ x, int T, int H, int I, int k, int E, const int* __restrict__ perm_src,
                   const int* __restrict__ offsets, const int* __restrict__ counts, const moe_expert* __restrict__ experts,
                   bool identity, const int* __restrict__ active, float* __restrict__ h_out, WsHeader* hdr) {
  extern __shared__ float xs[];  // [kTB][H]
  int cur_row0 = -1, cur_expert = -1;  // identical in every thread: no divergence at the barriers
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrb = I / kRB;
  const long long total = identity ? (long long)((T + kTB - 1) / kTB) * nrb : (long long)active[1] * nrb;
  const long long per = (total + gridDim.x - 1) / gridDim.x;
  const long long i0 = blockIdx.x * per, i1 = min(total, i0 + per);
  for (long long item = i0; item < i1; ++item) {
    const ItemMap m = map_item(item, nrb, identity, T, active, E, offsets, counts);
    const moe_expert ex = experts[m.expert];
    if (!expert_ok(ex, H, I)) {
      if (threadIdx.x == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 1000000 + m.expert);
      continue;
    }
    if (m.row0 != cur_row0 || m.expert != cur_expert) {
      __syncthreads();
      for (int i = threadIdx.x; i < kTB * H; i += blockDim.x) {
        const int t = i / H, c = i % H;
        xs[i] = t < m.nrows ? bf16_to_f32(x[size_t(row_token(m.row0 + t, identity, perm_src, k)) * H + c]) : 0.f;
      }
      __syncthreads();
      cur_row0 = m.row0;
      cur_expert = m.expert;
    }
    const int rowbytes = row_code_bytes(ex.gate.qtype, H);
    const int ne = chunk_elems(ex.gate.qtype);
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int i = m.rb * kRB + warp * kRowsPerWarp + rr;
      float ag[kTB], au[kTB];
#pragma unroll
      for (int t = 0; t < kTB; ++t) ag[t] = au[t] = 0.f;
      for (int c = lane; c < rowbytes / 16; c += 32) {
        const uint4 rg = __ldg(reinterpret_cast<const uint4*>(ex.gate.codes + size_t(i) * rowbytes) + c);
        const uint4 ru = __ldg(reinterpret_cast<const uint4*>(ex.up.codes + size_t(i) * rowbytes) + c);
        float wg[64], wu[64];
        dequant_chunk(ex.gate, i, c, rg, wg);
        dequant_chunk(ex.up, i, c, ru, wu);
        const int kb = c * ne;
#pragma unroll
        for (int t = 0; t < kTB; ++t) {
          if (t < m.nrows) {
            const float* xt = xs + t * H + kb;
            for (int q = 0; q < ne; ++q) {
              ag[t] = fmaf(wg[q], xt[q], ag[t]);
              au[t] = fmaf(wu[q], xt[q], au[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kTB; ++t) {
        if (t < m.nrows) {
          const float g = warp_sum(ag[t]), u = warp_sum(au[t]);
          if (lane == 0) h_out[size_t(m.row0 + t) * I + i] = silu_f32(g) * u;
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kFW * 32)
ffn_down_kernel(int T, int H, int I, int E, const int* __restrict__ offsets, const int* __restrict__ counts,
                const moe_expert* __restrict__ experts, bool identity, const int* __restrict__ active,
                const float* __restrict__ h_in, uint16_t* __restrict__ y_bf16, float* __restrict__ y_f32, WsHeader* hdr) {
  extern __shared__ float hs[];  // [kTB][I]
  int cur_row0 = -1, cur_expert = -1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrb = H / kRB;
  const long long total = identity ? (long long)((T + kTB - 1) / kTB) * nrb : (long long)active[1] * nrb;
  const long long per = (total + gridDim.x - 1) / gridDim.x;
  const long long i0 = blockIdx.x * per, i1 = min(total, i0 + per);
  for (long long item = i0; item < i1; ++item) {
    const ItemMap m = map_item(item, nrb, identity, T, active, E, offsets, counts);
    const moe_expert ex = experts[m.expert];
    if (!expert_ok(ex, H, I)) continue;  // flagged by the gate/up pass
    if (m.row0 != cur_row0 || m.expert != cur_expert) {
      __syncthreads();
      for (int i = threadIdx.x; i < kTB * I; i += blockDim.x) {
        const int t = i / I;
        hs[i] = t < m.nrows ? h_in[size_t(m.row0) * I + i] : 0.f;
      }
      __syncthreads();
      cur_row0 = m.row0;
      cur_expert = m.expert;
    }
    const int rowbytes = row_code_bytes(ex.down.qtype, I);
    const int ne = chunk_elems(ex.down.qtype);
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int n = m.rb * kRB + warp * kRowsPerWarp + rr;
      float acc[kTB];
#pragma unroll
      for (int t = 0; t < kTB; ++t) acc[t] = 0.f;
      for (int c = lane; c < rowbytes / 16; c += 32) {
        const uint4 rd = __ldg(reinterpret_cast<const uint4*>(ex.down.codes + size_t(n) * rowbytes) + c);
        float wd[64];
        dequant_chunk(ex.down, n, c, rd, wd);
        const int kb = c * ne;
#pragma unroll
        for (int t = 0; t < kTB; ++t) {
          if (t < m.nrows) {
            const float* ht = hs + t * I + kb;
            for (int q = 0; q < ne; ++q) acc[t] = fmaf(wd[q], ht[q], acc[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kTB; ++t) {
        if (t < m.nrows) {
          const float y = warp_sum(acc[t]);
          if (lane == 0) {
            const size_t o = size_t(m.row0 + t) * H + n;
            if (y_bf16) y_bf16[o] = f32_to_bf16_rn(y);
            else y_f32[o] = y;
          }
        }
      }
    }
  }
}

static int g_num_sms = 0;
static int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

cudaError_t launch_expert_ffn(const uint16_t* x, int T, int H, int I, int k, int E, const int* perm_src,
                              const int* offsets, const int* counts, const moe_expert* experts, bool identity,
                              float* h_ws, int* active_ws, uint16_t* y_bf16, float* y_f32, WsHeader* hdr,
                              cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (!identity) active_list_kernel<<<1, 256, 0, st>>>(counts, E, active_ws);
  const int grid = num_sms() * 4;
  const size_t smem_gu = size_t(kTB) * H * sizeof(float);
  const size_t smem_dn = size_t(kTB) * I * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(ffn_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_gu));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ffn_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_dn));
  if (e != cudaSuccess) return e;
  ffn_gate_up_kernel<<<grid, kFW * 32, smem_gu, st>>>(x, T, H, I, k, E, perm_src, offsets, counts, experts, identity,
                                                      active_ws, h_ws, hdr);
  ffn_down_kernel<<<grid, kFW * 32, smem_dn, st>>>(T, H, I, E, offsets, counts, experts, identity, active_ws, h_ws,
                                                   y_bf16, y_f32, hdr);
  count_launches(identity ? 2 : 3);
  return cudaGetLastError();
}

}  // namespace moe
