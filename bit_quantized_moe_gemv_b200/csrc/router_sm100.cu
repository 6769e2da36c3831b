// Prefill router on the tensor cores: logits[t, e] = sum_h x[t,h] W_r[e,h] + b,
// fp32-accurate.
//
// The router is a dense [T x H] x [H x E] contraction at prefill (the telli.sh
// page "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
// "稀疏架构创造了机会": 512 routed experts scored per token). W_r is fp32; it is
// split exactly into three bf16 pieces, w = w1 + w2 + w3 (8 significant bits
// each cover fp32's 24), and x is bf16 already, so every product x * w_i is
// exact in fp32 and the three accumulating bf16 MMAs per k-block give the
// fp32 dot product up to accumulation order.
//
// Both operands are first laid out as 16 KiB tiles of 128 rows x 64 bf16 in
// the 128-byte-swizzled K-major shared-memory image, so one 1-D bulk copy
// fills each operand of a stage. Tile (eb, tb): experts eb*128.. on the MMA's
// M side (TMEM lanes), tokens tb*128.. on N; the epilogue adds the bias and
// writes fp32 logits. Warp 0 copies, warp 1 issues MMAs, warps 2-5 drain TMEM.
#include <cuda_bf16.h>

#include "moe_common.cuh"
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace rtc {

constexpr int BM = 128, BN = 128, BK = 64;
constexpr int kTileBytes = 128 * 64 * 2;
constexpr int kStages = 3;
constexpr int kStageBytes = 4 * kTileBytes;  // three W pieces + one x tile
constexpr int kThreads = 6 * 32;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return uint32_t(row) * 128u + (uint32_t(chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float f) { return f32_to_bf16_rn(f); }

// W_r [E, H] fp32 -> three tiled bf16 arrays (each [E/128][H/64][16 KiB]).
__global__ void __launch_bounds__(256) split_w_kernel(const float* __restrict__ w, int E, int H,
                                                      uint8_t* __restrict__ w3) {
  const int KB = H / BK;
  const size_t piece = size_t(E / BM) * KB * kTileBytes;
  const long long n8 = (long long)E * H / 8;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const int e = int(i / (H / 8)), c = int(i % (H / 8));
    const float4 a = __ldg(reinterpret_cast<const float4*>(w + size_t(e) * H) + 2 * c);
    const float4 b = __ldg(reinterpret_cast<const float4*>(w + size_t(e) * H) + 2 * c + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint16_t p[3][8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint16_t h1 = bf16_rn_bits(v[q]);
      const float r1 = v[q] - __uint_as_float(uint32_t(h1) << 16);  // exact
      const uint16_t h2 = bf16_rn_bits(r1);
      const float r2 = r1 - __uint_as_float(uint32_t(h2) << 16);   // exact
      p[0][q] = h1;
      p[1][q] = h2;
      p[2][q] = bf16_rn_bits(r2);
    }
    const int eb = e / BM, row = e % BM, kb = c / 8, chunk = c % 8;
    const size_t off = (size_t(eb) * KB + kb) * kTileBytes + swz(row, chunk);
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      uint4 o;
      o.x = uint32_t(p[s][0]) | (uint32_t(p[s][1]) << 16);
      o.y = uint32_t(p[s][2]) | (uint32_t(p[s][3]) << 16);
      o.z = uint32_t(p[s][4]) | (uint32_t(p[s][5]) << 16);
      o.w = uint32_t(p[s][6]) | (uint32_t(p[s][7]) << 16);
      *reinterpret_cast<uint4*>(w3 + s * piece + off) = o;
    }
  }
}

// x [T, H] bf16 -> tiles [ceil(T/128)][H/64][16 KiB] (rows past T left as is).
__global__ void __launch_bounds__(256) tile_x_kernel(const uint16_t* __restrict__ x, int T, int H,
                                                     uint8_t* __restrict__ xt) {
  const int KB = H / BK;
  const long long n8 = (long long)T * H / 8;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const int t = int(i / (H / 8)), c = int(i % (H / 8));
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + size_t(t) * H) + c);
    const int tb = t / BN, row = t % BN, kb = c / 8, chunk = c % 8;
    *reinterpret_cast<uint4*>(xt + (size_t(tb) * KB + kb) * kTileBytes + swz(row, chunk)) = v;
  }
}

struct Args {
  const uint8_t* w3;  // three W pieces
  const uint8_t* xt;  // x tiles
  const float* bias;
  long long bstride;
  float* logits;      // [T][E]
  int T, H, E;
  WsHeader* hdr;
};

__global__ void __launch_bounds__(kThreads, 1) router_tc_kernel(Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], accf_bar[2], acce_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int EB = a.E / BM, TB = (a.T + BN - 1) / BN, KB = a.H / BK;
  const long long ntiles = (long long)EB * TB;
  const size_t piece = size_t(EB) * KB * kTileBytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(ptx::smem_addr(&full_bar[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_addr(&accf_bar[b]), 1);
      ptx::mbar_init(ptx::smem_addr(&acce_bar[b]), 4);
    }
    ptx::mbar_init(ptx::smem_addr(&drain_bar), 1);
    abort_sh = 0;
    ptx::mbar_init_fence();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&tmem_base_sh), 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_p = &abort_sh;
  auto fail = [&](int where) {
    flag_error(a.hdr, MOE_ERR_TIMEOUT, where);
    *abort_p = 1;
  };

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x) {
        const int eb = int(t % EB), tb = int(t / EB);
        const int nrows = min(BN, a.T - tb * BN);
        const uint32_t xbytes = uint32_t((nrows + 15) & ~15) * 128u;
        for (int kb = 0; kb < KB; ++kb) {
          if (!ptx::mbar_wait(ptx::smem_addr(&empty_bar[s]), ph ^ 1u, abort_p)) {
            fail(8000001);
            break;
          }
          uint8_t* st = smem + size_t(s) * kStageBytes;
          const uint32_t bar = ptx::smem_addr(&full_bar[s]);
          ptx::mbar_arrive_expect_tx(bar, 3u * kTileBytes + xbytes);
          const size_t wo = (size_t(eb) * KB + kb) * kTileBytes;
#pragma unroll
          for (int p = 0; p < 3; ++p)
            ptx::bulk_g2s(ptx::smem_addr(st + p * kTileBytes), a.w3 + p * piece + wo, kTileBytes, bar);
          ptx::bulk_g2s(ptx::smem_addr(st + 3 * kTileBytes), a.xt + (size_t(tb) * KB + kb) * kTileBytes, xbytes, bar);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int s = 0, it = 0;
      uint32_t ph = 0;
      for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x, ++it) {
        const int tb = int(t / EB);
        const int nrows = min(BN, a.T - tb * BN);
        const uint32_t idesc = ptx::idesc_bf16(BM, (nrows + 15) & ~15);
        const int buf = it & 1;
        if (!ptx::mbar_wait(ptx::smem_addr(&acce_bar[buf]), (uint32_t(it >> 1) & 1u) ^ 1u, abort_p)) {
          fail(8000002);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + uint32_t(buf * 128);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!ptx::mbar_wait(ptx::smem_addr(&full_bar[s]), ph, abort_p)) {
            fail(8000003);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t st = ptx::smem_addr(smem + size_t(s) * kStageBytes);
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t bdesc = ptx::smem_desc_k128(st + 3 * kTileBytes + 32 * ks);
#pragma unroll
            for (int p = 0; p < 3; ++p)
              ptx::mma_f16(d, ptx::smem_desc_k128(st + p * kTileBytes + 32 * ks), bdesc, idesc,
                           (kb | ks | p) != 0);
          }
          ptx::mma_commit(ptx::smem_addr(&empty_bar[s]));
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&accf_bar[buf]));
      }
      ptx::mma_commit(ptx::smem_addr(&drain_bar));
      ptx::mbar_wait(ptx::smem_addr(&drain_bar), 0, nullptr);
    }
  } else {
    const int q = warp & 3;
    int it = 0;
    for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x, ++it) {
      const int eb = int(t % EB), tb = int(t / EB);
      const int nrows = min(BN, a.T - tb * BN);
      const int buf = it & 1;
      if (!ptx::mbar_wait(ptx::smem_addr(&accf_bar[buf]), uint32_t(it >> 1) & 1u, abort_p)) {
        fail(8000004);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * 128);
      const int e = eb * BM + 32 * q + lane;
      for (int c0 = 0; c0 < nrows; c0 += 16) {
        uint32_t v[16];
        ptx::tmem_ld16(taddr + uint32_t(c0), v);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n < nrows) {
            const int tok = tb * BN + n;
            const float bv = a.bias ? a.bias[tok * a.bstride + e] : 0.f;
            a.logits[size_t(tok) * a.E + e] = __uint_as_float(v[j]) + bv;
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&acce_bar[buf]));
    }
  }
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
}

}  // namespace rtc

bool router_tc_eligible(int T, int H, int E) { return T > 4 && (E % 128) == 0 && (H % 64) == 0; }

size_t router_tc_ws_bytes(long long T, int H, int E) {
  return align256(3 * size_t(E) * H * 2) + align256(size_t((T + 127) / 128) * 128 * H * 2);
}

cudaError_t launch_router_tc(const uint16_t* x, int T, int H, const float* W, int E, const float* bias,
                             long long bstride, float* logits, void* scratch, WsHeader* hdr, cudaStream_t st) {
  using namespace rtc;
  uint8_t* w3 = static_cast<uint8_t*>(scratch);
  uint8_t* xt = w3 + align256(3 * size_t(E) * H * 2);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  split_w_kernel<<<sms * 4, 256, 0, st>>>(W, E, H, w3);
  tile_x_kernel<<<sms * 4, 256, 0, st>>>(x, T, H, xt);
  const size_t smem = size_t(kStages) * kStageBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const long long ntiles = (long long)(E / BM) * ((T + BN - 1) / BN);
  const int grid = int(ntiles < sms ? ntiles : sms);
  Args a{w3, xt, bias, bstride, logits, T, H, E, hdr};
  router_tc_kernel<<<grid, kThreads, smem, st>>>(a);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace moe
