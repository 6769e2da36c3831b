// Fused decode step: route -> top-k -> dequant-fused SwiGLU experts -> combine
// in ONE persistent cooperative launch, for small batches (T <= 4).
//
// Decode reads every selected expert's weights once per step, so it is bound
// by memory bandwidth (the lcz.me forum thread "Halogen Flash Server配置與實測",
// comment section: decode reads a fixed set of weights each step, and its
// ceiling scales with bandwidth). The telli.sh page "Strata 与 Qwen3.8-Flash-Next：
// 如何在个人电脑上运行 180B 级模型", section "稀疏架构创造了机会", gives the step:
// 10 of 512 routed experts plus one shared expert per token; section
// "GPU、RAM 和 SSD 各司其职" keeps decode separate from batched prefill.
//
// One CTA per SM, three phases split by two grid barriers (bounded spins):
//  A  router GEMV rows split over all CTAs (partial sums per K-quarter), the
//     shared expert's gate/up rows (independent of routing), and an L2
//     prefetch of the shared expert's down rows.
//  B  every CTA rebuilds the logits from the partials and runs the top-k
//     itself (no extra barrier), then computes the routed gate/up rows of its
//     slice of the intermediate dimension, and prefetches into L2 the down
//     rows it will need in phase C.
//  C  each CTA owns a slice of the output rows: down projections of all
//     (token, slot) pairs and the shared expert from L2, then the gate-weighted
//     sum in slot order, rounded once to bf16.
//
// Dequantisation: a code c (0..15 or 0..3) is placed by one byte-permute in
// bits 16..23 of the float 0x3F000000, which reads as f = 0.5 + c/256 exactly;
// products f*x are exact for bf16 x, so per quantisation group
//   sum_k c_k x_k = 256 * (sum_k f_k x_k - 0.5 * X_g),   X_g = sum_k x_k,
// with packed fp32x2 FMAs doing two codes per instruction.
#include <cuda_fp16.h>
#include <math_constants.h>

#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace dec {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRQ = 4;  // router K-quarters
constexpr int kMaxT = 4;
constexpr long long kSpinCycles = 2000000000LL;  // ~1 s at B200 clocks

struct Params {
  const uint16_t* x;
  int T, H, I, E, k;
  const float* w_router;
  const float* bias;
  long long bstride;
  const moe_expert* experts;
  const moe_expert* shared;
  int* topk_idx;
  float* topk_w;
  uint16_t* out;
  float* partial;  // [T][E][kRQ]
  float* h;        // [T*k + T][I]: routed pairs, then the shared expert's rows
  WsHeader* hdr;
};

// ---------------------------------------------------------------- helpers
// Packed fp32x2 FMA (sm_100): two lanes of work per instruction.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Code byte b of `w` (a nibble or crumb already isolated in the low bits of
// each byte) -> 0.5 + c/256.
template <int B>
__device__ __forceinline__ float code_f(uint32_t w) {
  return __uint_as_float(__byte_perm(w, 0x3F000000u, 0x7044u | (B << 8)));
}

__device__ __forceinline__ void split_range(int n, int parts, int i, int& lo, int& hi) {
  lo = int((long long)n * i / parts);
  hi = int((long long)n * (i + 1) / parts);
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ---------------------------------------------------------------- dot engine
// One warp computes dot products of whole rows of a packed matrix with one
// activation vector kept in registers. Lane l owns chunks c = l + 32 j
// (j < CPL, c < CPR) of 16 bytes; its activations sit in registers in the
// byte-permute order of the codes.
template <int QT>
struct QT_;
template <>
struct QT_<MOE_Q_INT4_SYM_G32> {
  static constexpr int EPC = 32;  // elements per 16-byte chunk
  static constexpr int GPC = 1;   // quantisation groups per chunk
};
template <>
struct QT_<MOE_Q_INT2_ASYM_G16> {
  static constexpr int EPC = 64;
  static constexpr int GPC = 4;
};
template <>
struct QT_<MOE_Q_INT8_PER_CHANNEL> {
  static constexpr int EPC = 16;
  static constexpr int GPC = 1;
};

template <bool kGlobal>
__device__ __forceinline__ float4 ld4(const float* p) {
  if (kGlobal) return __ldcg(reinterpret_cast<const float4*>(p));
  return *reinterpret_cast<const float4*>(p);
}

template <int QT, int CPL>
struct XRegs {
  static constexpr int EPC = QT_<QT>::EPC, GPC = QT_<QT>::GPC;
  float v[CPL][EPC];   // permuted order
  float gsum[CPL][GPC];

  // Load the lane's chunks of x (length K, fp32; shared memory, or global
  // memory written by other CTAs when kGlobal).
  template <bool kGlobal = false>
  __device__ __forceinline__ void load(const float* xs, int CPR) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = lane + 32 * j;
      const bool ok = c < CPR;
      const float* src = xs + size_t(ok ? c : 0) * EPC;
#pragma unroll
      for (int g = 0; g < GPC; ++g) gsum[j][g] = 0.f;
      if (QT == MOE_Q_INT4_SYM_G32) {
        // word w holds elements 8w..8w+7; order: 0,2,4,6,1,3,5,7
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 a = ok ? ld4<kGlobal>(src + 8 * w) : make_float4(0, 0, 0, 0);
          const float4 b = ok ? ld4<kGlobal>(src + 8 * w + 4) : make_float4(0, 0, 0, 0);
          float* d = v[j] + 8 * w;
          d[0] = a.x; d[1] = a.z; d[2] = b.x; d[3] = b.z;
          d[4] = a.y; d[5] = a.w; d[6] = b.y; d[7] = b.w;
          gsum[j][0] += (a.x + a.y) + (a.z + a.w) + (b.x + b.y) + (b.z + b.w);
        }
      } else if (QT == MOE_Q_INT2_ASYM_G16) {
        // word w (one group of 16) holds elements 16w..16w+15; byte i has
        // elements 4i..4i+3 at bit pairs 0..3; order: m-major then byte
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float e[16];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 a = ok ? ld4<kGlobal>(src + 16 * w + 4 * q) : make_float4(0, 0, 0, 0);
            e[4 * q] = a.x; e[4 * q + 1] = a.y; e[4 * q + 2] = a.z; e[4 * q + 3] = a.w;
          }
          float s = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v[j][16 * w + 4 * m + i] = e[4 * i + m];
              s += e[4 * i + m];
            }
          gsum[j][w] = s;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 a = ok ? ld4<kGlobal>(src + 4 * q) : make_float4(0, 0, 0, 0);
          v[j][4 * q] = a.x; v[j][4 * q + 1] = a.y; v[j][4 * q + 2] = a.z; v[j][4 * q + 3] = a.w;
        }
      }
    }
  }
};

__device__ __forceinline__ void prefetch_l2(const void* base, size_t lo, size_t hi) {
  // L2 prefetch of [lo, hi) bytes from base; only whole 16-byte blocks inside
  // the range are touched.
  const uintptr_t a = (reinterpret_cast<uintptr_t>(base) + lo + 15) & ~uintptr_t(15);
  const uintptr_t b = (reinterpret_cast<uintptr_t>(base) + hi) & ~uintptr_t(15);
  if (b <= a) return;
  uint32_t left = uint32_t(b - a);
  uintptr_t p = a;
  while (left) {
    const uint32_t n = left > (1u << 20) ? (1u << 20) : left;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(n) : "memory");
    p += n;
    left -= n;
  }
}

// Bounded grid barrier. Returns false (on every thread of the CTA) if the
// wait expired or another CTA gave up; the status word then reads TIMEOUT.
__device__ bool grid_sync(WsHeader* hdr, uint32_t target) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    // release: the CTA's writes (ordered before this thread by the CTA
    // barrier above) become visible before the arrival is counted
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&hdr->bar_count) : "memory");
    const long long t0 = clock64();
    for (uint32_t it = 1; ld_acquire(&hdr->bar_count) < target; ++it) {
      if ((it & 31) == 0 && *reinterpret_cast<volatile int*>(&hdr->abort)) {
        ok = 0;
        break;
      }
      if (clock64() - t0 > kSpinCycles) {
        flag_error(hdr, MOE_ERR_TIMEOUT, int(target));
        atomicExch(&hdr->abort, 1);
        ok = 0;
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__host__ __device__ __forceinline__ int bits_of(int qt) {
  return qt == MOE_Q_INT4_SYM_G32 ? 4 : qt == MOE_Q_INT2_ASYM_G16 ? 2 : 8;
}
// Chunks (16 bytes of codes) per row of K inputs.
__host__ __device__ __forceinline__ int chunks_per_row(int qt, int K) { return K * bits_of(qt) / 128; }
__host__ __device__ __forceinline__ int scale_row_bytes(int qt, int K) {
  return qt == MOE_Q_INT4_SYM_G32 ? K / 16 : qt == MOE_Q_INT2_ASYM_G16 ? K / 8 : 2;
}

// ---------------------------------------------------------------- lane-private staging ring
// Each lane copies (cp.async, 16/8/4 bytes) exactly the chunks of the rows it
// will itself consume into its own slots of shared memory, so no cross-lane
// synchronisation is needed: cp.async.wait_group is the only wait. A warp
// keeps kSlots batches in flight; one batch is at most 8 chunks of codes per
// lane (4 KiB per warp) plus their scales and mins.
constexpr int kSlots = 3;
constexpr int kSlotCodeBytes = 4096;  // 8 items x 32 lanes x 16 B
constexpr int kSlotAuxBytes = 2048;   // 8 aux words x 32 lanes x 8 B
constexpr int kSlotBytes = kSlotCodeBytes + kSlotAuxBytes;

__device__ __forceinline__ void cp_async16(uint8_t* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async8(uint8_t* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint8_t* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint8_t* code_item(uint8_t* slot, int item, int lane) {
  return slot + (item * 32 + lane) * 16;
}
__device__ __forceinline__ uint8_t* aux_word(uint8_t* slot, int a, int lane) {
  return slot + kSlotCodeBytes + (a * 32 + lane) * 8;
}

// Rows per batch for a qtype, chunks per lane and matrices per row (gate+up
// = 2, down = 1): at most 8 code items per lane, int2 at most 4 (its aux
// holds 8 scales and 8 mins per item).
__host__ __device__ constexpr int batch_rows(int qt, int cpl, int m) {
  return qt == MOE_Q_INT2_ASYM_G16 ? (4 / (m * cpl) > 0 ? 4 / (m * cpl) : 1) : (8 / (m * cpl) > 0 ? 8 / (m * cpl) : 1);
}

// A batch: rows [row0, row0 + nrow) of M matrices (W0, W1) sharing a qtype.
struct Batch {
  const moe_qmatrix* W0;
  const moe_qmatrix* W1;
  int qt;
  int row0, nrow;
  int dest;  // phase-specific destination (pair index)
};

template <int QT, int CPL, int M>
__device__ __forceinline__ void issue_batch_t(uint8_t* slot, const Batch& b, int K) {
  constexpr int R = batch_rows(QT, CPL, M);
  const int lane = threadIdx.x & 31;
  const int CPR = chunks_per_row(QT, K);
#pragma unroll 1
  for (int r = 0; r < R; ++r) {
    if (r >= b.nrow) continue;
    const int row = b.row0 + r;
#pragma unroll 1
    for (int m = 0; m < M; ++m) {
      const moe_qmatrix& W = m == 0 ? *b.W0 : *b.W1;
      const uint8_t* sc = reinterpret_cast<const uint8_t*>(W.scales);
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = lane + 32 * j;
        if (c >= CPR) continue;
        const int item = (r * M + m) * CPL + j;
        cp_async16(code_item(slot, item, lane), W.codes + (size_t(row) * CPR + c) * 16);
        if (QT == MOE_Q_INT4_SYM_G32) {
          cp_async4(aux_word(slot, item, lane), sc + size_t(row) * (K / 16) + 4 * (c >> 1));
        } else if (QT == MOE_Q_INT2_ASYM_G16) {
          cp_async8(aux_word(slot, 2 * item, lane), sc + (size_t(row) * (K / 16) + 4 * c) * 2);
          cp_async8(aux_word(slot, 2 * item + 1, lane),
                    reinterpret_cast<const uint8_t*>(W.mins) + (size_t(row) * (K / 16) + 4 * c) * 2);
        }
      }
      if (QT == MOE_Q_INT8_PER_CHANNEL) cp_async4(aux_word(slot, r * M + m, lane), sc + 4 * size_t(row >> 1));
    }
  }
}

// int8 activations in natural order read straight from shared memory (used
// where keeping them in registers would exhaust the register file).
template <int CPL>
struct XPtr {
  const float* v[CPL];
  float gsum[CPL][1];
  __device__ __forceinline__ void load(const float* xs, int CPR) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = lane + 32 * j;
      v[j] = xs + size_t(c < CPR ? c : 0) * 16;
      gsum[j][0] = 0.f;
    }
  }
};

// Partial dot products (this lane's chunks) of the batch's R x M rows with x.
// The partial of item (r, m) goes to red[(r M + m) * 32 + lane] (this warp's
// shared scratch); the item loop is kept rolled so the executed code stays
// small (this kernel is latency-bound and runs each code path once per step).
template <int QT, int CPL, int M, class X>
__device__ __forceinline__ void compute_batch_t(uint8_t* slot, const Batch& b, int K, const X& x, float* red) {
  constexpr int R = batch_rows(QT, CPL, M);
  // two independent items per iteration: the gate and up rows of one row
  // index (M = 2), or two consecutive rows (M = 1)
  constexpr int U = (M == 2 || R == 1) ? 1 : 2;
  const int lane = threadIdx.x & 31;
  const int CPR = chunks_per_row(QT, K);
#pragma unroll 1
  for (int r0i = 0; r0i < R; r0i += U) {
#pragma unroll
    for (int it = 0; it < U * M; ++it) {
      const int r = r0i + it / M, m = it % M;
      float acc = 0.f;
      if (r < b.nrow) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          const int c = lane + 32 * j;
          if (c >= CPR) continue;
          const int item = (r * M + m) * CPL + j;
          const uint4 raw = *reinterpret_cast<const uint4*>(code_item(slot, item, lane));
          const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
          if (QT == MOE_Q_INT4_SYM_G32) {
            // one accumulator per 32-bit word: four independent FMA chains
            float2 a4[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t lo = wd[w] & 0x0F0F0F0Fu, hi = (wd[w] >> 4) & 0x0F0F0F0Fu;
              const float* xv = x.v[j] + 8 * w;
              float2 t2 = __fmul2_rn(make_float2(code_f<0>(lo), code_f<1>(lo)), make_float2(xv[0], xv[1]));
              t2 = ffma2(make_float2(code_f<2>(lo), code_f<3>(lo)), make_float2(xv[2], xv[3]), t2);
              t2 = ffma2(make_float2(code_f<0>(hi), code_f<1>(hi)), make_float2(xv[4], xv[5]), t2);
              a4[w] = ffma2(make_float2(code_f<2>(hi), code_f<3>(hi)), make_float2(xv[6], xv[7]), t2);
            }
            const float2 s2 = make_float2((a4[0].x + a4[1].x) + (a4[2].x + a4[3].x),
                                          (a4[0].y + a4[1].y) + (a4[2].y + a4[3].y));
            const uint32_t sw = *reinterpret_cast<const uint32_t*>(aux_word(slot, item, lane));
            const float s = f16_to_f32(uint16_t((c & 1) ? (sw >> 16) : (sw & 0xffffu)));
            // sum (c - 8) x = 256 S - 136 X
            acc = fmaf(s, fmaf(256.f, s2.x + s2.y, -136.f * x.gsum[j][0]), acc);
          } else if (QT == MOE_Q_INT2_ASYM_G16) {
            const uint2 scw = *reinterpret_cast<const uint2*>(aux_word(slot, 2 * item, lane));
            const uint2 mnw = *reinterpret_cast<const uint2*>(aux_word(slot, 2 * item + 1, lane));
            const uint32_t sv[4] = {scw.x & 0xffffu, scw.x >> 16, scw.y & 0xffffu, scw.y >> 16};
            const uint32_t mv[4] = {mnw.x & 0xffffu, mnw.x >> 16, mnw.y & 0xffffu, mnw.y >> 16};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t b0 = wd[w] & 0x03030303u, b1 = (wd[w] >> 2) & 0x03030303u;
              const uint32_t b2 = (wd[w] >> 4) & 0x03030303u, b3 = (wd[w] >> 6) & 0x03030303u;
              const float* xv = x.v[j] + 16 * w;
              float2 s2 = make_float2(0.f, 0.f);
              s2 = ffma2(make_float2(code_f<0>(b0), code_f<1>(b0)), make_float2(xv[0], xv[1]), s2);
              s2 = ffma2(make_float2(code_f<2>(b0), code_f<3>(b0)), make_float2(xv[2], xv[3]), s2);
              s2 = ffma2(make_float2(code_f<0>(b1), code_f<1>(b1)), make_float2(xv[4], xv[5]), s2);
              s2 = ffma2(make_float2(code_f<2>(b1), code_f<3>(b1)), make_float2(xv[6], xv[7]), s2);
              s2 = ffma2(make_float2(code_f<0>(b2), code_f<1>(b2)), make_float2(xv[8], xv[9]), s2);
              s2 = ffma2(make_float2(code_f<2>(b2), code_f<3>(b2)), make_float2(xv[10], xv[11]), s2);
              s2 = ffma2(make_float2(code_f<0>(b3), code_f<1>(b3)), make_float2(xv[12], xv[13]), s2);
              s2 = ffma2(make_float2(code_f<2>(b3), code_f<3>(b3)), make_float2(xv[14], xv[15]), s2);
              const float s = f16_to_f32(uint16_t(sv[w])), mn = f16_to_f32(uint16_t(mv[w]));
              // sum (c s + m) x = 256 s S + (m - 128 s) X
              acc = fmaf(256.f * s, s2.x + s2.y, fmaf(mn - 128.f * s, x.gsum[j][w], acc));
            }
          } else {
            float2 a4[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t u = wd[w] ^ 0x80808080u;  // q + 128 in each byte
              const float* xv = x.v[j] + 4 * w;
              float q[4];
#pragma unroll
              for (int bb = 0; bb < 4; ++bb)
                q[bb] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u | bb)) - 8388736.0f;  // - (2^23+128)
              a4[w] = ffma2(make_float2(q[2], q[3]), make_float2(xv[2], xv[3]),
                            __fmul2_rn(make_float2(q[0], q[1]), make_float2(xv[0], xv[1])));
            }
            acc += ((a4[0].x + a4[1].x) + (a4[2].x + a4[3].x)) + ((a4[0].y + a4[1].y) + (a4[2].y + a4[3].y));
          }
        }
        if (QT == MOE_Q_INT8_PER_CHANNEL) {
          const uint32_t sw = *reinterpret_cast<const uint32_t*>(aux_word(slot, r * M + m, lane));
          acc *= f16_to_f32(uint16_t(((b.row0 + r) & 1) ? (sw >> 16) : (sw & 0xffffu)));
        }
      }
      red[(r * M + m) * 32 + lane] = acc;
    }
  }
  __syncwarp();
}

// Butterfly reduce-scatter of V (power of two) per-lane partials: lane l ends
// with the warp-wide sum of value (l >> (5 - log2 V)). V-1 + log2(32/V)
// shuffles instead of 5 V.
template <int V>
__device__ __forceinline__ float reduce_scatter(float* v) {
  const int lane = threadIdx.x & 31;
  int w = 16;
#pragma unroll
  for (int cnt = V; cnt > 1; cnt >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < cnt / 2; ++i) {
      const float send = upper ? v[i] : v[i + cnt / 2];
      const float keep = upper ? v[i + cnt / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
    w >>= 1;
  }
  float r = v[0];
#pragma unroll
  for (; w >= 1; w >>= 1) r += __shfl_xor_sync(0xffffffffu, r, w);
  return r;
}

// Sum the 32 lane partials of each of V outputs held in red[V][32]: lane l
// ends with the total of output l >> (5 - log2 V). Fixed summation order.
template <int V>
__device__ __forceinline__ float reduce_smem(const float* red) {
  constexpr int G = 32 / V;  // lanes per output
  const int lane = threadIdx.x & 31;
  const int o = lane / G, sidx = lane % G;
  float acc = 0.f;
#pragma unroll 1
  for (int i = 0; i < V; ++i) acc += red[o * 32 + sidx * V + i];
#pragma unroll
  for (int w = G / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
  __syncwarp();
  return acc;
}

template <int V>
struct Log2;
template <>
struct Log2<1> { static constexpr int v = 0; };
template <>
struct Log2<2> { static constexpr int v = 1; };
template <>
struct Log2<4> { static constexpr int v = 2; };
template <>
struct Log2<8> { static constexpr int v = 3; };

// ---------------------------------------------------------------- job lists
// The descriptors a step uses are copied into shared memory once, with a
// per-pair table of rows per batch and a prefix over the pairs' batch counts,
// so mapping a batch index to its rows never touches global memory.
//
// Gate/up batches: pairs j in [0, npair) with descriptors desc[j], rows
// [r0, r0 + nr) of each, cut into batches of rpb[j] rows; pre[j] = first
// batch of pair j (pre[npair] = total).
struct GateUpJobs {
  const moe_expert* desc;
  const int* pre;
  const int* rpb;
  int npair, r0, nr, H;
  int dest0;  // h row block of pair 0
  __device__ int total() const { return pre[npair]; }
  __device__ Batch get(int b) const {
    int j = 0;
    while (j + 1 < npair && pre[j + 1] <= b) ++j;
    const int R = rpb[j], lb = b - pre[j];
    const moe_expert& e = desc[j];
    return Batch{&e.gate, &e.up, e.gate.qtype, r0 + lb * R, min(R, nr - lb * R), dest0 + j};
  }
};

// Down batches: pairs p in [0, npair) (routed picks, then the shared expert's
// T rows: desc index min(p, nrouted)), rows [n0, n0 + nn).
struct DownJobs {
  const moe_expert* desc;
  const int* pre;
  const int* rpb;
  int nrouted, npair, n0, nn, I;
  __device__ int total() const { return pre[npair]; }
  __device__ Batch get(int b) const {
    int p = 0;
    while (p + 1 < npair && pre[p + 1] <= b) ++p;
    const int R = rpb[p], lb = b - pre[p];
    const moe_qmatrix& m = desc[p < nrouted ? p : nrouted].down;
    return Batch{&m, nullptr, m.qtype, n0 + lb * R, min(R, nn - lb * R), p};
  }
};

__device__ __forceinline__ int gu_rows_per_batch(const moe_expert& e, int H) {
  const int qt = e.gate.qtype;
  return batch_rows(qt, (chunks_per_row(qt, H) + 31) / 32, 2);
}
__device__ __forceinline__ int dn_rows_per_batch(const moe_qmatrix& m, int I) {
  return batch_rows(m.qtype, (chunks_per_row(m.qtype, I) + 31) / 32, 1);
}

// Runtime qtype / chunks-per-lane dispatch of a batch issue. Unsupported
// combinations issue nothing (the caller checks support up front).
template <int M>
__device__ __forceinline__ void issue_any(uint8_t* slot, const Batch& b, int K) {
  if (b.nrow > 0) {
    const int cpl = (chunks_per_row(b.qt, K) + 31) / 32;
    if (b.qt == MOE_Q_INT4_SYM_G32) {
      if (cpl == 1) issue_batch_t<MOE_Q_INT4_SYM_G32, 1, M>(slot, b, K);
      else if (cpl == 2) issue_batch_t<MOE_Q_INT4_SYM_G32, 2, M>(slot, b, K);
    } else if (b.qt == MOE_Q_INT2_ASYM_G16) {
      if (cpl == 1) issue_batch_t<MOE_Q_INT2_ASYM_G16, 1, M>(slot, b, K);
    } else if (b.qt == MOE_Q_INT8_PER_CHANNEL) {
      if (cpl == 1) issue_batch_t<MOE_Q_INT8_PER_CHANNEL, 1, M>(slot, b, K);
      else if (cpl == 2) issue_batch_t<MOE_Q_INT8_PER_CHANNEL, 2, M>(slot, b, K);
      else if (cpl <= 4) issue_batch_t<MOE_Q_INT8_PER_CHANNEL, 4, M>(slot, b, K);
    }
  }
  cp_commit();  // one group per batch, empty or not
}

__device__ __forceinline__ bool qt_supported(int qt, int K) {
  const int cpl = (chunks_per_row(qt, K) + 31) / 32;
  if (qt == MOE_Q_INT4_SYM_G32) return cpl <= 2;
  if (qt == MOE_Q_INT2_ASYM_G16) return cpl <= 1;
  if (qt == MOE_Q_INT8_PER_CHANNEL) return cpl <= 4;
  return false;
}
// Down matrices (K = I) keep activations in registers: int8 up to 2 chunks per lane.
__device__ __forceinline__ bool qt_supported_down(int qt, int K) {
  const int cpl = (chunks_per_row(qt, K) + 31) / 32;
  return qt == MOE_Q_INT8_PER_CHANNEL ? cpl <= 2 : qt_supported(qt, K);
}

// Stream this warp's gate/up batches [b, b1) of one qtype through its ring:
// h[dest * I + row] = silu(W_g x) * (W_u x). xs: the token's activations
// (shared memory, fp32). Returns the first batch of a different qtype.
template <int QT, int CPL, class X = XRegs<QT, CPL>>
__device__ __noinline__ int gate_up_run(uint8_t* ring, float* red, const GateUpJobs& J, int b, int b0, int b1,
                                        const float* xs, float* h, int I) {
  constexpr int R = batch_rows(QT, CPL, 2), V = 2 * R, SH = 5 - Log2<V>::v;
  const int lane = threadIdx.x & 31;
  X x;
  x.load(xs, chunks_per_row(QT, J.H));
  for (; b < b1; ++b) {
    const Batch bt = J.get(b);
    if (bt.qt != QT) break;
    uint8_t* slot = ring + ((b - b0) % kSlots) * kSlotBytes;
    cp_wait<kSlots - 1>();
    compute_batch_t<QT, CPL, 2, X>(slot, bt, J.H, x, red);
    const float sum = reduce_smem<V>(red);
    const float u = __shfl_down_sync(0xffffffffu, sum, 32 / V);
    const int idx = lane >> SH;  // = 2 r + m
    if ((lane & ((32 / V) - 1)) == 0 && (idx & 1) == 0 && (idx >> 1) < bt.nrow)
      h[size_t(bt.dest) * I + bt.row0 + (idx >> 1)] = silu_f32(sum) * u;
    const int nb = b + kSlots;
    issue_any<2>(slot, nb < b1 ? J.get(nb) : Batch{nullptr, nullptr, 0, 0, 0, 0}, J.H);
  }
  return b;
}

__device__ __noinline__ void gate_up_stream(uint8_t* ring, float* red, const GateUpJobs& J, int b0, int b1,
                                            const float* xs, float* h, int I, bool primed) {
  if (!primed)
    for (int i = 0; i < kSlots; ++i)
      issue_any<2>(ring + i * kSlotBytes, b0 + i < b1 ? J.get(b0 + i) : Batch{nullptr, nullptr, 0, 0, 0, 0}, J.H);
  int b = b0;
  while (b < b1) {
    const int qt = J.get(b).qt;
    const int cpl = (chunks_per_row(qt, J.H) + 31) / 32;
    int nb = b1;
    if (qt == MOE_Q_INT4_SYM_G32 && cpl == 1) nb = gate_up_run<MOE_Q_INT4_SYM_G32, 1>(ring, red, J, b, b0, b1, xs, h, I);
    else if (qt == MOE_Q_INT4_SYM_G32 && cpl == 2) nb = gate_up_run<MOE_Q_INT4_SYM_G32, 2>(ring, red, J, b, b0, b1, xs, h, I);
    else if (qt == MOE_Q_INT2_ASYM_G16 && cpl == 1) nb = gate_up_run<MOE_Q_INT2_ASYM_G16, 1>(ring, red, J, b, b0, b1, xs, h, I);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 1) nb = gate_up_run<MOE_Q_INT8_PER_CHANNEL, 1>(ring, red, J, b, b0, b1, xs, h, I);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 2) nb = gate_up_run<MOE_Q_INT8_PER_CHANNEL, 2>(ring, red, J, b, b0, b1, xs, h, I);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl <= 4)
      nb = gate_up_run<MOE_Q_INT8_PER_CHANNEL, 4, XPtr<4>>(ring, red, J, b, b0, b1, xs, h, I);
    if (nb == b) {  // unsupported batch: consume its (empty) group and move on
      cp_wait<kSlots - 1>();
      const int nx = b + kSlots;
      issue_any<2>(ring + ((b - b0) % kSlots) * kSlotBytes, nx < b1 ? J.get(nx) : Batch{nullptr, nullptr, 0, 0, 0, 0},
                   J.H);
      nb = b + 1;
    }
    b = nb;
  }
  cp_wait<0>();
}

// Down batches [b, b1) of one qtype: ys[dest * nn + row - n0] = W_d h_dest.
template <int QT, int CPL>
__device__ __noinline__ int down_run(uint8_t* ring, float* red, const DownJobs& J, int b, int b0, int b1,
                                     const float* h, float* ys) {
  constexpr int R = batch_rows(QT, CPL, 1), V = R, SH = 5 - Log2<V>::v;
  const int lane = threadIdx.x & 31;
  XRegs<QT, CPL> x;
  int xp = -1;
  for (; b < b1; ++b) {
    const Batch bt = J.get(b);
    if (bt.qt != QT) break;
    if (bt.dest != xp) {
      x.template load<true>(h + size_t(bt.dest) * J.I, chunks_per_row(QT, J.I));
      xp = bt.dest;
    }
    uint8_t* slot = ring + ((b - b0) % kSlots) * kSlotBytes;
    cp_wait<kSlots - 1>();
    compute_batch_t<QT, CPL, 1, XRegs<QT, CPL>>(slot, bt, J.I, x, red);
    const float sum = reduce_smem<V>(red);
    const int r = lane >> SH;
    if ((lane & ((32 / V) - 1)) == 0 && r < bt.nrow) ys[size_t(bt.dest) * J.nn + (bt.row0 - J.n0) + r] = sum;
    const int nb = b + kSlots;
    issue_any<1>(slot, nb < b1 ? J.get(nb) : Batch{nullptr, nullptr, 0, 0, 0, 0}, J.I);
  }
  return b;
}

__device__ __noinline__ void down_stream(uint8_t* ring, float* red, const DownJobs& J, int b0, int b1, const float* h,
                                         float* ys) {
  for (int i = 0; i < kSlots; ++i)
    issue_any<1>(ring + i * kSlotBytes, b0 + i < b1 ? J.get(b0 + i) : Batch{nullptr, nullptr, 0, 0, 0, 0}, J.I);
  int b = b0;
  while (b < b1) {
    const int qt = J.get(b).qt;
    const int cpl = (chunks_per_row(qt, J.I) + 31) / 32;
    int nb = b1;
    if (qt == MOE_Q_INT4_SYM_G32 && cpl == 1) nb = down_run<MOE_Q_INT4_SYM_G32, 1>(ring, red, J, b, b0, b1, h, ys);
    else if (qt == MOE_Q_INT4_SYM_G32 && cpl == 2) nb = down_run<MOE_Q_INT4_SYM_G32, 2>(ring, red, J, b, b0, b1, h, ys);
    else if (qt == MOE_Q_INT2_ASYM_G16 && cpl == 1) nb = down_run<MOE_Q_INT2_ASYM_G16, 1>(ring, red, J, b, b0, b1, h, ys);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 1) nb = down_run<MOE_Q_INT8_PER_CHANNEL, 1>(ring, red, J, b, b0, b1, h, ys);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 2) nb = down_run<MOE_Q_INT8_PER_CHANNEL, 2>(ring, red, J, b, b0, b1, h, ys);
    if (nb == b) {
      cp_wait<kSlots - 1>();
      const int nx = b + kSlots;
      issue_any<1>(ring + ((b - b0) % kSlots) * kSlotBytes, nx < b1 ? J.get(nx) : Batch{nullptr, nullptr, 0, 0, 0, 0},
                   J.I);
      nb = b + 1;
    }
    b = nb;
  }
  cp_wait<0>();
}

// ---------------------------------------------------------------- top-k
__device__ __forceinline__ uint32_t f2key(float f) {
  if (f != f) f = -CUDART_INF_F;  // NaN loses to every number
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Warp selection of the best `k` of n (key, id) candidates, NPL per lane
// (candidate i at lane i % 32, slot i / 32): larger key first, ties to the
// lower id. Writes keys and ids of the picks in order.
template <int NPL>
__device__ void warp_select(const uint32_t* keys, const int* ids, int n, int k, uint32_t* out_key, int* out_id) {
  const int lane = threadIdx.x & 31;
  uint32_t kk[NPL];
  int id[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int c = lane + 32 * i;
    kk[i] = c < n ? keys[c] : 0u;
    id[i] = c < n ? ids[c] : 0x7fffffff;
  }
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u;
    int bi = 0x7fffffff, bs = -1;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (id[i] != 0x7fffffff && (bs < 0 || kk[i] > bk || (kk[i] == bk && id[i] < bi))) {
        bk = kk[i];
        bi = id[i];
        bs = i;
      }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bs >= 0 ? bk : 0u);
    const uint32_t wi = __reduce_min_sync(0xffffffffu, (bs >= 0 && bk == wk) ? uint32_t(bi) : 0xffffffffu);
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (i == bs && uint32_t(bi) == wi) id[i] = 0x7fffffff;
    if (lane == 0) {
      out_key[j] = wk;
      out_id[j] = int(wi);
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- kernel

struct Smem {
  // carved from dynamic shared memory
  uint8_t* ring;  // kWarps x kSlots x kSlotBytes
  float* xs;      // [T][H]
  float* lg;      // [T][E]
  uint32_t* ck;   // [T][kWarps][k] candidate keys
  int* ci;        // [T][kWarps][k] candidate ids
  float* ys;      // [npairs][nn_max]
  moe_expert* desc;  // [T k + 1]: the picks' descriptors, then the shared expert's
  int* gpre;      // [T][k + 1] gate/up batch prefix per token
  int* grpb;      // [T][k]     gate/up rows per batch
  int* dpre;      // [T k + T + 1] down batch prefix
  int* drpb;      // [T k + T]     down rows per batch
  int* spre;      // [2] shared gate/up prefix
  int* srpb;      // [1]
};

__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ int s_idx[kMaxT * kMaxK];
  __shared__ float s_w[kMaxT * kMaxK];
  __shared__ uint32_t s_key[kMaxT * kMaxK];
  __shared__ float s_red[kWarps][8 * 32];  // per-warp partials of one batch
  const int T = P.T, H = P.H, I = P.I, E = P.E, k = P.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  const bool has_shared = P.shared != nullptr;
  WsHeader* hdr = P.hdr;

  int n0, n1;
  split_range(H, G, b, n0, n1);
  const int nn = n1 - n0;
  const int nn_max = (H + G - 1) / G;
  Smem S;
  S.ring = smem;
  S.xs = reinterpret_cast<float*>(smem + size_t(kWarps) * kSlots * kSlotBytes);
  S.lg = S.xs + size_t(T) * H;
  S.ck = reinterpret_cast<uint32_t*>(S.lg + size_t(T) * E);
  S.ci = reinterpret_cast<int*>(S.ck + size_t(T) * kWarps * k);
  S.ys = reinterpret_cast<float*>(S.ci + size_t(T) * kWarps * k);
  {
    uintptr_t q = reinterpret_cast<uintptr_t>(S.ys + size_t(T * k + T) * nn_max);
    q = (q + 15) & ~uintptr_t(15);
    S.desc = reinterpret_cast<moe_expert*>(q);
    S.gpre = reinterpret_cast<int*>(S.desc + T * k + 1);
    S.grpb = S.gpre + T * (k + 1);
    S.dpre = S.grpb + T * k;
    S.drpb = S.dpre + T * k + T + 1;
    S.spre = S.drpb + T * k + T;
    S.srpb = S.spre + 2;
  }
  __shared__ int s_bad;
  uint8_t* ring = S.ring + size_t(warp) * kSlots * kSlotBytes;
  float* red = s_red[warp];

  // Warps are pinned to tokens (warp w serves token w % T) for gate/up, so the
  // activation registers are loaded once per phase.
  const int my_t = warp % T;
  const int grp = warp / T, ngrp = (kWarps - my_t + T - 1) / T;

  // ------------------------------------------------ phase A
  // 1) issue this warp's router loads (registers) and shared gate/up copies
  //    before waiting for anything.
  int u0, u1;
  split_range(E * kRQ, G, b, u0, u1);
  const int qlen = H / kRQ;          // floats per router quarter-row
  const int q4 = qlen / 128;         // float4 per lane per quarter-row (qlen multiple of 128)
  bool shared_ok = false;
  GateUpJobs SJ{};
  int sb0 = 0, sb1 = 0;
  // The shared expert's descriptor into shared memory; the routed table into
  // L2 (its rows are read right after the top-k).
  if (has_shared && threadIdx.x < int(sizeof(moe_expert) / 4))
    reinterpret_cast<uint32_t*>(S.desc + T * k)[threadIdx.x] = reinterpret_cast<const uint32_t*>(P.shared)[threadIdx.x];
  if (threadIdx.x == 32) {
    int e0, e1;
    split_range(E, G, b, e0, e1);
    prefetch_l2(P.experts, size_t(e0) * sizeof(moe_expert), size_t(e1) * sizeof(moe_expert));
  }
  // Router: this CTA's quarter-rows, two at a time per warp, loads first.
  float4 wv[2][4];
  int ucur = u0 + warp;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int u = ucur + s * kWarps;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (u < u1 && c < q4) {
        const float4* wr = reinterpret_cast<const float4*>(P.w_router + size_t(u / kRQ) * H + (u % kRQ) * qlen);
        wv[s][c] = __ldg(wr + lane + 32 * c);
      }
    }
  }
  for (int i = threadIdx.x; i < T * H; i += kThreads) S.xs[i] = bf16_to_f32(P.x[i]);
  __syncthreads();
  if (has_shared) {
    const moe_expert& sd = S.desc[T * k];
    shared_ok = expert_ok(sd, H, I) && qt_supported(sd.gate.qtype, H) && qt_supported_down(sd.down.qtype, I);
    if (!shared_ok && b == 0 && threadIdx.x == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 2000000);
  }
  if (shared_ok) {
    int r0, r1;
    split_range(I, G, b, r0, r1);
    const int R = gu_rows_per_batch(S.desc[T * k], H);
    if (threadIdx.x == 0) {
      S.spre[0] = 0;
      S.spre[1] = (r1 - r0 + R - 1) / R;
      S.srpb[0] = R;
    }
    __syncthreads();
    SJ = GateUpJobs{S.desc + T * k, S.spre, S.srpb, 1, r0, r1 - r0, H, T * k + my_t};
    split_range(SJ.total(), ngrp, grp, sb0, sb1);
    for (int i = 0; i < kSlots; ++i)
      issue_any<2>(ring + i * kSlotBytes, sb0 + i < sb1 ? SJ.get(sb0 + i) : Batch{nullptr, nullptr, 0, 0, 0, 0}, H);
  }
  for (; ucur < u1; ucur += 2 * kWarps) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int u = ucur + s * kWarps;
      if (u >= u1) continue;
      const int e = u / kRQ, q = u % kRQ;
      float acc[kMaxT] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c >= q4) continue;
        const float4 w4 = wv[s][c];
#pragma unroll
        for (int t = 0; t < kMaxT; ++t)
          if (t < T) {
            const float4 x4 = *reinterpret_cast<const float4*>(S.xs + t * H + q * qlen + 4 * (lane + 32 * c));
            acc[t] = fmaf(w4.x, x4.x, fmaf(w4.y, x4.y, fmaf(w4.z, x4.z, fmaf(w4.w, x4.w, acc[t]))));
          }
      }
#pragma unroll
      for (int t = 0; t < kMaxT; ++t)
        if (t < T) {
          const float sum = warp_sum(acc[t]);
          if (lane == 0) P.partial[(size_t(t) * E + e) * kRQ + q] = sum;
        }
    }
    // loads of the next pair of units (rare: more than 16 units per CTA)
    const int un = ucur + 2 * kWarps;
    if (un < u1) {
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int u = un + s * kWarps;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (u < u1 && c < q4) {
            const float4* wr = reinterpret_cast<const float4*>(P.w_router + size_t(u / kRQ) * H + (u % kRQ) * qlen);
            wv[s][c] = __ldg(wr + lane + 32 * c);
          }
      }
    }
  }
  // 2) shared expert gate/up, already in flight
  if (shared_ok) gate_up_stream(ring, red, SJ, sb0, sb1, S.xs + my_t * H, P.h, I, true);
  // 3) L2 prefetch of the shared down rows this CTA uses in phase C
  if (shared_ok && threadIdx.x == kThreads - 32) {  // not the barrier thread
    const moe_qmatrix& d = S.desc[T * k].down;
    const size_t rb = size_t(chunks_per_row(d.qtype, I)) * 16, sb = size_t(scale_row_bytes(d.qtype, I));
    prefetch_l2(d.codes, n0 * rb, n1 * rb);
    if (d.qtype != MOE_Q_INT8_PER_CHANNEL) prefetch_l2(d.scales, n0 * sb, n1 * sb);
    if (d.mins) prefetch_l2(d.mins, n0 * sb, n1 * sb);
  }
  if (!grid_sync(hdr, uint32_t(G))) goto done;

  // ------------------------------------------------ phase B
  {
    for (int i = threadIdx.x; i < T * E; i += kThreads) {
      const int t = i / E, e = i % E;
      const float4 p4 = __ldcg(reinterpret_cast<const float4*>(P.partial + size_t(i) * kRQ));
      S.lg[i] = ((p4.x + p4.y) + (p4.z + p4.w)) + (P.bias ? P.bias[t * P.bstride + e] : 0.f);
    }
    __syncthreads();
    // Top-k, stage 1: warp w selects the best k of its slice of the experts
    // (loop-based, so the code stays small: it runs once per launch, cold).
    const int chunk = (E + kWarps - 1) / kWarps;  // <= 128
    for (int t = 0; t < T; ++t) {
      const int e0 = min(E, warp * chunk), e1 = min(E, e0 + chunk);
      const int n = e1 - e0, kk = min(k, n);
      uint32_t* ck = S.ck + (size_t(t) * kWarps + warp) * k;
      int* ci = S.ci + (size_t(t) * kWarps + warp) * k;
      uint32_t keys[4];
      int ids[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = lane + 32 * i;
        keys[i] = c < n ? f2key(S.lg[size_t(t) * E + e0 + c]) : 0u;
        ids[i] = c < n ? e0 + c : 0x7fffffff;
      }
      for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int bi = 0x7fffffff, bs = -1;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (ids[i] != 0x7fffffff && (bs < 0 || keys[i] > bk || (keys[i] == bk && ids[i] < bi))) {
            bk = keys[i];
            bi = ids[i];
            bs = i;
          }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bs >= 0 ? bk : 0u);
        const uint32_t wi = __reduce_min_sync(0xffffffffu, (bs >= 0 && bk == wk) ? uint32_t(bi) : 0xffffffffu);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i == bs && uint32_t(bi) == wi) ids[i] = 0x7fffffff;
        if (lane == 0) {
          ck[j] = j < kk ? wk : 0u;
          ci[j] = j < kk ? int(wi) : 0x7fffffff;
        }
      }
    }
    __syncthreads();
    // Stage 2: warp t picks the best k of the kWarps * k candidates.
    if (warp < T) {
      const int t = warp;
      const int nc = kWarps * k;
      if (nc <= 256) warp_select<8>(S.ck + size_t(t) * nc, S.ci + size_t(t) * nc, nc, k, s_key + t * k, s_idx + t * k);
      else warp_select<16>(S.ck + size_t(t) * nc, S.ci + size_t(t) * nc, nc, k, s_key + t * k, s_idx + t * k);
      // renormalised softmax over the picks
      const float v0 = key2f(s_key[t * k]);
      float part = 0.f;
      for (int j = lane; j < k; j += 32) part += expf(key2f(s_key[t * k + j]) - v0);
      const float denom = warp_sum(part);
      for (int j = lane; j < k; j += 32) s_w[t * k + j] = expf(key2f(s_key[t * k + j]) - v0) / denom;
    }
    __syncthreads();
    if (b == 0)
      for (int i = threadIdx.x; i < T * k; i += kThreads) {
        P.topk_idx[i] = s_idx[i];
        P.topk_w[i] = s_w[i];
      }
    // The picks' descriptors into shared memory, then the batch tables.
    {
      constexpr int W = int(sizeof(moe_expert) / 4);
      const uint32_t* src = reinterpret_cast<const uint32_t*>(P.experts);
      uint32_t* dst = reinterpret_cast<uint32_t*>(S.desc);
      for (int i = threadIdx.x; i < T * k * W; i += kThreads) dst[i] = src[size_t(s_idx[i / W]) * W + (i % W)];
    }
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    int r0, r1;
    split_range(I, G, b, r0, r1);
    const int nr = r1 - r0;
    const int nrouted = T * k, npairs = nrouted + (shared_ok ? T : 0);
    for (int p = threadIdx.x; p < npairs; p += kThreads) {
      const moe_expert& e = S.desc[p < nrouted ? p : nrouted];
      if (p < nrouted) {
        if (!expert_ok(e, H, I) || !qt_supported(e.gate.qtype, H) || !qt_supported_down(e.down.qtype, I)) {
          s_bad = 1;
          continue;
        }
        S.grpb[p] = gu_rows_per_batch(e, H);
      }
      S.drpb[p] = dn_rows_per_batch(e.down, I);
    }
    __syncthreads();
    if (s_bad) {
      if (threadIdx.x == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 1000000);
    } else {
      if (threadIdx.x < T) {  // gate/up prefix per token
        const int t = threadIdx.x;
        int acc = 0;
        for (int j = 0; j < k; ++j) {
          S.gpre[t * (k + 1) + j] = acc;
          const int R = S.grpb[t * k + j];
          acc += (nr + R - 1) / R;
        }
        S.gpre[t * (k + 1) + k] = acc;
      }
      if (threadIdx.x == 32) {  // down prefix over all pairs
        int acc = 0;
        for (int p = 0; p < npairs; ++p) {
          S.dpre[p] = acc;
          const int R = S.drpb[p];
          acc += (nn + R - 1) / R;
        }
        S.dpre[npairs] = acc;
      }
      __syncthreads();
      GateUpJobs RJ{S.desc + my_t * k, S.gpre + my_t * (k + 1), S.grpb + my_t * k, k, r0, nr, H, my_t * k};
      int b0, b1;
      split_range(RJ.total(), ngrp, grp, b0, b1);
      gate_up_stream(ring, red, RJ, b0, b1, S.xs + my_t * H, P.h, I, false);
    }
    // L2 prefetch of the routed down rows this CTA owns in phase C.
    for (int p = threadIdx.x - (kThreads - 64); p >= 0 && p < T * k && !s_bad; p += 64) {  // last two warps
      const moe_qmatrix& d = S.desc[p].down;
      const size_t rb = size_t(chunks_per_row(d.qtype, I)) * 16, sb = size_t(scale_row_bytes(d.qtype, I));
      prefetch_l2(d.codes, n0 * rb, n1 * rb);
      if (d.qtype != MOE_Q_INT8_PER_CHANNEL) prefetch_l2(d.scales, n0 * sb, n1 * sb);
      if (d.mins) prefetch_l2(d.mins, n0 * sb, n1 * sb);
    }
  }
  if (__syncthreads_or(0) || !grid_sync(hdr, uint32_t(2 * G))) goto done;

  // ------------------------------------------------ phase C
  {
    const int nrouted = T * k;
    const int npairs = nrouted + (shared_ok ? T : 0);
    const bool bad = s_bad != 0;
    if (!bad) {
      DownJobs D{S.desc, S.dpre, S.drpb, nrouted, npairs, n0, nn, I};
      int b0, b1;
      split_range(D.total(), kWarps, warp, b0, b1);
      down_stream(ring, red, D, b0, b1, P.h, S.ys);
    }
    __syncthreads();
    // Gate-weighted sum in slot order plus the shared expert; one rounding.
    if (!bad)
      for (int i = threadIdx.x; i < T * nn; i += kThreads) {
        const int t = i / nn, n = i % nn;
        float acc = 0.f;
        for (int j = 0; j < k; ++j) acc = fmaf(s_w[t * k + j], S.ys[size_t(t * k + j) * nn + n], acc);
        if (shared_ok) acc += S.ys[size_t(nrouted + t) * nn + n];
        P.out[size_t(t) * H + n0 + n] = f32_to_bf16_rn(acc);
      }
    (void)nn_max;
  }

done:
  // The last CTA out resets the barrier words for the next launch.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&hdr->exit_count, 1u);
    if (prev == uint32_t(G) - 1) {
      hdr->bar_count = 0;
      hdr->exit_count = 0;
      hdr->abort = 0;
      __threadfence();
    }
  }
}

}  // namespace dec

// Host side -----------------------------------------------------------------
static size_t decode_fused_smem(int T, int H, int I, int E, int k, int grid) {
  const size_t ring = size_t(dec::kWarps) * dec::kSlots * dec::kSlotBytes;
  const int nn = (H + grid - 1) / grid;
  const size_t floats = size_t(T) * H + size_t(T) * E + size_t(T * k + T) * nn;
  const size_t cand = 2 * 4 * size_t(T) * dec::kWarps * k;
  const size_t tables = 16 + sizeof(moe_expert) * size_t(T * k + 1) + 4 * size_t(T * (k + 1) + T * k + 2 * (T * k + T) + 4);
  return ring + 4 * floats + cand + tables;
}

bool decode_fused_eligible(int T, int H, int I, int E, int k) {
  if (T < 1 || T > dec::kMaxT || E > kMaxE || k > kMaxK) return false;
  if (H > 2048 || I > 1024 || (H % 512) || (I % 256)) return false;
  if (E > dec::kWarps * 128) return false;
  return decode_fused_smem(T, H, I, E, k, 148) <= 220 * 1024;
}

cudaError_t launch_decode_fused(const uint16_t* x, int T, int H, int I, int E, int k, const float* w_router,
                                const float* bias, long long bstride, const moe_expert* experts,
                                const moe_expert* shared, int* topk_idx, float* topk_w, uint16_t* out,
                                float* partial, float* h, WsHeader* hdr, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = sms > 0 ? sms : 148;
  const size_t smem = decode_fused_smem(T, H, I, E, k, grid);
  e = cudaFuncSetAttribute(dec::decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dec::Params P{x, T, H, I, E, k, w_router, bias, bstride, experts, shared, topk_idx, topk_w, out, partial, h, hdr};
  void* args[] = {&P};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(dec::decode_fused_kernel), dim3(grid), dim3(dec::kThreads),
                                  args, smem, st);
  count_launches(1);
  return e;
}

}  // namespace moe
