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
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

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
    __threadfence();
    atomicAdd(&hdr->bar_count, 1u);
    const long long t0 = clock64();
    while (ld_acquire(&hdr->bar_count) < target) {
      if (*reinterpret_cast<volatile int*>(&hdr->abort)) {
        ok = 0;
        break;
      }
      if (clock64() - t0 > kSpinCycles) {
        flag_error(hdr, MOE_ERR_TIMEOUT, int(target));
        atomicExch(&hdr->abort, 1);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
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

// Partial dot product of this lane's chunks of one row with x. `codes` is
// the row's packed codes (shared memory), `sc`/`mn` its fp16 group scales and
// mins (shared memory; int8 rows take their scale from the caller instead).
template <int QT, int CPL>
__device__ __forceinline__ float row_dot(const uint8_t* codes, const uint16_t* sc, const uint16_t* mn, int CPR,
                                         const XRegs<QT, CPL>& x) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = lane + 32 * j;
    if (c >= CPR) continue;
    const uint4 raw = *reinterpret_cast<const uint4*>(codes + 16 * c);
    const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
    if (QT == MOE_Q_INT4_SYM_G32) {
      float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t lo = wd[w] & 0x0F0F0F0Fu, hi = (wd[w] >> 4) & 0x0F0F0F0Fu;
        const float* xv = x.v[j] + 8 * w;
        s2 = ffma2(make_float2(code_f<0>(lo), code_f<1>(lo)), make_float2(xv[0], xv[1]), s2);
        s2 = ffma2(make_float2(code_f<2>(lo), code_f<3>(lo)), make_float2(xv[2], xv[3]), s2);
        s2 = ffma2(make_float2(code_f<0>(hi), code_f<1>(hi)), make_float2(xv[4], xv[5]), s2);
        s2 = ffma2(make_float2(code_f<2>(hi), code_f<3>(hi)), make_float2(xv[6], xv[7]), s2);
      }
      const float s = f16_to_f32(sc[c]);
      // sum (c - 8) x = 256 S - 136 X
      acc = fmaf(s, fmaf(256.f, s2.x + s2.y, -136.f * x.gsum[j][0]), acc);
    } else if (QT == MOE_Q_INT2_ASYM_G16) {
      const uint2 scw = *reinterpret_cast<const uint2*>(sc + 4 * c);
      const uint2 mnw = *reinterpret_cast<const uint2*>(mn + 4 * c);
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
        const float s = f16_to_f32(uint16_t(sv[w])), m = f16_to_f32(uint16_t(mv[w]));
        // sum (c s + m) x = 256 s S + (m - 128 s) X
        acc = fmaf(256.f * s, s2.x + s2.y, fmaf(m - 128.f * s, x.gsum[j][w], acc));
      }
    } else {
      float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t u = wd[w] ^ 0x80808080u;  // q + 128 in each byte
        const float* xv = x.v[j] + 4 * w;
        float q[4];
#pragma unroll
        for (int b = 0; b < 4; ++b)
          q[b] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u | b)) - 8388736.0f;  // - (2^23 + 128)
        s2 = ffma2(make_float2(q[0], q[1]), make_float2(xv[0], xv[1]), s2);
        s2 = ffma2(make_float2(q[2], q[3]), make_float2(xv[2], xv[3]), s2);
      }
      acc += s2.x + s2.y;  // the row scale is applied by the caller
    }
  }
  return acc;
}

__host__ __device__ __forceinline__ int bits_of(int qt) {
  return qt == MOE_Q_INT4_SYM_G32 ? 4 : qt == MOE_Q_INT2_ASYM_G16 ? 2 : 8;
}
// Chunks (16 bytes of codes) per row of K inputs.
__host__ __device__ __forceinline__ int chunks_per_row(int qt, int K) { return K * bits_of(qt) / 128; }
// Bytes of group scales (and of mins) per row; 0 for int8 (scale per row,
// read from global memory at use).
__host__ __device__ __forceinline__ int scale_row_bytes(int qt, int K) {
  return qt == MOE_Q_INT4_SYM_G32 ? K / 16 : qt == MOE_Q_INT2_ASYM_G16 ? K / 8 : 0;
}

// ---------------------------------------------------------------- staging ring
// Every warp owns kSlots shared-memory slots filled by 1-D bulk (TMA) copies
// that complete on one mbarrier per slot. Lane 0 issues, all lanes wait.
constexpr int kSlots = 4;
constexpr int kSlotBytes = 4608;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Bounded wait for the phase with the given parity. false = gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (true) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > kSpinCycles) return false;
  }
}

struct Ring {
  uint8_t* slots;       // kSlots x kSlotBytes, this warp's
  uint32_t bar0;        // shared address of this warp's first mbarrier
  uint32_t parity;      // bit s: parity of the next completion of slot s
  uint32_t pending;     // bit s: a copy into slot s is in flight
  __device__ uint32_t bar(int s) const { return bar0 + 8u * s; }
  __device__ uint8_t* slot(int s) const { return slots + size_t(s) * kSlotBytes; }
};

// Copy up to 6 (src, bytes) segments into consecutive 16-byte aligned places
// of slot s. Lane 0 only. Segments with bytes == 0 are skipped.
struct Seg {
  const void* src;
  uint32_t bytes;
};

__device__ __forceinline__ void ring_issue(Ring& r, int s, const Seg* segs, int nseg) {
  uint32_t total = 0;
  for (int i = 0; i < nseg; ++i) total += segs[i].bytes;
  if ((threadIdx.x & 31) == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // earlier generic reads of the slot
    mbar_expect_tx(r.bar(s), total);
    uint32_t off = 0;
    for (int i = 0; i < nseg; ++i) {
      if (segs[i].bytes) bulk_g2s(smem_u32(r.slot(s)) + off, segs[i].src, segs[i].bytes, r.bar(s));
      off += segs[i].bytes;
    }
  }
  r.pending |= 1u << s;
}

// Wait for slot s (all lanes). false = the bounded wait expired.
__device__ __forceinline__ bool ring_wait(Ring& r, int s) {
  const bool ok = mbar_wait(r.bar(s), (r.parity >> s) & 1u);
  if (ok) {
    r.parity ^= 1u << s;
    r.pending &= ~(1u << s);
  }
  return ok;
}

// Segments of one gate/up unit: row `row` of gate and of up (codes, then
// scales, then mins). Returns the number of segments (0 = unit skipped).
__device__ __forceinline__ int gate_up_segs(const moe_expert& ex, int H, int row, Seg* segs) {
  const int qt = ex.gate.qtype;
  const uint32_t cb = uint32_t(chunks_per_row(qt, H)) * 16u, sb = uint32_t(scale_row_bytes(qt, H));
  segs[0] = {ex.gate.codes + size_t(row) * cb, cb};
  segs[1] = {ex.up.codes + size_t(row) * cb, cb};
  segs[2] = {reinterpret_cast<const uint8_t*>(ex.gate.scales) + size_t(row) * sb, sb};
  segs[3] = {reinterpret_cast<const uint8_t*>(ex.up.scales) + size_t(row) * sb, sb};
  const bool mins = qt == MOE_Q_INT2_ASYM_G16;
  segs[4] = {mins ? reinterpret_cast<const uint8_t*>(ex.gate.mins) + size_t(row) * sb : nullptr, mins ? sb : 0u};
  segs[5] = {mins ? reinterpret_cast<const uint8_t*>(ex.up.mins) + size_t(row) * sb : nullptr, mins ? sb : 0u};
  return 6;
}

// Segments of one down unit: rows [n0, n0 + nr) of matrix m (K = I).
__device__ __forceinline__ int down_segs(const moe_qmatrix& m, int I, int n0, int nr, Seg* segs) {
  const int qt = m.qtype;
  const uint32_t cb = uint32_t(chunks_per_row(qt, I)) * 16u, sb = uint32_t(scale_row_bytes(qt, I));
  segs[0] = {m.codes + size_t(n0) * cb, cb * nr};
  segs[1] = {reinterpret_cast<const uint8_t*>(m.scales) + size_t(n0) * sb, sb * nr};
  const bool mins = qt == MOE_Q_INT2_ASYM_G16;
  segs[2] = {mins ? reinterpret_cast<const uint8_t*>(m.mins) + size_t(n0) * sb : nullptr, mins ? sb * nr : 0u};
  return 3;
}

// Rows of a down matrix that fit one slot.
__host__ __device__ __forceinline__ int down_rows_per_slot(int qt, int I) {
  const int per = chunks_per_row(qt, I) * 16 + scale_row_bytes(qt, I) * (qt == MOE_Q_INT2_ASYM_G16 ? 2 : 1);
  return kSlotBytes / per;
}
// ---------------------------------------------------------------- top-k
__device__ __forceinline__ uint32_t f2key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp top-k over logits lg[0..E) (smem, E <= 1024): repeated warp-wide
// argmax (larger value, then lower index) with redux.sync.
__device__ void warp_topk(const float* lg, int E, int k, int* sidx, float* sw) {
  const int lane = threadIdx.x & 31;
  const int nper = (E + 31) / 32;
  uint32_t key[32];
  uint32_t avail = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (i < nper && e < E) {
      float v = lg[e];
      if (v != v) v = -CUDART_INF_F;
      key[i] = f2key(v);
      avail |= 1u << i;
    }
  }
  float sel0 = 0.f, denom = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (((avail >> i) & 1u) && (bi < 0 || key[i] > best)) {
        best = key[i];
        bi = i;
      }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, bi >= 0 ? best : 0u);
    const uint32_t cand = (bi >= 0 && best == wmax) ? uint32_t(lane + 32 * bi) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if (int(win & 31) == lane) avail &= ~(1u << (win >> 5));
    // recover the float value of the winning key
    const uint32_t u = (wmax & 0x80000000u) ? (wmax & 0x7fffffffu) : ~wmax;
    const float v = __uint_as_float(u);
    if (j == 0) sel0 = v;
    const float ev = expf(v - sel0);
    denom += ev;
    if (lane == 0) {
      sidx[j] = int(win);
      sw[j] = ev;
    }
  }
  __syncwarp();
  for (int j = lane; j < k; j += 32) sw[j] = sw[j] / denom;
  __syncwarp();
}

// ---------------------------------------------------------------- unit runners
// Issue the copy of gate/up unit (expert ex, row) into slot s.
__device__ __forceinline__ void issue_gate_up(Ring& R, int s, const moe_expert& ex, int H, int row) {
  Seg segs[6];
  gate_up_segs(ex, H, row, segs);
  ring_issue(R, s, segs, 6);
}

// A warp's list of gate/up units: unit i (0 <= i < n) is row
// r0 + (q0 + i) % nr of the expert of pair pidx[(q0 + i) / nr]; results go to
// h[(pair_base + (q0 + i) / nr) * I + row]. expert_of(i) gives the descriptor.
struct GateUpList {
  const moe_expert* experts;  // routed table, or the shared descriptor
  const int* pidx;            // expert id per local pair (nullptr: always experts[0])
  int q0, n, nr, r0, pair_base;
  float* h;
  int H, I;
  __device__ int pair(int i) const { return (q0 + i) / nr; }
  __device__ int row(int i) const { return r0 + (q0 + i) % nr; }
  __device__ const moe_expert& ex(int i) const { return experts[pidx ? pidx[pair(i)] : 0]; }
};

__device__ __forceinline__ bool unit_ok(const GateUpList& L, int i) { return expert_ok(L.ex(i), L.H, L.I); }

template <int QT, int CPL>
__device__ int gate_up_run(Ring& R, const GateUpList& L, int i, const float* xs, WsHeader* hdr, bool& failed) {
  const int CPR = chunks_per_row(QT, L.H);
  const uint32_t cb = uint32_t(CPR) * 16u, sb = uint32_t(scale_row_bytes(QT, L.H));
  XRegs<QT, CPL> x;
  x.load(xs, CPR);
  for (; i < L.n; ++i) {
    const moe_expert& ex = L.ex(i);
    if (ex.gate.qtype != QT) break;
    const int s = i % kSlots;
    if (unit_ok(L, i)) {
      if (!ring_wait(R, s)) {
        if ((threadIdx.x & 31) == 0) {
          flag_error(hdr, MOE_ERR_TIMEOUT, 4000000);
          atomicExch(&hdr->abort, 1);
        }
        failed = true;
        return L.n;
      }
      const uint8_t* base = R.slot(s);
      const int row = L.row(i);
      const uint16_t* gs = reinterpret_cast<const uint16_t*>(base + 2 * cb);
      const uint16_t* us = reinterpret_cast<const uint16_t*>(base + 2 * cb + sb);
      const uint16_t* gm = reinterpret_cast<const uint16_t*>(base + 2 * cb + 2 * sb);
      const uint16_t* um = reinterpret_cast<const uint16_t*>(base + 2 * cb + 3 * sb);
      float g = warp_sum(row_dot<QT, CPL>(base, gs, gm, CPR, x));
      float u = warp_sum(row_dot<QT, CPL>(base + cb, us, um, CPR, x));
      if (QT == MOE_Q_INT8_PER_CHANNEL) {
        g *= f16_to_f32(ex.gate.scales[row]);
        u *= f16_to_f32(ex.up.scales[row]);
      }
      if ((threadIdx.x & 31) == 0) L.h[size_t(L.pair_base + L.pair(i)) * L.I + row] = silu_f32(g) * u;
      __syncwarp();
    } else if ((threadIdx.x & 31) == 0) {
      flag_error(hdr, MOE_ERR_DEVICE_FAULT, 1000000 + L.pair(i));
    }
    const int nx = i + kSlots;
    if (nx < L.n && unit_ok(L, nx)) issue_gate_up(R, s, L.ex(nx), L.H, L.row(nx));
  }
  return i;
}

__device__ void gate_up_prime(Ring& R, const GateUpList& L) {
  for (int i = 0; i < L.n && i < kSlots; ++i)
    if (unit_ok(L, i)) issue_gate_up(R, i % kSlots, L.ex(i), L.H, L.row(i));
}

// Consume a primed list (units stream through the ring, kSlots ahead).
__device__ void gate_up_consume(Ring& R, const GateUpList& L, const float* xs, WsHeader* hdr, bool& failed) {
  int i = 0;
  while (i < L.n && !failed) {
    const int qt = L.ex(i).gate.qtype;
    const int cpl = (chunks_per_row(qt, L.H) + 31) / 32;
    int j = L.n;
    if (qt == MOE_Q_INT4_SYM_G32 && cpl == 1) j = gate_up_run<MOE_Q_INT4_SYM_G32, 1>(R, L, i, xs, hdr, failed);
    else if (qt == MOE_Q_INT4_SYM_G32 && cpl == 2) j = gate_up_run<MOE_Q_INT4_SYM_G32, 2>(R, L, i, xs, hdr, failed);
    else if (qt == MOE_Q_INT2_ASYM_G16 && cpl == 1) j = gate_up_run<MOE_Q_INT2_ASYM_G16, 1>(R, L, i, xs, hdr, failed);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 1) j = gate_up_run<MOE_Q_INT8_PER_CHANNEL, 1>(R, L, i, xs, hdr, failed);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 2) j = gate_up_run<MOE_Q_INT8_PER_CHANNEL, 2>(R, L, i, xs, hdr, failed);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl <= 4) j = gate_up_run<MOE_Q_INT8_PER_CHANNEL, 4>(R, L, i, xs, hdr, failed);
    else {
      // Malformed or unsupported: the descriptor check flags it; drain the unit.
      if ((threadIdx.x & 31) == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 5000000 + qt);
      const int s = i % kSlots;
      if ((R.pending >> s) & 1u) ring_wait(R, s);
      const int nx = i + kSlots;
      if (nx < L.n && unit_ok(L, nx)) issue_gate_up(R, s, L.ex(nx), L.H, L.row(nx));
      j = i + 1;
    }
    i = j;
  }
}

// Down units of one warp: unit i covers pair p = (u0 + i) / nsub, rows
// n0 + sub*rpu .. (clipped to n1), sub = (u0 + i) % nsub.
struct DownList {
  const moe_expert* experts;
  const moe_expert* shared;
  const int* pidx;  // expert ids of the routed pairs
  int nrouted;      // pairs < nrouted are routed, the rest shared (token p - nrouted)
  int u0, n, nsub, rpu, n0, n1, nn;
  const float* h;   // [npairs][I] (global, written by other CTAs)
  float* ys;        // [npairs][nn] (shared)
  int H, I;
  __device__ int pair(int i) const { return (u0 + i) / nsub; }
  __device__ int rlo(int i) const { return n0 + ((u0 + i) % nsub) * rpu; }
  __device__ int rhi(int i) const { return min(n1, rlo(i) + rpu); }
  __device__ const moe_qmatrix& mat(int i) const {
    const int p = pair(i);
    return p < nrouted ? experts[pidx[p]].down : shared->down;
  }
};

__device__ __forceinline__ void issue_down(Ring& R, int s, const DownList& L, int i) {
  Seg segs[3];
  down_segs(L.mat(i), L.I, L.rlo(i), L.rhi(i) - L.rlo(i), segs);
  ring_issue(R, s, segs, 3);
}

template <int QT, int CPL>
__device__ int down_run(Ring& R, const DownList& L, int i, WsHeader* hdr, bool& failed) {
  const int CPR = chunks_per_row(QT, L.I);
  const uint32_t cb = uint32_t(CPR) * 16u, sb = uint32_t(scale_row_bytes(QT, L.I));
  XRegs<QT, CPL> x;
  int xp = -1;
  for (; i < L.n; ++i) {
    const moe_qmatrix& m = L.mat(i);
    if (m.qtype != QT) break;
    const int s = i % kSlots;
    const int p = L.pair(i);
    if (qmatrix_ok(m, L.H, L.I)) {
      if (p != xp) {
        x.template load<true>(L.h + size_t(p) * L.I, CPR);
        xp = p;
      }
      if (!ring_wait(R, s)) {
        if ((threadIdx.x & 31) == 0) {
          flag_error(hdr, MOE_ERR_TIMEOUT, 4000001);
          atomicExch(&hdr->abort, 1);
        }
        failed = true;
        return L.n;
      }
      const uint8_t* base = R.slot(s);
      const int lo = L.rlo(i), hi = L.rhi(i), nr = hi - lo;
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(base + nr * cb);
      const uint16_t* mn = reinterpret_cast<const uint16_t*>(base + nr * cb + nr * sb);
      for (int r = 0; r < nr; ++r) {
        float y = warp_sum(row_dot<QT, CPL>(base + r * cb, sc + r * (sb / 2), mn + r * (sb / 2), CPR, x));
        if (QT == MOE_Q_INT8_PER_CHANNEL) y *= f16_to_f32(m.scales[lo + r]);
        if ((threadIdx.x & 31) == 0) L.ys[size_t(p) * L.nn + (lo - L.n0) + r] = y;
      }
      __syncwarp();
    }
    const int nx = i + kSlots;
    if (nx < L.n && qmatrix_ok(L.mat(nx), L.H, L.I)) issue_down(R, s, L, nx);
  }
  return i;
}

__device__ void down_list(Ring& R, const DownList& L, WsHeader* hdr, bool& failed) {
  if (L.n <= 0) return;
  for (int i = 0; i < L.n && i < kSlots; ++i)
    if (qmatrix_ok(L.mat(i), L.H, L.I)) issue_down(R, i % kSlots, L, i);
  int i = 0;
  while (i < L.n && !failed) {
    const int qt = L.mat(i).qtype;
    const int cpl = (chunks_per_row(qt, L.I) + 31) / 32;
    int j;
    if (qt == MOE_Q_INT4_SYM_G32 && cpl == 1) j = down_run<MOE_Q_INT4_SYM_G32, 1>(R, L, i, hdr, failed);
    else if (qt == MOE_Q_INT4_SYM_G32 && cpl == 2) j = down_run<MOE_Q_INT4_SYM_G32, 2>(R, L, i, hdr, failed);
    else if (qt == MOE_Q_INT2_ASYM_G16 && cpl == 1) j = down_run<MOE_Q_INT2_ASYM_G16, 1>(R, L, i, hdr, failed);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 1) j = down_run<MOE_Q_INT8_PER_CHANNEL, 1>(R, L, i, hdr, failed);
    else if (qt == MOE_Q_INT8_PER_CHANNEL && cpl == 2) j = down_run<MOE_Q_INT8_PER_CHANNEL, 2>(R, L, i, hdr, failed);
    else {
      const int s = i % kSlots;
      if ((R.pending >> s) & 1u) ring_wait(R, s);
      const int nx = i + kSlots;
      if (nx < L.n && qmatrix_ok(L.mat(nx), L.H, L.I)) issue_down(R, s, L, nx);
      j = i + 1;
    }
    i = j;
  }
}

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[kWarps * kSlots];
  __shared__ int s_idx[kMaxT * kMaxK];
  __shared__ float s_w[kMaxT * kMaxK];
  const int T = P.T, H = P.H, I = P.I, E = P.E, k = P.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  const bool has_shared = P.shared != nullptr;
  WsHeader* hdr = P.hdr;
  bool failed = false;

  uint8_t* ring_base = smem;                                      // kWarps x kSlots x kSlotBytes
  float* xs = reinterpret_cast<float*>(smem + kWarps * kSlots * kSlotBytes);  // [T][H]
  float* lg = xs + T * H;                                         // [T][E] (phase B), ys (phase C)

  Ring R;
  R.slots = ring_base + size_t(warp) * kSlots * kSlotBytes;
  R.bar0 = smem_u32(&bars[warp * kSlots]);
  R.parity = 0;
  R.pending = 0;
  if (lane == 0)
    for (int s = 0; s < kSlots; ++s) mbar_init(R.bar(s));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  for (int i = threadIdx.x; i < T * H; i += kThreads) xs[i] = bf16_to_f32(P.x[i]);
  bool shared_ok = false;
  if (has_shared) {
    shared_ok = expert_ok(*P.shared, H, I);
    if (!shared_ok && b == 0 && threadIdx.x == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 2000000);
  }
  __syncthreads();

  // Warps are pinned to tokens (warp w serves token w % T): the activation
  // registers are loaded once per phase.
  const int my_t = warp % T;
  const int grp = warp / T, ngrp = (kWarps - my_t + T - 1) / T;

  // ------------------------------------------------ phase A
  {
    // Shared expert gate/up of this CTA's intermediate rows (through the ring).
    GateUpList L{};
    if (shared_ok) {
      int r0, r1;
      split_range(I, G, b, r0, r1);
      const int nr = r1 - r0;
      int q0, q1;
      split_range(nr, ngrp, grp, q0, q1);
      L = GateUpList{P.shared, nullptr, q0, q1 - q0, nr > 0 ? nr : 1, r0, T * k + my_t, P.h, H, I};
      gate_up_prime(R, L);  // the copies overlap the router below
    }
    // Router quarter-rows of this CTA, loaded straight into registers.
    int u0, u1;
    split_range(E * kRQ, G, b, u0, u1);
    const int qlen = H / kRQ;
    for (int u = u0 + warp; u < u1; u += kWarps) {
      const int e = u / kRQ, q = u % kRQ;
      const float4* wr = reinterpret_cast<const float4*>(P.w_router + size_t(e) * H + q * qlen);
      float acc[kMaxT] = {0.f, 0.f, 0.f, 0.f};
      for (int c = lane; c < qlen / 4; c += 32) {
        const float4 w4 = __ldg(wr + c);
#pragma unroll
        for (int t = 0; t < kMaxT; ++t)
          if (t < T) {
            const float4 x4 = *reinterpret_cast<const float4*>(xs + t * H + q * qlen + 4 * c);
            acc[t] = fmaf(w4.x, x4.x, fmaf(w4.y, x4.y, fmaf(w4.z, x4.z, fmaf(w4.w, x4.w, acc[t]))));
          }
      }
#pragma unroll
      for (int t = 0; t < kMaxT; ++t)
        if (t < T) {
          const float s = warp_sum(acc[t]);
          if (lane == 0) P.partial[(size_t(t) * E + e) * kRQ + q] = s;
        }
    }
    if (shared_ok) gate_up_consume(R, L, xs + my_t * H, hdr, failed);
    // L2 prefetch of the shared down rows this CTA will use in phase C.
    if (shared_ok && threadIdx.x == 0) {
      int n0, n1;
      split_range(H, G, b, n0, n1);
      const moe_qmatrix& d = P.shared->down;
      const size_t rb = size_t(chunks_per_row(d.qtype, I)) * 16, sb = size_t(scale_row_bytes(d.qtype, I));
      prefetch_l2(d.codes, n0 * rb, n1 * rb);
      if (sb) prefetch_l2(d.scales, n0 * sb, n1 * sb);
      if (d.mins) prefetch_l2(d.mins, n0 * sb, n1 * sb);
    }
  }
  if (__syncthreads_or(failed) || !grid_sync(hdr, uint32_t(G))) goto done;

  // ------------------------------------------------ phase B
  {
    for (int i = threadIdx.x; i < T * E; i += kThreads) {
      const int t = i / E, e = i % E;
      const float4 p4 = __ldcg(reinterpret_cast<const float4*>(P.partial + size_t(i) * kRQ));
      lg[i] = ((p4.x + p4.y) + (p4.z + p4.w)) + (P.bias ? P.bias[t * P.bstride + e] : 0.f);
    }
    __syncthreads();
    if (warp < T) warp_topk(lg + warp * E, E, k, s_idx + warp * k, s_w + warp * k);
    __syncthreads();
    if (b == 0)
      for (int i = threadIdx.x; i < T * k; i += kThreads) {
        P.topk_idx[i] = s_idx[i];
        P.topk_w[i] = s_w[i];
      }
    // Routed gate/up: this CTA's intermediate rows, this warp's token.
    int r0, r1;
    split_range(I, G, b, r0, r1);
    const int nr = r1 - r0;
    int q0, q1;
    split_range(k * nr, ngrp, grp, q0, q1);
    GateUpList L{P.experts, s_idx + my_t * k, q0, q1 - q0, nr > 0 ? nr : 1, r0, my_t * k, P.h, H, I};
    gate_up_prime(R, L);
    gate_up_consume(R, L, xs + my_t * H, hdr, failed);
    // L2 prefetch of the routed down rows this CTA owns in phase C.
    int n0, n1;
    split_range(H, G, b, n0, n1);
    for (int p = threadIdx.x; p < T * k; p += kThreads) {
      const moe_qmatrix& d = P.experts[s_idx[p]].down;
      if (!qmatrix_ok(d, H, I)) continue;
      const size_t rb = size_t(chunks_per_row(d.qtype, I)) * 16, sb = size_t(scale_row_bytes(d.qtype, I));
      prefetch_l2(d.codes, n0 * rb, n1 * rb);
      if (sb) prefetch_l2(d.scales, n0 * sb, n1 * sb);
      if (d.mins) prefetch_l2(d.mins, n0 * sb, n1 * sb);
    }
  }
  if (__syncthreads_or(failed) || !grid_sync(hdr, uint32_t(2 * G))) goto done;

  // ------------------------------------------------ phase C
  {
    int n0, n1;
    split_range(H, G, b, n0, n1);
    const int nn = n1 - n0;
    const int nrouted = T * k;
    const int npairs = nrouted + (shared_ok ? T : 0);
    float* ys = lg;  // [npairs][nn]
    const int rpu = down_rows_per_slot(MOE_Q_INT8_PER_CHANNEL, I);  // fits every qtype
    const int nsub = (nn + rpu - 1) / rpu;
    int u0, u1;
    split_range(npairs * nsub, kWarps, warp, u0, u1);
    DownList D{P.experts, P.shared, s_idx, nrouted, u0, u1 - u0, nsub, rpu, n0, n1, nn, P.h, ys, H, I};
    down_list(R, D, hdr, failed);
    __syncthreads();
    // Gate-weighted sum in slot order plus the shared expert; one rounding.
    for (int i = threadIdx.x; i < T * nn; i += kThreads) {
      const int t = i / nn, n = i % nn;
      float acc = 0.f;
      for (int j = 0; j < k; ++j) acc = fmaf(s_w[t * k + j], ys[size_t(t * k + j) * nn + n], acc);
      if (shared_ok) acc += ys[size_t(nrouted + t) * nn + n];
      P.out[size_t(t) * H + n0 + n] = f32_to_bf16_rn(acc);
    }
  }

done:
  // Copies still in flight (only after a failure) are waited for, bounded.
  for (int s = 0; s < kSlots; ++s)
    if ((R.pending >> s) & 1u) mbar_wait(R.bar(s), (R.parity >> s) & 1u);
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
  const size_t lgc = std::max(size_t(T) * E, size_t(T * k + T) * nn);
  return ring + 4 * (size_t(T) * H + lgc);
}

bool decode_fused_eligible(int T, int H, int I, int E, int k) {
  if (T < 1 || T > dec::kMaxT || E > kMaxE || k > kMaxK) return false;
  if (H > 2048 || I > 2048 || (H % 256) || (I % 256)) return false;
  if (dec::down_rows_per_slot(MOE_Q_INT8_PER_CHANNEL, I) < 1) return false;
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
