// Shared device helpers and the workspace layout of the MoE library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 64;
constexpr int kDispatchMaxBlocks = 256;  // multi-block dispatch histogram rows
constexpr int kTicketSlots = 16;

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
  int32_t status;        // first device-side error code (MOE_OK = none)
  int32_t detail;        // code-specific detail (e.g. the bad expert id)
  int32_t abort;         // set when a bounded grid barrier gave up
  uint32_t bar_count;    // grid-barrier arrivals of the running fused launch
  uint32_t exit_count;   // CTAs that left the running fused launch
  int32_t pad[11];
  uint32_t tickets[kTicketSlots];  // last-CTA tickets, always left at 0
};
static_assert(sizeof(WsHeader) <= 256, "header must fit in 256 bytes");

// Counters of the fused decode launch (finished gate/up tiles and the
// largest |h| per expert slot and token), right after the header. They must
// be zero when a launch starts; the launch leaves them zero again, and
// moe_reset_status clears them with the header.
constexpr size_t kDecodeCounterBytes = 8448;  // 65 expert slots x 128 bytes, rounded to 256
constexpr size_t kWsResetBytes = 256 + kDecodeCounterBytes;

// Offsets (bytes from the workspace base) of every workspace segment.
struct WsLayout {
  size_t dcnt, counts, offsets, perm, inv, hist, active, topk_idx, topk_w, logits, logits_u, sgate, h, dh,
      shared_y, y_perm, gemm, router;
  size_t total;
};
size_t decode_fused_ws_bytes(int T, int I);

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

size_t grouped_ws_bytes(long long T, int H, int I, int k, int E, bool with_shared);
size_t router_tc_ws_bytes(long long T, int H, int E);

inline WsLayout ws_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  WsLayout L{};
  size_t o = 256;
  auto take = [&](size_t bytes) { size_t r = o; o = align256(o + bytes); return r; };
  const int64_t n = T * k;
  L.dcnt = take(kDecodeCounterBytes);
  L.counts = take(4 * E);
  L.offsets = take(4 * (E + 1));
  L.perm = take(4 * n);
  L.inv = take(4 * n);
  L.hist = take(4 * E * kDispatchMaxBlocks);
  L.active = take(4 * (2 * E + 4));
  L.topk_idx = take(4 * n);
  L.topk_w = take(4 * n);
  L.logits = take(4 * T * E);
  L.logits_u = take(4 * T * E);  // unbiased logits (bias used for the selection only)
  L.sgate = take(4 * T);         // the shared expert's per-token sigmoid gate
  L.h = take(size_t(4 * (n + T) * I));  // fp32 intermediate rows of the multi-launch path
  L.dh = take(T >= 1 && T <= 4 ? decode_fused_ws_bytes(int(T), int(I)) : 0);  // fused decode: h per expert slot
  L.shared_y = take(4 * T * H);
  L.y_perm = take(4 * n * H);  // fp32 routed rows inside moe_layer
  L.gemm = take(grouped_ws_bytes(T, int(H), int(I), int(k), int(E), true));  // tcgen05 prefill scratch
  L.router = take(router_tc_ws_bytes(T, int(H), int(E)));                   // tcgen05 router scratch
  L.total = o;
  return L;
}

template <typename P>
__host__ __device__ inline P* ws_at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

__device__ inline void flag_error(WsHeader* hdr, int code, int detail) {
  if (atomicCAS(&hdr->status, 0, code) == 0) atomicExch(&hdr->detail, detail);
}

// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}
// fp32 -> bf16, round to nearest even (finite inputs; NaN stays NaN).
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return uint16_t((u >> 16) | 0x40);
  u += 0x7fffu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// Validate one packed matrix descriptor against the expected shape.
__device__ inline bool qmatrix_ok(const moe_qmatrix& m, int rows, int cols) {
  if (m.rows != rows || m.cols != cols || m.codes == nullptr || m.scales == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(m.codes) & 15) || (reinterpret_cast<uintptr_t>(m.scales) & 15)) return false;
  switch (m.qtype) {
    case MOE_Q_INT4_SYM_G32: return m.group == 32 && (cols % 64) == 0;
    case MOE_Q_INT2_ASYM_G16:
      return m.group == 16 && (cols % 64) == 0 && m.mins != nullptr && !(reinterpret_cast<uintptr_t>(m.mins) & 15);
    case MOE_Q_INT8_PER_CHANNEL: return m.group == 0 && (cols % 64) == 0;
    default: return false;
  }
}

__device__ inline bool expert_ok(const moe_expert& e, int H, int I) {
  return qmatrix_ok(e.gate, I, H) && qmatrix_ok(e.up, I, H) && qmatrix_ok(e.down, H, I) &&
         e.gate.qtype == e.up.qtype && e.gate.qtype == e.down.qtype;
}

// Bytes of packed codes per row of a K-column matrix.
__host__ __device__ inline int row_code_bytes(int qtype, int K) {
  return qtype == MOE_Q_INT4_SYM_G32 ? K / 2 : qtype == MOE_Q_INT2_ASYM_G16 ? K / 4 : K;
}
// Elements per 16-byte chunk of codes.
__host__ __device__ inline int chunk_elems(int qtype) {
  return qtype == MOE_Q_INT4_SYM_G32 ? 32 : qtype == MOE_Q_INT2_ASYM_G16 ? 64 : 16;
}

// Dequantise one 16-byte chunk c of row n into 32/64/16 fp32 weights w[].
// Returns the element count. Exact: q*s is a product of a <=8-bit integer and
// an fp16 value, representable in fp32.
__device__ __forceinline__ int dequant_chunk(const moe_qmatrix& m, int n, int c, uint4 raw, float* w) {
  const uint8_t* b = reinterpret_cast<const uint8_t*>(&raw);
  const int K = m.cols;
  if (m.qtype == MOE_Q_INT4_SYM_G32) {
    const float s = f16_to_f32(m.scales[size_t(n) * (K / 32) + c]);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      w[2 * i] = float(int(b[i] & 15) - 8) * s;
      w[2 * i + 1] = float(int(b[i] >> 4) - 8) * s;
    }
    return 32;
  } else if (m.qtype == MOE_Q_INT2_ASYM_G16) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const size_t gi = size_t(n) * (K / 16) + 4 * c + g;
      const float s = f16_to_f32(m.scales[gi]);
      const float mn = f16_to_f32(m.mins[gi]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint8_t v = b[4 * g + i];
#pragma unroll
        for (int q = 0; q < 4; ++q) w[16 * g + 4 * i + q] = fmaf(float((v >> (2 * q)) & 3), s, mn);
      }
    }
    return 64;
  } else {
    const float s = f16_to_f32(m.scales[n]);
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = float(int8_t(b[i])) * s;
    return 16;
  }
}

}  // namespace moe
