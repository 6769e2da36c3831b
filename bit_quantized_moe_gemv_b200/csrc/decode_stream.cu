// Decode step (T <= 4 tokens) as ONE persistent cooperative launch fed by two
// producer warps through a ring of shared-memory slots.
//
// Decode reads every picked expert's weights once per step, so it is bound by
// memory bandwidth (the lcz.me forum thread "Halogen Flash Server配置與實測",
// comment section: decode reads a fixed set of weights per step and its
// ceiling follows bandwidth). The telli.sh page "Strata 与 Qwen3.8-Flash-Next：
// 如何在个人电脑上运行 180B 级模型", section "稀疏架构创造了机会", gives the step:
// 10 of 512 routed experts plus one shared expert per token.
//
// One CTA per SM: 8 consumer warps and 2 producer warps (unit q is issued by
// producer q mod 2; the slot count is even, so each slot keeps one producer).
// A producer copies each unit of work (a 16-row tile piece of weight codes and
// its scales, with cp.async 16 bytes per lane into rows padded for ldmatrix;
// router rows, and for down tiles their activations, with 1-D bulk copies)
// and the slot's mbarrier completes when every copy has landed. Router units
// and the tiles of phase A are shared by all eight consumer warps; every
// later tile goes to one of four groups of two warps, which split its K; the
// last warp to finish writes the tile's result, and the warps that worked on
// the unit release the slot. Work per CTA, in order:
//   A  router quarter-rows (partial logits to global) and the shared expert's
//      gate/up tiles dealt round-robin over the CTAs;
//      -- grid barrier; every CTA rebuilds the logits, takes the top-k and
//         lists the distinct picked experts in ascending id order --
//   B  the shared expert's down rows this CTA owns, then the routed gate/up
//      tiles dealt round-robin (tile = 8 intermediate rows of gate and of up);
//      -- grid barrier, awaited by the producer only: the down tiles'
//         activations are copied in after it, their weights before it --
//   C  the routed down rows this CTA owns, then the combine of those rows.
//
// Dot products use mma.sync m16n8k16 (fp16 operands, fp32 accumulate) with the
// weights as A (16 rows) and the tokens as the columns of B. A 4-, 2- or 8-bit
// code becomes an exact fp16 value with one lop3 that ORs the code bits under
// a fixed exponent ("magic" value base + c); the K order inside a fragment is
// permuted so each thread dequantises whole 32-bit words, and B is stored in
// the same permuted order. The MMA's cost per weight does not depend on T,
// where fp32 FMAs need one per token per weight.
//   int4 g32: A = (c - 8) per group, scale applied to the group's fp32 result
//             (gate/up: the base + 8 offset is removed through the MMA's C
//             input instead of a subtraction per pair);
//   int2 g16: A = c*s + m in fp16 (one rounding), summed over all groups;
//   int8:     A = q exactly, the row scale applied once at the end.
// The intermediate activations h of the down projection are kept in fp16.
#include <cuda_fp16.h>
#include <math_constants.h>

#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace dks {

constexpr int kCW = 8;                    // consumer warps
constexpr int kProducers = 2;             // producer warps: unit q is issued by warp kCW + q % kProducers
constexpr int kThreads = (kCW + kProducers) * 32;
constexpr int kProducer = kCW;
constexpr int kGroups = 4;               // consumer groups: tile i goes to group i % kGroups
constexpr int kGW = kCW / kGroups;       // warps per group
constexpr int kMaxT = 4;
constexpr int kMaxK = 16;
constexpr int kMaxSlots = 14;
constexpr int kMaxUnits = 384;
constexpr int kSlotBytes = 19456;
constexpr long long kSpin = 2000000000LL;  // ~1 s
constexpr int kSmemLimit = 227 * 1024;

enum : short { kRouter = 0, kGateUp = 1, kDown = 2 };

// One unit of work = one slot load. 16 bytes.
struct Unit {
  short kind, fmt, last, nrows;  // nrows: real rows of a tile (<= 16); router: quarter-rows in the slot
  short e;                       // descriptor index (routed 0..U-1; shared = T*k); router: unused
  short row0;                    // gate/up: first intermediate row; down: first output row; router: first quarter-row
  short k0, kn;                  // K range of this piece
};
static_assert(sizeof(Unit) == 16, "unit record");

__host__ __device__ inline int bits_of(int fmt) {
  return fmt == MOE_Q_INT4_SYM_G32 ? 4 : fmt == MOE_Q_INT2_ASYM_G16 ? 2 : 8;
}
__host__ __device__ inline int group_of(int fmt) {
  return fmt == MOE_Q_INT4_SYM_G32 ? 32 : fmt == MOE_Q_INT2_ASYM_G16 ? 16 : 0;
}
// Round a row length up to 16 bytes and make its 16-byte count odd, so eight
// rows at that stride start in eight different 16-byte bank groups.
__host__ __device__ inline int pad_odd16(int b) {
  const int r = (b + 15) & ~15;
  return ((r >> 4) & 1) ? r : r + 16;
}

// Slot layout of a 16-row tile piece covering K range [k0, k0 + kn).
struct Geo {
  int cb, cs;    // code bytes per row, code row stride
  int ab, as;    // scale (and min) bytes per row, their row stride (int4/int2)
  int aux0;      // scales: 16 rows at stride as (int8: two 16-byte blocks or one <= 48-byte run)
  int aux1;      // mins (int2)
  int bofs;      // activations in fragment order (down tiles)
  int bbytes;
  int bytes;
};
__host__ __device__ inline Geo geo(int fmt, int kn, int T, bool withB) {
  Geo g{};
  g.cb = kn * bits_of(fmt) / 8;
  g.cs = pad_odd16(g.cb);
  int o = 16 * g.cs;
  g.aux0 = o;
  if (fmt == MOE_Q_INT8_PER_CHANNEL) {
    g.ab = 0;
    g.as = 0;
    g.aux1 = o;
    o += 64;
  } else {
    g.ab = kn / group_of(fmt) * 2;
    g.as = pad_odd16(g.ab);
    o += 16 * g.as;
    g.aux1 = o;
    if (fmt == MOE_Q_INT2_ASYM_G16) o += 16 * g.as;
  }
  g.bofs = o;
  g.bbytes = withB ? T * (kn / 16) * 32 : 0;
  g.bytes = o + g.bbytes;
  return g;
}
// Pieces a K-long tile is cut into so one piece fits a slot (0 = none fits).
__host__ __device__ inline int npieces(int fmt, int K, int T, bool withB) {
  for (int np = 1; np <= 8; ++np) {
    if (K % (np * 256)) continue;
    if (geo(fmt, K / np, T, withB).bytes <= kSlotBytes) return np;
  }
  return 0;
}

// Byte offset of activation (k, token t) inside a fragment-ordered buffer for
// weights of format fmt. Per MMA k-step, per token, per thread of a quad: 8
// bytes = (b0, b1), each a pair of fp16, matching how that thread's A pairs
// are cut from its 32-bit code word.
__host__ __device__ inline int frag_off(int fmt, int k, int t, int T) {
  int ks, q, reg, half;
  if (fmt == MOE_Q_INT4_SYM_G32) {  // word = nibbles 8q..8q+7 of a group; pairs (0,4) (1,5) | (2,6) (3,7)
    const int p = k & 31, r = p & 7;
    q = p >> 3;
    ks = 2 * (k >> 5) + ((r & 3) >> 1);
    reg = r & 1;
    half = r >> 2;
  } else if (fmt == MOE_Q_INT2_ASYM_G16) {  // word = group q of a 64-wide chunk; pairs (i, i+8)
    const int p = k & 63, i = p & 15;
    q = p >> 4;
    ks = 4 * (k >> 6) + ((i & 7) >> 1);
    reg = i & 1;
    half = i >> 3;
  } else {  // int8: word = bytes 4q..4q+3 of a k-step; pairs (0,2) (1,3)
    const int p = k & 15, r = p & 3;
    q = p >> 2;
    ks = k >> 4;
    reg = r & 1;
    half = r >> 1;
  }
  return ((ks * T + t) * 4 + q) * 8 + reg * 4 + half * 2;
}
__host__ __device__ inline int frag_bytes(int K, int T) { return (K / 16) * T * 32; }

// Router: quarter-rows of RQ per row, KP floats each.
__host__ __device__ inline int router_rq(int H) { return H >= 1024 ? H / 512 : 1; }

// Shared-memory plan (offsets from the dynamic base).
struct Plan {
  int slots;
  int o_slots, o_x32, o_f0, o_corr, o_y, o_s, o_red, o_units, o_desc, o_bias, total;
};
__host__ __device__ inline Plan make_plan(int T, int H, int E, int k, int slots) {
  Plan p{};
  p.slots = slots;
  int o = 0;
  auto take = [&](int bytes, int al) { o = (o + al - 1) & ~(al - 1); const int r = o; o += bytes; return r; };
  p.o_slots = take(slots * kSlotBytes, 1024);
  const int x32 = 4 * T * (H > E ? H : E);
  p.o_x32 = take(x32 > 4 * T * H ? x32 : 4 * T * H, 128);  // router x, then logits, then two fragment buffers
  p.o_f0 = take(2 * T * H, 128);
  p.o_corr = take(3 * (H / 32) * 16, 16);
  const int U = T * k < E ? T * k : E;
  p.o_y = take(U * 16 * 16, 16);
  p.o_s = take(16 * 16, 16);
  p.o_red = take(slots * kCW * 16 * 16, 16);
  p.o_units = take(kMaxUnits * int(sizeof(Unit)), 16);
  p.o_desc = take((T * k + 1) * int(sizeof(moe_expert)), 16);
  p.o_bias = take(4 * T * E, 16);
  p.total = o;
  return p;
}

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
  float* logits_out;  // [T][E] or null
  uint16_t* out;
  float* partial;   // [T][E][RQ]
  uint8_t* hfrag;   // (T*k + 1) fragment buffers of the down activations
  WsHeader* hdr;
  int slots;
  int np_gu[4], np_dn[4];  // pieces of a gate/up (K = H) and a down (K = I) tile per format
};

// ---------------------------------------------------------------- PTX bits
__device__ __forceinline__ uint32_t lop_or(uint32_t a, uint32_t mask, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));  // (a & mask) | magic
  return d;
}
// ((a ^ 0x80) & 0xFF) | 0x6400 in each half: int8 q -> fp16 1024 + (q + 128).
__device__ __forceinline__ uint32_t lop_i8(uint32_t a) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(0x00FF00FFu), "r"(0x64806480u));
  return d;
}
__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c) {
  const __half2 r = __hfma2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b),
                            *reinterpret_cast<const __half2*>(&c));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1, const float (&c)[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}
__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Arrival counted n times.
__device__ __forceinline__ void mbar_arrive_n(uint32_t bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(n) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory"); }
__device__ __forceinline__ bool test_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ uint32_t h2dup(uint16_t h) { return uint32_t(h) | (uint32_t(h) << 16); }

// ---------------------------------------------------------------- tile math
// This warp's share (16-byte code columns [c0, c1)) of one 16-row piece.
// frag: activations in fragment order for the piece's format, k-step 0 = K 0;
// ks0 = first k-step of the piece. corr (int4 with kCorr): per group, per
// token padded to 4, sum over the group of (base + 8) * x.
template <int F, bool kCorr>
__device__ __forceinline__ void tile_mma(const uint8_t* slot, const Geo& g, int c0, int c1, const uint8_t* frag,
                                         int ks0, const float* corr, int T, float (&acc)[4]) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const bool bval = gq < T;
  const int lm = lane >> 3, lr = lane & 7;
  const uint32_t lrow = ptx::smem_addr(slot) + uint32_t((lr + 8 * (lm & 1)) * g.cs + (lm >> 1) * 16);
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(slot + g.aux0);
  const uint16_t* mn = reinterpret_cast<const uint16_t*>(slot + g.aux1);
  const int asw = g.as >> 1;
#pragma unroll 1
  for (int c = c0; c < c1; c += 2) {
    const bool two = c + 1 < c1;
    uint32_t R[4];
    if (two) ldsm4(lrow + uint32_t(c) * 16u, R[0], R[1], R[2], R[3]);
    else {
      ldsm2(lrow + uint32_t(c) * 16u, R[0], R[1]);
      R[2] = R[3] = 0u;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      if (hh == 1 && !two) break;
      const uint32_t w = R[2 * hh], v = R[2 * hh + 1];
      const int cc = c + hh;
      if (F == MOE_Q_INT4_SYM_G32) {
        const float sg = f16_to_f32(sc[gq * asw + cc]), sg8 = f16_to_f32(sc[(gq + 8) * asw + cc]);
        uint32_t p0 = lop_or(w, 0x000F000Fu, 0x64006400u), p1 = lop_or(w, 0x00F000F0u, 0x54005400u);
        uint32_t q0 = lop_or(v, 0x000F000Fu, 0x64006400u), q1 = lop_or(v, 0x00F000F0u, 0x54005400u);
        const uint32_t w8 = w >> 8, v8 = v >> 8;
        uint32_t p2 = lop_or(w8, 0x000F000Fu, 0x64006400u), p3 = lop_or(w8, 0x00F000F0u, 0x54005400u);
        uint32_t q2 = lop_or(v8, 0x000F000Fu, 0x64006400u), q3 = lop_or(v8, 0x00F000F0u, 0x54005400u);
        float cin[4] = {0.f, 0.f, 0.f, 0.f};
        if (kCorr) {
          const float2 cr = tq < 2 ? *reinterpret_cast<const float2*>(corr + (ks0 / 2 + cc) * 4 + 2 * tq)
                                   : make_float2(0.f, 0.f);
          cin[0] = -cr.x;
          cin[1] = -cr.y;
          cin[2] = -cr.x;
          cin[3] = -cr.y;
        } else {  // c - 8: subtract 1032 (low nibble) or 72 (high nibble, base 64)
          p0 = hsub2u(p0, 0x64086408u);
          q0 = hsub2u(q0, 0x64086408u);
          p2 = hsub2u(p2, 0x64086408u);
          q2 = hsub2u(q2, 0x64086408u);
          p1 = hsub2u(p1, 0x54805480u);
          q1 = hsub2u(q1, 0x54805480u);
          p3 = hsub2u(p3, 0x54805480u);
          q3 = hsub2u(q3, 0x54805480u);
        }
        const int s = ks0 + 2 * cc;
        const uint2 b0 = bval ? lds64(frag + ((s * T + gq) * 4 + tq) * 8) : make_uint2(0u, 0u);
        const uint2 b1 = bval ? lds64(frag + (((s + 1) * T + gq) * 4 + tq) * 8) : make_uint2(0u, 0u);
        float d[4];
        mma16816(d, p0, q0, p1, q1, b0.x, b0.y, cin);
        mma16816(d, p2, q2, p3, q3, b1.x, b1.y, d);
        acc[0] = fmaf(sg, d[0], acc[0]);
        acc[1] = fmaf(sg, d[1], acc[1]);
        acc[2] = fmaf(sg8, d[2], acc[2]);
        acc[3] = fmaf(sg8, d[3], acc[3]);
      } else if (F == MOE_Q_INT8_PER_CHANNEL) {
        const uint32_t a0 = hsub2u(lop_i8(w), 0x64806480u), a2 = hsub2u(lop_i8(w >> 8), 0x64806480u);
        const uint32_t a1 = hsub2u(lop_i8(v), 0x64806480u), a3 = hsub2u(lop_i8(v >> 8), 0x64806480u);
        const int s = ks0 + cc;
        const uint2 b = bval ? lds64(frag + ((s * T + gq) * 4 + tq) * 8) : make_uint2(0u, 0u);
        mma16816(acc, a0, a1, a2, a3, b.x, b.y, acc);
      } else {  // int2: A = c*s + m, one rounding
        const int gi = 4 * cc + tq;
        const uint32_t s2 = h2dup(sc[gq * asw + gi]), m2 = h2dup(mn[gq * asw + gi]);
        const uint32_t s28 = h2dup(sc[(gq + 8) * asw + gi]), m28 = h2dup(mn[(gq + 8) * asw + gi]);
        uint32_t A[8], B[8];
        const uint32_t w8 = w >> 8, v8 = v >> 8;
        A[0] = hfma2u(hsub2u(lop_or(w, 0x00030003u, 0x64006400u), 0x64006400u), s2, m2);
        A[1] = hfma2u(hsub2u(lop_or(w, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u), s2, m2);
        A[2] = hfma2u(hsub2u(lop_or(w, 0x00300030u, 0x54005400u), 0x54005400u), s2, m2);
        A[3] = hfma2u(hsub2u(lop_or(w, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u), s2, m2);
        A[4] = hfma2u(hsub2u(lop_or(w, 0x03000300u, 0x44004400u), 0x44004400u), s2, m2);
        A[5] = hfma2u(hsub2u(lop_or(w8, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u), s2, m2);
        A[6] = hfma2u(hsub2u(lop_or(w8, 0x00300030u, 0x54005400u), 0x54005400u), s2, m2);
        A[7] = hfma2u(hsub2u(lop_or(w8, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u), s2, m2);
        B[0] = hfma2u(hsub2u(lop_or(v, 0x00030003u, 0x64006400u), 0x64006400u), s28, m28);
        B[1] = hfma2u(hsub2u(lop_or(v, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u), s28, m28);
        B[2] = hfma2u(hsub2u(lop_or(v, 0x00300030u, 0x54005400u), 0x54005400u), s28, m28);
        B[3] = hfma2u(hsub2u(lop_or(v, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u), s28, m28);
        B[4] = hfma2u(hsub2u(lop_or(v, 0x03000300u, 0x44004400u), 0x44004400u), s28, m28);
        B[5] = hfma2u(hsub2u(lop_or(v8, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u), s28, m28);
        B[6] = hfma2u(hsub2u(lop_or(v8, 0x00300030u, 0x54005400u), 0x54005400u), s28, m28);
        B[7] = hfma2u(hsub2u(lop_or(v8, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u), s28, m28);
        const int s = ks0 + 4 * cc;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint2 b = bval ? lds64(frag + (((s + j) * T + gq) * 4 + tq) * 8) : make_uint2(0u, 0u);
          mma16816(acc, A[2 * j], B[2 * j], A[2 * j + 1], B[2 * j + 1], b.x, b.y, acc);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- top-k keys
__device__ __forceinline__ uint32_t f2key(float f) {
  if (f != f) f = -CUDART_INF_F;  // NaN loses to every number
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Best k (k <= 16) of up to 128 candidates held 4 per lane, each packed as
// key << 32 | ~id so that a larger value is a better candidate (key desc, id
// asc); 0 = no candidate. Each lane sorts its four (five compare-exchanges);
// each of the k rounds takes the best lane head (a reduction on the key, one
// on the low word among equal keys) and the winning lane pops it. A missing
// pick reads key 0, id INT_MAX. One small instantiation: code that runs once
// per launch pays an instruction-cache miss per line.
__device__ __forceinline__ void cx(uint64_t& a, uint64_t& b) {
  const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
  a = hi;
  b = lo;
}
__device__ __forceinline__ void warp_topk4(uint64_t (&c)[4], int k, uint32_t* okey, int* oid) {
  const int lane = threadIdx.x & 31;
  cx(c[0], c[1]);
  cx(c[2], c[3]);
  cx(c[0], c[2]);
  cx(c[1], c[3]);
  cx(c[1], c[2]);
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    const uint32_t bk = uint32_t(c[0] >> 32), bl = uint32_t(c[0]);
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t wl = __reduce_max_sync(0xffffffffu, bk == wk ? bl : 0u);
    if (lane == 0) {
      okey[j] = wk;
      oid[j] = wk ? int(~wl) : 0x7fffffff;
    }
    if (wk != 0u && bk == wk && bl == wl) {
      c[0] = c[1];
      c[1] = c[2];
      c[2] = c[3];
      c[3] = 0ull;
    }
  }
}

// ---------------------------------------------------------------- the kernel
// Slot protocol: full[s] completes after 33 arrivals: one cp.async-tracked
// arrival per producer lane (its weight copies landed) plus one more, made
// right away for units without activations and, for down units, by the bulk
// copy of their activations once the barrier they need has passed. empty[s]
// completes after 8 arrivals: one per consumer warp for shared units, or kCW /
// kGW from each warp of the group that owns a tile.
constexpr int kFullCount = 33;

struct Ctx {
  const Params* P;
  uint8_t* slots;
  Unit* units;
  moe_expert* desc;
  uint64_t* full;
  uint64_t* empty;
  int S;         // slot count
  int n0, nr;    // output rows this CTA owns
  int RQ, KP, nper;
  int kShared;   // descriptor index of the shared expert
  const Geo* geo;  // [2][4]: slot layout of a gate/up (0) or down (1) piece per format
  volatile int* issued;  // [kProducers]: one past the last unit each producer has taken a slot for
  __device__ uint8_t* slot(int q) const { return slots + (q % S) * kSlotBytes; }
  __device__ uint32_t full_bar(int q) const { return ptx::smem_addr(&full[q % S]); }
  __device__ uint32_t empty_bar(int q) const { return ptx::smem_addr(&empty[q % S]); }
};

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on `bar` once this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// 16-byte int8 row-scale run covering rows [row0, row0 + n).
__device__ __forceinline__ void i8_scale_run(int row0, int n, int& lo, int& hi) {
  lo = (row0 & ~7) * 2;
  hi = ((row0 + n) * 2 + 15) & ~15;
}

// All producer lanes: rows (<= 16) x bytes (multiple of 16) into shared rows
// at `stride`. Lanes are split over the rows (2 lanes per row for up to 16
// rows, 4 for up to 8, ...), each walking every lpr-th 16-byte chunk of its
// row; row r is read from a + r * rs for r < split, else b + (r - split) * rs.
__device__ __forceinline__ void copy_rows(uint32_t dst, int stride, int rows, int bytes, const uint8_t* a,
                                          const uint8_t* b, int split, size_t rs) {
  const int lane = threadIdx.x & 31;
  const int lpr = rows > 8 ? 2 : rows > 4 ? 4 : rows > 2 ? 8 : rows > 1 ? 16 : 32;  // lanes per row
  const int r = lane / lpr, part = lane - r * lpr;
  if (r >= rows) return;
  const uint8_t* src = (r < split ? a + size_t(r) * rs : b + size_t(r - split) * rs) + part * 16;
  uint32_t d = dst + uint32_t(r * stride + part * 16);
  const int n = ((bytes >> 4) - part + lpr - 1) / lpr;  // chunks of this lane
  const int step = lpr * 16;
  int i = 0;
#pragma unroll 1
  for (; i + 4 <= n; i += 4) {
    cp16(d, src);
    cp16(d + step, src + step);
    cp16(d + 2 * step, src + 2 * step);
    cp16(d + 3 * step, src + 3 * step);
    d += 4 * step;
    src += 4 * step;
  }
  for (; i < n; ++i) {
    cp16(d, src);
    d += step;
    src += step;
  }
}

// Producer warp: the weight copies of unit u into its slot.
__device__ __forceinline__ void issue_weights(const Ctx& C, const Unit& u, uint8_t* slot, uint32_t bar) {
  const Params& P = *C.P;
  const uint32_t base = ptx::smem_addr(slot);
  if (u.kind == kRouter) {
    // consecutive quarter-rows are one contiguous run: one bulk copy, and
    // lane 0's arrival on the slot carries its byte count
    if ((threadIdx.x & 31) == 0) {
      const uint32_t bytes = uint32_t(u.nrows * C.KP * 4);
      ptx::mbar_arrive_expect_tx(bar, bytes);
      ptx::bulk_g2s(base, P.w_router + size_t(u.row0) * C.KP, bytes, bar);
    }
    return;
  }
  const bool gu = u.kind == kGateUp;
  const Geo& g = C.geo[(!gu) * 4 + u.fmt];
  const moe_expert& d = C.desc[u.e];
  const moe_qmatrix& m0 = gu ? d.gate : d.down;
  const moe_qmatrix& m1 = gu ? d.up : d.down;
  const int K = gu ? P.H : P.I;
  const int bits = bits_of(u.fmt);
  const size_t rowb = size_t(K) * bits / 8, k0b = size_t(u.k0) * bits / 8;
  const int rows = gu ? 16 : u.nrows, split = gu ? 8 : 16;
  copy_rows(base, g.cs, rows, g.cb, m0.codes + size_t(u.row0) * rowb + k0b, m1.codes + size_t(u.row0) * rowb + k0b,
            split, rowb);
  if (u.fmt == MOE_Q_INT8_PER_CHANNEL) {
    const int lane = threadIdx.x & 31;
    if (gu) {
      if (lane < 2)
        cp16(base + g.aux0 + 16 * lane,
             reinterpret_cast<const uint8_t*>(lane ? m1.scales : m0.scales) + size_t(u.row0) * 2);
    } else {
      int lo, hi;
      i8_scale_run(u.row0, u.nrows, lo, hi);
      if (lane * 16 < hi - lo) cp16(base + g.aux0 + 16 * lane, reinterpret_cast<const uint8_t*>(m0.scales) + lo + 16 * lane);
    }
    return;
  }
  const int grp = group_of(u.fmt);
  const size_t srow = size_t(K / grp) * 2, sk0 = size_t(u.k0 / grp) * 2;
  const uint8_t* s0 = reinterpret_cast<const uint8_t*>(m0.scales) + size_t(u.row0) * srow + sk0;
  const uint8_t* s1 = reinterpret_cast<const uint8_t*>(m1.scales) + size_t(u.row0) * srow + sk0;
  copy_rows(base + g.aux0, g.as, rows, g.ab, s0, s1, split, srow);
  if (u.fmt == MOE_Q_INT2_ASYM_G16) {
    const uint8_t* n0 = reinterpret_cast<const uint8_t*>(m0.mins) + size_t(u.row0) * srow + sk0;
    const uint8_t* n1 = reinterpret_cast<const uint8_t*>(m1.mins) + size_t(u.row0) * srow + sk0;
    copy_rows(base + g.aux1, g.as, rows, g.ab, n0, n1, split, srow);
  }
}

// Producer lane 0: a down unit's activations (fragment order), the slot's
// last arrival.
__device__ __forceinline__ void issue_acts(const Ctx& C, const Unit& u, uint8_t* slot, uint32_t bar) {
  const Params& P = *C.P;
  const Geo& g = C.geo[4 + u.fmt];
  const uint8_t* src = P.hfrag + size_t(u.e) * frag_bytes(P.I, P.T) + size_t(u.k0 / 16) * P.T * 32;
  ptx::mbar_arrive_expect_tx(bar, uint32_t(g.bbytes));
  ptx::bulk_g2s(ptx::smem_addr(slot + g.bofs), src, uint32_t(g.bbytes), bar);
}

__device__ __forceinline__ void router_range(const Params& P, int RQ, int b, int G, int& u0, int& u1) {
  const int n = P.E * RQ, q = n / G, r = n % G;
  u0 = b * q + (b < r ? b : r);
  u1 = u0 + q + (b < r ? 1 : 0);
}

__device__ __forceinline__ Unit router_unit(const Ctx& C, int u0, int u1, int i) {
  Unit x{};
  x.kind = kRouter;
  x.row0 = short(u0 + i * C.nper);
  x.nrows = short(min(C.nper, u1 - (u0 + i * C.nper)));
  x.last = 1;
  return x;
}

__device__ __forceinline__ int gateup_pieces(const Params& P, int fmt, int e, int i0, Unit* out) {
  const int np = P.np_gu[fmt];
  const int kn = P.H / np;
  for (int p = 0; p < np; ++p) {
    Unit x{};
    x.kind = kGateUp;
    x.fmt = short(fmt);
    x.e = short(e);
    x.row0 = short(i0);
    x.nrows = 16;
    x.k0 = short(p * kn);
    x.kn = short(kn);
    x.last = short(p == np - 1);
    out[p] = x;
  }
  return np;
}

__device__ __forceinline__ int down_pieces(const Params& P, int fmt, int e, int n0, int nr, Unit* out) {
  const int np = P.np_dn[fmt];
  const int kn = P.I / np;
  for (int p = 0; p < np; ++p) {
    Unit x{};
    x.kind = kDown;
    x.fmt = short(fmt);
    x.e = short(e);
    x.row0 = short(n0);
    x.nrows = short(nr);
    x.k0 = short(p * kn);
    x.kn = short(kn);
    x.last = short(p == np - 1);
    out[p] = x;
  }
  return np;
}

// The tokens' activations in fragment order for weights of format fmt, read
// from the bf16 input (consumer warps; one warp per 32-wide group and token,
// one element per lane). int4 also gets its corrections: corr[G][t] = sum over
// group G of (base + 8) * x, base 1024 at even positions (low nibbles) and 64
// at odd ones; tokens padded to 4 with zeros.
__device__ __forceinline__ void build_frag(const Params& P, int fmt, uint8_t* frag, float* corr) {
  const int T = P.T, H = P.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool i4 = fmt == MOE_Q_INT4_SYM_G32;
  if (i4)
    for (int i = threadIdx.x; i < (H / 32) * (4 - T); i += kCW * 32) corr[(i / (4 - T)) * 4 + T + i % (4 - T)] = 0.f;
#pragma unroll 1
  for (int gt = warp; gt < (H / 32) * T; gt += kCW) {
    const int G = gt / T, t = gt - G * T;
    const int kk = 32 * G + lane;
    const __half hv = __float2half_rn(bf16_to_f32(P.x[t * H + kk]));
    *reinterpret_cast<__half*>(frag + frag_off(fmt, kk, t, T)) = hv;
    if (i4) {
      const float s = warp_sum(((lane & 1) ? 72.f : 1032.f) * __half2float(hv));
      if (lane == 0) corr[G * 4 + t] = s;
    }
  }
}

// Bounded wait of all lanes of a consumer warp on a slot's full barrier.
__device__ __forceinline__ bool wait_full(const Ctx& C, int q, WsHeader* hdr) {
  // A group that skips the other group's tiles can run a ring ahead, where
  // the slot's phase parity would match an older, completed phase: first
  // wait until the producer of unit q has taken its slot.
  volatile int* iss = C.issued + q % kProducers;
  if (*iss <= q) {
    const long long t0 = clock64();
    while (*iss <= q) {
      __nanosleep(32);
      if (*reinterpret_cast<volatile int*>(&hdr->abort) || clock64() - t0 > kSpin) {
        if (!hdr->abort) flag_error(hdr, MOE_ERR_TIMEOUT, 3500000 + q);
        atomicExch(&hdr->abort, 1);
        return false;
      }
    }
  }
  if (ptx::mbar_wait(C.full_bar(q), uint32_t((q / C.S) & 1), &hdr->abort)) return true;
  if (!hdr->abort) flag_error(hdr, MOE_ERR_TIMEOUT, 3000000 + q);
  atomicExch(&hdr->abort, 1);
  return false;
}

// Sum of a group's partials of one tile, in warp order.
__device__ __forceinline__ float red_sum(const float* rs, int r, int t, int nw) {
  float v = 0.f;
#pragma unroll 1
  for (int w = 0; w < nw; ++w) v += rs[w * 64 + r * 4 + t];
  return v;
}

// One consumer warp's part of a router slot: quarter-row `warp` of the slot.
__device__ __forceinline__ void router_unit_dot(const Ctx& C, const Unit& u, const uint8_t* slot, const float* x32) {
  const Params& P = *C.P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= u.nrows) return;
  const int T = P.T, H = P.H, E = P.E;
  const int uq = u.row0 + warp, e = uq / C.RQ, q = uq - e * C.RQ;
  const float4* W4 = reinterpret_cast<const float4*>(slot + warp * C.KP * 4);
  float a[kMaxT] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
  for (int c = 0; c < C.KP / 128; ++c) {
    const float4 w = W4[lane + 32 * c];
#pragma unroll
    for (int t = 0; t < kMaxT; ++t)
      if (t < T) {
        const float4 xv = *reinterpret_cast<const float4*>(x32 + t * H + q * C.KP + 4 * (lane + 32 * c));
        a[t] = fmaf(w.x, xv.x, fmaf(w.y, xv.y, fmaf(w.z, xv.z, fmaf(w.w, xv.w, a[t]))));
      }
  }
#pragma unroll
  for (int t = 0; t < kMaxT; ++t)
    if (t < T) {
      const float sum = warp_sum(a[t]);
      if (lane == 0) P.partial[(size_t(t) * E + e) * C.RQ + q] = sum;
    }
}

// Producer state (lane 0 owns the bookkeeping; all lanes issue copies).
struct Producer {
  const Ctx& C;
  WsHeader* hdr;
  int G;
  int p;  // this producer's units are those with q % kProducers == p
  int bq = 0;       // next unit whose activations may still be due
  bool b1 = false;  // barrier 1 passed (shared down activations exist)
  bool b2 = false;  // barrier 2 passed (routed down activations exist)

  // lane 0: the activations of every issued down unit whose barrier passed.
  __device__ __forceinline__ void pump(int issued) {
    while (bq < issued) {
      const Unit& u = C.units[bq];
      if (bq % kProducers == p && u.kind == kDown) {
        const bool ready = u.e == C.kShared ? b1 : b2;
        if (!ready) break;
        issue_acts(C, u, C.slot(bq), C.full_bar(bq));
      }
      ++bq;
    }
  }
  __device__ __forceinline__ void poll_b2(int issued) {
    if (!b2 && bq < issued && ld_acquire_u32(&hdr->bar_count) >= uint32_t(2 * G)) {
      b2 = true;
      fence_proxy_async_global();
      pump(issued);
    }
  }
  // lane 0: wait until the slot of unit q is free (bounded), pumping meanwhile.
  __device__ __forceinline__ bool wait_empty(int q) {
    if (q < C.S) return true;
    const uint32_t bar = C.empty_bar(q), par = uint32_t(((q / C.S) - 1) & 1);
    const long long t0 = clock64();
    for (uint32_t it = 0;; ++it) {
      if (test_wait(bar, par)) return true;
      poll_b2(q);
      __nanosleep(64);
      if ((it & 15) == 15 && *reinterpret_cast<volatile int*>(&hdr->abort)) return false;
      if (clock64() - t0 > kSpin) {
        flag_error(hdr, MOE_ERR_TIMEOUT, 4000000 + q);
        atomicExch(&hdr->abort, 1);
        return false;
      }
    }
  }
  // all lanes: unit q into its slot. Returns false after an expired wait.
  __device__ __forceinline__ bool issue(int q) {
    const int lane = threadIdx.x & 31;
    int good = 1;
    if (lane == 0) {
      good = wait_empty(q);
      if (good) C.issued[p] = q + 1;  // unit q's full phase is now its slot's current one
    }
    good = __shfl_sync(0xffffffffu, good, 0);
    if (!good) return false;
    // The second barrier's count, loaded before the copies are issued and
    // looked at after them, so its latency hides behind them: activations
    // are due as soon as the barrier passes, not when a slot next runs out.
    uint32_t seen = 0;
    if (lane == 0 && !b2) seen = ld_relaxed_u32(&hdr->bar_count);
    const Unit u = C.units[q];
    issue_weights(C, u, C.slot(q), C.full_bar(q));
    cp_arrive(C.full_bar(q));
    __syncwarp();
    if (lane == 0) {
      if (u.kind == kGateUp) ptx::mbar_arrive(C.full_bar(q));  // router: arrived with its copy
      if (!b2 && seen >= uint32_t(2 * G)) {
        b2 = true;
        asm volatile("fence.acq_rel.gpu;" ::: "memory");  // the relaxed read above, made an acquire
        fence_proxy_async_global();
      }
      pump(q + 1);
    }
    return true;
  }
  // lane 0: wait for barrier 2 while activations are still due.
  __device__ __forceinline__ void finish(int issued) {
    const long long t0 = clock64();
    for (uint32_t it = 0; bq < issued && !b2; ++it) {
      poll_b2(issued);
      if (b2) break;
      __nanosleep(64);
      if ((it & 15) == 15 && *reinterpret_cast<volatile int*>(&hdr->abort)) return;
      if (clock64() - t0 > kSpin) {
        flag_error(hdr, MOE_ERR_TIMEOUT, 5000000);
        atomicExch(&hdr->abort, 1);
        return;
      }
    }
    pump(issued);
  }
};

__global__ void __launch_bounds__(kThreads, 1) decode_stream_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t s_full[kMaxSlots];
  __shared__ __align__(8) uint64_t s_empty[kMaxSlots];
  __shared__ int s_cnt[kMaxSlots];
  __shared__ Geo s_geo[8];
  __shared__ int s_nA, s_nSD, s_nB, s_nC, s_U, s_bad, s_fail;
  __shared__ volatile int s_issued[kProducers];
  __shared__ int s_fmap[4];  // weight format -> fragment buffer
  __shared__ int s_uniq[kMaxT * kMaxK];
  __shared__ int s_slotmap[kMaxT * kMaxK];
  __shared__ uint32_t s_bits[kMaxE / 32];
  __shared__ uint32_t s_bpre[kMaxE / 32];
  __shared__ int s_idx[kMaxT * kMaxK];
  __shared__ float s_w[kMaxT * kMaxK];
  __shared__ uint32_t s_key[kMaxT * kMaxK];
  __shared__ uint32_t s_ck[kMaxT * kCW * kMaxK];
  __shared__ int s_ci[kMaxT * kCW * kMaxK];

  const int T = P.T, H = P.H, I = P.I, E = P.E, k = P.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  WsHeader* hdr = P.hdr;
  const Plan L = make_plan(T, H, E, k, P.slots);
  const bool has_shared = P.shared != nullptr;

  Ctx C;
  C.P = &P;
  C.slots = smem + L.o_slots;
  C.units = reinterpret_cast<Unit*>(smem + L.o_units);
  C.desc = reinterpret_cast<moe_expert*>(smem + L.o_desc);
  C.full = s_full;
  C.empty = s_empty;
  C.S = P.slots;
  {
    const int q = H / G, r = H % G;
    C.n0 = b * q + (b < r ? b : r);
    C.nr = q + (b < r ? 1 : 0);
  }
  C.RQ = router_rq(H);
  C.KP = H / C.RQ;
  C.nper = min(kCW, kSlotBytes / (C.KP * 4));
  C.kShared = T * k;
  C.geo = s_geo;
  C.issued = s_issued;
  if (threadIdx.x < 8) {
    const int dn = threadIdx.x >> 2, f = threadIdx.x & 3;
    const int np = f == 0 ? 1 : (dn ? P.np_dn[f] : P.np_gu[f]);
    s_geo[threadIdx.x] = f == 0 || np == 0 ? Geo{} : geo(f, (dn ? I : H) / np, T, dn != 0);
  }
  float* x32 = reinterpret_cast<float*>(smem + L.o_x32);
  uint8_t* f0 = smem + L.o_f0;
  float* corr = reinterpret_cast<float*>(smem + L.o_corr);
  float* Y = reinterpret_cast<float*>(smem + L.o_y);
  float* Sy = reinterpret_cast<float*>(smem + L.o_s);
  float* red = reinterpret_cast<float*>(smem + L.o_red);
  int u0, u1;
  router_range(P, C.RQ, b, G, u0, u1);
  const int nR = (u1 - u0 + C.nper - 1) / C.nper;

  if (threadIdx.x == 0) {
    s_bad = 0;
    s_fail = 0;
    s_U = 0;
    s_nB = 0;
    s_nC = 0;
    for (int i = 0; i < 4; ++i) s_fmap[i] = -1;
  }
  if (threadIdx.x < kMaxSlots) s_cnt[threadIdx.x] = 0;

  // ---------------------------------------------------------- start
  if (warp > kProducer) {
    // the second producer warp has nothing to do before S1
  } else if (warp == kProducer) {
    // mbarriers, then the router loads before anything else (the consumers
    // list the same units in the same order).
    if (lane == 0) {
      for (int i = 0; i < C.S; ++i) {
        ptx::mbar_init(ptx::smem_addr(&s_full[i]), kFullCount);
        ptx::mbar_init(ptx::smem_addr(&s_empty[i]), kCW);
      }
      ptx::mbar_init_fence();
    }
    __syncwarp();
    for (int i = 0; i < nR && i < C.S; ++i) {
      const Unit u = router_unit(C, u0, u1, i);
      issue_weights(C, u, C.slot(i), C.full_bar(i));
      cp_arrive(C.full_bar(i));
      __syncwarp();
      // (router units: lane 0 arrived with the copy's byte count)
    }
    if (lane == 0)
      for (int p = 0; p < kProducers; ++p) s_issued[p] = nR < C.S ? nR : C.S;
  } else {
    if (threadIdx.x == 32) {  // the routed descriptors into L2 for after the top-k
      const uintptr_t a = reinterpret_cast<uintptr_t>(P.experts) & ~uintptr_t(15);
      const uintptr_t e = (reinterpret_cast<uintptr_t>(P.experts + E) + 15) & ~uintptr_t(15);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(uint32_t(e - a)) : "memory");
    }
    if (has_shared && threadIdx.x < int(sizeof(moe_expert) / 4))
      reinterpret_cast<uint32_t*>(C.desc + C.kShared)[threadIdx.x] =
          reinterpret_cast<const uint32_t*>(P.shared)[threadIdx.x];
    for (int i = threadIdx.x; i < T * H; i += kCW * 32) x32[i] = bf16_to_f32(P.x[i]);
    {  // the router bias, read after the barrier
      float* bs = reinterpret_cast<float*>(smem + L.o_bias);
      for (int i = threadIdx.x; i < T * E; i += kCW * 32) {
        const int t = i / E, e = i - t * E;
        bs[i] = P.bias ? P.bias[t * P.bstride + e] : 0.f;
      }
    }
    consumer_sync();
    if (threadIdx.x == 0) {
      int n = 0;
      for (int i = 0; i < nR; ++i) C.units[n++] = router_unit(C, u0, u1, i);
      int nsd = 0;
      if (has_shared) {
        const moe_expert& sd = C.desc[C.kShared];
        const int f = sd.gate.qtype;
        const bool good = expert_ok(sd, H, I) && P.np_gu[f & 3] > 0 && P.np_dn[f & 3] > 0;
        if (!good) {
          s_bad = 1;
          flag_error(hdr, MOE_ERR_DEVICE_FAULT, 2000000);
        } else {
          for (int j = b; j < I / 8; j += G) n += gateup_pieces(P, f, C.kShared, 8 * j, C.units + n);
          if (C.nr > 0) nsd = down_pieces(P, f, C.kShared, C.n0, C.nr, C.units + n);
        }
      }
      s_nA = n;
      s_nSD = nsd;
    }
  }
  __syncthreads();  // S1: phase-A list ready
  const int nA = s_nA, nSD = s_nSD;

  if (warp >= kProducer) {
    // ------------------------------------------------ producers: unit q is issued by warp kCW + q % kProducers
    // (the slot count is a multiple of kProducers, so each slot is only ever
    // filled by one producer warp, in order: a slot's phases never run more
    // than one ahead of its producer's waits)
    const int pw = warp - kProducer;
    Producer PR{C, hdr, G, pw};
    const int q0 = nR < C.S ? nR : C.S;
    int q = q0 + (pw - q0 % kProducers + kProducers) % kProducers;  // the first own unit from q0 on
    int total = nA + nSD;
    bool ok = true, s2 = false;
    for (;; q += kProducers) {
      if (!s2 && q >= nA + nSD) {
        __syncthreads();  // S2: routed lists ready, barrier 1 passed
        s2 = true;
        total = nA + nSD + s_nB + s_nC;
        if (lane == 0) {
          fence_proxy_async_global();
          PR.b1 = true;
          PR.pump(q);
        }
      }
      if (q >= total) break;
      if (ok) ok = PR.issue(q);
    }
    if (lane == 0 && ok) PR.finish(total);
    __syncwarp();
  } else {
    // ------------------------------------------------ consumers: one pass over all units
    // Every consumer thread passes every barrier below exactly once, in the
    // same order; after an expired wait a warp stops working (dead) but keeps
    // walking the unit indices so the barriers still line up.
    int total = nA + nSD;
    bool dead = false;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int grp = warp / kGW, gw = warp % kGW;  // consumer group, warp within it
    int ti = -1;  // index of the current tile (the same count on every warp)
    for (int q = 0;; ++q) {
      if (q == nR) {
        // the shared expert's activations in fragment order (buffer 0), once
        // the router rows (already in flight) have been consumed
        if (has_shared && !s_bad) {
          const int f = C.desc[C.kShared].gate.qtype;
          build_frag(P, f, f0, corr);
          if (threadIdx.x == 0) s_fmap[f] = 0;
        }
        consumer_sync();
      }
      if (q == nA) {
        // ---------------------------------------- barrier 1, top-k, routed lists
        consumer_sync();  // every warp's phase-A results are written
        if (threadIdx.x == 0) {
          if (!s_fail) {
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&hdr->bar_count) : "memory");
            const long long t0 = clock64();
            for (uint32_t it = 1; ld_acquire_u32(&hdr->bar_count) < uint32_t(G); ++it) {
              if ((it & 31) == 0 && *reinterpret_cast<volatile int*>(&hdr->abort)) {
                s_fail = 1;
                break;
              }
              if (clock64() - t0 > kSpin) {
                flag_error(hdr, MOE_ERR_TIMEOUT, int(G));
                atomicExch(&hdr->abort, 1);
                s_fail = 1;
                break;
              }
            }
          } else {
            atomicExch(&hdr->abort, 1);
          }
        }
        consumer_sync();
        const bool live = !s_fail;
        float* lg = x32;  // the router activations are no longer needed
        if (live) {
          // eight of this thread's partial loads in flight at once
          const float* bs = reinterpret_cast<const float*>(smem + L.o_bias);
          constexpr int kPer = 8;
#pragma unroll 1
          for (int i0 = threadIdx.x; i0 < T * E; i0 += kPer * kCW * 32) {
            float v[kPer];
            if (C.RQ == 4) {
#pragma unroll
              for (int j = 0; j < kPer; ++j) {
                const int i = i0 + j * kCW * 32;
                if (i < T * E) {
                  const float4 p4 = __ldcg(reinterpret_cast<const float4*>(P.partial) + i);
                  v[j] = (p4.x + p4.y) + (p4.z + p4.w);
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < kPer; ++j) {
                const int i = i0 + j * kCW * 32;
                if (i < T * E) {
                  const float* pp = P.partial + size_t(i) * C.RQ;
                  float a = __ldcg(pp);
                  for (int qq = 1; qq < C.RQ; ++qq) a += __ldcg(pp + qq);
                  v[j] = a;
                }
              }
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
              const int i = i0 + j * kCW * 32;
              if (i < T * E) lg[i] = v[j] + bs[i];
            }
          }
        }
        consumer_sync();
        // two rounds of warp top-k: first one job per (token, 128 logits), the
        // jobs dealt over the warps, each keeping its chunk's best k; then one
        // warp per token over those picks (at most 8 chunks x 16 = 128)
        const int nch = (E + 127) >> 7;
#pragma unroll 1
        for (int stage = 0; stage < 2; ++stage) {
          const int njobs = live ? (stage == 0 ? T * nch : T) : 0;
#pragma unroll 1
          for (int job = warp; job < njobs; job += kCW) {
            const int t = stage == 0 ? job / nch : job, ch = stage == 0 ? job - t * nch : 0;
            const int nc = stage == 0 ? min(128, E - (ch << 7)) : nch * k;
            const uint32_t* ck = s_ck + t * kCW * kMaxK;
            const int* ci = s_ci + t * kCW * kMaxK;
            uint64_t cand[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int c = lane + 32 * i;
              const uint32_t key = c >= nc ? 0u : stage == 0 ? f2key(lg[t * E + (ch << 7) + c]) : ck[c];
              const int id = stage == 0 ? (ch << 7) + c : ci[c < nc ? c : 0];
              cand[i] = key ? (uint64_t(key) << 32) | uint64_t(~uint32_t(id)) : 0ull;
            }
            uint32_t* okey = stage == 0 ? s_ck + t * kCW * kMaxK + ch * k : s_key + t * k;
            int* oid = stage == 0 ? s_ci + t * kCW * kMaxK + ch * k : s_idx + t * k;
            warp_topk4(cand, k, okey, oid);
          }
          consumer_sync();
        }
        if (live && warp < T) {
          const int t = warp;
          __syncwarp();
          // renormalised softmax over the picks
          const float v0 = key2f(s_key[t * k]);
          float part = 0.f;
          for (int j = lane; j < k; j += 32) part += expf(key2f(s_key[t * k + j]) - v0);
          const float den = warp_sum(part);
          for (int j = lane; j < k; j += 32) s_w[t * k + j] = expf(key2f(s_key[t * k + j]) - v0) / den;
        }
        // distinct picked experts, ascending, through a bitmap of expert ids:
        // rank of an id = set bits below it
        const int nk = T * k;
        if (threadIdx.x < kMaxE / 32) s_bits[threadIdx.x] = 0u;
        consumer_sync();
        if (live && threadIdx.x < nk) atomicOr(&s_bits[s_idx[threadIdx.x] >> 5], 1u << (s_idx[threadIdx.x] & 31));
        consumer_sync();
        if (warp == 0) {
          uint32_t pre = 0;
#pragma unroll
          for (int i = 0; i < kMaxE / 32 / 32; ++i) {
            const uint32_t c = __popc(s_bits[i * 32 + lane]);
            uint32_t inc = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
              if (lane >= o) inc += y;
            }
            s_bpre[i * 32 + lane] = pre + inc - c;
            pre += __shfl_sync(0xffffffffu, inc, 31);
          }
          if (lane == 0) s_U = int(pre);
        }
        consumer_sync();
        if (live && threadIdx.x < nk) {
          const int id = s_idx[threadIdx.x], w = id >> 5;
          const int rank = int(s_bpre[w] + __popc(s_bits[w] & ((1u << (id & 31)) - 1u)));
          s_slotmap[threadIdx.x] = rank;
          s_uniq[rank] = id;
        }
        consumer_sync();
        const int U = s_U;
        if (live) {
          constexpr int W = int(sizeof(moe_expert) / 4);
          const uint32_t* src = reinterpret_cast<const uint32_t*>(P.experts);
          uint32_t* dst = reinterpret_cast<uint32_t*>(C.desc);
          for (int i = threadIdx.x; i < U * W; i += kCW * 32) {
            const int id = s_uniq[i / W];
            dst[i] = (id >= 0 && id < E) ? src[size_t(id) * W + (i % W)] : 0u;
          }
          if (b == 0) {
            for (int i = threadIdx.x; i < nk; i += kCW * 32) {
              P.topk_idx[i] = s_idx[i];
              P.topk_w[i] = s_w[i];
            }
            if (P.logits_out)
              for (int i = threadIdx.x; i < T * E; i += kCW * 32) P.logits_out[i] = lg[i];
          }
        }
        consumer_sync();
        // validate the picked experts' descriptors (one thread per expert)
        if (live && threadIdx.x < U) {
          const moe_expert& d = C.desc[threadIdx.x];
          const int f = d.gate.qtype, id = s_uniq[threadIdx.x];
          if (id < 0 || id >= E || !expert_ok(d, H, I) || P.np_gu[f & 3] == 0 || P.np_dn[f & 3] == 0) s_bad = 1;
        }
        consumer_sync();
        if (live && !s_bad && warp == 0) {
          // formats -> fragment buffers (the shared expert's format already has 0)
          {
            const int fa = lane < U ? C.desc[lane].gate.qtype : 0;
            const int fb = lane + 32 < U ? C.desc[lane + 32].gate.qtype : 0;
            int next = 1;
            for (int f = 1; f <= 3; ++f) {
              const bool used = __any_sync(0xffffffffu, fa == f || fb == f);
              if (used && s_fmap[f] < 0) {
                if (lane == 0) s_fmap[f] = next;
                ++next;
              }
            }
          }
          // routed gate/up jobs b, b + G, ... (8 intermediate rows each), then
          // this CTA's down rows of every picked expert; offsets by warp scan
          Unit* out = C.units + nA + nSD;
          const int J = U * (I / 8);
          int n = 0;
          for (int m0 = 0; b + m0 * G < J; m0 += 32) {
            const int j = b + (m0 + lane) * G;
            const bool v = j < J;
            const int u = v ? j / (I / 8) : 0;
            const int f = v ? C.desc[u].gate.qtype : 0;
            const int np = v ? P.np_gu[f] : 0;
            int inc = np;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(0xffffffffu, inc, o);
              if (lane >= o) inc += y;
            }
            if (v && n + inc <= kMaxUnits / 2) gateup_pieces(P, f, u, (j % (I / 8)) * 8, out + n + inc - np);
            n += __shfl_sync(0xffffffffu, inc, 31);
          }
          const int nB = n < kMaxUnits / 2 ? n : kMaxUnits / 2;
          n = 0;
          if (C.nr > 0)
            for (int uu = 0; uu < U; uu += 32) {
              const int u = uu + lane;
              const bool v = u < U;
              const int f = v ? C.desc[u].down.qtype : 0;
              const int np = v ? P.np_dn[f] : 0;
              int inc = np;
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
              }
              if (v) down_pieces(P, f, u, C.n0, C.nr, out + nB + n + inc - np);
              n += __shfl_sync(0xffffffffu, inc, 31);
            }
          if (lane == 0) {
            s_nB = nB;
            s_nC = n;
          }
        }
        if (live && s_bad && threadIdx.x == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 1000000);
        consumer_sync();
        // activations of the routed formats not built yet (buffers 1, 2 replace
        // the logits, which are no longer read)
        if (live && !s_bad)
          for (int f = 1; f <= 3; ++f) {
            const int fb = s_fmap[f];
            if (fb > 0) build_frag(P, f, smem + L.o_x32 + (fb - 1) * 2 * T * H, corr + fb * (H / 32) * 4);
          }
        __syncthreads();  // S2: lists and activations ready
        total = s_fail ? nA : nA + nSD + s_nB + s_nC;
      }
      if (q == nA + nSD + s_nB) {
        // ---------------------------------------- barrier 2: arrival only
        consumer_sync();
        if (threadIdx.x == 0) {
          if (!s_fail) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&hdr->bar_count) : "memory");
          else atomicExch(&hdr->abort, 1);
        }
      }
      if (q >= total) break;
      // ---------------------------------------------------- unit q
      // Router units are shared by all 8 warps (one quarter-row each); tile i
      // (all pieces of one 16-row tile) after phase A belongs to warp group
      // i % kGroups, whose kGW warps split its K; each of them releases the
      // slot for kCW / kGW warps.
      const Unit u = C.units[q];
      const bool tile = u.kind != kRouter;
      if (tile && u.k0 == 0) ++ti;
      // phase-A tiles (before the first barrier, on every CTA's critical
      // path) are shared by all eight warps like router units
      const bool all8 = q < nA;
      const int nw = all8 ? kCW : kGW, wi = all8 ? warp : gw;  // warps on this unit, this warp's share
      if (dead || (tile && !all8 && (ti % kGroups) != grp)) continue;
      if (!wait_full(C, q, hdr)) {
        s_fail = 1;
        dead = true;
        continue;
      }
      const uint8_t* slot = C.slot(q);
      if (!tile) {
        router_unit_dot(C, u, slot, x32);
      } else {
        const bool dn = u.kind == kDown;
        if (u.k0 == 0) acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        const Geo g = C.geo[dn * 4 + u.fmt];
        const int nch = g.cb / 16;
        const int c0 = wi * nch / nw, c1 = (wi + 1) * nch / nw;
        {  // one call site per instantiation (down tiles: activations in the slot)
          const int fb = dn ? 0 : s_fmap[u.fmt];
          const uint8_t* frag = dn ? slot + g.bofs : fb == 0 ? f0 : smem + L.o_x32 + (fb - 1) * 2 * T * H;
          const int ks0 = dn ? 0 : u.k0 / 16;
          if (u.fmt == MOE_Q_INT4_SYM_G32) {
            if (dn) tile_mma<MOE_Q_INT4_SYM_G32, false>(slot, g, c0, c1, frag, 0, nullptr, T, acc);
            else tile_mma<MOE_Q_INT4_SYM_G32, true>(slot, g, c0, c1, frag, ks0, corr + fb * (H / 32) * 4, T, acc);
          } else if (u.fmt == MOE_Q_INT2_ASYM_G16) {
            tile_mma<MOE_Q_INT2_ASYM_G16, false>(slot, g, c0, c1, frag, ks0, nullptr, T, acc);
          } else {
            tile_mma<MOE_Q_INT8_PER_CHANNEL, false>(slot, g, c0, c1, frag, ks0, nullptr, T, acc);
          }
        }
        if (u.last) {
          // partials of this warp -> red; the last warp to arrive finishes the tile
          const int gq = lane >> 2, tq = lane & 3, s = q % C.S;
          float* rs = red + size_t(s) * kCW * 64;
          if (tq < 2) {
            *reinterpret_cast<float2*>(rs + wi * 64 + gq * 4 + 2 * tq) = make_float2(acc[0], acc[1]);
            *reinterpret_cast<float2*>(rs + wi * 64 + (gq + 8) * 4 + 2 * tq) = make_float2(acc[2], acc[3]);
          }
          __syncwarp();
          int prev = 0;
          if (lane == 0) {
            __threadfence_block();
            prev = atomicAdd(&s_cnt[s], 1);
          }
          prev = __shfl_sync(0xffffffffu, prev, 0);
          if (prev == nw - 1) {
            __threadfence_block();
            __syncwarp();
            if (lane == 0) s_cnt[s] = 0;
            if (!dn) {
              const int r = lane >> 2, t = lane & 3;
              if (t < T) {
                float gs = red_sum(rs, r, t, nw), us = red_sum(rs, 8 + r, t, nw);
                if (u.fmt == MOE_Q_INT8_PER_CHANNEL) {
                  const uint16_t* sc = reinterpret_cast<const uint16_t*>(slot + g.aux0);
                  gs *= f16_to_f32(sc[r]);
                  us *= f16_to_f32(sc[8 + r]);
                }
                const float h = silu_f32(gs) * us;
                const int dfmt = C.desc[u.e].down.qtype;
                uint8_t* hf = P.hfrag + size_t(u.e) * frag_bytes(I, T);
                *reinterpret_cast<__half*>(hf + frag_off(dfmt, u.row0 + r, t, T)) = __float2half_rn(h);
              }
            } else {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const int idx = lane + 32 * hh, r = idx >> 2, t = idx & 3;
                if (r < u.nrows && t < T) {
                  float y = red_sum(rs, r, t, nw);
                  if (u.fmt == MOE_Q_INT8_PER_CHANNEL)
                    y *= f16_to_f32(reinterpret_cast<const uint16_t*>(slot + g.aux0)[(u.row0 & 7) + r]);
                  if (u.e == C.kShared) Sy[r * 4 + t] = y;
                  else Y[(u.e * 16 + r) * 4 + t] = y;
                }
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        if (tile && !all8) mbar_arrive_n(C.empty_bar(q), kCW / kGW);  // the other groups' share too
        else ptx::mbar_arrive(C.empty_bar(q));
      }
    }
    consumer_sync();
    // ------------------------------------------------ combine of the owned rows
    if (!s_fail && !s_bad)
      for (int i = threadIdx.x; i < T * C.nr; i += kCW * 32) {
        const int t = i / C.nr, r = i - t * C.nr;
        float a = 0.f;
        for (int j = 0; j < k; ++j) a = fmaf(s_w[t * k + j], Y[(s_slotmap[t * k + j] * 16 + r) * 4 + t], a);
        if (has_shared) a += Sy[r * 4 + t];
        P.out[size_t(t) * H + C.n0 + r] = f32_to_bf16_rn(a);
      }
  }
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

// ---------------------------------------------------------------- host side
constexpr int kStaticSmem = 8 * 1024;  // upper bound of the kernel's static shared memory

int units_bound(int T, int H, int I, int E, int k, int G, int nper, int RQ) {
  int gu = 0, dn = 0;
  for (int f = 1; f <= 3; ++f) {
    const int a = npieces(f, H, T, false), d = npieces(f, I, T, true);
    if (a == 0 || d == 0) return 1 << 30;
    gu = a > gu ? a : gu;
    dn = d > dn ? d : dn;
  }
  const int U = T * k < E ? T * k : E;
  const int rpc = (E * RQ + G - 1) / G;
  const int A = (rpc + nper - 1) / nper + ((I / 8 + G - 1) / G) * gu;
  const int B = dn + ((U * (I / 8) + G - 1) / G) * gu;
  const int Cn = U * dn;
  return A + B + Cn;
}

int pick_slots(int T, int H, int E, int k) {
  // a multiple of kProducers: each slot has one producer warp
  for (int s = kMaxSlots - kMaxSlots % kProducers; s >= 4 && s >= kProducers; s -= kProducers)
    if (make_plan(T, H, E, k, s).total + kStaticSmem <= kSmemLimit) return s;
  return 0;
}

int grid_size() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

}  // namespace dks

bool decode_stream_eligible(int T, int H, int I, int E, int k) {
  using namespace dks;
  if (T < 1 || T > kMaxT || k < 1 || k > dks::kMaxK || E < k || E > moe::kMaxE) return false;
  if (H < 256 || I < 256 || H > 2048 || I > 2048 || (H % 256) || (I % 256)) return false;
  const int G = grid_size();
  if ((H + G - 1) / G > 16) return false;
  const int RQ = router_rq(H), KP = H / RQ;
  if (H % RQ || KP % 128 || KP * 4 > kSlotBytes) return false;
  const int nper = std::min(kCW, kSlotBytes / (KP * 4));
  const int S = pick_slots(T, H, E, k);
  if (S == 0) return false;
  for (int f = 1; f <= 3; ++f)
    if (npieces(f, I, T, true) >= S) return false;
  return units_bound(T, H, I, E, k, G, nper, RQ) <= kMaxUnits / 2;
}

size_t decode_stream_hfrag_bytes(int T, int I, int k) {
  return size_t(T * k + 1) * size_t(dks::frag_bytes(I, T));
}

cudaError_t launch_decode_stream(const uint16_t* x, int T, int H, int I, int E, int k, const float* w_router,
                                 const float* bias, long long bstride, const moe_expert* experts,
                                 const moe_expert* shared, int* topk_idx, float* topk_w, float* logits_out,
                                 uint16_t* out, float* partial, void* hfrag, WsHeader* hdr, cudaStream_t st) {
  using namespace dks;
  const int grid = grid_size();
  const int S = pick_slots(T, H, E, k);
  const size_t smem = size_t(make_plan(T, H, E, k, S).total);
  cudaError_t e = cudaFuncSetAttribute(decode_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  Params P{x, T, H, I, E, k, w_router, bias, bstride, experts, shared, topk_idx, topk_w, logits_out, out, partial,
           static_cast<uint8_t*>(hfrag), hdr, S, {0, 0, 0, 0}, {0, 0, 0, 0}};
  for (int f = 1; f <= 3; ++f) {
    P.np_gu[f] = npieces(f, H, T, false);
    P.np_dn[f] = npieces(f, I, T, true);
  }
  void* args[] = {&P};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(decode_stream_kernel), dim3(grid), dim3(kThreads), args,
                                  smem, st);
  count_launches(1);
  return e;
}

}  // namespace moe
