// Decode step (1 <= T <= 4 tokens) as ONE persistent cooperative launch in
// which every warp fetches and dequantises its own weight rows.
//
// Decode reads each picked expert's weights once per step, so its floor is
// memory bandwidth (the lcz.me forum thread "Halogen Flash Server配置與實測",
// comment section: decode re-reads a fixed set of weights every step and its
// ceiling follows bandwidth). The step itself is the one the telli.sh page
// "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
// "稀疏架构创造了机会", describes: 10 of 512 routed experts plus one shared
// expert per token.
//
// Structure (one CTA of 16 warps per SM, all CTAs co-resident):
//   A  router rows of this CTA (whole logits, one publication per CTA; the
//      weights are loaded at the kernel's entry); the CTA then arrives on a
//      grid counter, and while every CTA's logits gather it converts x for
//      the tensor cores and prefetches its rows of the shared expert;
//   -  every CTA, all warps, reads all logits and takes the top-k itself
//      (identical inputs, identical code, identical picks): 32-logit chunks
//      sorted per warp, a cutoff at each token's k-th best chunk winner, the
//      survivors ranked; then the gates, the distinct picked experts (slots)
//      and their descriptors;
//   B  the gate/up tiles of this CTA in the list "shared expert, then the
//      picked ones" (tile g goes to CTA g mod G, so each expert's tiles
//      finish early and together); finishing a tile publishes its 8
//      intermediate values h per token and bumps that expert's tile counter;
//   C  this CTA's slice of output rows of every expert's down projection,
//      each waiting only for ITS expert's counter (no second grid barrier);
//      then the gate-weighted combine of those rows.
// Jobs are numbered per CTA and computed from their numbers; warp w takes
// jobs w, w + 16, ... (B jobs before C jobs, so a warp waiting in C never
// holds back a tile that another waits for). A job is 16 weight rows over a
// K range. int4 and int2 rows are copied into the warp's own shared-memory
// buffer by per-lane cp.async (all of the job at once) when the buffers fit,
// else each lane loads 16 bytes of its two rows per iteration straight into
// registers, several iterations ahead; the codes are dequantised in
// registers and fed to mma.sync m16n8k16 (fp16 operands, fp32 accumulation)
// with the T <= 4 tokens as the MMA's columns, read from shared memory in the
// order the dequantisation produces pairs.
//
// Numerics: int4 and int2 weights become fp16 with one rounding (code times
// the group scale, plus the min for int2), int8 codes are exact and their
// row scale multiplies the fp32 result. Activations enter the MMA as fp16
// after an exact power-of-two scaling that keeps them inside the fp16 range
// (x per token; h per expert and token, from the largest |h| of that expert),
// undone on the fp32 results: any finite bf16 input stays finite.
#include <cuda_fp16.h>
#include <math_constants.h>

#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace dfx {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxT = 4;
constexpr int kMaxK = 16;
constexpr int kMaxSlots = kMaxT * kMaxK + 1;  // routed slots + the shared expert
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMaxH = 2048;     // largest hidden size of the fused kernel
constexpr int kMaxI = 2048;     // largest expert intermediate size
constexpr int kMaxBias = 64;    // router bias values of one CTA's rows (rows x tokens)

enum : uint8_t { kRouter = 0, kGateUp = 1, kDown = 2 };

// One warp's job. 8 bytes.
struct Job {
  uint8_t kind;
  uint8_t slot;   // expert slot (shared = kSharedSlot); router: local row
  uint8_t nrows;  // down: output rows (<= 16)
  uint8_t part;   // gate/up: K part of nsplit; router: segment
  uint16_t row0;  // gate/up: first intermediate row; down: first output row
  uint16_t tile;  // gate/up: local tile index (reduction slot)
};
static_assert(sizeof(Job) == 8, "job record");
constexpr int kSharedSlot = kMaxSlots - 1;
// Counters of an expert slot, each slot on a 128-byte line of its own (so
// the warps polling one expert do not contend with another's): word 0 =
// finished gate/up tiles, words 1..kMaxT = bits of the largest |h| per token.
constexpr int kCntStride = 32;

// ---------------------------------------------------------------- formats
// A 16-byte column of codes holds kc(F) weights of one row; its activations
// for one token take wb(F) bytes per 32-bit word of codes, 4 words per column.
__host__ __device__ constexpr int kc(int F) { return F == MOE_Q_INT4_SYM_G32 ? 32 : F == MOE_Q_INT2_ASYM_G16 ? 64 : 16; }
__host__ __device__ constexpr int wbytes(int F) { return F == MOE_Q_INT4_SYM_G32 ? 16 : F == MOE_Q_INT2_ASYM_G16 ? 32 : 8; }
__host__ __device__ constexpr int colbytes(int F) { return 4 * wbytes(F); }  // = 2 * kc(F)

// Byte offset of activation (k, token t) in a buffer laid out for format F:
// [column][token][word][pairs]. The dequantisation of a 32-bit code word
// yields fp16 pairs, and MMA k-columns (2tq, 2tq+1) / (2tq+8, 2tq+9) take
// them in this order:
//   int4 word (8 nibbles i = 0..7):  (0,4) (1,5) | (2,6) (3,7)   two MMAs
//   int2 word (16 codes i = 0..15):  (0,8) (1,9) | (2,10) (3,11) | ...  four MMAs
//   int8 word (4 bytes i = 0..3):    (0,2) (1,3)                  one MMA
__host__ __device__ inline int frag_pos(int F, int k, int t, int T) {
  const int c = k / kc(F), p = k % kc(F);
  int j, pos;
  if (F == MOE_Q_INT4_SYM_G32) {
    j = p >> 3;
    const int i = p & 7;
    pos = (i & 3) * 2 + (i >> 2);
  } else if (F == MOE_Q_INT2_ASYM_G16) {
    j = p >> 4;
    const int i = p & 15;
    pos = (i & 7) * 2 + (i >> 3);
  } else {
    j = p >> 2;
    const int i = p & 3;
    pos = (i & 1) * 2 + (i >> 1);
  }
  return (c * T + t) * colbytes(F) + j * wbytes(F) + pos * 2;
}

// Byte offsets of activations k0 .. k0 + 3 (k0 % 4 == 0) of one token within
// its fragment-order word: frag_pos(F, k0, t, T) + quad_off<F>(i). int4 and
// int2 put four consecutive k in every other fp16 slot, int8 in slots
// 0, 2, 1, 3.
template <int F>
__host__ __device__ constexpr int quad_off(int i) {
  return F == MOE_Q_INT8_PER_CHANNEL ? 2 * ((i & 1) * 2 + (i >> 1)) : 4 * i;
}

// K parts of a gate/up tile, the same for every format: two halves when each
// half is a whole number of iterations (4 columns of 16 bytes) in every
// format (H % 512 == 0), else one.
__host__ __device__ inline int gu_parts(int H) { return H % 512 == 0 ? 2 : 1; }

// ---------------------------------------------------------------- plan
// Dynamic shared memory, offsets from the base.
struct Plan {
  int o_x32;   // fp32 x [T][H] (router input, phase A only)
  int o_cand;  // top-k candidates of the routing [T][E / 32][k] and their survivors [T][k k], 8 bytes each (over x32)
  int o_hf;    // per-warp activations of a down job, 2 T I bytes each (phase C; over x32)
  int o_xf;    // 3 activation buffers in fragment order, 2 T H bytes each
  int o_rp;    // router partials [rows][segs][T]
  int o_red;   // gate/up K-split sums [tiles][16][T]
  int o_td;    // gate/up K-split arrivals [tiles]
  int o_y;     // down results [kMaxSlots][16][T]
  int o_desc;  // expert descriptors of the picked slots and the shared one
  int o_stage;      // per-warp staging buffers of int4/int2 job rows, or -1
  int stage_bytes;  // bytes of one warp's staging buffer
  int total;
};
__host__ __device__ inline int router_rows(int E, int G) { return (E + G - 1) / G; }
__host__ __device__ inline int router_seg(int H) { return H % 512 == 0 ? 512 : 256; }
__host__ __device__ inline int max_tiles(int T, int I, int E, int k, int G) {
  const int U = T * k < E ? T * k : E;
  return ((U + 1) * (I / 8) + G - 1) / G;  // routed experts and the shared one
}
// Row pitches of a staged job with ncol 16-byte code columns per row: codes
// ncol * 16 + 16 (one spare 16-byte unit, so consecutive rows start on
// different banks), scales (and int2 mins) of those columns rounded up to 16.
__host__ __device__ inline void stage_pitches(int f, int ncol, int& cp, int& sp) {
  cp = ncol * 16 + 16;
  const int s = f == MOE_Q_INT2_ASYM_G16 ? ncol * 8 : ncol * 2;
  sp = (s + 15) / 16 * 16;
}
constexpr int kStaticSmemBound = 12 * 1024;  // bound on the kernel's static shared memory


__host__ __device__ inline Plan make_plan(int T, int H, int I, int E, int k, int G) {
  Plan p{};
  int o = 0;
  auto take = [&](int bytes, int al) {
    o = (o + al - 1) / al * al;
    const int r = o;
    o += bytes;
    return r;
  };
  // routing candidates: [T][E / 32][k], then up to k^2 survivors per token
  const int x32 = 4 * T * H, hf = kWarps * 2 * T * I, cand = 8 * T * (((E + 31) / 32) * k + k * k);
  const int big = hf > cand ? hf : cand;
  p.o_x32 = take(x32 > big ? x32 : big, 16);
  p.o_cand = p.o_x32;
  p.o_hf = p.o_x32;
  p.o_xf = take(3 * 2 * T * H, 16);
  p.o_rp = take(4 * (router_rows(E, G) + 1) * (H / router_seg(H)) * T, 16);
  p.o_red = take(4 * max_tiles(T, I, E, k, G) * 16 * T, 16);
  p.o_td = take(4 * max_tiles(T, I, E, k, G), 16);
  p.o_y = take(4 * kMaxSlots * 16 * T, 16);
  p.o_desc = take(int(sizeof(moe_expert)) * kMaxSlots, 16);
  // staging: the largest int4 or int2 job (16 rows of a gate/up part or of
  // a down slice) with the row pitches of stage_pitches, when it fits
  int sb = 0;
  for (int f = MOE_Q_INT4_SYM_G32; f <= MOE_Q_INT2_ASYM_G16; ++f) {
    const int nm = f == MOE_Q_INT2_ASYM_G16 ? 2 : 1;
    int cp, sp;
    stage_pitches(f, H / kc(f) / gu_parts(H), cp, sp);
    sb = sb > 16 * (cp + nm * sp) ? sb : 16 * (cp + nm * sp);
    stage_pitches(f, I / kc(f), cp, sp);
    sb = sb > 16 * (cp + nm * sp) ? sb : 16 * (cp + nm * sp);
  }
  p.stage_bytes = sb;
  p.o_stage = -1;
  if (o + 16 + kWarps * sb + kStaticSmemBound <= kSmemLimit) p.o_stage = take(kWarps * sb, 16);
  p.total = o;
  return p;
}

// Output rows [n0, n0 + nr) of CTA b: H split as evenly as possible.
__host__ __device__ inline void out_rows(int H, int G, int b, int& n0, int& nr) {
  const int q = H / G, r = H % G;
  n0 = b * q + (b < r ? b : r);
  nr = q + (b < r ? 1 : 0);
}
// Router rows [e0, e0 + n) of CTA b.
__host__ __device__ inline void router_range(int E, int G, int b, int& e0, int& n) {
  const int rr = router_rows(E, G);
  e0 = b * rr < E ? b * rr : E;
  n = (e0 + rr < E ? e0 + rr : E) - e0;
}
// Gate/up tiles of CTA b in phases B and C: tiles g = b, b + G, ... of the
// step's expert-major list of `ne` experts (I / 8 tiles each).
__host__ __device__ inline int bc_tiles(int I, int G, int b, int ne) {
  const int J = ne * (I / 8);
  return J > b ? (J - 1 - b) / G + 1 : 0;
}

// Router rows of CTA b, plus one for the shared expert's gate vector on the
// last CTA when the gated variant is on (its local row index is the last).
__host__ __device__ inline int router_rows_of(int E, int G, int b, bool gate_row) {
  int e0, n;
  router_range(E, G, b, e0, n);
  return n + (gate_row && b == G - 1 ? 1 : 0);
}

// Jobs are numbered per CTA and computed from their number (no lists):
// warp w takes jobs w, w + 16, ...
//
// Phase A of CTA b: router parts (local row j / nseg, segment j % nseg).
__host__ __device__ inline int phase_a_count(int H, int E, int G, int b, bool gate_row) {
  return router_rows_of(E, G, b, gate_row) * (H / router_seg(H));
}
__host__ __device__ inline Job phase_a_job(int H, int j) {
  const int nseg = H / router_seg(H);
  return Job{kRouter, uint8_t(j / nseg), 0, uint8_t(j % nseg), 0, 0};
}
// Phases B and C of CTA b, over the list of ne = U (+ 1) experts, the shared
// one first (slot kSharedSlot), then the U picked ones (slots 0 .. U - 1):
// first the gate/up parts of this CTA's tiles (tile-major, gu_parts(H) K
// parts each; local tile index = position among this CTA's tiles), then one
// down job per expert for this CTA's output rows.
__host__ __device__ inline int phase_bc_count(int H, int I, int G, int b, int U, bool with_shared) {
  int n0, nr;
  out_rows(H, G, b, n0, nr);
  const int ne = U + (with_shared ? 1 : 0);
  return gu_parts(H) * bc_tiles(I, G, b, ne) + (nr > 0 ? ne : 0);
}
__host__ __device__ inline Job phase_bc_job(int H, int I, int G, int b, int U, bool with_shared, int j) {
  const int ns = gu_parts(H), nt = I / 8, sh = with_shared ? 1 : 0;
  const int ngu = ns * bc_tiles(I, G, b, U + sh);
  if (j < ngu) {
    const int i = j / ns, p = j - i * ns, g = b + G * i;
    const int e = g / nt, r = g - e * nt;
    return Job{kGateUp, uint8_t(sh && e == 0 ? kSharedSlot : e - sh), 16, uint8_t(p), uint16_t(8 * r), uint16_t(i)};
  }
  int n0, nr;
  out_rows(H, G, b, n0, nr);
  const int d = j - ngu;
  return Job{kDown, uint8_t(sh && d == 0 ? kSharedSlot : d - sh), uint8_t(nr), 0, uint16_t(n0), 0};
}

struct Params {
  Plan L;  // shared-memory plan of the launch
  const uint16_t* x;
  int T, H, I, E, k;
  const float* w_router;
  const float* bias;
  long long bstride;
  const moe_expert* experts;
  const moe_expert* shared;
  int* topk_idx;
  float* topk_w;
  float* logits_out;
  uint16_t* out;
  WsHeader* hdr;
  float* logits;   // [T][E] workspace
  float* h;        // [kMaxSlots][T][I] workspace
  __half* h16;     // [kMaxSlots][2 T I bytes]: h as fp16 in the down format's fragment order (workspace)
  uint32_t* cnt;   // [kMaxSlots][kCntStride]: finished tiles, then max |h| bits per token
  long long wait_cycles;
  uint32_t flags;            // MOE_BIAS_SELECTION_ONLY
  const float* shared_gate;  // fp32 [H] or null: sigmoid-gated shared expert
  float* logits_u;           // [T][E] unbiased logits (selection-only bias)
  float* sgate;              // [T] shared_gate . x
  uint32_t* heat;            // [E] routing heat, or null
  // Experts only (the moe_expert_ffn call at decode sizes): the routing is
  // given as dispatch arrays, nothing is routed or combined, and every
  // dispatched row's expert output goes to y_perm. Null otherwise.
  const int* perm_src;  // [T k] token * k + pick of each row
  const int* offsets;   // [E + 1] first row of each expert
  const int* counts;    // [E] rows of each expert
  uint16_t* y_perm;     // bf16 [T k, H]
};

// ---------------------------------------------------------------- PTX bits
__device__ __forceinline__ uint32_t lop_or(uint32_t a, uint32_t mask, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));  // (a & mask) | magic
  return d;
}
// ((a ^ 0x80) & 0xFF) | 0x6400 in each 16-bit half: byte q -> fp16 1024 + (q + 128).
__device__ __forceinline__ uint32_t lop_i8(uint32_t a) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(0x00FF00FFu), "r"(0x64806480u));
  return d;
}
__device__ __forceinline__ uint32_t h2sub(uint32_t a, uint32_t b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2mul(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2fma(uint32_t a, uint32_t b, uint32_t c) {
  const __half2 r = __hfma2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b),
                            *reinterpret_cast<const __half2*>(&c));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t dup16(uint32_t h) { return (h & 0xffffu) | (h << 16); }
__device__ __forceinline__ void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                    uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint4 ldg16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg8(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg2(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return uint32_t(v);
}
__device__ __forceinline__ uint32_t ldg4(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
// The warp's staging copies have landed and every lane may read them.
__device__ __forceinline__ void stage_wait() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
// Bulk prefetch of [p, p + bytes) into L2 (a hint: skipped unless the range
// is 16-byte aligned and a whole number of 16 bytes).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  if (bytes > 0 && ((reinterpret_cast<uintptr_t>(p) | bytes) & 15u) == 0)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// 2^e as a float for -126 <= e <= 127 (the range scaling uses |e| <= 114):
// multiplying by it is exact up to the one rounding of the product.
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }
__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
  return uint32_t(__half_as_ushort(lo)) | (uint32_t(__half_as_ushort(hi)) << 16);
}
// Activations k0 .. k0 + 3 (k0 % 4 == 0) of token t into a buffer in format
// F's fragment order.
template <int F>
__device__ __forceinline__ void store4(uint8_t* buf, int k0, int t, int T, float a, float b, float c, float d) {
  uint8_t* p = buf + frag_pos(F, k0, t, T);
  const __half ha = __float2half_rn(a), hb = __float2half_rn(b), hc = __float2half_rn(c), hd = __float2half_rn(d);
  if (F == MOE_Q_INT8_PER_CHANNEL) {
    static_assert(quad_off<MOE_Q_INT8_PER_CHANNEL>(1) == 4 && quad_off<MOE_Q_INT8_PER_CHANNEL>(2) == 2, "int8 quad");
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_h2(ha, hc), pack_h2(hb, hd));
  } else {
    *reinterpret_cast<__half*>(p + quad_off<F>(0)) = ha;
    *reinterpret_cast<__half*>(p + quad_off<F>(1)) = hb;
    *reinterpret_cast<__half*>(p + quad_off<F>(2)) = hc;
    *reinterpret_cast<__half*>(p + quad_off<F>(3)) = hd;
  }
}

// Power-of-two exponent that brings a magnitude below 2^15 (fp16 max 65504):
// 0 for anything already below.
__device__ __forceinline__ int range_exp(uint32_t abs_bits) {
  const int e = int((abs_bits >> 23) & 0xff) - 127;  // floor(log2) of a finite positive float
  return e >= 15 ? min(e - 14, 250) : 0;
}

// ---------------------------------------------------------------- tiles
// Pointers of one lane's two rows in a matrix (A rows gq and gq + 8).
struct Rows {
  const uint8_t* c_lo;
  const uint8_t* c_hi;
  const uint16_t* s_lo;
  const uint16_t* s_hi;
  const uint16_t* m_lo;
  const uint16_t* m_hi;
  bool lo, hi;  // rows present
};

// Loads of one iteration (this lane's 16-byte column of both rows).
struct Ld {
  uint4 a, b;
  uint2 sa, sb, ma, mb;  // int4: sa.x / sb.x = scale; int2: 4 scales / 4 mins each
};

// Weight loads from global memory (streamed, not kept in L1) or from this
// warp's staging buffer in shared memory (kSmem: generic loads).
template <bool kSmem>
__device__ __forceinline__ uint4 ldw16(const void* p) {
  if constexpr (kSmem) return *reinterpret_cast<const uint4*>(p);
  else return ldg16(p);
}
template <bool kSmem>
__device__ __forceinline__ uint2 ldw8(const void* p) {
  if constexpr (kSmem) return *reinterpret_cast<const uint2*>(p);
  else return ldg8(p);
}
template <bool kSmem>
__device__ __forceinline__ uint32_t ldw4(const void* p) {
  if constexpr (kSmem) return *reinterpret_cast<const uint32_t*>(p);
  else return ldg4(p);
}
template <bool kSmem>
__device__ __forceinline__ uint32_t ldw2(const void* p) {
  if constexpr (kSmem) return uint32_t(*reinterpret_cast<const uint16_t*>(p));
  else return ldg2(p);
}

template <int F, bool kSmem>
__device__ __forceinline__ void load_it(const Rows& R, int c, Ld& L) {
  L.a = R.lo ? ldw16<kSmem>(R.c_lo + size_t(c) * 16) : make_uint4(0u, 0u, 0u, 0u);
  L.b = R.hi ? ldw16<kSmem>(R.c_hi + size_t(c) * 16) : make_uint4(0u, 0u, 0u, 0u);
  if (F == MOE_Q_INT4_SYM_G32) {
    L.sa.x = R.lo ? ldw2<kSmem>(R.s_lo + c) : 0u;
    L.sb.x = R.hi ? ldw2<kSmem>(R.s_hi + c) : 0u;
  } else if (F == MOE_Q_INT2_ASYM_G16) {
    L.sa = R.lo ? ldw8<kSmem>(R.s_lo + 4 * c) : make_uint2(0u, 0u);
    L.sb = R.hi ? ldw8<kSmem>(R.s_hi + 4 * c) : make_uint2(0u, 0u);
    L.ma = R.lo ? ldw8<kSmem>(R.m_lo + 4 * c) : make_uint2(0u, 0u);
    L.mb = R.hi ? ldw8<kSmem>(R.m_hi + 4 * c) : make_uint2(0u, 0u);
  }
}

__device__ __forceinline__ uint32_t word(const uint4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t half_of(const uint2& v, int g) {  // g-th fp16 of four
  const uint32_t w = g < 2 ? v.x : v.y;
  return (g & 1) ? (w >> 16) : (w & 0xffffu);
}

// Code -> fp16 by the published "magic number" conversion (as in the int4
// kernels of FasterTransformer and Marlin): OR the code bits into the
// mantissa of an fp16 constant whose exponent makes one unit of those bits
// worth 1, then subtract the constant. Here the low nibble of a byte sits
// under 1024 (0x6400) and the high nibble under 64 (0x5400, where bits 4-7
// are worth 1 each), so neither needs a shift.
// int4 word -> four fp16 pairs (c - 8) * s in the order of frag_pos.
__device__ __forceinline__ void deq4(uint32_t w, uint32_t s2, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = h2mul(h2sub(lop_or(w, 0x000F000Fu, 0x64006400u), 0x64086408u), s2);   // (n0, n4): 1024 + n - 1032
  p[1] = h2mul(h2sub(lop_or(w, 0x00F000F0u, 0x54005400u), 0x54805480u), s2);   // (n1, n5): 64 + n - 72
  p[2] = h2mul(h2sub(lop_or(w8, 0x000F000Fu, 0x64006400u), 0x64086408u), s2);  // (n2, n6)
  p[3] = h2mul(h2sub(lop_or(w8, 0x00F000F0u, 0x54005400u), 0x54805480u), s2);  // (n3, n7)
}
// int2 word (one group) -> eight fp16 pairs c * s + m, pair i = codes (i, i + 8).
__device__ __forceinline__ void deq2(uint32_t w, uint32_t s2, uint32_t m2, uint32_t (&p)[8]) {
  const uint32_t w8 = w >> 8;
  p[0] = h2fma(h2sub(lop_or(w, 0x00030003u, 0x64006400u), 0x64006400u), s2, m2);   // bits 0-1: 1024 + c
  p[1] = h2fma(h2sub(lop_or(w, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u), s2, m2);   // bits 2-3: 256 + c
  p[2] = h2fma(h2sub(lop_or(w, 0x00300030u, 0x54005400u), 0x54005400u), s2, m2);   // bits 4-5: 64 + c
  p[3] = h2fma(h2sub(lop_or(w, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u), s2, m2);   // bits 6-7: 16 + c
  p[4] = h2fma(h2sub(lop_or(w, 0x03000300u, 0x44004400u), 0x44004400u), s2, m2);   // bits 8-9: 4 + c
  p[5] = h2fma(h2sub(lop_or(w8, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u), s2, m2);  // bits 10-11
  p[6] = h2fma(h2sub(lop_or(w8, 0x00300030u, 0x54005400u), 0x54005400u), s2, m2);  // bits 12-13
  p[7] = h2fma(h2sub(lop_or(w8, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u), s2, m2);  // bits 14-15
}
// int8 word -> two exact fp16 pairs (q0, q2), (q1, q3).
__device__ __forceinline__ void deq8(uint32_t w, uint32_t (&p)[2]) {
  p[0] = h2sub(lop_i8(w), 0x64806480u);
  p[1] = h2sub(lop_i8(w >> 8), 0x64806480u);
}

// MMAs of one iteration: this lane's column c of both rows against the
// activations of column c in `bf` (fragment order); only lanes gq < T read B.
template <int F>
__device__ __forceinline__ void mma_it(const Ld& L, const uint8_t* bf, int c, int T, float (&acc)[2][4]) {
  const int lane = threadIdx.x & 31, gq = lane >> 2;
  const bool bv = gq < T;
  const uint8_t* bp = bf + (size_t(c) * T + gq) * colbytes(F);
  // int4: this column's activation fragments first (64 bytes of shared
  // memory), so their latency overlaps the dequantisation
  // (int2 and int8 load each word's piece in its turn: fewer registers)
  constexpr int kNb = F == MOE_Q_INT4_SYM_G32 ? 4 : 1;
  uint4 bq[kNb];
#pragma unroll
  for (int i = 0; i < kNb; ++i) bq[i] = bv ? reinterpret_cast<const uint4*>(bp)[i] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wa = word(L.a, j), wb = word(L.b, j);
    if (F == MOE_Q_INT4_SYM_G32) {
      uint32_t pa[4], pb[4];
      deq4(wa, dup16(L.sa.x), pa);
      deq4(wb, dup16(L.sb.x), pb);
      mma(acc[0], pa[0], pb[0], pa[1], pb[1], bq[j].x, bq[j].y);
      mma(acc[1], pa[2], pb[2], pa[3], pb[3], bq[j].z, bq[j].w);
    } else if (F == MOE_Q_INT2_ASYM_G16) {
      uint32_t pa[8], pb[8];
      deq2(wa, dup16(half_of(L.sa, j)), dup16(half_of(L.ma, j)), pa);
      deq2(wb, dup16(half_of(L.sb, j)), dup16(half_of(L.mb, j)), pb);
      const uint4 b0 = bv ? *reinterpret_cast<const uint4*>(bp + j * 32) : make_uint4(0u, 0u, 0u, 0u);
      const uint4 b1 = bv ? *reinterpret_cast<const uint4*>(bp + j * 32 + 16) : make_uint4(0u, 0u, 0u, 0u);
      mma(acc[0], pa[0], pb[0], pa[1], pb[1], b0.x, b0.y);
      mma(acc[1], pa[2], pb[2], pa[3], pb[3], b0.z, b0.w);
      mma(acc[0], pa[4], pb[4], pa[5], pb[5], b1.x, b1.y);
      mma(acc[1], pa[6], pb[6], pa[7], pb[7], b1.z, b1.w);
    } else {
      uint32_t pa[2], pb[2];
      deq8(wa, pa);
      deq8(wb, pb);
      const uint2 b = bv ? *reinterpret_cast<const uint2*>(bp + j * 8) : make_uint2(0u, 0u);
      mma(acc[j & 1], pa[0], pb[0], pa[1], pb[1], b.x, b.y);
    }
  }
}

// Iterations of loads in flight per lane (int2 carries 4 scales and 4 mins
// per row and iteration, so it keeps fewer in registers). The rows of every
// job are on their way into L2 since the routing, so these loads mostly wait
// for L2, not DRAM.
__host__ __device__ constexpr int depth(int F) { return F == MOE_Q_INT2_ASYM_G16 ? 2 : 4; }

// One warp's share of a tile: iterations it = 0..nit-1, lane column
// wc = wcol0 + 4 it + tq of the weights (global, or the staged copy) against
// activation column c = col0 + 4 it + tq; the loads of depth(F) iterations
// are in flight while one is computed. Returns this lane's four accumulators
// (D rows gq, gq + 8; token columns 2 tq, 2 tq + 1). One function per format
// and source, so each gets its own register allocation.
template <int F, bool kSmem>
__device__ __noinline__ float4 run_tile(const Rows R, int wcol0, int col0, int nit, const uint8_t* bf, int T) {
  const int tq = threadIdx.x & 3;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  if constexpr (kSmem) {
    // staged rows: once they have landed, one iteration at a time
    // (shared-memory latency) in a small loop
    stage_wait();
#pragma unroll 1
    for (int it = 0; it < nit; ++it) {
      Ld L;
      load_it<F, true>(R, wcol0 + 4 * it + tq, L);
      mma_it<F>(L, bf, col0 + 4 * it + tq, T, acc);
    }
    return make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
  }
  constexpr int kDepth = kSmem ? 1 : depth(F);
  Ld L[kDepth];
#pragma unroll
  for (int s = 0; s < kDepth; ++s)
    if (s < nit) load_it<F, kSmem>(R, wcol0 + 4 * s + tq, L[s]);
#pragma unroll 1
  for (int it0 = 0; it0 < nit; it0 += kDepth) {
#pragma unroll
    for (int s = 0; s < kDepth; ++s) {
      const int it = it0 + s;
      if (it < nit) {
        mma_it<F>(L[s], bf, col0 + 4 * it + tq, T, acc);
        if (it + kDepth < nit) load_it<F, kSmem>(R, wcol0 + 4 * (it + kDepth) + tq, L[s]);
      }
    }
  }
  return make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
}
template <bool kSmem>
__device__ __forceinline__ void run_any(int f, const Rows& R, int wcol0, int col0, int nit, const uint8_t* bf, int T,
                                        float (&acc)[4]) {
  const float4 v = f == MOE_Q_INT4_SYM_G32 ? run_tile<MOE_Q_INT4_SYM_G32, kSmem>(R, wcol0, col0, nit, bf, T)
                   : f == MOE_Q_INT2_ASYM_G16
                       ? run_tile<MOE_Q_INT2_ASYM_G16, kSmem>(R, wcol0, col0, nit, bf, T)
                       : run_tile<MOE_Q_INT8_PER_CHANNEL, false>(R, wcol0, col0, nit, bf, T);  // int8: never staged
  acc[0] = v.x;
  acc[1] = v.y;
  acc[2] = v.z;
  acc[3] = v.w;
}

// int4 tile for T <= 2 tokens with the group scales applied to fp32 sums
// instead of to every fp16 weight: the A fragments are the exact codes
// (c - 8), and B column n of the MMA carries only the activations that A
// lane tq = n & 3 contributes (token n >> 2), so D column n is the sum over
// group n & 3 of the iteration's four 16-byte columns (one int4 group each).
// Each lane then scales its two columns by their group scales (loaded as one
// 32-bit pair) and adds them to fp32 accumulators. Same four results per
// lane as run_tile. Needs 4-byte aligned scale rows.
struct Ld4 {
  uint4 a, b;      // codes of rows gq and gq + 8, this lane's column
  uint32_t sa, sb;  // fp16 scales of this lane's two D columns, rows gq and gq + 8
};
template <bool kSmem>
__device__ __forceinline__ void load_i4(const Rows& R, int c, int cs, Ld4& L) {
  L.a = R.lo ? ldw16<kSmem>(R.c_lo + size_t(c) * 16) : make_uint4(0u, 0u, 0u, 0u);
  L.b = R.hi ? ldw16<kSmem>(R.c_hi + size_t(c) * 16) : make_uint4(0u, 0u, 0u, 0u);
  L.sa = R.lo ? ldw4<kSmem>(R.s_lo + cs) : 0u;
  L.sb = R.hi ? ldw4<kSmem>(R.s_hi + cs) : 0u;
}
// int4 word -> four fp16 pairs (c - 8), exact, in the order of frag_pos.
__device__ __forceinline__ void deq4_codes(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = h2sub(lop_or(w, 0x000F000Fu, 0x64006400u), 0x64086408u);
  p[1] = h2sub(lop_or(w, 0x00F000F0u, 0x54005400u), 0x54805480u);
  p[2] = h2sub(lop_or(w8, 0x000F000Fu, 0x64006400u), 0x64086408u);
  p[3] = h2sub(lop_or(w8, 0x00F000F0u, 0x54005400u), 0x54805480u);
}
template <bool kSmem>
__device__ __noinline__ float4 run_tile_i4(const Rows R, int wcol0, int col0, int nit, const uint8_t* bf, int T) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const int dt = gq - tq;
  const bool bv = dt == 0 || (dt == 4 && T == 2);  // B column gq takes A lane tq's activations
  const int bt = dt == 4 ? 1 : 0;                   // of this token
  const int g0 = (2 * tq) & 3;                      // groups of this lane's D columns 2 tq, 2 tq + 1
  constexpr int kDepth = kSmem ? 1 : 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  Ld4 L[kDepth];
  if constexpr (kSmem) stage_wait();  // the staged rows have landed
#pragma unroll
  for (int s = 0; s < kDepth; ++s)
    if (s < nit) load_i4<kSmem>(R, wcol0 + 4 * s + tq, wcol0 + 4 * s + g0, L[s]);
#pragma unroll 1
  for (int it0 = 0; it0 < nit; it0 += kDepth) {
#pragma unroll
    for (int s = 0; s < kDepth; ++s) {
      const int it = it0 + s;
      if (it < nit) {
        const uint4* bp = reinterpret_cast<const uint4*>(bf + (size_t(col0 + 4 * it + tq) * T + bt) * 64);
        uint4 bq[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) bq[j] = bv ? bp[j] : make_uint4(0u, 0u, 0u, 0u);
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t pa[4], pb[4];
          deq4_codes(word(L[s].a, j), pa);
          deq4_codes(word(L[s].b, j), pb);
          float (&d)[4] = j < 2 ? d0 : d1;
          mma(d, pa[0], pb[0], pa[1], pb[1], bq[j].x, bq[j].y);
          mma(d, pa[2], pb[2], pa[3], pb[3], bq[j].z, bq[j].w);
        }
        const float2 sa = __half22float2(*reinterpret_cast<const __half2*>(&L[s].sa));
        const float2 sb = __half22float2(*reinterpret_cast<const __half2*>(&L[s].sb));
        acc[0] = fmaf(sa.x, d0[0] + d1[0], acc[0]);
        acc[1] = fmaf(sa.y, d0[1] + d1[1], acc[1]);
        acc[2] = fmaf(sb.x, d0[2] + d1[2], acc[2]);
        acc[3] = fmaf(sb.y, d0[3] + d1[3], acc[3]);
        if (it + kDepth < nit)
          load_i4<kSmem>(R, wcol0 + 4 * (it + kDepth) + tq, wcol0 + 4 * (it + kDepth) + g0, L[s]);
      }
    }
  }
  // lane (gq, tq) holds groups g0, g0 + 1 of token tq >> 1: add the other
  // two groups (lane tq ^ 1), then give lane tq = 0 both tokens (token 1
  // from lane tq = 2), the layout of run_tile (tokens 2 tq, 2 tq + 1)
  float lo = acc[0] + acc[1], hi = acc[2] + acc[3];
  lo += __shfl_xor_sync(0xffffffffu, lo, 1);
  hi += __shfl_xor_sync(0xffffffffu, hi, 1);
  const float lo1 = __shfl_xor_sync(0xffffffffu, lo, 2), hi1 = __shfl_xor_sync(0xffffffffu, hi, 2);
  return tq == 0 ? make_float4(lo, lo1, hi, hi1) : make_float4(0.f, 0.f, 0.f, 0.f);
}
// The int4 path of a tile: run_tile_i4 where it applies, else run_tile.
__device__ __forceinline__ bool i4_grouped(int f, int T, const Rows& R) {
  return f == MOE_Q_INT4_SYM_G32 && T <= 2 &&
         ((reinterpret_cast<uintptr_t>(R.s_lo) | reinterpret_cast<uintptr_t>(R.s_hi)) & 3u) == 0;
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
// ---------------------------------------------------------------- bounded waits
// Spin (one thread) until *p >= target, the abort flag is raised or the
// cycle budget runs out (checked before every new poll: with a budget of 0 a
// wait not met at its first poll gives up). Returns true when the target
// was reached; an expired budget leaves MOE_ERR_TIMEOUT with `detail` in the
// status word and raises the abort flag, which ends every other wait of the
// launch.
__device__ bool wait_counter(const uint32_t* p, uint32_t target, WsHeader* hdr, long long budget, int detail) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (clock64() - t0 >= budget) {
      flag_error(hdr, MOE_ERR_TIMEOUT, detail);
      atomicExch(&hdr->abort, 1);
      return false;
    }
    if (ld_acquire(p) >= target) return true;
    if ((it & 15) == 0 && *reinterpret_cast<volatile int*>(&hdr->abort)) return false;
    __nanosleep(it < 8 ? 32 : 256);  // back off: many warps may poll, and the counter's writers need its line
  }
}

// ---------------------------------------------------------------- job context
// What every job reads: set up once per launch in shared memory.
struct Ctx {
  const Params* P;
  uint8_t* smem;
  Plan L;
  int T, H, I, E, k, G, b;
  int e0, nrr, seg, nseg;   // router rows [e0, e0 + nrr) (+ the gate row last), segments per row
  int nreal;                // rows of W_r among them
  int n0, nr;               // output rows of this CTA
  int xexp[kMaxT];          // power-of-two scaling of x per token
  float bias[kMaxBias];     // router bias of this CTA's rows, [row][token]
  int fail;                 // a wait of this CTA gave up
  int rdone;                // router jobs finished
  moe_expert* desc;         // descriptors: slots 0..U-1, kSharedSlot
};

// ---------------------------------------------------------------- staging
// int4 and int2 job rows come into the warp's own shared-memory buffer by
// per-lane asynchronous copies (cp.async, 16 bytes each): all of a job's
// bytes are in flight at once and none of them occupies registers. Job row r
// (A rows 0-15) lies at r * cp, its scales at 16 cp + r * sp and its int2
// mins at 16 cp + 16 sp + r * sp (stage_pitches).
__device__ __forceinline__ bool stage_aligned(const moe_qmatrix& m) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(m.codes) | reinterpret_cast<uintptr_t>(m.scales) |
                      (m.qtype == MOE_Q_INT2_ASYM_G16 ? reinterpret_cast<uintptr_t>(m.mins) : 0u);
  return (a & 15u) == 0;
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
// Rows [row_lo, row_lo + n_lo) of m_lo become job rows 0.., rows [row_hi,
// row_hi + n_hi) of m_hi job rows 8..; columns [col0, col0 + ncol) of 16
// code bytes each, of a K-column matrix. The 16-byte pieces are dealt to the
// lanes row-major; one commit group for the whole job.
__device__ __noinline__ void stage_issue(const moe_qmatrix& m_lo, int row_lo, int n_lo, const moe_qmatrix& m_hi,
                                         int row_hi, int n_hi, int K, int col0, int ncol, uint8_t* sb, int cp,
                                         int sp) {
  const int lane = threadIdx.x & 31;
  const bool i2 = m_lo.qtype == MOE_Q_INT2_ASYM_G16;
  const int rb = K >> (i2 ? 2 : 1);    // code bytes per row
  const int sper = K >> (i2 ? 4 : 5);  // scales per row
  // codes: piece (r, c) for c < ncol
  {
    int r = 0, c = lane;
    while (c >= ncol) c -= ncol, ++r;
    for (; r < 16;) {
      const bool lo = r < 8;
      const int rr = r & 7;
      if (rr < (lo ? n_lo : n_hi)) {
        const moe_qmatrix& m = lo ? m_lo : m_hi;
        cp_async16(sb + r * cp + c * 16, m.codes + size_t((lo ? row_lo : row_hi) + rr) * rb + size_t(col0 + c) * 16);
      }
      c += 32;
      while (c >= ncol) c -= ncol, ++r;
    }
  }
  // scales, then int2 mins: su pieces per row
  const int su = ncol * (i2 ? 8 : 2) / 16;
  for (int mi = 0; mi < (i2 ? 2 : 1); ++mi) {
    int r = 0, c = lane;
    while (c >= su) c -= su, ++r;
    for (; r < 16;) {
      const bool lo = r < 8;
      const int rr = r & 7;
      if (rr < (lo ? n_lo : n_hi)) {
        const moe_qmatrix& m = lo ? m_lo : m_hi;
        const uint16_t* base = (mi ? m.mins : m.scales) + size_t((lo ? row_lo : row_hi) + rr) * sper +
                               size_t(col0) * (i2 ? 4 : 1);
        cp_async16(sb + 16 * cp + mi * 16 * sp + r * sp + c * 16, reinterpret_cast<const uint8_t*>(base) + c * 16);
      }
      c += 32;
      while (c >= su) c -= su, ++r;
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Rows of a staged job for run_tile / run_tile_i4 (weight columns from 0).
__device__ __forceinline__ Rows staged_rows(uint8_t* sb, int cp, int sp, bool lo, bool hi) {
  const int gq = (threadIdx.x & 31) >> 2;
  Rows R;
  R.lo = lo;
  R.hi = hi;
  R.c_lo = sb + gq * cp;
  R.c_hi = sb + (gq + 8) * cp;
  R.s_lo = reinterpret_cast<const uint16_t*>(sb + 16 * cp + gq * sp);
  R.s_hi = reinterpret_cast<const uint16_t*>(sb + 16 * cp + (gq + 8) * sp);
  R.m_lo = reinterpret_cast<const uint16_t*>(sb + 16 * cp + 16 * sp + gq * sp);
  R.m_hi = reinterpret_cast<const uint16_t*>(sb + 16 * cp + 16 * sp + (gq + 8) * sp);
  return R;
}

// gate/up tile part: 8 intermediate rows of gate (A rows 0-7) and of up
// (A rows 8-15) over part p of K. The last part to finish sums the parts
// (two fp32 values: the same sum in either order), applies SwiGLU and
// publishes h, its largest |h| per token and one more finished tile of its
// expert.
__device__ __noinline__ void job_gate_up(Ctx& C, const Job jb) {
  const Params& P = *C.P;
  const int T = C.T, H = C.H, I = C.I;
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3, warp = threadIdx.x >> 5;
  const int slot = jb.slot;
  const moe_expert& d = C.desc[slot];
  const int f = d.gate.qtype, ns = gu_parts(H);
  const int ncol = H / kc(f) / ns, col0 = jb.part * ncol, nit = ncol / 4;
  const int rb = row_code_bytes(f, H);
  const int row = jb.row0 + gq;
  const int sper = f == MOE_Q_INT8_PER_CHANNEL ? 1 : H / (f == MOE_Q_INT4_SYM_G32 ? 32 : 16);
  Rows R;
  R.lo = R.hi = true;
  R.c_lo = d.gate.codes + size_t(row) * rb;
  R.c_hi = d.up.codes + size_t(row) * rb;
  R.s_lo = d.gate.scales + size_t(row) * sper;
  R.s_hi = d.up.scales + size_t(row) * sper;
  R.m_lo = f == MOE_Q_INT2_ASYM_G16 ? d.gate.mins + size_t(row) * sper : nullptr;
  R.m_hi = f == MOE_Q_INT2_ASYM_G16 ? d.up.mins + size_t(row) * sper : nullptr;
  const uint8_t* bf = C.smem + C.L.o_xf + (f - 1) * 2 * T * H;  // formats 1..3 -> buffers 0..2
  float acc[4];
  if (C.L.o_stage >= 0 && f != MOE_Q_INT8_PER_CHANNEL && stage_aligned(d.gate) && stage_aligned(d.up)) {
    uint8_t* sb = C.smem + C.L.o_stage + warp * C.L.stage_bytes;
    int cp, sp;
    stage_pitches(f, ncol, cp, sp);
    stage_issue(d.gate, jb.row0, 8, d.up, jb.row0, 8, H, col0, ncol, sb, cp, sp);
    const Rows S = staged_rows(sb, cp, sp, true, true);  // the tile loop waits for the copies
    if (i4_grouped(f, T, S)) {
      const float4 v = run_tile_i4<true>(S, 0, col0, nit, bf, T);
      acc[0] = v.x, acc[1] = v.y, acc[2] = v.z, acc[3] = v.w;
    } else {
      run_any<true>(f, S, 0, col0, nit, bf, T, acc);
    }
  } else if (i4_grouped(f, T, R)) {
    const float4 v = run_tile_i4<false>(R, col0, col0, nit, bf, T);
    acc[0] = v.x, acc[1] = v.y, acc[2] = v.z, acc[3] = v.w;
  } else {
    run_any<false>(f, R, col0, col0, nit, bf, T, acc);
  }
  // D rows gq (gate) / gq + 8 (up), tokens 2 tq, 2 tq + 1
  if (ns > 1) {
    float* rs = reinterpret_cast<float*>(C.smem + C.L.o_red) + size_t(jb.tile) * 16 * T;
    int* td = reinterpret_cast<int*>(C.smem + C.L.o_td) + jb.tile;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = gq + 8 * (i >> 1), t = 2 * tq + (i & 1);
      if (t < T) atomicAdd(rs + r * T + t, acc[i]);
    }
    __syncwarp();
    int prev = 0;
    if (lane == 0) {
      __threadfence_block();
      prev = atomicAdd(td, 1);
    }
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != ns - 1) return;
    __threadfence_block();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = gq + 8 * (i >> 1), t = 2 * tq + (i & 1);
      acc[i] = t < T ? *reinterpret_cast<volatile float*>(rs + r * T + t) : 0.f;
    }
  }
  float* hs = P.h + size_t(slot) * T * I;
  uint32_t* am = P.cnt + slot * kCntStride + 1;
  float gsc = 1.f, usc = 1.f;
  if (f == MOE_Q_INT8_PER_CHANNEL) {
    gsc = f16_to_f32(d.gate.scales[row]);
    usc = f16_to_f32(d.up.scales[row]);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int t = 2 * tq + i;
    float h = 0.f;
    if (t < T) {
      const float sc = exp2i(C.xexp[t]);
      const float g = acc[i] * gsc * sc, u = acc[2 + i] * usc * sc;
      h = silu_f32(g) * u;
      __stcg(hs + size_t(t) * I + row, h);
      // also in fp16, unscaled, where the down job's activations go: used
      // as they are when no token of the expert needs range scaling
      P.h16[size_t(slot) * T * I + frag_pos(f, row, t, T) / 2] = __float2half_rn(h);
    }
    // largest |h| of the tile per token: lanes of equal tq hold the same token
    uint32_t a = t < T ? __float_as_uint(fabsf(h)) : 0u;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (gq == 0 && t < T) atomicMax(am + t, a);
  }
  // the warp barrier orders every lane's stores before lane 0's release
  __syncwarp();
  if (lane == 0) red_release(P.cnt + slot * kCntStride, 1u);
}

// L2 prefetch of piece w (0..5) of gate/up tile r (intermediate rows
// 8r .. 8r + 7, whole K) of an expert: 0/1 the gate/up codes, 2/3 their
// scales, 4/5 their mins (int2).
__device__ __noinline__ void prefetch_tile_piece(const moe_expert& d, int H, int r, int w) {
  const moe_qmatrix& m = (w & 1) ? d.up : d.gate;
  const int f = m.qtype;
  const int rb = H >> (f == MOE_Q_INT4_SYM_G32 ? 1 : f == MOE_Q_INT2_ASYM_G16 ? 2 : 0);
  const int sper = f == MOE_Q_INT8_PER_CHANNEL ? 1 : H >> (f == MOE_Q_INT4_SYM_G32 ? 5 : 4);
  const size_t row = size_t(8) * r;
  if (w < 2) prefetch_l2(m.codes + row * rb, uint32_t(8 * rb));
  else if (w < 4) prefetch_l2(m.scales + row * sper, uint32_t(16 * sper));
  else if (f == MOE_Q_INT2_ASYM_G16) prefetch_l2(m.mins + row * sper, uint32_t(16 * sper));
}
// L2 prefetch of output rows [n0, n0 + nr) of a down matrix: piece 0 codes,
// 1 scales, 2 mins (int2).
__device__ __noinline__ void prefetch_down_piece(const moe_qmatrix& m, int I, int n0, int nr, int w) {
  const int f = m.qtype;
  const int rb = I >> (f == MOE_Q_INT4_SYM_G32 ? 1 : f == MOE_Q_INT2_ASYM_G16 ? 2 : 0);
  const int sper = f == MOE_Q_INT8_PER_CHANNEL ? 1 : I >> (f == MOE_Q_INT4_SYM_G32 ? 5 : 4);
  if (w == 0) prefetch_l2(m.codes + size_t(n0) * rb, uint32_t(nr * rb));
  else if (w == 1) prefetch_l2(m.scales + size_t(n0) * sper, uint32_t(nr * sper * 2));
  else if (m.qtype == MOE_Q_INT2_ASYM_G16) prefetch_l2(m.mins + size_t(n0) * sper, uint32_t(nr * sper * 2));
}

// h of one expert (fp32 [T][I] in the workspace) into a warp's activation
// buffer in format F's fragment order, scaled by 2^-eh[t] per token; 8 loads
// per lane in flight at a time.
template <int F>
__device__ __noinline__ void h_to_frag(const float4* hs, int T, int I, const int* eh, uint8_t* hf) {
  const int lane = threadIdx.x & 31, n4 = T * I / 4;  // I % 4 == 0: a float4 holds four values of one token
  for (int base = lane; base < n4; base += 8 * 32) {
    float4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = base + 32 * j < n4 ? __ldcg(hs + base + 32 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = 4 * (base + 32 * j);
      if (i < T * I) {
        const int t = int(i >= I) + int(i >= 2 * I) + int(i >= 3 * I);  // T <= 4
        const float sc = exp2i(-eh[t]);
        store4<F>(hf, i - t * I, t, T, v[j].x * sc, v[j].y * sc, v[j].z * sc, v[j].w * sc);
      }
    }
  }
}

// down job: this CTA's output rows [n0, n0 + nr) of one expert (already on
// their way into L2 since the top-k). The warp waits for the expert's
// gate/up tiles, converts h (scaled into the fp16 range) into its own
// activation buffer and runs the MMAs. Results go to Y[slot].
__device__ __noinline__ void job_down(Ctx& C, const Job jb) {
  const Params& P = *C.P;
  const int T = C.T, I = C.I;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const int slot = jb.slot;
  const moe_expert& d = C.desc[slot];
  const int f = d.down.qtype;
  const int nit = I / kc(f) / 4;
  const int rb = row_code_bytes(f, I);
  const int sper = f == MOE_Q_INT8_PER_CHANNEL ? 1 : I / (f == MOE_Q_INT4_SYM_G32 ? 32 : 16);
  const int rlo = jb.row0 + gq, rhi = jb.row0 + gq + 8;
  Rows R;
  R.lo = gq < jb.nrows;
  R.hi = gq + 8 < jb.nrows;
  R.c_lo = d.down.codes + size_t(R.lo ? rlo : 0) * rb;
  R.c_hi = d.down.codes + size_t(R.hi ? rhi : 0) * rb;
  R.s_lo = d.down.scales + size_t(R.lo ? rlo : 0) * sper;
  R.s_hi = d.down.scales + size_t(R.hi ? rhi : 0) * sper;
  R.m_lo = f == MOE_Q_INT2_ASYM_G16 ? d.down.mins + size_t(R.lo ? rlo : 0) * sper : nullptr;
  R.m_hi = f == MOE_Q_INT2_ASYM_G16 ? d.down.mins + size_t(R.hi ? rhi : 0) * sper : nullptr;
  uint8_t* hf = C.smem + C.L.o_hf + warp * 2 * T * I;
  __shared__ int s_eh[kWarps][kMaxT];
  // this job's rows on their way while its expert's gate/up tiles finish:
  // into the warp's staging buffer (int4, int2), else into L2 (the shared
  // expert's are in L2 since phase A)
  const bool staged = C.L.o_stage >= 0 && f != MOE_Q_INT8_PER_CHANNEL && stage_aligned(d.down);
  uint8_t* sb = C.smem + C.L.o_stage + warp * C.L.stage_bytes;
  int cp = 0, sp = 0;
  if (staged) {
    stage_pitches(f, I / kc(f), cp, sp);
    stage_issue(d.down, jb.row0, min(int(jb.nrows), 8), d.down, jb.row0 + 8, max(int(jb.nrows) - 8, 0), I, 0,
                I / kc(f), sb, cp, sp);
  } else if (slot != kSharedSlot && lane < 3) {
    prefetch_down_piece(d.down, I, jb.row0, jb.nrows, lane);
  }
  int ok = 1;
  if (lane == 0)
    ok = wait_counter(P.cnt + slot * kCntStride, uint32_t(I / 8), P.hdr, P.wait_cycles, 7100000 + slot) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (!ok) {
    if (lane == 0) C.fail = 1;
    if (staged) stage_wait();  // the copies land before the warp moves on
    return;
  }
  (void)ld_acquire(P.cnt + slot * kCntStride);  // every lane orders its reads of h after the counter
  if (lane < T) s_eh[warp][lane] = range_exp(__ldcg(P.cnt + slot * kCntStride + 1 + lane));
  __syncwarp();
  bool unscaled = true;
  for (int t = 0; t < T; ++t) unscaled &= s_eh[warp][t] == 0;
  if (unscaled) {
    // every |h| of the expert fits fp16: its tiles' fp16 copy is exactly what
    // the conversion below would produce; 8 loads per lane in flight
    const uint4* src = reinterpret_cast<const uint4*>(P.h16 + size_t(slot) * T * I);
    uint4* dst = reinterpret_cast<uint4*>(hf);
    const int n16 = T * I / 8;  // 16-byte pieces
    for (int base = lane; base < n16; base += 8 * 32) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = base + 32 * j < n16 ? __ldcg(src + base + 32 * j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (base + 32 * j < n16) dst[base + 32 * j] = v[j];
    }
  } else {
    const float4* hs = reinterpret_cast<const float4*>(P.h + size_t(slot) * T * I);
    if (f == MOE_Q_INT4_SYM_G32) h_to_frag<MOE_Q_INT4_SYM_G32>(hs, T, I, s_eh[warp], hf);
    else if (f == MOE_Q_INT2_ASYM_G16) h_to_frag<MOE_Q_INT2_ASYM_G16>(hs, T, I, s_eh[warp], hf);
    else h_to_frag<MOE_Q_INT8_PER_CHANNEL>(hs, T, I, s_eh[warp], hf);
  }
  __syncwarp();
  float acc[4];
  if (staged) {
    const Rows S = staged_rows(sb, cp, sp, R.lo, R.hi);  // the tile loop waits for the copies
    if (i4_grouped(f, T, S)) {
      const float4 v = run_tile_i4<true>(S, 0, 0, nit, hf, T);
      acc[0] = v.x, acc[1] = v.y, acc[2] = v.z, acc[3] = v.w;
    } else {
      run_any<true>(f, S, 0, 0, nit, hf, T, acc);
    }
  } else if (i4_grouped(f, T, R)) {
    const float4 v = run_tile_i4<false>(R, 0, 0, nit, hf, T);
    acc[0] = v.x, acc[1] = v.y, acc[2] = v.z, acc[3] = v.w;
  } else {
    run_any<false>(f, R, 0, 0, nit, hf, T, acc);
  }
  float* y = reinterpret_cast<float*>(C.smem + C.L.o_y) + size_t(slot) * 16 * T;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = gq + 8 * (i >> 1), t = 2 * tq + (i & 1);
    if (r < jb.nrows && t < T) {
      float v = acc[i] * exp2i(s_eh[warp][t]);
      if (f == MOE_Q_INT8_PER_CHANNEL) v *= f16_to_f32(d.down.scales[jb.row0 + r]);
      y[r * T + t] = v;
    }
  }
  __syncwarp();
}

// The weights of router part (row e0 + r, floats [s seg, (s + 1) seg)) for
// this lane: 4 (or 2) 16-byte loads. Issued before anything else of the
// launch, so the router's bytes are on their way while the prologue runs.
__device__ __forceinline__ void router_load(const Params& P, int e0, int nreal, int seg, const Job& jb,
                                            uint4 (&w)[4]) {
  const int lane = threadIdx.x & 31;
  const bool gate_row = jb.slot >= nreal;  // the shared expert's gate vector
  const float* wr = (gate_row ? P.shared_gate : P.w_router + size_t(e0 + jb.slot) * P.H) + jb.part * seg;
  const int nv = seg / 128;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (i < nv) w[i] = ldg16(wr + 4 * lane + 128 * i);
}

// router part: row e0 + r, floats [s seg, (s + 1) seg) of it, with its
// weights already loaded; the last part of the CTA to finish sums each row's
// parts in order, adds the bias, publishes the logits and arrives on the
// grid counter.
__device__ __noinline__ void job_router(Ctx& C, const Job jb, const uint4 w0, const uint4 w1, const uint4 w2,
                                        const uint4 w3) {
  const Params& P = *C.P;
  const int T = C.T, H = C.H, E = C.E, seg = C.seg, nseg = C.nseg;
  const int lane = threadIdx.x & 31;
  const float* x32 = reinterpret_cast<const float*>(C.smem + C.L.o_x32);
  float* rp = reinterpret_cast<float*>(C.smem + C.L.o_rp);
  const int nv = seg / 128;  // 16-byte loads per lane (4 or 2)
  const uint4 w[4] = {w0, w1, w2, w3};
#pragma unroll 1
  for (int t = 0; t < T; ++t) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < nv) {
        const float4 xv = *reinterpret_cast<const float4*>(x32 + t * H + jb.part * seg + 4 * lane + 128 * i);
        a = fmaf(__uint_as_float(w[i].x), xv.x,
                 fmaf(__uint_as_float(w[i].y), xv.y, fmaf(__uint_as_float(w[i].z), xv.z, fmaf(__uint_as_float(w[i].w), xv.w, a))));
      }
    a = warp_sum(a);
    if (lane == 0) rp[(jb.slot * nseg + jb.part) * T + t] = a;
  }
  __syncwarp();
  int prev = 0;
  if (lane == 0) {
    __threadfence_block();
    prev = atomicAdd(&C.rdone, 1);
  }
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != C.nrr * nseg - 1) return;
  __threadfence_block();
  for (int i = lane; i < C.nrr * T; i += 32) {
    const int r = i / T, t = i - r * T;
    float a = 0.f;
    for (int s = 0; s < nseg; ++s) a += *reinterpret_cast<volatile float*>(rp + (r * nseg + s) * T + t);
    if (r >= C.nreal) {
      __stcg(P.sgate + t, a);
      continue;
    }
    const float bv = C.bias[r * T + t];
    __stcg(P.logits + size_t(t) * E + C.e0 + r, a + bv);
    if (P.flags & MOE_BIAS_SELECTION_ONLY) __stcg(P.logits_u + size_t(t) * E + C.e0 + r, a);
  }
  // the warp barrier orders every lane's stores before lane 0's release
  __syncwarp();
  if (lane == 0) red_release(&P.hdr->bar_count, 1u);
}

// ---------------------------------------------------------------- routing
// Routing of one CTA, by all its warps once phase A is done: wait for every
// CTA's logits; top-k per token in two rounds (each warp sorts 32-logit
// chunks and keeps the best k of each; then every kept candidate's rank
// among its token's candidates, the best k by rank); gates; the distinct
// picked experts in ascending id order (slots) and their descriptors.
// Returns whether phases B and C run (the same answer on every CTA:
// identical inputs, identical code).
struct RouteShared {
  int idx[kMaxT * kMaxK];
  float w[kMaxT * kMaxK];
  uint32_t key[kMaxT * kMaxK];
  int slot[kMaxT * kMaxK];  // (t, j) -> slot
  int uniq[kMaxT * kMaxK];  // slot -> expert id
  uint32_t bits[kMaxE / 32];
  uint32_t bpre[kMaxE / 32];  // set bits in the words before
  uint64_t best[kMaxT * kMaxE / 32];  // each chunk's best candidate
  uint64_t cut[kMaxT];                // the k-th best chunk winner of each token
  int nsurv[kMaxT];                   // candidates at or above it
  int U, bad;
};

// Bitonic sort of 32 keys, one per lane, into descending lane order.
__device__ __forceinline__ uint64_t warp_sort32_desc(uint64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, v, stride);
      // the lower lane of a pair keeps the larger key in a descending run
      const bool keep_max = ((lane & size) == 0) == ((lane & stride) == 0);
      v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
    }
  return v;
}

__device__ __noinline__ bool route_all(Ctx& C, RouteShared& R, bool has_shared) {
  const Params& P = *C.P;
  const int T = C.T, E = C.E, k = C.k, H = C.H, I = C.I, G = C.G, b = C.b;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool given = P.counts != nullptr;  // experts only: the picks are the dispatched experts
  if (threadIdx.x == 0 && !given) {
    if (!wait_counter(&P.hdr->bar_count, uint32_t(G), P.hdr, P.wait_cycles, 7000000 + b)) C.fail = 1;
  }
  if (threadIdx.x < kMaxE / 32) R.bits[threadIdx.x] = 0u;
  __syncthreads();
  const bool live = !C.fail;
  if (given) {
    // the experts with rows (at most T k of them, each used by at most T rows)
    for (int e = threadIdx.x; e < E; e += kThreads) {
      const int c = __ldg(P.counts + e);
      if (c < 0 || c > T) R.bad = 1;
      else if (c > 0) atomicOr(&R.bits[e >> 5], 1u << (e & 31));
    }
  } else {
  // first round: chunk ch of token t = logits [32 ch, 32 ch + 32); CTA 0 also
  // exports the logits
  const int n32 = (E + 31) / 32, nc = n32 * k;
  uint64_t* cand = reinterpret_cast<uint64_t*>(C.smem + C.L.o_cand);  // [T][n32][k]
  if (live)
    for (int q = warp; q < T * n32; q += kWarps) {
      const int t = q / n32, e = (q - t * n32) * 32 + lane;
      uint64_t v = 0ull;
      if (e < E) {
        const float l = __ldcg(P.logits + size_t(t) * E + e);
        if (b == 0 && P.logits_out) P.logits_out[size_t(t) * E + e] = l;
        v = (uint64_t(f2key(l)) << 32) | uint64_t(~uint32_t(e));  // key descending, then id ascending
      }
      v = warp_sort32_desc(v);
      if (lane < k) cand[size_t(q) * k + lane] = v;
      if (lane == 0) R.best[q] = v;
    }
  __syncthreads();
  // cutoff of each token: its k-th best chunk winner. Those k winners are k
  // logits at or above it, so every one of the token's top k is too; and
  // only the k chunks they head can hold candidates at or above it, so at
  // most k^2 candidates survive (all of them when there are fewer than k
  // chunks: cutoff 0)
  if (live && warp < T) {
    const int t = warp;
    uint64_t v = lane < n32 ? R.best[t * n32 + lane] : 0ull;
    v = warp_sort32_desc(v);
    const uint64_t cut = __shfl_sync(0xffffffffu, v, k - 1);
    if (lane == 0) {
      R.cut[t] = n32 >= k ? cut : 0ull;
      R.nsurv[t] = 0;
    }
  }
  __syncthreads();
  uint64_t* surv = cand + size_t(T) * nc;  // [T][k k]
  if (live)
    for (int q = threadIdx.x; q < T * nc; q += kThreads) {
      const int t = q / nc;
      const uint64_t v = cand[q];
      if (v != 0ull && v >= R.cut[t]) surv[t * k * k + atomicAdd(&R.nsurv[t], 1)] = v;  // v == 0: no logit
    }
  __syncthreads();
  // second round: a survivor's rank among its token's survivors (keys are
  // distinct: the low word is the id); the best k go to their rank's place
  if (live)
    for (int q = threadIdx.x; q < T * k * k; q += kThreads) {
      const int t = q / (k * k), i = q - t * (k * k), ns = R.nsurv[t];
      if (i >= ns) continue;
      const uint64_t* c = surv + size_t(t) * k * k;
      const uint64_t v = c[i];
      int rank = 0;
      for (int j = 0; j < ns; ++j) rank += c[j] > v ? 1 : 0;
      if (rank < k) {
        R.key[t * k + rank] = uint32_t(v >> 32);
        R.idx[t * k + rank] = int(~uint32_t(v));
      }
    }
  __syncthreads();
  // gates (one warp per token): the softmax over all logits restricted to the
  // picks and renormalised = a softmax over the picked logits (of the
  // unbiased ones when the bias only selects)
  if (live && warp < T) {
    const int t = warp;
    const bool sel_only = (P.flags & MOE_BIAS_SELECTION_ONLY) != 0;
    float v = -CUDART_INF_F;
    if (lane < k) v = sel_only ? __ldcg(P.logits_u + size_t(t) * E + R.idx[t * k + lane]) : key2f(R.key[t * k + lane]);
    float v0 = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v0 = fmaxf(v0, __shfl_xor_sync(0xffffffffu, v0, o));
    const float ev = lane < k ? expf(v - v0) : 0.f;
    const float den = warp_sum(ev);
    if (lane < k) {
      R.w[t * k + lane] = ev / den;
      const int id = R.idx[t * k + lane];
      if (id >= 0 && id < E) atomicOr(&R.bits[id >> 5], 1u << (id & 31));
      else R.bad = 1;
    }
  }
  }
  __syncthreads();
  moe_expert* desc = C.desc;
  if (warp == 0) {
    // slots: the slot of an id = set bits below it (warp scan over the bitmap)
    static_assert(kMaxE / 32 == 32, "one bitmap word per lane");
    const uint32_t c = __popc(R.bits[lane]);
    uint32_t inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    R.bpre[lane] = inc - c;
    if (lane == 31) {
      R.U = int(inc);
      if (int(inc) > T * k) R.bad = 1;  // more experts than rows (experts only: bad counts)
    }
  }
  __syncthreads();
  const int U = R.U;
  if (live && R.bad == 0) {
    // slot of an expert = picked experts below it; routing: slot of each pick
    for (int e = threadIdx.x; e < E; e += kThreads) {
      const uint32_t wb = R.bits[e >> 5];
      if ((wb >> (e & 31)) & 1u) R.uniq[R.bpre[e >> 5] + __popc(wb & ((1u << (e & 31)) - 1u))] = e;
    }
    if (!given)
      for (int i = threadIdx.x; i < T * k; i += kThreads) {
        const int id = R.idx[i], wd = id >> 5;
        R.slot[i] = int(R.bpre[wd] + __popc(R.bits[wd] & ((1u << (id & 31)) - 1u)));
      }
  }
  __syncthreads();
  // descriptors of the picked experts (the table is in L2 since the entry):
  // U W <= kMaxT kMaxK W words over all threads, loads first
  constexpr int W = int(sizeof(moe_expert) / 4);
  constexpr int kPer = (kMaxT * kMaxK * W + kThreads - 1) / kThreads;
  if (live && R.bad == 0) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(P.experts);
    uint32_t* dst = reinterpret_cast<uint32_t*>(desc);
    uint32_t v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = threadIdx.x + j * kThreads;
      v[j] = i < U * W ? src[size_t(R.uniq[i / W]) * W + (i % W)] : 0u;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      if (threadIdx.x + j * kThreads < U * W) dst[threadIdx.x + j * kThreads] = v[j];
  }
  __syncthreads();
  if (live && R.bad == 0 && threadIdx.x < U && !expert_ok(desc[threadIdx.x], H, I)) R.bad = 1;
  __syncthreads();
  const bool work = live && R.bad == 0;
  if (live && !work && threadIdx.x == 0) flag_error(P.hdr, MOE_ERR_DEVICE_FAULT, 1000000);
  return work;
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ Ctx C;
  __shared__ RouteShared R;
  __shared__ uint32_t s_xamax[kMaxT];
  __shared__ int s_bad;

  const int T = P.T, H = P.H, I = P.I, E = P.E, k = P.k;
  const int G = gridDim.x, b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = P.hdr;
  const bool has_shared = P.shared != nullptr;
  const bool gate_row = P.shared_gate != nullptr && has_shared;
  const bool given = P.counts != nullptr;  // experts only: no router, no combine
  const Plan& L = P.L;

  // ---------------------------------------------------------- loads first
  // This warp's router part (phase-A job `warp`, when there is one), then
  // everything else the prologue reads, all in flight together: x (this
  // thread's 8-element groups), the bias of this CTA's router rows and the
  // shared expert's descriptor; the expert table goes into L2 for the routing.
  int e0, nreal;
  router_range(E, G, b, e0, nreal);
  const int seg = router_seg(H), nseg = H / seg;
  const int nrr = given ? 0 : router_rows_of(E, G, b, gate_row);
  const int nA = nrr * nseg;
  uint4 w0[4] = {};
  if (warp < nA) router_load(P, e0, nreal, seg, phase_a_job(H, warp), w0);
  constexpr int kXg = kMaxT * kMaxH / 8 / kThreads;
  const int ng = T * H / 8;
  uint4 xg[kXg];
#pragma unroll
  for (int j = 0; j < kXg; ++j) {
    const int g = threadIdx.x + j * kThreads;
    xg[j] = g < ng ? ldg16(P.x + size_t(g) * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
  float bias_v = 0.f;
  if (P.bias && threadIdx.x < nreal * T) {
    const int r = threadIdx.x / T, t = threadIdx.x - r * T;
    bias_v = P.bias[t * P.bstride + e0 + r];
  }
  constexpr int kDescWords = int(sizeof(moe_expert) / 4);
  uint32_t sdesc_v = 0u;
  if (has_shared && threadIdx.x < kDescWords) sdesc_v = reinterpret_cast<const uint32_t*>(P.shared)[threadIdx.x];
  {
    const size_t tbytes = size_t(E) * sizeof(moe_expert);
    const size_t l = size_t(b) * kThreads + threadIdx.x;
    const char* tb = reinterpret_cast<const char*>(P.experts);
    if (l * 128 < tbytes) prefetch_line_l2(tb + l * 128);
    if (l == 0) prefetch_line_l2(tb + tbytes - 1);
  }

  // ---------------------------------------------------------- prologue
  moe_expert* desc = reinterpret_cast<moe_expert*>(smem + L.o_desc);
  if (threadIdx.x == 0) {
    C.P = &P;
    C.smem = smem;
    C.L = L;
    C.T = T, C.H = H, C.I = I, C.E = E, C.k = k, C.G = G, C.b = b;
    C.e0 = e0;
    C.nreal = nreal;
    C.nrr = nrr;
    C.seg = seg;
    C.nseg = nseg;
    out_rows(H, G, b, C.n0, C.nr);
    C.fail = 0;
    C.rdone = 0;
    C.desc = desc;
    s_bad = 0;
    R.bad = 0;
    R.U = 0;
  }
  if (threadIdx.x < kMaxT) s_xamax[threadIdx.x] = 0u;
  __syncthreads();
  if (has_shared && threadIdx.x < kDescWords) reinterpret_cast<uint32_t*>(desc + kSharedSlot)[threadIdx.x] = sdesc_v;
  if (threadIdx.x < kMaxBias) C.bias[threadIdx.x] = bias_v;  // zero beyond the CTA's rows
  {
    const int ntl = max_tiles(T, I, E, k, G);
    float* Y = reinterpret_cast<float*>(smem + L.o_y);
    float* red = reinterpret_cast<float*>(smem + L.o_red);
    int* tdone = reinterpret_cast<int*>(smem + L.o_td);
    for (int i = threadIdx.x; i < kMaxSlots * 16 * T; i += kThreads) Y[i] = 0.f;
    for (int i = threadIdx.x; i < ntl * 16 * T; i += kThreads) red[i] = 0.f;
    for (int i = threadIdx.x; i < ntl; i += kThreads) tdone[i] = 0;
  }
  // x in fp32 (router) and the largest |x| per token
  {
    float* x32 = reinterpret_cast<float*>(smem + L.o_x32);
#pragma unroll
    for (int j = 0; j < kXg; ++j) {
      const int g = threadIdx.x + j * kThreads;
      // a warp's 32 groups (256 elements) belong to one token (H % 256 == 0)
      // and are all in range together (T H % 256 == 0)
      if (g < ng) {
        const uint32_t wv[4] = {xg[j].x, xg[j].y, xg[j].z, xg[j].w};
        float v[8];
        uint32_t m = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[e] = bf16_to_f32(uint16_t(e & 1 ? wv[e >> 1] >> 16 : wv[e >> 1] & 0xffffu));
          m = max(m, __float_as_uint(fabsf(v[e])));
        }
        reinterpret_cast<float4*>(x32)[2 * g] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(x32)[2 * g + 1] = make_float4(v[4], v[5], v[6], v[7]);
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) atomicMax(&s_xamax[g * 8 / H], m);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < T) C.xexp[threadIdx.x] = range_exp(s_xamax[threadIdx.x]);
  if (threadIdx.x == 0 && has_shared && !expert_ok(desc[kSharedSlot], H, I)) {
    s_bad = 1;
    flag_error(hdr, MOE_ERR_DEVICE_FAULT, 2000000);
  }
  __syncthreads();
  if (nrr == 0 && threadIdx.x == 0) red_release(&hdr->bar_count, 1u);  // no router rows: arrive at once
  __syncthreads();

  // ---------------------------------------------------------- phase A
  for (int j = warp; j < nA; j += kWarps) {
    const Job jb = phase_a_job(H, j);
    uint4 w[4] = {};
    if (j == warp) {
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = w0[i];
    } else {
      router_load(P, e0, nreal, seg, jb, w);
    }
    job_router(C, jb, w[0], w[1], w[2], w[3]);
  }
  // While the grid gathers the logits: the shared expert's gate/up tiles of
  // this CTA and its down rows into L2 (needed whatever the routing), and the
  // activations in fragment order for all three formats (so routed experts
  // of any format need no further barrier).
  if (has_shared && !s_bad) {
    const int nsh = bc_tiles(I, G, b, 1);  // its tiles come first in the B/C list
    for (int q = threadIdx.x; q < nsh * 6; q += kThreads)
      prefetch_tile_piece(desc[kSharedSlot], H, b + G * (q / 6), q % 6);
    if (C.nr > 0 && threadIdx.x >= kThreads - 3)
      prefetch_down_piece(desc[kSharedSlot].down, I, C.n0, C.nr, threadIdx.x - (kThreads - 3));
  }
#pragma unroll
  for (int j = 0; j < kXg; ++j) {
    const int g = threadIdx.x + j * kThreads;
    if (g < ng) {
      const int t = g * 8 / H, k0 = g * 8 - t * H;
      const float sc = exp2i(-C.xexp[t]);
      const uint32_t wv[4] = {xg[j].x, xg[j].y, xg[j].z, xg[j].w};
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = bf16_to_f32(uint16_t(e & 1 ? wv[e >> 1] >> 16 : wv[e >> 1] & 0xffffu)) * sc;
      uint8_t* xf = smem + L.o_xf;
      store4<MOE_Q_INT4_SYM_G32>(xf, k0, t, T, v[0], v[1], v[2], v[3]);
      store4<MOE_Q_INT4_SYM_G32>(xf, k0 + 4, t, T, v[4], v[5], v[6], v[7]);
      store4<MOE_Q_INT2_ASYM_G16>(xf + 2 * T * H, k0, t, T, v[0], v[1], v[2], v[3]);
      store4<MOE_Q_INT2_ASYM_G16>(xf + 2 * T * H, k0 + 4, t, T, v[4], v[5], v[6], v[7]);
      store4<MOE_Q_INT8_PER_CHANNEL>(xf + 4 * T * H, k0, t, T, v[0], v[1], v[2], v[3]);
      store4<MOE_Q_INT8_PER_CHANNEL>(xf + 4 * T * H, k0 + 4, t, T, v[4], v[5], v[6], v[7]);
    }
  }

  // ---------------------------------------------------------- routing
  const bool work = route_all(C, R, has_shared) && !s_bad;

  // ---------------------------------------------------------- phases B, C
  if (work) {
    const int U = R.U;
    const int nJ = phase_bc_count(H, I, G, b, U, has_shared);
    for (int j = warp; j < nJ; j += kWarps) {
      const Job jb = phase_bc_job(H, I, G, b, U, has_shared, j);
      if (jb.kind == kGateUp) job_gate_up(C, jb);
      else job_down(C, jb);
    }
  }
  __syncthreads();

  // ---------------------------------------------------------- combine
  if (work && !C.fail && given) {
    // experts only: this CTA's columns [n0, n0 + nr) of every dispatched row,
    // rounded once to bf16 (the rows of an expert are [offsets[e],
    // offsets[e] + counts[e]); a row's token is perm_src / k)
    const float* Y = reinterpret_cast<const float*>(smem + L.o_y);
    const int nr = C.nr, n0 = C.n0, U = R.U;
    for (int r = threadIdx.x; r < T * k; r += kThreads) R.slot[r] = -1;
    __syncthreads();
    for (int u = threadIdx.x; u < U; u += kThreads) {
      const int e = R.uniq[u], r0 = __ldg(P.offsets + e), c = __ldg(P.counts + e);
      for (int j = 0; j < c; ++j)
        if (r0 + j >= 0 && r0 + j < T * k) R.slot[r0 + j] = u;
    }
    __syncthreads();
    for (int q = threadIdx.x; q < T * k * nr; q += kThreads) {
      const int r = q / nr, i = q - r * nr;
      const int u = R.slot[r], ps = __ldg(P.perm_src + r), t = ps / k;
      if (u >= 0 && ps >= 0 && t < T) P.y_perm[size_t(r) * H + n0 + i] = f32_to_bf16_rn(Y[(u * 16 + i) * T + t]);
    }
  } else if (work && !C.fail) {
    const float* Y = reinterpret_cast<const float*>(smem + L.o_y);
    const int nr = C.nr, n0 = C.n0;
    for (int i = threadIdx.x; i < T * nr; i += kThreads) {
      const int t = i / nr, r = i - t * nr;
      float a = 0.f;
      for (int j = 0; j < k; ++j) a = fmaf(R.w[t * k + j], Y[(R.slot[t * k + j] * 16 + r) * T + t], a);
      if (has_shared) {
        const float ys = Y[(kSharedSlot * 16 + r) * T + t];
        a = P.shared_gate ? fmaf(1.f / (1.f + expf(-__ldcg(P.sgate + t))), ys, a) : a + ys;
      }
      P.out[size_t(t) * H + n0 + r] = f32_to_bf16_rn(a);
    }
    if (b == 0) {
      for (int i = threadIdx.x; i < T * k; i += kThreads) {
        P.topk_idx[i] = R.idx[i];
        P.topk_w[i] = R.w[i];
        if (P.heat) atomicAdd(P.heat + R.idx[i], 1u);
      }
    }
  }

  // ---------------------------------------------------------- exit
  // The last CTA out clears the launch's counters for the next launch.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&hdr->exit_count, 1u);
    if (prev == uint32_t(G) - 1) {
      __threadfence();
      for (int i = 0; i < kMaxSlots; ++i)
        for (int j = 0; j <= kMaxT; ++j) P.cnt[i * kCntStride + j] = 0u;
      hdr->bar_count = 0;
      hdr->abort = 0;
      hdr->exit_count = 0;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------- host side
constexpr int kStaticSmem = kStaticSmemBound;

int grid_size() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

// Whether the shape runs as one fused launch on a grid of G CTAs.
bool eligible_on(int T, int H, int I, int E, int k, int G) {
  if (T < 1 || T > kMaxT || k < 1 || k > kMaxK || E < k || E > kMaxE) return false;
  if (H < 256 || I < 256 || H > kMaxH || I > kMaxI || (H % 256) || (I % 256)) return false;
  if (router_rows(E, G) * T > kMaxBias) return false;
  if ((H + G - 1) / G > 16) return false;             // output rows per CTA fit one 16-row tile
  return make_plan(T, H, I, E, k, G).total + kStaticSmem <= kSmemLimit;
}

}  // namespace dfx

bool decode_fused_eligible(int T, int H, int I, int E, int k) {
  return dfx::eligible_on(T, H, I, E, k, dfx::grid_size());
}

size_t decode_fused_ws_bytes(int T, int I) {
  // h of every expert slot in fp32, then in fp16 (fragment order)
  return size_t(dfx::kMaxSlots) * size_t(T) * size_t(I) * (sizeof(float) + sizeof(__half));
}

cudaError_t launch_decode_fused(const uint16_t* x, int T, int H, int I, int E, int k, const float* w_router,
                                const float* bias, long long bstride, const moe_expert* experts,
                                const moe_expert* shared, int* topk_idx, float* topk_w, float* logits_out,
                                uint16_t* out, float* logits_ws, float* h_ws, uint32_t* counters, WsHeader* hdr,
                                long long wait_cycles, uint32_t flags, const float* shared_gate, float* logits_u_ws,
                                float* sgate_ws, uint32_t* heat, const int32_t* perm_src, const int32_t* offsets,
                                const int32_t* counts, uint16_t* y_perm, cudaStream_t st) {
  using namespace dfx;
  const int grid = grid_size();
  const size_t smem = size_t(make_plan(T, H, I, E, k, grid).total);
  // the kernel's dynamic shared-memory cap: raised once per device to the
  // most any plan may take
  static int s_cap_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !s_cap_set[dev]) {
    e = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemLimit - kStaticSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) s_cap_set[dev] = 1;
  }
  Params P{make_plan(T, H, I, E, k, grid), x, T, H, I, E, k, w_router, bias,
           bstride, experts, shared, topk_idx, topk_w, logits_out, out, hdr,
           logits_ws, h_ws, reinterpret_cast<__half*>(h_ws + size_t(kMaxSlots) * T * I), counters, wait_cycles, flags,
           shared_gate, logits_u_ws,
           sgate_ws, heat, perm_src, offsets, counts, y_perm};
  void* args[] = {&P};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(decode_fused_kernel), dim3(grid), dim3(kThreads), args,
                                  smem, st);
  count_launches(1);
  return e;
}

}  // namespace moe
