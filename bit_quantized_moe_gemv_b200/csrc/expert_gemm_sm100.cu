// Prefill experts: grouped GEMM on the 5th-generation tensor cores (tcgen05,
// accumulators in TMEM), dequantising the packed weights to 16-bit floats in
// shared memory.
//
// Operand type: fp16 for both A and B (kind::f16 needs them equal). An int4
// or int2 code maps exactly to an fp16 integer and the fp16 group scale is
// used as stored, so each weight rounds once, at 2^-11; bf16 would round the
// scale and then the product at 2^-8 each, which breaks the 2e-2 x rms
// max-error bound on long dot products. The bf16 activations convert to fp16
// exactly after a per-row power-of-two scaling into fp16's range, and the
// SwiGLU output is scaled the same way (kHShift below), both undone on the
// fp32 results.
//
// Prefill pushes many tokens through each expert at once (the telli.sh page
// "Strata 与 Qwen3.8-Flash-Next：如何在个人电脑上运行 180B 级模型", section
// "GPU、RAM 和 SSD 各司其职": larger batches, kernels separate from decode), so
// the expert FFN is a dense contraction per expert:
//   gate/up:  H_e = silu(X_e Wg_e^T) * (X_e Wu_e^T)     [n_e x I]
//   down:     Y_e = H_e Wd_e^T                          [n_e x H]
// over the rows X_e the dispatch grouped for expert e (the shared expert is
// one more group holding every token).
//
// Layout ("swap AB"): the weight rows are the MMA's M side (128 per tile),
// tokens its N side (up to 128 per row tile), so a small expert wastes no M.
// Activations are stored once, by `gather_rows_kernel`, as 16 KiB tiles of
// 128 rows x 64 fp16 already in the 128-byte-swizzled K-major shared-memory
// image, so one 1-D bulk copy loads a B tile. Inside every 8-element group
// the K order is (0,4,1,5,2,6,3,7): the order in which a byte-free lop3
// unpacks eight int4 codes of one 32-bit word. Weights (A) are produced by
// 8 dequant warps straight into the swizzled image in the same K order, so
// the MMA's sum over K is unchanged. The gate/up epilogue writes H in the
// same tiled form, which is the down GEMM's B operand.
//
// Heavy groups (at least two row tiles) are dequantised once, before the
// GEMMs, by `predequant_kernel` into A tiles of that same image, and run in
// `wide_gemm_kernel`: tiles of two A tiles x 256 tokens (two row tiles), A
// and B both taken by bulk copies. An MMA of N = 256 reads each A tile of
// shared memory once for twice the tokens, which halves the A bytes per
// multiply-add that come from L2 and that the tensor core reads from shared
// memory (at 128 x 128 both streams are near their limits together).
// The other groups' row tiles run in `grouped_gemm_kernel`, whose warps
// dequantise A per tile:
//   warp 0      bulk-copy producer of B tiles, TMEM allocation
//   warp 1      MMA issuer (one thread)
//   warps 2-5   epilogue (TMEM -> registers -> global)
//   warps 6-13  dequant producers of A tiles
// Both kernels are persistent (one CTA per SM over their tile lists). Every
// wait is bounded; an expired wait flags MOE_ERR_TIMEOUT, stops the CTA's
// loops, drains what it issued and frees TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "moe_common.cuh"
#include "moe_internal.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace gemm {

constexpr int BM = 128, BN = 128, BK = 64;
constexpr int kTileBytes = BN * BK * 2;  // 16 KiB: one A or B tile
constexpr int kThreads = 14 * 32;
constexpr int kDqWarps = 8;
// A group with at least kHeavyRows rows (two or more row tiles) has its
// weights dequantised once, into A tiles in global memory, which its GEMM
// tiles then load like B instead of dequantising per row tile. At most
// kMaxHeavy groups (the first ones in group order) take this path.
constexpr int kHeavyRows = BN + 1;
constexpr int kMaxHeavy = 64;
// Int4 groups of at most kMmaRows rows run on mma.sync (one pass of two
// 8-token column blocks per job); larger single-tile groups on tcgen05.
constexpr int kMmaRows = 16;

// ---------------------------------------------------------------- plan
// Row tiles: every group (routed expert e < E, or the shared expert = E) is
// cut into tiles of at most BN rows. For each tile: group, first row (a
// dispatched row, or a token for the shared group) and row count. Heavy
// groups get a slot of pre-dequantised weights (hslot[g], -1 for none). The
// row tiles of a heavy group are paired into wide tiles (rows 2j and 2j + 1
// of the group; wlist holds the first), which `wide_gemm_kernel` runs. A
// group of one row tile whose three matrices are int4 is listed in mlist for
// `light_mma_kernel`; the row tiles of the remaining groups are listed in
// llist for `grouped_gemm_kernel`. A row tile is also the unit of the
// gathered activations and of the gate/up output tiles, whichever kernel
// made them.
struct Plan {
  int* count;   // [0] row tiles, [1] heavy slots used, [2] wide tiles, [3] llist tiles, [4] mlist tiles
  int* group;   // [max]
  int* row0;    // [max]
  int* nrows;   // [max]
  int* wlist;   // [max] first row tile of each wide tile
  int* llist;   // [max] row tiles for the dequantising tcgen05 GEMM
  int* mlist;   // [max] row tiles for the mma.sync GEMV
  int* hslot;   // [groups] heavy slot or -1
  int* hlist;   // [heavy slots] group of each slot
  int* tscaled; // [max] nonzero when a row of the tile has its x scaled (set by the gather)
};

// Exclusive prefix sum over the 1024 threads of the block; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  __syncthreads();  // wsum free (a previous scan may still read it)
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  int wb = 0, tot = 0;
  for (int i = 0; i < 32; ++i) {
    if (i < w) wb += wsum[i];
    tot += wsum[i];
  }
  *total = tot;
  return wb + incl - v;
}

// The GEMM that takes a group of n rows: its numbers of wide tiles (pairs of
// row tiles, when it has a heavy slot), of row tiles for the dequantising
// GEMM and of row tiles for the mma.sync GEMV (one tile of at most kMmaRows
// rows whose matrices are all int4). Every row tile lands in exactly one list.
struct GroupLists {
  int nw, nl, nm;
};
__host__ __device__ inline GroupLists group_lists(int n, bool heavy_slot, bool all_int4) {
  const int nt = (n + BN - 1) / BN;
  const bool mma = !heavy_slot && nt == 1 && n <= kMmaRows && all_int4;
  return GroupLists{heavy_slot ? (nt + 1) / 2 : 0, (heavy_slot || mma) ? 0 : nt, mma ? 1 : 0};
}

// A group's three matrices are all well-formed int4 (the mma.sync path).
__device__ __forceinline__ bool all_int4(const moe_expert& ex, int H, int I) {
  return ex.gate.qtype == MOE_Q_INT4_SYM_G32 && ex.up.qtype == MOE_Q_INT4_SYM_G32 &&
         ex.down.qtype == MOE_Q_INT4_SYM_G32 && qmatrix_ok(ex.gate, I, H) && qmatrix_ok(ex.up, I, H) &&
         qmatrix_ok(ex.down, H, I);
}

__global__ void __launch_bounds__(1024) plan_kernel(const int* __restrict__ counts, const int* __restrict__ offsets,
                                                    const moe_expert* __restrict__ experts,
                                                    const moe_expert* __restrict__ shared, int H, int I, int E,
                                                    int shared_rows, int max_tiles, int max_heavy, Plan plan,
                                                    WsHeader* hdr) {
  __shared__ int wsum[32];
  const int ngroups = E + (shared_rows > 0 ? 1 : 0);
  const int g = threadIdx.x;
  for (int i = g; i < max_tiles; i += blockDim.x) plan.tscaled[i] = 0;
  int nt = 0;
  if (g < ngroups) {
    const int n = g < E ? counts[g] : shared_rows;
    nt = (n + BN - 1) / BN;
  }
  int total, htotal, wtotal, ltotal, mtotal;
  const int excl = block_excl_scan(nt, wsum, &total);
  // heavy groups: slots in group order
  const int hv = (g < ngroups && nt >= 2) ? 1 : 0;  // n >= kHeavyRows
  const int hslot = block_excl_scan(hv, wsum, &htotal);
  const bool heavy = hv && hslot < max_heavy;
  const int n_g = g < ngroups ? (g < E ? counts[g] : shared_rows) : 0;
  // descriptors are read only for the groups that could take the mma.sync path
  const bool int4 = !heavy && nt == 1 && n_g <= kMmaRows && all_int4(g < E ? experts[g] : *shared, H, I);
  const GroupLists gl = group_lists(n_g, heavy, int4);
  const int nw = gl.nw, nl = gl.nl, nm = gl.nm;
  const int wexcl = block_excl_scan(nw, wsum, &wtotal);
  const int lexcl = block_excl_scan(nl, wsum, &ltotal);
  const int mexcl = block_excl_scan(nm, wsum, &mtotal);
  const bool fits = total <= max_tiles;  // the host's bound covers every routing
  if (g < ngroups) {
    plan.hslot[g] = heavy ? hslot : -1;
    if (heavy) plan.hlist[hslot] = g;
  }
  if (g == 0) {
    plan.count[0] = fits ? total : 0;
    plan.count[1] = min(htotal, max_heavy);
    plan.count[2] = fits ? wtotal : 0;
    plan.count[3] = fits ? ltotal : 0;
    plan.count[4] = fits ? mtotal : 0;
    if (!fits) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 7000002);
  }
  if (g < ngroups && fits) {
    const int n = g < E ? counts[g] : shared_rows;
    const int r0 = g < E ? offsets[g] : 0;
    for (int t = 0; t < nt; ++t) {
      plan.group[excl + t] = g;
      plan.row0[excl + t] = r0 + t * BN;
      plan.nrows[excl + t] = min(BN, n - t * BN);
    }
    for (int j = 0; j < nw; ++j) plan.wlist[wexcl + j] = excl + 2 * j;
    for (int t = 0; t < nl; ++t) plan.llist[lexcl + t] = excl + t;
    if (nm) plan.mlist[mexcl] = excl;
  }
}

// Byte offset of element (row, k) inside a swizzled 128-row x 64-col 16-bit tile,
// with the (0,4,1,5,2,6,3,7) order inside each 8-element group.
__device__ __forceinline__ uint32_t tile_off(int row, int k) {
  const int chunk = k >> 3, e = k & 7;
  const int pos = e < 4 ? 2 * e : 2 * (e - 4) + 1;
  return uint32_t(row) * 128u + (uint32_t((chunk ^ (row & 7))) << 4) + uint32_t(pos) * 2u;
}

// ---------------------------------------------------------------- fp16 helpers
__device__ __forceinline__ float sat_f16(float v) { return fminf(fmaxf(v, -65504.f), 65504.f); }

// Range of the fp16 operands. Each gathered row of x is scaled by 2^-e
// (e >= 0, exact) so that |x| < 2^8; the SwiGLU output h of that row is
// stored as h 2^-(kHShift + 2e) and the down GEMM's result multiplied back.
// For ordinary rows (|x| < 256) e = 0 and only the fixed 2^-kHShift applies,
// which moves fp16's overflow from 65504 to 2^kHShift x 65504 and costs h
// values below 2^(kHShift - 14) some relative precision (absolute error
// under 2^(kHShift - 24)).
constexpr int kHShift = 8;
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // -126 <= e <= 127
// The exponents of 16 consecutive rows (a 64-byte aligned run); returns
// whether any is nonzero.
__device__ __forceinline__ bool row_exps(const int* p, int (&e)[16]) {
  const int4* q = reinterpret_cast<const int4*>(p);
  int any = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int4 v = q[i];
    e[4 * i] = v.x;
    e[4 * i + 1] = v.y;
    e[4 * i + 2] = v.z;
    e[4 * i + 3] = v.w;
    any |= v.x | v.y | v.z | v.w;
  }
  return any != 0;
}
__device__ __forceinline__ int row_exp(uint32_t amax_bf16) {  // bf16 magnitude bits
  const int ex = int((amax_bf16 >> 7) & 0xff) - 127;          // floor(log2 |x|) of the largest element
  return ex >= 8 ? (ex - 7 < 119 ? ex - 7 : 119) : 0;
}
__device__ __forceinline__ uint32_t h2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------- gather
__device__ __forceinline__ uint32_t bf16x8_absmax(const uint4& v) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) m = max(m, max(in[q] & 0x7fffu, (in[q] >> 16) & 0x7fffu));
  return m;
}
// Eight bf16 values (16-byte chunk c of the row) -> fp16 after scaling by
// sc (|x sc| < 2^8; inf saturates at +-65504), K order (0,4,1,5,2,6,3,7),
// into the row's place in its swizzled 16 KiB tile.
__device__ __forceinline__ void store_x8(uint8_t* dst_row, int c, int row, const uint4& v, float sc) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = sat_f16(__uint_as_float(in[i] << 16) * sc);
    f[2 * i + 1] = sat_f16(__uint_as_float(in[i] & 0xffff0000u) * sc);
  }
  uint4 o;
  o.x = h2_bits(f[0], f[4]);
  o.y = h2_bits(f[1], f[5]);
  o.z = h2_bits(f[2], f[6]);
  o.w = h2_bits(f[3], f[7]);
  const int kb = c >> 3, chunk = c & 7;
  *reinterpret_cast<uint4*>(dst_row + size_t(kb) * kTileBytes + ((chunk ^ (row & 7)) << 4)) = o;
}
// One warp per tile row: token row -> 16 KiB swizzled tiles of X (K = H).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x, int H, int k,
                                                          const int* __restrict__ perm_src, int E, Plan plan,
                                                          uint8_t* __restrict__ xt, int* __restrict__ xexp) {
  const int ntiles = plan.count[0];
  const int KB = H / BK;
  const int lane = threadIdx.x & 31;
  for (long long wr = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); wr < (long long)ntiles * BN;
       wr += (long long)gridDim.x * 8) {
    const int rt = int(wr / BN), row = int(wr % BN);
    if (row >= plan.nrows[rt]) {  // padding rows of a partial tile: no scaling
      if (lane == 0) xexp[size_t(rt) * BN + row] = 0;
      continue;
    }
    const int g = plan.group[rt];
    const int r = plan.row0[rt] + row;
    const int tok = g < E ? perm_src[r] / k : r;
    const uint4* src = reinterpret_cast<const uint4*>(x + size_t(tok) * H);
    uint8_t* dst_row = xt + size_t(rt) * KB * kTileBytes + size_t(row) * 128;
    // the row's largest |x| (bf16 magnitude bits compare as integers); rows
    // of up to 2048 elements stay in registers for the conversion
    constexpr int kRegChunks = 8;
    uint4 keep[kRegChunks];
    uint32_t am = 0;
    if (H / 8 <= 32 * kRegChunks) {
#pragma unroll
      for (int i = 0; i < kRegChunks; ++i) {
        const int c = lane + 32 * i;
        keep[i] = c < H / 8 ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        am = max(am, bf16x8_absmax(keep[i]));
      }
      am = __reduce_max_sync(0xffffffffu, am);
      const int e = row_exp(am);
      if (lane == 0) {
        xexp[size_t(rt) * BN + row] = e;
        if (e) atomicOr(&plan.tscaled[rt], 1);
      }
      const float sc = pow2f(-e);
#pragma unroll
      for (int i = 0; i < kRegChunks; ++i) {
        const int c = lane + 32 * i;
        if (c < H / 8) store_x8(dst_row, c, row, keep[i], sc);
      }
    } else {
      for (int c = lane; c < H / 8; c += 32) am = max(am, bf16x8_absmax(__ldg(src + c)));
      am = __reduce_max_sync(0xffffffffu, am);
      const int e = row_exp(am);
      if (lane == 0) {
        xexp[size_t(rt) * BN + row] = e;
        if (e) atomicOr(&plan.tscaled[rt], 1);
      }
      const float sc = pow2f(-e);
      for (int c = lane; c < H / 8; c += 32) store_x8(dst_row, c, row, __ldg(src + c), sc);
    }
  }
}

// ---------------------------------------------------------------- dequant
// (a & mask) | magic in one instruction: the first step of the published
// "magic number" code -> fp16 conversion (OR the code under an fp16 exponent
// whose mantissa unit is worth 1, then subtract that constant)
__device__ __forceinline__ uint32_t lop_or(uint32_t a, uint32_t mask, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
  return d;
}
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b),
                      *reinterpret_cast<__half2*>(&c));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_splat(uint16_t h) { return uint32_t(h) | (uint32_t(h) << 16); }

// Raw data one dequant thread needs for one k-block of one matrix: 32
// consecutive K elements of one weight row.
struct RawK {
  uint4 c0, c1;      // codes (int4: c0; int2: c0.x,c0.y; int8: c0,c1)
  uint32_t s, m;     // scale(s) / min(s) as fp16 bit patterns
};

__device__ __forceinline__ void load_raw(const moe_qmatrix& W, int row, int k0, RawK& r) {
  const int K = W.cols;
  if (W.qtype == MOE_Q_INT4_SYM_G32) {
    r.c0 = __ldg(reinterpret_cast<const uint4*>(W.codes + size_t(row) * (K / 2) + k0 / 2));
    r.s = W.scales[size_t(row) * (K / 32) + k0 / 32];
  } else if (W.qtype == MOE_Q_INT2_ASYM_G16) {
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(W.codes + size_t(row) * (K / 4) + k0 / 4));
    r.c0 = make_uint4(c.x, c.y, 0, 0);
    const size_t gi = size_t(row) * (K / 16) + k0 / 16;
    r.s = __ldg(reinterpret_cast<const unsigned int*>(W.scales + gi));
    r.m = __ldg(reinterpret_cast<const unsigned int*>(W.mins + gi));
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(W.codes + size_t(row) * K + k0);
    r.c0 = __ldg(p);
    r.c1 = __ldg(p + 1);
    r.s = W.scales[row];
  }
}

// 32 weights -> 4 x 16-byte chunks of fp16, K order (0,4,1,5,2,6,3,7) per 8.
// A code c sits in the mantissa of the fp16 1024 + c (0x6400 | c), so the
// code-to-integer step is exact and the scale product rounds once.
__device__ __forceinline__ void dequant32(int qtype, const RawK& r, uint4 (&o)[4]) {
  if (qtype == MOE_Q_INT4_SYM_G32) {
    const uint32_t s2 = h2_splat(uint16_t(r.s));
    const uint32_t w[4] = {r.c0.x, r.c0.y, r.c0.z, r.c0.w};
    const uint32_t k1032 = 0x64086408u;  // fp16x2 (1032, 1032): 1024 + 8
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      // nibbles (0,4) and (2,6) as 1024 + c, (1,5) and (3,7) as 64 + c: one
      // lop3 each (no shift for the odd nibbles), then c - 8 exactly
      const uint32_t x = w[c], x8 = x >> 8;
      const uint32_t v0 = h2_sub(lop_or(x, 0x000F000Fu, 0x64006400u), k1032);
      const uint32_t v1 = h2_sub(lop_or(x, 0x00F000F0u, 0x54005400u), 0x54805480u);  // 64 + 8
      const uint32_t v2 = h2_sub(lop_or(x8, 0x000F000Fu, 0x64006400u), k1032);
      const uint32_t v3 = h2_sub(lop_or(x8, 0x00F000F0u, 0x54005400u), 0x54805480u);
      o[c] = make_uint4(h2_mul(v0, s2), h2_mul(v1, s2), h2_mul(v2, s2), h2_mul(v3, s2));
    }
  } else if (qtype == MOE_Q_INT2_ASYM_G16) {
    const uint32_t sA = h2_splat(uint16_t(r.s & 0xffffu)), sB = h2_splat(uint16_t(r.s >> 16));
    const uint32_t mA = h2_splat(uint16_t(r.m & 0xffffu)), mB = h2_splat(uint16_t(r.m >> 16));
    const uint32_t k1024 = 0x64006400u;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t word = c < 2 ? r.c0.x : r.c0.y;
      const uint32_t t = __byte_perm(word, 0u, (c & 1) ? 0x4342u : 0x4140u);
      const uint32_t s2 = c < 2 ? sA : sB, m2 = c < 2 ? mA : mB;
      uint32_t v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = h2_fma(h2_sub(((t >> (2 * j)) & 0x00030003u) | 0x64006400u, k1024), s2, m2);
      o[c] = make_uint4(v[0], v[1], v[2], v[3]);
    }
  } else {
    const float s = __half2float(__ushort_as_half(uint16_t(r.s)));
    const uint32_t w[8] = {r.c0.x, r.c0.y, r.c0.z, r.c0.w, r.c1.x, r.c1.y, r.c1.z, r.c1.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t a = w[2 * c] ^ 0x80808080u, b = w[2 * c + 1] ^ 0x80808080u;  // elements 0-3, 4-7
      float q[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        q[j] = __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7540u | j)) - 8388736.0f;
        q[4 + j] = __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7540u | j)) - 8388736.0f;
      }
      uint32_t v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = h2_bits(q[j] * s, q[4 + j] * s);
      o[c] = make_uint4(v[0], v[1], v[2], v[3]);
    }
  }
}

// ---------------------------------------------------------------- heavy groups
// Pre-dequantised weights of heavy slot h: the gate/up A tiles [I/128][H/64]
// [gate, up], then the down A tiles [H/128][I/64]; each a 16 KiB tile laid
// out exactly as the dequant warps write one into shared memory, so a GEMM
// stage takes it with one bulk copy.
__host__ __device__ inline size_t heavy_gu_bytes(int H, int I) { return size_t(2) * I * H * 2; }
__host__ __device__ inline size_t heavy_slot_bytes(int H, int I) { return size_t(3) * I * H * 2; }

// One CTA of 256 threads per group of kPD tiles; thread (row, half) takes 32
// K of one row of each tile. All kPD loads of a thread are issued before any
// dequantisation, so they are in flight together; four CTAs per SM (at most
// 64 registers per thread) keep more of them in flight than two CTAs with
// twice the tiles each.
constexpr int kPD = 2;
__global__ void __launch_bounds__(256, 4) predequant_kernel(const moe_expert* __restrict__ experts,
                                                         const moe_expert* __restrict__ shared, int E, int H, int I,
                                                         Plan plan, uint8_t* __restrict__ img, WsHeader* hdr) {
  const int nslots = plan.count[1];
  const int kbg = H / BK, kbd = I / BK;
  const int gu_tiles = (I / BM) * kbg * 2, per_slot = gu_tiles + (H / BM) * kbd;
  const int n = nslots * per_slot;
  const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
  for (int it0 = blockIdx.x * kPD; it0 < n; it0 += gridDim.x * kPD) {
    RawK raw[kPD];
    int qt[kPD];
    uint8_t* tile[kPD];
#pragma unroll
    for (int j = 0; j < kPD; ++j) {
      qt[j] = 0;
      tile[j] = nullptr;
      const int it = it0 + j;
      if (it >= n) continue;
      const int hs = it / per_slot, r = it - hs * per_slot;
      const int g = plan.hlist[hs];
      const moe_expert& ex = g < E ? experts[g] : *shared;
      const moe_qmatrix* W;
      int K, M, mt, kb;
      size_t off;
      if (r < gu_tiles) {  // r = (mt * kbg + kb) * 2 + (0 gate | 1 up)
        const int q = r >> 1;
        mt = q / kbg;
        kb = q - mt * kbg;
        W = (r & 1) ? &ex.up : &ex.gate;
        K = H;
        M = I;
        off = size_t(r) * kTileBytes;
      } else {  // down: q = mt * kbd + kb
        const int q = r - gu_tiles;
        mt = q / kbd;
        kb = q - mt * kbd;
        W = &ex.down;
        K = I;
        M = H;
        off = heavy_gu_bytes(H, I) + size_t(q) * kTileBytes;
      }
      if (!qmatrix_ok(*W, M, K)) {
        if (threadIdx.x == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 7000001);
        continue;
      }
      load_raw(*W, mt * BM + row, kb * BK + half * 32, raw[j]);
      qt[j] = W->qtype;
      tile[j] = img + size_t(hs) * heavy_slot_bytes(H, I) + off;
    }
#pragma unroll
    for (int j = 0; j < kPD; ++j) {
      if (tile[j] == nullptr) continue;
      uint4 o[4];
      dequant32(qt[j], raw[j], o);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int chunk = 4 * half + c;
        *reinterpret_cast<uint4*>(tile[j] + row * 128 + ((chunk ^ (row & 7)) << 4)) = o[c];
      }
    }
  }
}

// ---------------------------------------------------------------- GEMM kernel
struct Args {
  Plan plan;
  const moe_expert* experts;  // routed table
  const moe_expert* shared;   // shared descriptor or nullptr
  int E;
  int K;              // reduction length (H for gate/up, I for down)
  int M;              // weight rows (I for gate/up, H for down)
  int I, H;
  const uint8_t* bt;  // B tiles [tiles][K/64][16 KiB]
  const int* xexp;    // per gathered row (tile * 128 + row): the power-of-two scaling of x
  uint8_t* ht;        // gate/up: H tiles out [tiles][I/64][16 KiB]
  float* y_f32;       // down: fp32 rows out (routed rows), or nullptr
  uint16_t* y_bf16;   // down: bf16 rows out, or nullptr
  float* ys_f32;      // down: shared expert rows out (fp32 [T][H])
  const uint8_t* aimg;  // pre-dequantised weights of the heavy slots
  size_t aslot;         // bytes per heavy slot
  size_t aoff;          // this GEMM's A tiles within a slot
  WsHeader* hdr;
};

// ---------------------------------------------------------------- epilogues
// Gate/up: 16 columns (rows c0 .. c0 + 15 of row tile rt) of weight row m,
// g in v0 and u in v1 -> h = silu(g) u in fp16 into the H tiles (the down
// GEMM's B: row c of tile rt, K index m), at tile_off(c0 + j, m & 63): c0 is
// a multiple of 16, so the row's swizzle term (row & 7) is j & 7 and the
// offsets are c0 * 128 plus constants of j.
__device__ __forceinline__ void epi_h16(const Args& a, int rt, int m, int c0, int nrows, bool tile_scaled,
                                        const uint32_t (&v0)[16], const uint32_t (&v1)[16]) {
  const int kc = (m & 63) >> 3, e = m & 7;
  uint8_t* base = a.ht + (size_t(rt) * (a.I / BK) + (m >> 6)) * kTileBytes + size_t(c0) * 128 +
                  (e < 4 ? 4 * e : 4 * (e - 4) + 2);
  const int nv = nrows - c0 < 16 ? nrows - c0 : 16;
  int xe[16] = {};
  const bool scaled = tile_scaled && row_exps(a.xexp + size_t(rt) * BN + c0, xe);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j < nv) {
      // the row's x was scaled by 2^-e: g = g_s 2^e, u = u_s 2^e, and
      // h 2^-(kHShift + 2e) = silu(g) 2^-e u_s 2^-kHShift
      float gv = __uint_as_float(v0[j]), uv = __uint_as_float(v1[j]) * (1.0f / (1 << kHShift));
      if (scaled) {
        gv *= pow2f(xe[j]);
        uv *= pow2f(-xe[j]);
      }
      *reinterpret_cast<__half*>(base + j * 128 + ((kc ^ (j & 7)) << 4)) =
          __float2half_rn(sat_f16(__fdividef(gv, 1.0f + __expf(-gv)) * uv));
    }
  }
}

// Down: 16 columns (rows c0 .. c0 + 15 of row tile rt, dispatched rows
// row0 + c0 .. of group g) of output column m -> y, undoing the scaling of h:
// y = y_s 2^(kHShift + 2e) for the row's e.
__device__ __forceinline__ void epi_y16(const Args& a, int rt, int g, int row0, int m, int c0, int nrows,
                                        bool tile_scaled, const uint32_t (&v0)[16]) {
  const int nv = nrows - c0 < 16 ? nrows - c0 : 16;
  int xe[16] = {};
  const bool scaled = tile_scaled && row_exps(a.xexp + size_t(rt) * BN + c0, xe);
  float yv[16];
  if (!scaled) {
#pragma unroll
    for (int j = 0; j < 16; ++j) yv[j] = __uint_as_float(v0[j]) * float(1 << kHShift);
  } else {  // 2^(kHShift + 2e) = 2^(kHShift + e) 2^e, each a normal float for e <= 119
#pragma unroll
    for (int j = 0; j < 16; ++j) yv[j] = __uint_as_float(v0[j]) * pow2f(kHShift + xe[j]) * pow2f(xe[j]);
  }
  if (g < a.E && a.y_f32 == nullptr) {
    uint16_t* yp = a.y_bf16 + size_t(row0 + c0) * a.H + m;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nv) yp[size_t(j) * a.H] = f32_to_bf16_rn(yv[j]);
  } else {  // fp32 rows: column m of rows row0 + c0 .. (one pointer step of H per row)
    float* yp = (g < a.E ? a.y_f32 : a.ys_f32) + size_t(row0 + c0) * a.H + m;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nv) yp[size_t(j) * a.H] = yv[j];
  }
}

// Staged epilogues for a warp's 32 weight rows m = mbase + lane (mbase a
// multiple of 32) and 16 tokens: the warp writes its outputs into its own
// shared-memory scratch in the destination's byte order and then stores them
// as 16-byte pieces, one store instruction per lane for 4 fp32 or 8 fp16/bf16
// values instead of one per value. fp32 rows first:
constexpr int kEpiScratch = 2048;  // bytes of scratch per epilogue warp

__device__ __forceinline__ void epi_y16_f32_staged(const Args& a, int rt, int g, int row0, int mbase, int c0,
                                                   int nrows, bool tile_scaled, const uint32_t (&v0)[16],
                                                   uint8_t* scr) {
  const int lane = threadIdx.x & 31;
  const int nv = nrows - c0 < 16 ? nrows - c0 : 16;
  int xe[16] = {};
  const bool scaled = tile_scaled && row_exps(a.xexp + size_t(rt) * BN + c0, xe);
  float* s32 = reinterpret_cast<float*>(scr);
#pragma unroll
  for (int j = 0; j < 16; ++j)  // undo the scaling of h: y = y_s 2^(kHShift + 2e) for the row's e
    s32[j * 32 + lane] = scaled ? __uint_as_float(v0[j]) * pow2f(kHShift + xe[j]) * pow2f(xe[j])
                                : __uint_as_float(v0[j]) * float(1 << kHShift);
  __syncwarp();
  float* y = g < a.E ? a.y_f32 : a.ys_f32;  // 128 contiguous bytes per token
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int p = lane + 32 * i;  // token p / 8, 4 values p % 8
    const int j = p >> 3, part = p & 7;
    if (j < nv)
      *reinterpret_cast<uint4*>(y + size_t(row0 + c0 + j) * a.H + mbase + part * 4) =
          *reinterpret_cast<const uint4*>(scr + j * 128 + part * 16);
  }
  __syncwarp();
}

// 16-bit outputs (fp16 h, bf16 y) in token pairs: each lane converts two
// tokens' values of its column with one paired conversion and stores them as
// one 32-bit word ([token pair][column] in the scratch); the read-back splits
// the pairs with byte permutes into one 16-byte piece for each of the two
// tokens.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void epi_h16_pairs(const Args& a, int rt, int mbase, int c0, int nrows, bool tile_scaled,
                                              const uint32_t (&v0)[16], const uint32_t (&v1)[16], uint8_t* scr) {
  const int lane = threadIdx.x & 31;
  const int nv = nrows - c0 < 16 ? nrows - c0 : 16;
  int xe[16] = {};
  const bool scaled = tile_scaled && row_exps(a.xexp + size_t(rt) * BN + c0, xe);
  uint32_t* s32 = reinterpret_cast<uint32_t*>(scr);
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    float h[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int j = 2 * jj + t;
      // the row's x was scaled by 2^-e: g = g_s 2^e, u = u_s 2^e, and
      // h 2^-(kHShift + 2e) = silu(g) 2^-e u_s 2^-kHShift
      float gv = __uint_as_float(v0[j]), uv = __uint_as_float(v1[j]) * (1.0f / (1 << kHShift));
      if (scaled) {
        gv *= pow2f(xe[j]);
        uv *= pow2f(-xe[j]);
      }
      h[t] = sat_f16(__fdividef(gv, 1.0f + __expf(-gv)) * uv);
    }
    s32[jj * 32 + lane] = h2_bits(h[0], h[1]);
  }
  __syncwarp();
  // lane: token pair jj, 16-byte chunk kcl = K values 8 kcl + (0..7) of its
  // 64-K block half, in the order (0,4,1,5,2,6,3,7)
  const int jj = lane >> 2, kcl = lane & 3;
  const uint4 w0 = *reinterpret_cast<const uint4*>(s32 + jj * 32 + kcl * 8);
  const uint4 w1 = *reinterpret_cast<const uint4*>(s32 + jj * 32 + kcl * 8 + 4);
  const uint4 ev = make_uint4(__byte_perm(w0.x, w1.x, 0x5410), __byte_perm(w0.y, w1.y, 0x5410),
                              __byte_perm(w0.z, w1.z, 0x5410), __byte_perm(w0.w, w1.w, 0x5410));
  const uint4 od = make_uint4(__byte_perm(w0.x, w1.x, 0x7632), __byte_perm(w0.y, w1.y, 0x7632),
                              __byte_perm(w0.z, w1.z, 0x7632), __byte_perm(w0.w, w1.w, 0x7632));
  const int kc = 4 * ((mbase & 63) >> 5) + kcl;
  uint8_t* tile = a.ht + (size_t(rt) * (a.I / BK) + (mbase >> 6)) * kTileBytes;
  const int r0 = c0 + 2 * jj;
  if (2 * jj < nv) *reinterpret_cast<uint4*>(tile + size_t(r0) * 128 + ((kc ^ (r0 & 7)) << 4)) = ev;
  if (2 * jj + 1 < nv) *reinterpret_cast<uint4*>(tile + size_t(r0 + 1) * 128 + ((kc ^ ((r0 + 1) & 7)) << 4)) = od;
  __syncwarp();
}

__device__ __forceinline__ void epi_y16_pairs(const Args& a, int rt, int g, int row0, int mbase, int c0, int nrows,
                                              bool tile_scaled, const uint32_t (&v0)[16], uint8_t* scr) {
  if (!(g < a.E && a.y_f32 == nullptr)) {  // fp32 rows
    epi_y16_f32_staged(a, rt, g, row0, mbase, c0, nrows, tile_scaled, v0, scr);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int nv = nrows - c0 < 16 ? nrows - c0 : 16;
  int xe[16] = {};
  const bool scaled = tile_scaled && row_exps(a.xexp + size_t(rt) * BN + c0, xe);
  uint32_t* s32 = reinterpret_cast<uint32_t*>(scr);
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    float y2[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int j = 2 * jj + t;
      // undo the scaling of h: y = y_s 2^(kHShift + 2e) for the row's e
      y2[t] = scaled ? __uint_as_float(v0[j]) * pow2f(kHShift + xe[j]) * pow2f(xe[j])
                     : __uint_as_float(v0[j]) * float(1 << kHShift);
    }
    s32[jj * 32 + lane] = pack_bf16x2(y2[0], y2[1]);
  }
  __syncwarp();
  // lane: token pair jj, columns mbase + 8 cg .. + 7
  const int jj = lane >> 2, cg = lane & 3;
  const uint4 w0 = *reinterpret_cast<const uint4*>(s32 + jj * 32 + cg * 8);
  const uint4 w1 = *reinterpret_cast<const uint4*>(s32 + jj * 32 + cg * 8 + 4);
  const uint4 ev = make_uint4(__byte_perm(w0.x, w0.y, 0x5410), __byte_perm(w0.z, w0.w, 0x5410),
                              __byte_perm(w1.x, w1.y, 0x5410), __byte_perm(w1.z, w1.w, 0x5410));
  const uint4 od = make_uint4(__byte_perm(w0.x, w0.y, 0x7632), __byte_perm(w0.z, w0.w, 0x7632),
                              __byte_perm(w1.x, w1.y, 0x7632), __byte_perm(w1.z, w1.w, 0x7632));
  uint16_t* y = a.y_bf16 + size_t(row0 + c0 + 2 * jj) * a.H + mbase + cg * 8;
  if (2 * jj < nv) *reinterpret_cast<uint4*>(y) = ev;
  if (2 * jj + 1 < nv) *reinterpret_cast<uint4*>(y + a.H) = od;
  __syncwarp();
}

// Raw-code staging: each dequant thread copies (cp.async) its own codes and
// scales kRawDepth k-blocks ahead into a private area of shared memory.
constexpr int kRawDepth = 3;
constexpr int kRawCodeBytes = 2 * 2 * 256 * 16;  // [matrix][16-B unit][thread] (int8 needs two units)
constexpr int kRawAuxBytes = 2 * 256 * 8;        // [matrix][thread] 8 B (scale / scales + mins)
constexpr int kRawSlotBytes = kRawCodeBytes + kRawAuxBytes;

template <bool kGateUp>
struct Cfg {
  static constexpr int kStages = kGateUp ? 3 : 5;
  static constexpr int kATiles = kGateUp ? 2 : 1;
  static constexpr int kStageBytes = (kATiles + 1) * kTileBytes;
  static constexpr int kAccCols = kGateUp ? 256 : 128;  // one accumulator buffer
  static constexpr int kTmemCols = 2 * kAccCols;
};

template <bool kGateUp>
__device__ __forceinline__ const moe_qmatrix& pick(const moe_expert& e, int which) {
  if (kGateUp) return which == 0 ? e.gate : e.up;
  return e.down;
}

// One job = one k-block of one tile: 128 weight rows x 64 K of each A matrix.
// Thread (row, half) of the 256 dequant threads handles 32 K elements of one
// row. The tile's matrix pointers are resolved once per tile into registers;
// the codes are staged in shared memory several k-blocks ahead.
struct DqMat {
  const uint8_t* codes;   // start of this thread's row
  const uint16_t* scales; // start of this thread's row of scales (int8: &scale[row])
  const uint16_t* mins;
  int qtype;
};

__device__ __forceinline__ DqMat dq_mat(const moe_qmatrix& W, int row, int M, int K, WsHeader* hdr) {
  DqMat d{nullptr, nullptr, nullptr, 0};
  if (!qmatrix_ok(W, M, K)) {
    if ((threadIdx.x & 31) == 0) flag_error(hdr, MOE_ERR_DEVICE_FAULT, 7000000);
    return d;
  }
  d.qtype = W.qtype;
  d.codes = W.codes + size_t(row) * row_code_bytes(W.qtype, K);
  if (W.qtype == MOE_Q_INT8_PER_CHANNEL) {
    d.scales = W.scales + row;
  } else {
    const int g = W.qtype == MOE_Q_INT4_SYM_G32 ? 32 : 16;
    d.scales = W.scales + size_t(row) * (K / g);
    d.mins = W.mins ? W.mins + size_t(row) * (K / g) : nullptr;
  }
  return d;
}

__device__ __forceinline__ void cp16(uint8_t* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp8(uint8_t* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(ptx::smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(uint8_t* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ptx::smem_addr(dst)), "l"(src) : "memory");
}

// Copy this thread's raw data of one k-block of matrix d into its slot.
__device__ __forceinline__ void raw_issue(const DqMat& d, int k0, uint8_t* slot, int w, int dt) {
  uint8_t* code0 = slot + ((w * 2 + 0) * 256 + dt) * 16;
  uint8_t* code1 = slot + ((w * 2 + 1) * 256 + dt) * 16;
  uint8_t* aux = slot + kRawCodeBytes + (w * 256 + dt) * 8;
  if (d.qtype == MOE_Q_INT4_SYM_G32) {
    cp16(code0, d.codes + k0 / 2);
    cp4(aux, d.scales + ((k0 / 32) & ~1));
  } else if (d.qtype == MOE_Q_INT2_ASYM_G16) {
    cp8(code0, d.codes + k0 / 4);
    cp4(aux, d.scales + k0 / 16);
    cp4(aux + 4, d.mins + k0 / 16);
  } else if (d.qtype == MOE_Q_INT8_PER_CHANNEL) {
    cp16(code0, d.codes + k0);
    cp16(code1, d.codes + k0 + 16);
    cp4(aux, reinterpret_cast<const uint16_t*>(reinterpret_cast<uintptr_t>(d.scales) & ~uintptr_t(3)));
  }
}

__device__ __forceinline__ void raw_read(const uint8_t* slot, int w, int dt, int qtype, int k0, bool odd_row_scale,
                                         RawK& r) {
  r.c0 = *reinterpret_cast<const uint4*>(slot + ((w * 2 + 0) * 256 + dt) * 16);
  if (qtype == MOE_Q_INT8_PER_CHANNEL) r.c1 = *reinterpret_cast<const uint4*>(slot + ((w * 2 + 1) * 256 + dt) * 16);
  const uint2 aux = *reinterpret_cast<const uint2*>(slot + kRawCodeBytes + (w * 256 + dt) * 8);
  if (qtype == MOE_Q_INT4_SYM_G32) {
    r.s = ((k0 / 32) & 1) ? (aux.x >> 16) : (aux.x & 0xffffu);
  } else if (qtype == MOE_Q_INT2_ASYM_G16) {
    r.s = aux.x;
    r.m = aux.y;
  } else {
    r.s = odd_row_scale ? (aux.x >> 16) : (aux.x & 0xffffu);
  }
}

template <bool kGateUp>
__device__ void dequant_role(const Args& a, uint8_t* smem, uint8_t* raw_smem, uint64_t* full_bar,
                             uint64_t* empty_bar, volatile int* abort_p, int MT, int KB, long long ntiles) {
  using C = Cfg<kGateUp>;
  constexpr int NW = kGateUp ? 2 : 1;
  const int dt = threadIdx.x - 6 * 32;  // 0 .. 255
  const int row = dt >> 1, half = dt & 1;
  // 32-bit job counters and cursors: no division per job
  const int per_cta = ntiles > blockIdx.x ? int((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
  const int njobs = per_cta * KB;
  DqMat ld[NW];
  int i_tile = -1, i_kb = KB - 1;  // issue cursor (local tile, k-block), one step before the first job
  int ld_wrow = 0;
  auto resolve = [&](int lt) {
    const int t = int(blockIdx.x) + lt * int(gridDim.x);
    const int li = t / MT, mt = t - li * MT;
    const int g = a.plan.group[a.plan.llist[li]];
    const moe_expert* ex = g < a.E ? a.experts + g : a.shared;
    ld_wrow = mt * BM + row;
    ld[0] = dq_mat(kGateUp ? ex->gate : ex->down, ld_wrow, a.M, a.K, a.hdr);
    if (kGateUp) ld[NW - 1] = dq_mat(ex->up, ld_wrow, a.M, a.K, a.hdr);
  };
  int qts[kRawDepth][NW];
  int odd[kRawDepth];
  auto issue = [&](int j, int p) {
    if (j < njobs) {
      if (++i_kb == KB) {
        i_kb = 0;
        resolve(++i_tile);
      }
      uint8_t* slot = raw_smem + size_t(p) * kRawSlotBytes;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        raw_issue(ld[w], i_kb * BK + half * 32, slot, w, dt);
        qts[p][w] = ld[w].qtype;
      }
      odd[p] = ld_wrow & 1;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int p = 0; p < kRawDepth; ++p) issue(p, p);
  int s = 0;
  uint32_t ph = 0;
  int c_kb = 0;  // consume cursor: k-block of job j
  for (int j0 = 0; j0 < njobs; j0 += kRawDepth) {
#pragma unroll
    for (int p = 0; p < kRawDepth; ++p) {
      const int j = j0 + p;
      if (j < njobs && !*abort_p) {
        asm volatile("cp.async.wait_group %0;" ::"n"(kRawDepth - 1) : "memory");
        RawK raw[NW];
        const uint8_t* slot = raw_smem + size_t(p) * kRawSlotBytes;
        const int k0 = c_kb * BK + half * 32;
        if (++c_kb == KB) c_kb = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) raw_read(slot, w, dt, qts[p][w], k0, odd[p] != 0, raw[w]);
        if (!ptx::mbar_wait(ptx::smem_addr(&empty_bar[s]), ph ^ 1u, abort_p)) {
          flag_error(a.hdr, MOE_ERR_TIMEOUT, 6000005);
          *abort_p = 1;
        } else {
          if (qts[p][0] != 0) {  // qtype 0: a flagged descriptor
#pragma unroll
            for (int w = 0; w < NW; ++w) {
              uint4 o[4];
              dequant32(qts[p][w], raw[w], o);
              uint8_t* tile = smem + size_t(s) * C::kStageBytes + size_t(w) * kTileBytes;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int chunk = 4 * half + c;
                *reinterpret_cast<uint4*>(tile + row * 128 + ((chunk ^ (row & 7)) << 4)) = o[c];
              }
            }
            ptx::fence_proxy_async_smem();
          }
          __syncwarp();
          if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(ptx::smem_addr(&full_bar[s]));
        }
        // refill this raw slot (its data is consumed: the dequant used the registers)
        issue(j + kRawDepth, p);
        if (++s == C::kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(Args a) {
  using C = Cfg<kGateUp>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[C::kStages], empty_bar[C::kStages], accf_bar[2], acce_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nlight = a.plan.count[3];
  const int MT = a.M / BM, KB = a.K / BK;
  const long long ntiles = (long long)nlight * MT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(ptx::smem_addr(&full_bar[s]), 1 + kDqWarps);
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
    ptx::tmem_alloc(ptx::smem_addr(&tmem_base_sh), C::kTmemCols);
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
  auto stage_a = [&](int s, int which) { return smem + size_t(s) * C::kStageBytes + size_t(which) * kTileBytes; };
  auto stage_b = [&](int s) { return smem + size_t(s) * C::kStageBytes + size_t(C::kATiles) * kTileBytes; };

  if (warp == 0) {
    // ------------------------------------------------ B producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x) {
        const int rt = a.plan.llist[int(t / MT)];
        const int nrows = a.plan.nrows[rt];
        const uint32_t bytes = uint32_t((nrows + 15) & ~15) * 128u;
        for (int kb = 0; kb < KB; ++kb) {
          if (!ptx::mbar_wait_sleep(ptx::smem_addr(&empty_bar[s]), ph ^ 1u, abort_p, 64)) {
            fail(6000001);
            break;
          }
          ptx::mbar_arrive_expect_tx(ptx::smem_addr(&full_bar[s]), bytes);
          ptx::bulk_g2s(ptx::smem_addr(stage_b(s)), a.bt + (size_t(rt) * KB + kb) * kTileBytes, bytes,
                        ptx::smem_addr(&full_bar[s]));
          if (++s == C::kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x, ++it) {
        const int rt = a.plan.llist[int(t / MT)];
        const int nrows = a.plan.nrows[rt];
        const int N = (nrows + 15) & ~15;
        const uint32_t idesc = ptx::idesc_f16(BM, N);
        const int buf = it & 1;
        const uint32_t use = uint32_t(it >> 1) & 1u;
        if (!ptx::mbar_wait(ptx::smem_addr(&acce_bar[buf]), use ^ 1u, abort_p)) {
          fail(6000002);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + uint32_t(buf * C::kAccCols);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!ptx::mbar_wait(ptx::smem_addr(&full_bar[s]), ph, abort_p)) {
            fail(6000003);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa0 = ptx::smem_addr(stage_a(s, 0));
          const uint32_t sb = ptx::smem_addr(stage_b(s));
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t bdesc = ptx::smem_desc_k128(sb + 32 * ks);
            const uint32_t acc = (kb | ks) != 0;
            ptx::mma_f16(d0, ptx::smem_desc_k128(sa0 + 32 * ks), bdesc, idesc, acc);
            if (kGateUp) {
              const uint32_t sa1 = ptx::smem_addr(stage_a(s, 1));
              ptx::mma_f16(d0 + 128, ptx::smem_desc_k128(sa1 + 32 * ks), bdesc, idesc, acc);
            }
          }
          ptx::mma_commit(ptx::smem_addr(&empty_bar[s]));
          if (++s == C::kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&accf_bar[buf]));
      }
      // Drain: wait (bounded) for every MMA this thread issued.
      ptx::mma_commit(ptx::smem_addr(&drain_bar));
      ptx::mbar_wait(ptx::smem_addr(&drain_bar), 0, nullptr);
    }
  } else if (warp < 6) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    int it = 0;
    for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x, ++it) {
      const int rt = a.plan.llist[int(t / MT)], mt = int(t % MT);
      const int nrows = a.plan.nrows[rt];
      const int g = a.plan.group[rt];
      const int row0 = a.plan.row0[rt];
      const int buf = it & 1;
      const uint32_t use = uint32_t(it >> 1) & 1u;
      // double-buffered accumulators: the epilogue's wake-up latency is hidden
      if (!ptx::mbar_wait_sleep(ptx::smem_addr(&accf_bar[buf]), use, abort_p, 256)) {
        fail(6000004);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * C::kAccCols);
      const int m = mt * BM + 32 * q + lane;  // weight row of this thread
      const bool tile_scaled = a.plan.tscaled[rt] != 0;  // any row of the tile has its x scaled
      for (int c0 = 0; c0 < nrows; c0 += 16) {
        uint32_t v0[16];
        ptx::tmem_ld16(taddr + uint32_t(c0), v0);
        if (kGateUp) {
          uint32_t v1[16];
          ptx::tmem_ld16(taddr + 128u + uint32_t(c0), v1);
          ptx::tmem_ld_wait();
          epi_h16(a, rt, m, c0, nrows, tile_scaled, v0, v1);
        } else {
          ptx::tmem_ld_wait();
          epi_y16(a, rt, g, row0, m, c0, nrows, tile_scaled, v0);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&acce_bar[buf]));
    }
  } else {
    // ------------------------------------------------ dequant producers
    dequant_role<kGateUp>(a, smem, smem + size_t(C::kStages) * C::kStageBytes, full_bar, empty_bar, abort_p, MT, KB,
                          ntiles);
  }
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}


// ---------------------------------------------------------------- wide tiles
// Heavy groups (weights pre-dequantised into A tiles) run in
// `wide_gemm_kernel<kGateUp, NA, NB>`: tiles of NA A tiles (128 weight rows
// each) x NB tokens (one or two row tiles of the group), both operands taken
// by bulk copies. gate/up: NA = 2, A0 = gate rows [128 mt, +128), A1 = the up
// rows of the same range; down: A0 (and A1) = down rows [128 NA mt, +128)
// (and the next 128). One MMA of N = 256 takes each A tile once for 256
// tokens, halving the A bytes per multiply-add that come from L2 and that the
// tensor core reads from shared memory, next to N = 128. The accumulators of a
// tile take NA x NB TMEM columns: with 512 a tile's MMAs start once the
// previous tile's epilogue has read them, with 256 they alternate between two
// buffers and the epilogue overlaps the next tile's main loop.
//
// Warp roles (320 threads, one CTA per SM, persistent over the tiles):
//   warp 0      bulk-copy producer (A tiles and the B rows), TMEM allocation
//   warp 1      MMA issuer (one thread)
//   warps 2-9   epilogue: warp 2 + 4 p + i reads TMEM lane quarter (warp % 4)
//               for token part p (of two) of the tile
template <int NA, int NB>
struct WCfg {
  static constexpr int kStageBytes = (NA + NB / BN) * kTileBytes;
  static constexpr int kAccCols = NA * NB;        // one tile's accumulators
  static constexpr int kBufs = 512 / kAccCols;    // 1 or 2
  static constexpr int kStages = (200 * 1024) / kStageBytes < 6 ? (200 * 1024) / kStageBytes : 6;
};
constexpr int kWEpiWarps = 8;
constexpr int kWThreads = (2 + kWEpiWarps) * 32;
// Tile shapes of the two GEMMs (A tiles x tokens).
constexpr int kGuNA = 2, kGuNB = 256;
constexpr int kDnNA = 1, kDnNB = 256;
template <int NA, int NB>
constexpr size_t wide_smem_bytes() {
  return size_t(WCfg<NA, NB>::kStages) * WCfg<NA, NB>::kStageBytes + size_t(kWEpiWarps) * kEpiScratch + 1024;
}

template <bool kGateUp, int NA, int NB>
__global__ void __launch_bounds__(kWThreads, 1) wide_gemm_kernel(Args a) {
  using C = WCfg<NA, NB>;
  static_assert(!kGateUp || NA == 2, "gate/up tiles hold the gate and the up rows");
  static_assert(C::kBufs * C::kAccCols == 512, "accumulators fill TMEM");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[C::kStages], empty_bar[C::kStages], accf_bar[C::kBufs],
      acce_bar[C::kBufs], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwide = a.plan.count[2], nrt = a.plan.count[0];
  // weight-row blocks: gate/up one 128-row block per tile; down NA blocks per
  // tile, the last holding only A0 when M / 128 is not a multiple of NA
  const int MT = kGateUp ? a.M / BM : (a.M / BM + NA - 1) / NA, KB = a.K / BK;
  constexpr int kParts = NB / BN;  // row tiles per tile: token slots of a wide tile
  const long long ntiles = (long long)nwide * (2 / kParts) * MT;
  auto has_a1 = [&](int mt) { return NA == 2 && (kGateUp || 2 * mt + 1 < a.M / BM); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(ptx::smem_addr(&full_bar[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&empty_bar[s]), 1);
    }
    for (int b = 0; b < C::kBufs; ++b) {
      ptx::mbar_init(ptx::smem_addr(&accf_bar[b]), 1);
      ptx::mbar_init(ptx::smem_addr(&acce_bar[b]), kWEpiWarps);
    }
    ptx::mbar_init(ptx::smem_addr(&drain_bar), 1);
    abort_sh = 0;
    ptx::mbar_init_fence();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_addr(&tmem_base_sh), 512);
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
  // Tile t: weight block mt and its tokens: the row tiles rt0 (n0 rows) and,
  // for NB = 256, its partner rt0 + 1 when that belongs to the same group (n1
  // rows, else 0). For NB = 128 a wide tile's two row tiles are two tiles (the
  // second skipped when empty).
  auto tile_of = [&](long long t, int& mt, int& rt0, int& n0, int& n1) {
    const long long u = t / MT;
    mt = int(t - u * MT);
    const int w = int(u / (2 / kParts)), second = int(u - (long long)w * (2 / kParts));
    const int r = a.plan.wlist[w];
    const bool pair = r + 1 < nrt && a.plan.group[r + 1] == a.plan.group[r];
    if (kParts == 2) {
      rt0 = r;
      n0 = a.plan.nrows[r];
      n1 = pair ? a.plan.nrows[r + 1] : 0;
    } else {
      rt0 = r + second;
      n0 = (second == 0 || pair) ? a.plan.nrows[rt0] : 0;
      n1 = 0;
    }
  };
  auto stage = [&](int s) { return smem + size_t(s) * C::kStageBytes; };

  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, armed = 0, armed_ph = 0;  // bit i: stage i armed, and its phase
      for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x) {
        int mt, rt0, n0, n1;
        tile_of(t, mt, rt0, n0, n1);
        if (n0 == 0) continue;  // the empty second row tile of a single one
        const uint32_t b0 = uint32_t((n0 + 15) & ~15) * 128u, b1 = uint32_t((n1 + 15) & ~15) * 128u;
        const int hs = a.plan.hslot[a.plan.group[rt0]];
        if (hs < 0) {  // a wide tile always belongs to a group with a slot
          flag_error(a.hdr, MOE_ERR_DEVICE_FAULT, 7000003);
          *abort_p = 1;
          break;
        }
        const uint8_t* img = a.aimg + size_t(hs) * a.aslot + a.aoff;
        const bool a1 = has_a1(mt);
        for (int kb = 0; kb < KB; ++kb) {
          if (!ptx::mbar_wait(ptx::smem_addr(&empty_bar[s]), ph ^ 1u, abort_p)) {
            fail(6000011);
            break;
          }
          armed |= 1u << s;
          armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
          const uint32_t bar = ptx::smem_addr(&full_bar[s]);
          const uint32_t dst = ptx::smem_addr(stage(s));
          ptx::mbar_arrive_expect_tx(bar, (a1 ? 2u : 1u) * kTileBytes + b0 + b1);
          if (kGateUp) {  // image [mt][kb][gate, up]
            ptx::bulk_g2s(dst, img + (size_t(mt) * KB + kb) * 2 * kTileBytes, 2u * kTileBytes, bar);
          } else {        // image [128-row block][kb]
            ptx::bulk_g2s(dst, img + (size_t(NA * mt) * KB + kb) * kTileBytes, kTileBytes, bar);
            if (a1)
              ptx::bulk_g2s(dst + kTileBytes, img + (size_t(NA * mt + 1) * KB + kb) * kTileBytes, kTileBytes, bar);
          }
          const uint32_t db = dst + uint32_t(NA) * kTileBytes;
          ptx::bulk_g2s(db, a.bt + (size_t(rt0) * KB + kb) * kTileBytes, b0, bar);
          if (b1) ptx::bulk_g2s(db + kTileBytes, a.bt + (size_t(rt0 + 1) * KB + kb) * kTileBytes, b1, bar);
          if (++s == C::kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // After an abort, let the copies already issued land (bounded) before the
      // CTA exits: a stage's full barrier waits for nothing but its bytes.
      if (*abort_p)
        for (int i = 0; i < C::kStages; ++i)
          if (armed & (1u << i)) ptx::mbar_wait(ptx::smem_addr(&full_bar[i]), (armed_ph >> i) & 1u, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x) {
        int mt, rt0, n0, n1;
        tile_of(t, mt, rt0, n0, n1);
        if (n0 == 0) continue;
        const bool a1 = has_a1(mt);
        const uint32_t idesc = ptx::idesc_f16(BM, (n0 + n1 + 15) & ~15);
        const int buf = it % C::kBufs;
        const uint32_t use = uint32_t(it / C::kBufs) & 1u;
        if (!ptx::mbar_wait(ptx::smem_addr(&acce_bar[buf]), use ^ 1u, abort_p)) {
          fail(6000012);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + uint32_t(buf * C::kAccCols);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!ptx::mbar_wait(ptx::smem_addr(&full_bar[s]), ph, abort_p)) {
            fail(6000013);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa0 = ptx::smem_addr(stage(s));
          const uint32_t sb = sa0 + uint32_t(NA) * kTileBytes;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t bdesc = ptx::smem_desc_k128(sb + 32 * ks);
            const uint32_t acc = (kb | ks) != 0;
            ptx::mma_f16(d0, ptx::smem_desc_k128(sa0 + 32 * ks), bdesc, idesc, acc);
            if (a1) ptx::mma_f16(d0 + uint32_t(NB), ptx::smem_desc_k128(sa0 + kTileBytes + 32 * ks), bdesc, idesc, acc);
          }
          ptx::mma_commit(ptx::smem_addr(&empty_bar[s]));
          if (++s == C::kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&accf_bar[buf]));
        ++it;
      }
      // Drain: wait (bounded) for every MMA this thread issued.
      ptx::mma_commit(ptx::smem_addr(&drain_bar));
      ptx::mbar_wait(ptx::smem_addr(&drain_bar), 0, nullptr);
    }
  } else {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int part = (warp - 2) >> 2;  // token part of the tile: NB / 2 tokens
    uint8_t* scr = smem + size_t(C::kStages) * C::kStageBytes + size_t(warp - 2) * kEpiScratch;
    int it = 0;
    for (long long t = blockIdx.x; t < ntiles && !*abort_p; t += gridDim.x) {
      int mt, rt0, n0, n1;
      tile_of(t, mt, rt0, n0, n1);
      if (n0 == 0) continue;
      const int buf = it % C::kBufs;
      const uint32_t use = uint32_t(it / C::kBufs) & 1u;
      if (!ptx::mbar_wait(ptx::smem_addr(&accf_bar[buf]), use, abort_p)) {
        fail(6000014);
        break;
      }
      ptx::tc_fence_after();
      // this warp's tokens: row tile rt, rows [c_lo, c_hi) of it, at TMEM column col0 + (row - c_lo)
      int rt, c_lo, c_hi, col0;
      if (kParts == 2) {
        rt = rt0 + part;
        c_lo = 0;
        c_hi = part ? n1 : n0;
        col0 = part * BN;
      } else {
        rt = rt0;
        c_lo = part * (BN / 2);
        c_hi = n0 < c_lo + BN / 2 ? n0 : c_lo + BN / 2;
        col0 = c_lo;
      }
      if (c_hi > c_lo) {
        const int g = a.plan.group[rt], row0 = a.plan.row0[rt];
        const bool tile_scaled = a.plan.tscaled[rt] != 0;
        const bool a1 = has_a1(mt);
        const uint32_t taddr = tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * C::kAccCols + col0 - c_lo);
        // weight rows of this warp: gate/up rows mbase + lane of A0 and A1;
        // down rows mbase + lane (and mbase + 128 + lane)
        const int mbase = (kGateUp ? mt * BM : mt * NA * BM) + 32 * q;
        for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
          uint32_t v0[16], v1[16];
          ptx::tmem_ld16(taddr + uint32_t(c0), v0);
          if (a1) ptx::tmem_ld16(taddr + uint32_t(NB + c0), v1);
          ptx::tmem_ld_wait();
          if (kGateUp) {
            epi_h16_pairs(a, rt, mbase, c0, c_hi, tile_scaled, v0, v1, scr);
          } else {
            epi_y16_pairs(a, rt, g, row0, mbase, c0, c_hi, tile_scaled, v0, scr);
            if (a1) epi_y16_pairs(a, rt, g, row0, mbase + BM, c0, c_hi, tile_scaled, v1, scr);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&acce_bar[buf]));
      ++it;
    }
  }
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}


// ---------------------------------------------------------------- int4 groups of a few rows
// An int4 group of at most kMmaRows rows streams its weights once for a
// handful of tokens (at 8K prefill 138 of the 185 single-tile groups): a
// GEMV more than a GEMM. Its row tile runs as warp jobs on mma.sync
// m16n8k16 (fp16 operands, fp32 accumulation)
// with the A fragments dequantised in registers straight from the codes, the
// way the decode kernel streams its experts: no shared-memory round trip of
// the weights. A job is 16 weight rows (of gate and up, or of down) against
// the row tile's tokens, 8 per MMA column block.
//
// Each lane takes one 16-byte code column (32 int4 codes along K, one group
// scale) of rows g and g + 8 (g = lane / 4) per iteration; the four lanes of
// a group take four consecutive columns. One 32-bit code word gives the
// fp16 pairs (n0, n4), (n1, n5), (n2, n6), (n3, n7) of its eight codes; the
// gathered activation tiles store each 8 K values in the order
// (0,4,1,5,2,6,3,7), so the 16-byte chunk of a token's row that holds the
// same 8 K values gives the matching B pairs in the same registers. The MMA
// sums over a permutation of K, which leaves the dot products unchanged.
constexpr int kLmWarps = 8;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// int4 word (codes n0..n7 of K 8i..8i+7) -> fp16 pairs (n_j, n_{j+4}) * s, j = 0..3
__device__ __forceinline__ void deq4_pairs(uint32_t w, uint32_t s2, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = h2_mul(h2_sub(lop_or(w, 0x000F000Fu, 0x64006400u), 0x64086408u), s2);
  p[1] = h2_mul(h2_sub(lop_or(w, 0x00F000F0u, 0x54005400u), 0x54805480u), s2);
  p[2] = h2_mul(h2_sub(lop_or(w8, 0x000F000Fu, 0x64006400u), 0x64086408u), s2);
  p[3] = h2_mul(h2_sub(lop_or(w8, 0x00F000F0u, 0x54005400u), 0x54805480u), s2);
}

struct LmRows {  // one matrix: this lane's rows g and g + 8 (codes, scales)
  const uint8_t* lo;
  const uint8_t* hi;
  const uint16_t* slo;
  const uint16_t* shi;
};
struct LmLd {  // one column of both rows
  uint4 a, b;
  uint32_t sa, sb;
};
__device__ __forceinline__ void lm_load(const LmRows& R, int c, LmLd& L) {
  L.a = __ldg(reinterpret_cast<const uint4*>(R.lo) + c);
  L.b = __ldg(reinterpret_cast<const uint4*>(R.hi) + c);
  L.sa = __ldg(R.slo + c);
  L.sb = __ldg(R.shi + c);
}
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// One matrix's share of a job: rows g, g + 8 of R against tokens
// n0 .. n0 + 8 NBP - 1 of the activation tile btile (K / 64 k-blocks), the
// loads of two iterations in flight.
template <int NBP>
__device__ __forceinline__ void lm_kloop(const LmRows& R, const uint8_t* btile, int nit, int n0,
                                         float (&acc)[NBP][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int b = 0; b < NBP; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
  LmLd L[2];
  lm_load(R, tig, L[0]);
  if (nit > 1) lm_load(R, 4 + tig, L[1]);
#pragma unroll 1
  for (int it0 = 0; it0 < nit; it0 += 2) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int it = it0 + s;
      if (it < nit) {
        const int c = 4 * it + tig;  // this lane's code column: K [32 c, 32 c + 32)
        const uint8_t* bk = btile + size_t(c >> 1) * kTileBytes;
        const uint32_t sa = h2_splat(uint16_t(L[s].sa)), sb = h2_splat(uint16_t(L[s].sb));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t pa[4], pb[4];
          deq4_pairs(u4_word(L[s].a, j), sa, pa);
          deq4_pairs(u4_word(L[s].b, j), sb, pb);
          const int ch = ((c & 1) << 2) + j;  // 16-byte chunk of K [32 c + 8 j, +8) in the k-block
#pragma unroll
          for (int b = 0; b < NBP; ++b) {
            const int r = n0 + 8 * b + g;  // token row of the tile (< 128; rows past n are unused columns)
            const uint4 bq = *reinterpret_cast<const uint4*>(bk + r * 128 + ((ch ^ (r & 7)) << 4));
            mma16816(acc[b], pa[0], pb[0], pa[1], pb[1], bq.x, bq.y);
            mma16816(acc[b], pa[2], pb[2], pa[3], pb[3], bq.z, bq.w);
          }
        }
        if (it + 2 < nit) lm_load(R, 4 * (it + 2) + tig, L[s]);
      }
    }
  }
}

__device__ __forceinline__ LmRows lm_rows(const moe_qmatrix& W, int m_lo, int K) {
  LmRows R;
  R.lo = W.codes + size_t(m_lo) * (K / 2);
  R.hi = W.codes + size_t(m_lo + 8) * (K / 2);
  R.slo = W.scales + size_t(m_lo) * (K / 32);
  R.shi = W.scales + size_t(m_lo + 8) * (K / 32);
  return R;
}

// One job: rows [16 rb, 16 rb + 16) of the weight matrices against the n
// tokens of row tile rt, NBP blocks of 8 tokens per pass over K (gate, then
// up, for gate/up).
template <bool kGateUp, int NBP>
__device__ void lm_job(const Args& a, int rt, int rb, int n) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const int K = a.K, KB = K / BK, nit = K / 128;
  const int grp = a.plan.group[rt];
  const moe_expert& ex = grp < a.E ? a.experts[grp] : *a.shared;
  const int m_lo = rb * 16 + g;
  const uint8_t* btile = a.bt + size_t(rt) * KB * kTileBytes;
  const bool tile_scaled = a.plan.tscaled[rt] != 0;
  for (int n0 = 0; n0 < n; n0 += 8 * NBP) {
    float acc[NBP][4], acu[NBP][4];
    lm_kloop<NBP>(lm_rows(kGateUp ? ex.gate : ex.down, m_lo, K), btile, nit, n0, acc);
    if (kGateUp) lm_kloop<NBP>(lm_rows(ex.up, m_lo, K), btile, nit, n0, acu);
    // D: (row m_lo, tokens 2 tig, 2 tig + 1), (row m_lo + 8, the same tokens)
#pragma unroll
    for (int b = 0; b < NBP; ++b)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int r = n0 + 8 * b + 2 * tig + (v & 1);
        if (r >= n) continue;
        const int m = m_lo + (v >> 1) * 8;
        const int e = tile_scaled ? a.xexp[size_t(rt) * BN + r] : 0;
        if (kGateUp) {
          // the row's x was scaled by 2^-e: g = g_s 2^e, u = u_s 2^e, and
          // h 2^-(kHShift + 2e) = silu(g) 2^-e u_s 2^-kHShift
          float gv = acc[b][v], uv = acu[b][v] * (1.0f / (1 << kHShift));
          if (e) {
            gv *= pow2f(e);
            uv *= pow2f(-e);
          }
          const int kc = (m & 63) >> 3, e8 = m & 7;
          uint8_t* dst = a.ht + (size_t(rt) * (a.I / BK) + (m >> 6)) * kTileBytes + size_t(r) * 128 +
                         ((kc ^ (r & 7)) << 4) + (e8 < 4 ? 4 * e8 : 4 * (e8 - 4) + 2);
          *reinterpret_cast<__half*>(dst) = __float2half_rn(sat_f16(__fdividef(gv, 1.0f + __expf(-gv)) * uv));
        } else {
          // undo the scaling of h: y = y_s 2^(kHShift + 2e)
          const float y = acc[b][v] * pow2f(kHShift + e) * pow2f(e);
          const size_t at = size_t(a.plan.row0[rt] + r) * a.H + m;
          if (grp < a.E && a.y_f32 == nullptr) a.y_bf16[at] = f32_to_bf16_rn(y);
          else (grp < a.E ? a.y_f32 : a.ys_f32)[at] = y;
        }
      }
  }
}

template <bool kGateUp>
__global__ void __launch_bounds__(kLmWarps * 32, 2) light_mma_kernel(Args a) {
  const int nm = a.plan.count[4];
  const int nrb = a.M / 16;  // 16-row weight blocks per matrix
  const long long njobs = (long long)nm * nrb;
  const long long nwarps = (long long)gridDim.x * kLmWarps;
  for (long long j = (long long)blockIdx.x * kLmWarps + (threadIdx.x >> 5); j < njobs; j += nwarps) {
    const int mi = int(j / nrb), rb = int(j - (long long)mi * nrb);
    const int rt = a.plan.mlist[mi];
    const int n = a.plan.nrows[rt];
    if (n <= 8) lm_job<kGateUp, 1>(a, rt, rb, n);
    else lm_job<kGateUp, 2>(a, rt, rb, n);  // n <= kMmaRows: one pass
  }
}
}  // namespace gemm
}  // namespace moe

namespace moe {

// Upper bound on row tiles: every group adds at most one partial tile.
long long grouped_max_tiles(long long T, int k, int E, bool with_shared) {
  // at most one partial tile per non-empty group, and at most T k non-empty groups
  const long long routed = (T * k + gemm::BN - 1) / gemm::BN + (E < T * k ? E : T * k);
  return routed + (with_shared ? (T + gemm::BN - 1) / gemm::BN + 1 : 0) + 1;
}

bool grouped_eligible(int H, int I, int E, bool with_shared) {
  return (H % 128) == 0 && (I % 128) == 0 && H <= 16384 && I <= 16384 && E + (with_shared ? 1 : 0) <= 1024;
}

// Heavy slots a launch may use: routed groups with at least kHeavyRows rows
// (at most T k / kHeavyRows of them) plus the shared group when T is that
// large, capped at kMaxHeavy and at 1 GiB of pre-dequantised weights.
int grouped_heavy_slots(long long T, int k, bool with_shared, int H, int I) {
  long long n = T * k / gemm::kHeavyRows + ((with_shared && T >= gemm::kHeavyRows) ? 1 : 0);
  n = n < gemm::kMaxHeavy ? n : gemm::kMaxHeavy;
  const long long by_bytes = (1ll << 30) / (long long)gemm::heavy_slot_bytes(H, I);
  return int(n < by_bytes ? n : by_bytes);
}

size_t grouped_ws_bytes(long long T, int H, int I, int k, int E, bool with_shared) {
  const long long mt = grouped_max_tiles(T, k, E, with_shared);
  return align256(24 * size_t(mt) + 32) + align256(4 * size_t(E + 1) + 4 * size_t(gemm::kMaxHeavy)) +
         align256(4 * size_t(mt)) + align256(4 * size_t(mt) * gemm::BN) + align256(size_t(mt) * (H / gemm::BK) * gemm::kTileBytes) +
         align256(size_t(mt) * (I / gemm::BK) * gemm::kTileBytes) +
         align256(size_t(grouped_heavy_slots(T, k, with_shared, H, I)) * gemm::heavy_slot_bytes(H, I));
}

cudaError_t launch_grouped_ffn(const uint16_t* x, int T, int H, int I, int k, int E, const int* perm_src,
                               const int* offsets, const int* counts, const moe_expert* experts,
                               const moe_expert* shared, float* y_f32, uint16_t* y_bf16, float* ys_f32,
                               void* scratch, WsHeader* hdr, cudaStream_t st) {
  using namespace gemm;
  if (T == 0) return cudaSuccess;
  const bool with_shared = shared != nullptr;
  const long long mt = grouped_max_tiles(T, k, E, with_shared);
  uint8_t* p = static_cast<uint8_t*>(scratch);
  Plan plan;
  plan.count = reinterpret_cast<int*>(p);
  plan.group = plan.count + 8;
  plan.row0 = plan.group + mt;
  plan.nrows = plan.row0 + mt;
  plan.wlist = plan.nrows + mt;
  plan.llist = plan.wlist + mt;
  plan.mlist = plan.llist + mt;
  p += align256(24 * size_t(mt) + 32);
  plan.hslot = reinterpret_cast<int*>(p);
  plan.hlist = plan.hslot + (E + 1);
  p += align256(4 * size_t(E + 1) + 4 * size_t(kMaxHeavy));
  plan.tscaled = reinterpret_cast<int*>(p);
  p += align256(4 * size_t(mt));
  int* xexp = reinterpret_cast<int*>(p);
  p += align256(4 * size_t(mt) * BN);
  uint8_t* xt = p;
  p += align256(size_t(mt) * (H / BK) * kTileBytes);
  uint8_t* ht = p;
  p += align256(size_t(mt) * (I / BK) * kTileBytes);
  uint8_t* aimg = p;
  const int max_heavy = grouped_heavy_slots(T, k, with_shared, H, I);

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

  plan_kernel<<<1, 1024, 0, st>>>(counts, offsets, experts, shared, H, I, E, with_shared ? T : 0, int(mt), max_heavy,
                                  plan, hdr);
  gather_rows_kernel<<<sms * 4, 256, 0, st>>>(x, H, k, perm_src, E, plan, xt, xexp);
  if (max_heavy > 0) predequant_kernel<<<sms * 4, 256, 0, st>>>(experts, shared, E, H, I, plan, aimg, hdr);
  const size_t smem_gu = size_t(Cfg<true>::kStages) * Cfg<true>::kStageBytes + size_t(kRawDepth) * kRawSlotBytes + 1024;
  const size_t smem_dn = size_t(Cfg<false>::kStages) * Cfg<false>::kStageBytes + size_t(kRawDepth) * kRawSlotBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem_gu));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_dn));
  if (e != cudaSuccess) return e;
  const size_t smem_wgu = wide_smem_bytes<kGuNA, kGuNB>(), smem_wdn = wide_smem_bytes<kDnNA, kDnNB>();
  e = cudaFuncSetAttribute(wide_gemm_kernel<true, kGuNA, kGuNB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem_wgu));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(wide_gemm_kernel<false, kDnNA, kDnNB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem_wdn));
  if (e != cudaSuccess) return e;
  Args a{};
  a.plan = plan;
  a.experts = experts;
  a.shared = shared;
  a.E = E;
  a.I = I;
  a.H = H;
  a.hdr = hdr;
  a.aimg = aimg;
  a.aslot = heavy_slot_bytes(H, I);
  a.xexp = xexp;
  // gate/up: K = H, M = I; B = gathered X tiles; out = H tiles
  a.K = H;
  a.M = I;
  a.bt = xt;
  a.ht = ht;
  a.aoff = 0;
  if (max_heavy > 0) wide_gemm_kernel<true, kGuNA, kGuNB><<<sms, kWThreads, smem_wgu, st>>>(a);
  grouped_gemm_kernel<true><<<sms, kThreads, smem_gu, st>>>(a);
  light_mma_kernel<true><<<sms * 2, kLmWarps * 32, 0, st>>>(a);
  // down: K = I, M = H; B = H tiles; out = rows
  a.K = I;
  a.M = H;
  a.bt = ht;
  a.ht = nullptr;
  a.aoff = heavy_gu_bytes(H, I);
  a.y_f32 = y_f32;
  a.y_bf16 = y_bf16;
  a.ys_f32 = ys_f32;
  if (max_heavy > 0) wide_gemm_kernel<false, kDnNA, kDnNB><<<sms, kWThreads, smem_wdn, st>>>(a);
  grouped_gemm_kernel<false><<<sms, kThreads, smem_dn, st>>>(a);
  light_mma_kernel<false><<<sms * 2, kLmWarps * 32, 0, st>>>(a);
  count_launches(max_heavy > 0 ? 9 : 6);
  return cudaGetLastError();
}

}  // namespace moe
