// prep.cuh -- fused SharQ preprocessing and weight quantization for sm_100a.
//
// SharQ (arXiv 2606.26587) abstract / Section 1: per activation row, an online
// N:M mask extracts an outlier-dominated sparse backbone that is quantized to
// FP4; the dense residual is taken against the QUANTIZED backbone and quantized
// to FP4 as well; mask selection, residual construction and the layer norm
// are done by one fused preprocessing operator.
//
// Work split: a thread owns 32 consecutive K elements (one "unit": 4 x
// 16-byte loads of bf16, 8 of fp32); a power-of-two number of threads (8..128)
// shares a row, several rows share a block of 128 threads when rows are short.
// For NVFP4 a unit is exactly one backbone block (16 kept values) and two
// residual blocks; for MXFP4 a backbone block spans the units of a lane pair
// (shuffle for its amax) and a residual block is one unit.  Every floating point step is an explicitly rounded fp32 op
// in a fixed order, so codes and scales are reproducible bit for bit.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace sharq {

enum { FMT_MX = 0, FMT_NV = 1 };
enum { PAT_24 = 0, PAT_48P = 1, PAT_816 = 2, PAT_816P = 3 };
// Patterns stored in the 4:8 pair layout (metadata, compressed backbone, scales):
// the 4:8 pair itself and the 8:16 selection re-packed into it.
__host__ __device__ constexpr bool pair_layout(int pat) { return pat == PAT_48P || pat == PAT_816P; }

// Byte offset of (row r, scale s) in the tiled scale layout with S scales per row.
__host__ __device__ __forceinline__ int64_t tiled_sf_offset(int64_t r, int64_t s, int64_t S) {
  const int64_t sblocks = (S + 3) >> 2;
  return ((r >> 7) * sblocks + (s >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (s & 3);
}
__host__ __device__ __forceinline__ int64_t tiled_sf_bytes(int64_t rows, int64_t S) {
  return ((rows + 127) / 128) * ((S + 3) / 4) * 512;
}

struct PrepParams {
  const void* x;     // activations (SwiGLU form: the gate input)
  const void* x2;    // SwiGLU form: the up input (same layout and dtype as x); else null
  const void* gamma;
  float eps;
  int64_t t, t_pad, k;
  uint8_t* meta;
  uint8_t* bb_codes;
  uint8_t* bb_scales;
  uint8_t* res_codes;
  uint8_t* res_scales;
  float* tensor;     // [amax, g_enc, g_dec]
  float act_amax;    // > 0: given by the caller
  const float* rstd; // per-row RMSNorm factors from the amax pass, or null
  int tpr;           // threads per row (a power of two, 8..128, set by the launcher)
};

// ------------------------------------------------------------- loading
template <bool XBF16>
__device__ __forceinline__ void load_unit(const void* base, int64_t off, float (&v)[32]) {
  if constexpr (XBF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + off);
#pragma unroll
    for (int q = 0; q < 4; q++) {
      uint4 w = __ldg(p + q);
      uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; j++) {
        v[8 * q + 2 * j] = __uint_as_float(ws[j] << 16);
        v[8 * q + 2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
#pragma unroll
    for (int q = 0; q < 8; q++) {
      float4 w = __ldg(p + q);
      v[4 * q] = w.x;
      v[4 * q + 1] = w.y;
      v[4 * q + 2] = w.z;
      v[4 * q + 3] = w.w;
    }
  }
}

// 32 bf16 values (4 x 16 bytes, element i in the low half first) -> fp32.
__device__ __forceinline__ void unpack_bf16_unit(const uint4 (&w4)[4], float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; q++) {
    const uint32_t ws[4] = {w4[q].x, w4[q].y, w4[q].z, w4[q].w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
      v[8 * q + 2 * j] = __uint_as_float(ws[j] << 16);
      v[8 * q + 2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
    }
  }
}

// --------------------------------------------------------------- SwiGLU
// h = SiLU(gate) * up with SiLU(a) = a / (1 + E(-a)), every step a single
// IEEE round-to-nearest fp32 operation.  E is this project's exponential:
// Cody and Waite's range reduction by ln 2 (split in two fp32 constants) and
// the degree-7 Taylor polynomial evaluated by Horner with fused multiply-adds,
// then an exact scaling by 2^n in two halves; the input is clamped to
// [-104, 89], beyond which e^x is 0 or infinite in fp32 anyway.
__device__ __forceinline__ float pow2i_dev(int e) {  // exact 2^e, -126 <= e <= 127
  return __int_as_float((e + 127) << 23);
}
__device__ __forceinline__ float dev_exp(float x) {
  x = fminf(fmaxf(x, -104.0f), 89.0f);
  const float nf = rintf(__fmul_rn(x, 1.44269502162933349609375f));  // log2(e) rounded to fp32
  const int n = (int)nf;
  float r = __fmaf_rn(-nf, 0.693145751953125f, x);                   // ln 2, high 15 bits
  r = __fmaf_rn(-nf, 1.428606765330187045037746429443359375e-06f, r);  // ln 2 - high part, rounded
  float p = 1.0f / 5040.0f;
  p = __fmaf_rn(p, r, 1.0f / 720.0f);
  p = __fmaf_rn(p, r, 1.0f / 120.0f);
  p = __fmaf_rn(p, r, 1.0f / 24.0f);
  p = __fmaf_rn(p, r, 1.0f / 6.0f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int n1 = n / 2, n2 = n - n1;
  return __fmul_rn(__fmul_rn(p, pow2i_dev(n1)), pow2i_dev(n2));
}
__device__ __forceinline__ float dev_silu(float a) { return __fdiv_rn(a, __fadd_rn(1.0f, dev_exp(-a))); }

// h of one unit in the SwiGLU form.
template <bool XBF16>
__device__ __forceinline__ void swiglu_unit(const void* gate, const void* up, int64_t off, float (&h)[32]) {
  float a[32], b[32];
  load_unit<XBF16>(gate, off, a);
  load_unit<XBF16>(up, off, b);
#pragma unroll
  for (int i = 0; i < 32; i++) h[i] = __fmul_rn(dev_silu(a[i]), b[i]);
}

// Eight E2M1 codes (nibbles of c, element i in nibble i) -> exact fp32 values.
__device__ __forceinline__ void e2m1x8_values(uint32_t c, float* out) {
#pragma unroll
  for (int b = 0; b < 4; b++) {
    uint32_t h2;
    const uint16_t byte = (uint16_t)((c >> (8 * b)) & 0xFF);
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u16 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "h"(byte));
    out[2 * b] = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
    out[2 * b + 1] = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
  }
}

// ------------------------------------------------------------------- mask
// keep bits (bit i = element i of the unit kept) and metadata for 32 values.
// Element (pair) i is kept iff fewer than N of its group beat it, where j
// beats i if |h_j| > |h_i|, or they are equal and j < i.
__device__ __forceinline__ uint32_t top2of4(float a0, float a1, float a2, float a3) {
  const int b01 = a0 >= a1, b02 = a0 >= a2, b03 = a0 >= a3, b12 = a1 >= a2, b13 = a1 >= a3, b23 = a2 >= a3;
  const int n0 = 3 - b01 - b02 - b03;
  const int n1 = b01 + 2 - b12 - b13;
  const int n2 = b02 + b12 + 1 - b23;
  const int n3 = b03 + b13 + b23;
  return (uint32_t)(n0 < 2) | ((uint32_t)(n1 < 2) << 1) | ((uint32_t)(n2 < 2) << 2) | ((uint32_t)(n3 < 2) << 3);
}
// 0xFFFFFFFF if a >= b, else 0: a comparison whose result can be combined bitwise.
__device__ __forceinline__ uint32_t ge_mask(float a, float b) {
  uint32_t r;
  asm("set.ge.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ uint32_t maj3(uint32_t a, uint32_t b, uint32_t c) { return (a & b) | (c & (a | b)); }
// The same top-2-of-4 rule as four masks (0 or ~0), from bitwise majorities of
// the comparison masks: entry p wins against q < p when s_p > s_q and against
// q > p when s_p >= s_q, and is kept iff it wins at least two of its three
// comparisons (used where byte masks are wanted, the 4:8 pair pattern).
__device__ __forceinline__ void top2of4_masks(float s0, float s1, float s2, float s3, uint32_t (&k)[4]) {
  const uint32_t b01 = ge_mask(s0, s1), b02 = ge_mask(s0, s2), b03 = ge_mask(s0, s3);
  const uint32_t b12 = ge_mask(s1, s2), b13 = ge_mask(s1, s3), b23 = ge_mask(s2, s3);
  k[0] = maj3(b01, b02, b03);
  k[1] = maj3(~b01, b12, b13);
  k[2] = maj3(~b02, ~b12, b23);
  k[3] = maj3(~b03, ~b13, ~b23);
}
// Metadata nibble i0 | i1 << 2 (kept indices i0 < i1) of two-of-four keep masks.
__device__ __forceinline__ uint32_t kept_nibble(const uint32_t (&k)[4]) {
  const uint32_t i0 = (~k[0] & 1u) + (~k[0] & ~k[1] & 1u);
  const uint32_t i1 = 1u + ((k[2] | k[3]) & 1u) + (k[3] & 1u);
  return i0 | (i1 << 2);
}
// metadata nibble (i0 | i1 << 2) of a 4-bit mask with exactly two bits set
__device__ __forceinline__ uint32_t pair_nibble(uint32_t kp) {
  // kp: 0b0011 -> 4, 0b0101 -> 8, 0b0110 -> 9, 0b1001 -> 12, 0b1010 -> 13, 0b1100 -> 14
  constexpr uint64_t LUT = (4ull << 12) | (8ull << 20) | (9ull << 24) | (12ull << 36) | (13ull << 40) | (14ull << 48);
  return (uint32_t)(LUT >> (4 * kp)) & 15u;
}

// Sorts 8 values in descending order with a 19-comparator network (each
// comparator: max to the lower position, min to the higher).
__device__ __forceinline__ void sort8_desc(float (&v)[8]) {
  auto ce = [&](int i, int j) {
    const float hi = fmaxf(v[i], v[j]), lo = fminf(v[i], v[j]);
    v[i] = hi;
    v[j] = lo;
  };
  ce(0, 2); ce(1, 3); ce(4, 6); ce(5, 7);
  ce(0, 4); ce(1, 5); ce(2, 6); ce(3, 7);
  ce(0, 1); ce(2, 3); ce(4, 5); ce(6, 7);
  ce(2, 4); ce(3, 5);
  ce(1, 4); ce(3, 6);
  ce(1, 2); ce(3, 4); ce(5, 6);
}

template <int PAT>
__device__ __forceinline__ uint32_t unit_mask(const float (&h)[32], uint32_t& meta) {
  uint32_t keep = 0;
  meta = 0;
  if constexpr (PAT == PAT_48P) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const float* hg = h + 8 * g;
      const uint32_t kp = top2of4(fmaxf(fabsf(hg[0]), fabsf(hg[1])), fmaxf(fabsf(hg[2]), fabsf(hg[3])),
                                  fmaxf(fabsf(hg[4]), fabsf(hg[5])), fmaxf(fabsf(hg[6]), fabsf(hg[7])));
      meta |= pair_nibble(kp) << (4 * g);
      // spread pair bits to element bits: pair p -> elements 2p, 2p+1
      uint32_t e = (kp & 1u) | ((kp & 2u) << 1) | ((kp & 4u) << 2) | ((kp & 8u) << 3);
      keep |= (e | (e << 1)) << (8 * g);
    }
  } else if constexpr (PAT == PAT_24) {
#pragma unroll
    for (int g = 0; g < 8; g++) {
      const float* hg = h + 4 * g;
      const uint32_t kg = top2of4(fabsf(hg[0]), fabsf(hg[1]), fabsf(hg[2]), fabsf(hg[3]));
      meta |= pair_nibble(kg) << (4 * g);
      keep |= kg << (4 * g);
    }
  } else {
    // top 8 of each group of 16 by magnitude, ties to the lower index: T, the
    // 8th largest magnitude, is the smallest of max(A_i, B_(7-i)) over the two
    // halves sorted in descending order (the first step of a bitonic merge);
    // every magnitude above T is kept, and of those equal to T the ones with
    // the lowest indices, as many as are still missing.  Equal to ranking each
    // element against the other 15.
#pragma unroll
    for (int g = 0; g < 2; g++) {
      float a[16], A[8], B[8];
#pragma unroll
      for (int i = 0; i < 16; i++) a[i] = fabsf(h[16 * g + i]);
#pragma unroll
      for (int i = 0; i < 8; i++) {
        A[i] = a[i];
        B[i] = a[8 + i];
      }
      sort8_desc(A);
      sort8_desc(B);
      float thr = fmaxf(A[0], B[7]);
#pragma unroll
      for (int i = 1; i < 8; i++) thr = fminf(thr, fmaxf(A[i], B[7 - i]));
      uint32_t gt = 0, eq = 0;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        gt |= (a[i] > thr ? 1u : 0u) << i;
        eq |= (a[i] == thr ? 1u : 0u) << i;
      }
      const int need = 8 - __popc(gt);  // >= 1: at most 7 magnitudes exceed the 8th largest
      uint32_t kg = gt;
#pragma unroll
      for (int q = 0; q < 8; q++) {  // the lowest `need` set bits of eq
        const uint32_t low = eq & (0u - eq);
        if (q < need) kg |= low;
        eq ^= low;
      }
      meta |= kg << (16 * g);
      keep |= kg << (16 * g);
    }
  }
  return keep;
}

// ------------------------------------------------------- block quantizers
// MXFP4 scale exponent: floor(log2 amax) - 2 clamped to [-127, 127]; amax = 0 -> -127.
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.0f)) return -127;
  const uint32_t bits = __float_as_uint(amax);
  const int ex = (int)((bits >> 23) & 0xFF);
  int fl = ex ? ex - 127 : (31 - __clz(bits & 0x7FFFFF)) - 149;
  int e = fl - 2;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}
__device__ __forceinline__ float pow2f(int e) {  // exact 2^e for e in [-127, 127]
  return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// amax / 6 rounded to nearest (the block's decode scale before the tensor
// scale: the largest E2M1 magnitude, 6, is mapped onto the block amax).  For
// amax >= 2^-125 one product with RN(1/6) is corrected by its remainder, which
// a fused multiply-add gives exactly (Markstein's correction step for division
// by a constant whose reciprocal is rounded to nearest); checked against IEEE
// division for every fp32 value in that range.  Below it the quotient is
// subnormal and the remainder inexact, so those (rare) inputs divide directly.
__device__ __forceinline__ float div6_rn(float a) {
  if (a < 0x1p-125f) return __fdiv_rn(a, 6.0f);
  constexpr float kSixth = 1.0f / 6.0f;  // RN(1/6)
  const float q0 = __fmul_rn(a, kSixth);
  return __fmaf_rn(__fmaf_rn(-q0, 6.0f, a), kSixth, q0);
}

// Block scale: returns the scale code, the multiplier that maps values onto the
// E2M1 grid (0 means "all codes +0") and the decoded scale (times g_dec for
// the dequantized value: deq = (e2m1 * sv) * g_dec for NVFP4, e2m1 * sv for MX).
// NVFP4: s = (amax / 6) * g_enc, each step rounded once, S = E4M3(s),
// mul = g_enc / S (exact table).
// NVFP4 also returns the decoded scale as an f16 value in both halves of sh
// (E4M3 values are exact in f16).
template <int FMT>
__device__ __forceinline__ uint32_t block_scale(float amax, float g_enc, const float* inv_tab, float& mul, float& sv,
                                                uint32_t& sh) {
  if constexpr (FMT == FMT_MX) {
    const int e = mx_exponent(amax);
    mul = pow2f(-e);
    sv = pow2f(e);
    sh = 0;
    return (uint32_t)(e + 127);
  } else {
    const uint32_t sc = cvt_e4m3(__fmul_rn(div6_rn(amax), g_enc));
    uint32_t h2;
    const uint16_t in = (uint16_t)(sc | (sc << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    sh = h2;
    sv = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
    mul = inv_tab[sc];  // 0 for code 0
    return sc;
  }
}
template <int FMT>
__device__ __forceinline__ uint32_t block_scale(float amax, float g_enc, const float* inv_tab, float& mul, float& sv) {
  uint32_t sh;
  return block_scale<FMT>(amax, g_enc, inv_tab, mul, sv, sh);
}

// Quantize 8 values: returns 8 codes (nibbles); mul = 0 gives +0 codes.
__device__ __forceinline__ uint32_t quant8(const float* v, float mul) {
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; i++) q[i] = __fmul_rn(v[i], mul);
  const uint32_t c = cvt_e2m1x8(q);
  return mul == 0.0f ? 0u : c;
}

// tensor scale from the amax (same rule as the weights'): g_enc = 2688 / A,
// g_dec = A / 2688; A = 0 gives 1; an overflowing g_enc is clamped.
__device__ __forceinline__ void tensor_scales(float amax, float& g_enc, float& g_dec) {
  if (!(amax > 0.0f)) {
    g_enc = 1.0f;
    g_dec = 1.0f;
    return;
  }
  g_enc = __fdiv_rn(2688.0f, amax);
  if (isinf(g_enc)) g_enc = 3.402823466e38f;
  g_dec = __fdiv_rn(amax, 2688.0f);
}

// Exact table of g_enc / value(code) for the E4M3 codes 1..126 (code 0 -> 0).
// Needs >= 128 threads in the block and a __syncthreads() after.
__device__ __forceinline__ void fill_inv_table(float* tab, float g_enc) {
  const int c = threadIdx.x;
  if (c < 128) tab[c] = (c >= 1 && c <= 126) ? __fdiv_rn(g_enc, e4m3_value((uint32_t)c)) : 0.0f;
}

// ------------------------------------------------------------ row mapping
// A block of 128 threads handles 128 / tpr rows at a time; tpr threads per row
// (a power of two, 8..128); thread t of a row owns the units t + tpr*j.
// Blocks stride over row groups.
struct RowMap {
  int tpr;    // threads per row
  int lg;     // log2(tpr)
  int units;  // units (32 elements) per row
  int nj;     // units per thread, <= 8
};

// Threads per row for a row of `units` 32-element units: the largest power of
// two in 8..128 that divides the units with at most 8 per thread, so that no
// thread of a row idles (5120 = 160 units: 32 threads x 5; 14336 = 448 units:
// 64 x 7); otherwise the smallest power of two covering them in <= 4 per thread.
__host__ __device__ __forceinline__ int rows_tpr(int64_t units) {
  for (int c = 128; c >= 8; c >>= 1)
    if (units % c == 0 && units / c <= 8) return c;
  int tpr = 8;
  while (tpr < units && tpr < 128) tpr <<= 1;
  return tpr;
}

// Few rows (all of them resident at once as one row per block) take 128 threads
// per row whenever that leaves at most 8 units per thread: the least serial work
// per thread.  When 128 threads per row would need a second round of blocks and
// 64 threads (two rows per block) fit every row in one round, 64 is taken (the
// same work per thread, no second launch wave: q_proj's 2048 rows on 1036
// resident blocks, 14.2 -> 13.6 us).  The reductions are the same fixed tree for
// every power-of-two tpr.
__host__ __device__ __forceinline__ int rows_tpr(int64_t units, int64_t rows, int64_t resident_blocks) {
  if (rows <= resident_blocks && units >= 128 && units <= 8 * 128) return 128;
  const int tpr = rows_tpr(units);
  if (tpr == 128 && units % 64 == 0 && units / 64 <= 8 && (rows + 1) / 2 <= resident_blocks) return 64;
  return tpr;
}

__device__ __forceinline__ RowMap row_map(int64_t k, int tpr) {
  RowMap m;
  m.units = (int)(k / 32);
  m.tpr = tpr;
  m.lg = 31 - __clz(tpr);
  m.nj = (m.units + tpr - 1) / tpr;
  return m;
}

// Sum of squares of the thread's row in the fixed order of the oracle:
// 16-element chunk sums by sequential FMA; then a pairwise tree of adjacent
// entries: the two chunks of a unit inside the thread, units across the row's
// threads by xor butterflies (inside a warp, then across the row's warps via
// shared memory), then the per-j slab sums pairwise, zero padded to 4.  This
// equals the tree over all chunks zero padded to a power of two.
// All threads of the block must call it (it contains __syncthreads()).
template <bool XBF16>
__device__ __forceinline__ float row_sumsq(const void* x, int64_t row_off, bool real, const RowMap& m, int t,
                                           int row_in_block, float* red /* [32 rows][4 warps][4 j] */) {
  float s[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  const int wlanes = m.tpr < 32 ? m.tpr : 32;
#pragma unroll
  for (int j = 0; j < 8; j++) {
    if (j < m.nj) {
      const int u = t + m.tpr * j;
      float c0 = 0.0f, c1 = 0.0f;
      if (real && u < m.units) {
        float v[32];
        load_unit<XBF16>(x, row_off + (int64_t)u * 32, v);
#pragma unroll
        for (int i = 0; i < 16; i++) c0 = __fmaf_rn(v[i], v[i], c0);
#pragma unroll
        for (int i = 16; i < 32; i++) c1 = __fmaf_rn(v[i], v[i], c1);
      }
      float a = __fadd_rn(c0, c1);
      for (int msk = 1; msk < wlanes; msk <<= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, msk));
      s[j] = a;
    }
  }
  if (m.tpr > 32) {
    const int w = t >> 5, nw = m.tpr >> 5;
    if ((t & 31) == 0) {
#pragma unroll
      for (int j = 0; j < 8; j++) red[(row_in_block * 4 + w) * 8 + j] = s[j];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const float w0 = red[(row_in_block * 4 + 0) * 8 + j], w1 = red[(row_in_block * 4 + 1) * 8 + j];
      if (nw == 2) {
        s[j] = __fadd_rn(w0, w1);
      } else {
        const float w2 = red[(row_in_block * 4 + 2) * 8 + j], w3 = red[(row_in_block * 4 + 3) * 8 + j];
        s[j] = __fadd_rn(__fadd_rn(w0, w1), __fadd_rn(w2, w3));
      }
    }
    __syncthreads();
  }
  return __fadd_rn(__fadd_rn(__fadd_rn(s[0], s[1]), __fadd_rn(s[2], s[3])),
                   __fadd_rn(__fadd_rn(s[4], s[5]), __fadd_rn(s[6], s[7])));
}

__device__ __forceinline__ float rstd_from_sumsq(float sumsq, int64_t k, float eps) {
  const float mean = __fdiv_rn(sumsq, (float)k);
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
}

// ---------------------------------------------------------- packed fp32
// Elementwise IEEE round-to-nearest on two fp32 lanes at once (sm_100 f32x2).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ void mul2(float& a, float& b, float c, float d) {  // (a, b) *= (c, d)
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk2(a, b)), "l"(pk2(c, d)));
  a = __uint_as_float((uint32_t)r);
  b = __uint_as_float((uint32_t)(r >> 32));
}
__device__ __forceinline__ void sub2(float& a, float& b, float c, float d) {  // (a, b) -= (c, d)
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk2(a, b)), "l"(pk2(c, d)));
  a = __uint_as_float((uint32_t)r);
  b = __uint_as_float((uint32_t)(r >> 32));
}

__device__ __forceinline__ void fma2(float& a, float& b, float c, float d, float e, float f) {  // (a,b)*(c,d)+(e,f)
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pk2(a, b)), "l"(pk2(c, d)), "l"(pk2(e, f)));
  a = __uint_as_float((uint32_t)r);
  b = __uint_as_float((uint32_t)(r >> 32));
}

// ------------------------------------------------------------ stats kernel
// Per row: rstd (RMSNorm) into rstd_out (if non-null) and max |h| folded into
// amax_out[0] (zeroed beforehand) with one atomic per block.
template <bool NORM, bool XBF16, bool ACT = false>
__global__ void __launch_bounds__(128) amax_kernel(const void* x, const void* gamma, float eps, int64_t t, int64_t k,
                                                   float* amax_out, float* rstd_out, const void* x2, int tpr) {
  static_assert(!(NORM && ACT), "the SwiGLU form has no RMSNorm");
  __shared__ float red[32 * 16];
  __shared__ float wmax[4];
  grid_dep_launch();
  const RowMap m = row_map(k, tpr);
  const int rpb = 128 / m.tpr;
  const int row_in_block = threadIdx.x >> m.lg, tt = threadIdx.x & (m.tpr - 1);
  float my = 0.0f;
  for (int64_t r0 = (int64_t)blockIdx.x * rpb; r0 < t; r0 += (int64_t)gridDim.x * rpb) {
    const int64_t r = r0 + row_in_block;
    const bool real = r < t;
    const int64_t off = r * k;
    float rs = 1.0f;
    if constexpr (NORM) {
      rs = rstd_from_sumsq(row_sumsq<XBF16>(x, off, real, m, tt, row_in_block, red), k, eps);
      if (rstd_out && real && tt == 0) rstd_out[r] = rs;
    }
    for (int j = 0; j < m.nj; j++) {
      const int u = tt + m.tpr * j;
      if (!real || u >= m.units) continue;
      float v[32];
      if constexpr (ACT) swiglu_unit<XBF16>(x, x2, off + (int64_t)u * 32, v);
      else load_unit<XBF16>(x, off + (int64_t)u * 32, v);
      if constexpr (NORM) {
        float g[32];
        load_unit<XBF16>(gamma, (int64_t)u * 32, g);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          mul2(v[i], v[i + 1], rs, rs);
          mul2(v[i], v[i + 1], g[i], g[i + 1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 32; i++) my = fmaxf(my, fabsf(v[i]));
    }
  }
#pragma unroll
  for (int msk = 16; msk >= 1; msk >>= 1) my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, msk));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = my;
  __syncthreads();
  if (threadIdx.x == 0) {
    const float mm = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    atomicMax(reinterpret_cast<unsigned int*>(amax_out), __float_as_uint(mm));
  }
}

// Amax pass for bf16 rows of k <= 4096 (at most 4 units per lane).  Two rows
// per block, two warps per row: lane l of warp h holds the units
// l + 32 (2h) and l + 32 (2h + 1), so each 32-unit slab is one coalesced
// 2 KB read, and all of a row's loads are issued before any arithmetic;
// gamma is copied into shared memory meanwhile.  The sum of squares follows
// row_sumsq's fixed order: 16-element chunk sums, the pair of a unit,
// butterflies over the 32 units of a slab, then the slab sums pairwise
// ((s0 + s1) + (s2 + s3), zero padded), the halves exchanged through
// shared memory at the one block barrier.
template <bool NORM>
__global__ void __launch_bounds__(128, 7) amax_rows_kernel(const void* x, const void* gamma, float eps, int64_t t,
                                                           int64_t k, float* amax_out, float* rstd_out) {
  __shared__ float wmax[4];
  __shared__ float ssum[4];
  __shared__ uint4 gs[4096 / 8];
  grid_dep_launch();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, hw = w & 1;
  const int64_t r = (int64_t)blockIdx.x * 2 + (w >> 1);
  const bool have = r < t;
  const int units = (int)(k / 32);
  const int nj = (units + 31) >> 5;
  const int64_t off = r * k;
  uint4 raw[2][4];
#pragma unroll
  for (int jj = 0; jj < 2; jj++) {
    const int j = 2 * hw + jj;
    const int u = lane + 32 * j;
    const bool on = have && j < nj && u < units;
    const uint4* p4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + (on ? off + (int64_t)u * 32 : 0));
#pragma unroll
    for (int q = 0; q < 4; q++) raw[jj][q] = on ? __ldg(p4 + q) : make_uint4(0u, 0u, 0u, 0u);
  }
  if constexpr (NORM) {
    const uint4* g4 = static_cast<const uint4*>(gamma);
    for (int i = threadIdx.x; i < (int)(k / 8); i += 128) gs[i] = __ldg(g4 + i);
  }
  float rs = 1.0f;
  if constexpr (NORM) {
    float sl[2];
#pragma unroll
    for (int jj = 0; jj < 2; jj++) {
      float v[32];
      unpack_bf16_unit(raw[jj], v);
      float c0 = 0.0f, c1 = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; i++) c0 = __fmaf_rn(v[i], v[i], c0);
#pragma unroll
      for (int i = 16; i < 32; i++) c1 = __fmaf_rn(v[i], v[i], c1);
      float a = __fadd_rn(c0, c1);
#pragma unroll
      for (int msk = 1; msk < 32; msk <<= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, msk));
      sl[jj] = (2 * hw + jj) < nj ? a : 0.0f;
    }
    if (lane == 0) ssum[w] = __fadd_rn(sl[0], sl[1]);
  }
  __syncthreads();  // every thread: gamma in shared memory, half-row sums exchanged
  float my = 0.0f;
  if (have) {
    if constexpr (NORM) {
      const int w0 = w & ~1;
      rs = rstd_from_sumsq(__fadd_rn(ssum[w0], ssum[w0 + 1]), k, eps);
      if (rstd_out && lane == 0 && hw == 0) rstd_out[r] = rs;
    }
#pragma unroll
    for (int jj = 0; jj < 2; jj++) {
      const int j = 2 * hw + jj;
      const int u = lane + 32 * j;
      if (j >= nj || u >= units) continue;
      float v[32];
      unpack_bf16_unit(raw[jj], v);
      if constexpr (NORM) {
        float g[32];
        const uint4 g4[4] = {gs[4 * u], gs[4 * u + 1], gs[4 * u + 2], gs[4 * u + 3]};
        unpack_bf16_unit(g4, g);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          mul2(v[i], v[i + 1], rs, rs);
          mul2(v[i], v[i + 1], g[i], g[i + 1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 32; i++) my = fmaxf(my, fabsf(v[i]));
    }
  }
#pragma unroll
  for (int msk = 16; msk >= 1; msk >>= 1) my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, msk));
  if (lane == 0) wmax[w] = my;
  __syncthreads();
  if (threadIdx.x == 0) {
    const float mm = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    if (__float_as_uint(mm) > *reinterpret_cast<volatile unsigned int*>(amax_out))
      atomicMax(reinterpret_cast<unsigned int*>(amax_out), __float_as_uint(mm));
  }
}

// Nibble mask of kept elements of a 2:4 quad pair (8 elements, two quads).
__device__ __forceinline__ uint32_t nibble_mask8(uint32_t keep8) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) m |= ((keep8 >> i) & 1u) ? (0xFu << (4 * i)) : 0u;
  return m;
}
// The same mask by bit spreading: bit i is moved to position 4i in three
// shift-or-mask steps, then each becomes a nibble by multiplying with 15 (no
// carries: every nibble holds 0 or 1).  Fewer instructions; used by the 8:16
// path, where it was measured faster (the 2:4 path keeps the loop above).
__device__ __forceinline__ uint32_t nibble_spread8(uint32_t keep8) {
  uint32_t x = keep8 & 0xFFu;
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  return x * 0xFu;
}
// Compact the codes of the two kept bytes (pairs p0 < p1) of a 4-byte word.
__device__ __forceinline__ uint32_t compact_pairs(uint32_t w, uint32_t p0, uint32_t p1) {
  return __byte_perm(w, 0u, p0 | (p1 << 4) | 0x4400u);  // bytes p0, p1 -> positions 0, 1; zeros above
}

// Residual of 8 values against their backbone codes, in place: h_i -= deq_i
// with deq = (e2m1(c_i) * S) * g (NVFP4) or e2m1(c_i) * 2^e (MXFP4).
//   NVFP4: e2m1 * S is exact (2-bit times 4-bit significands): one mixed
//   f16 x f16 -> f32 fused multiply-add with a -0 addend forms it from the f16
//   E2M1 pair and the f16 scale; times g is then one packed round-to-nearest
//   multiply, and h - deq one packed fused multiply-add with -1 (deq * -1 is
//   exact, so it rounds once, like the subtraction).  No multiply is followed
//   by a plain subtract that could be contracted into one rounding.
//   MXFP4: the product with 2^e is exact, so h - e2m1 * 2^e is one packed fused
//   multiply-add.
template <int FMT>
__device__ __forceinline__ void sub_deq8(float* h, uint32_t c, uint32_t sh, float sv, float g) {
  uint32_t e2[4];
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\tmov.b32 {t0, t1, t2, t3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t0;\n\tcvt.rn.f16x2.e2m1x2 %1, t1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, t2;\n\tcvt.rn.f16x2.e2m1x2 %3, t3;\n\t}"
      : "=r"(e2[0]), "=r"(e2[1]), "=r"(e2[2]), "=r"(e2[3])
      : "r"(c));
#pragma unroll
  for (int b = 0; b < 4; b++) {
    float d0, d1;
    if constexpr (FMT == FMT_NV) {
      asm("{\n\t.reg .f16 a0, a1, s0, s1;\n\tmov.b32 {a0, a1}, %2;\n\tmov.b32 {s0, s1}, %3;\n\t"
          "fma.rn.f32.f16 %0, a0, s0, %4;\n\tfma.rn.f32.f16 %1, a1, s0, %4;\n\t}"
          : "=f"(d0), "=f"(d1)
          : "r"(e2[b]), "r"(sh), "f"(-0.0f));
      mul2(d0, d1, g, g);
      fma2(d0, d1, -1.0f, -1.0f, h[2 * b], h[2 * b + 1]);
    } else {
      asm("{\n\t.reg .f16 a0, a1, one;\n\tmov.b32 {a0, a1}, %2;\n\tmov.b16 one, 0x3C00;\n\t"
          "fma.rn.f32.f16 %0, a0, one, %3;\n\tfma.rn.f32.f16 %1, a1, one, %3;\n\t}"
          : "=f"(d0), "=f"(d1)
          : "r"(e2[b]), "f"(-0.0f));
      fma2(d0, d1, -sv, -sv, h[2 * b], h[2 * b + 1]);
    }
    h[2 * b] = d0;
    h[2 * b + 1] = d1;
  }
}

// One unit of 32 values: mask, backbone quantization, residual (in place in
// h) and residual quantization.  Outputs: meta bits, backbone codes (k/2 kept
// codes: 2 words; 8:16 dense layout: 4 words) and scale, residual codes (4
// words) and scales.  The backbone is quantized in its expanded form (codes
// of dropped positions masked to +0), so R = h - deq needs no selects.
template <int FMT, int PAT>
__device__ __forceinline__ void quantize_unit(float (&h)[32], float g_enc, float g_dec, const float* inv_tab,
                                              uint32_t& meta, uint32_t (&bc)[4], uint32_t& bsc, uint32_t (&rc)[4],
                                              uint32_t& rsc0, uint32_t& rsc1) {
  uint32_t keepw[4];  // nibble mask of kept elements, per 8 elements
  meta = 0;
  float bamax = 0.0f;
  if constexpr (PAT == PAT_48P) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const float* hg = h + 8 * g;
      const float s0 = fmaxf(fabsf(hg[0]), fabsf(hg[1])), s1 = fmaxf(fabsf(hg[2]), fabsf(hg[3]));
      const float s2 = fmaxf(fabsf(hg[4]), fabsf(hg[5])), s3 = fmaxf(fabsf(hg[6]), fabsf(hg[7]));
      bamax = fmaxf(bamax, fmaxf(fmaxf(s0, s1), fmaxf(s2, s3)));
      uint32_t kk[4];
      top2of4_masks(s0, s1, s2, s3, kk);
      meta |= kept_nibble(kk) << (4 * g);
      keepw[g] = (kk[0] & 0x000000FFu) | (kk[1] & 0x0000FF00u) | (kk[2] & 0x00FF0000u) | (kk[3] & 0xFF000000u);
    }
  } else if constexpr (PAT == PAT_816P) {
    // the top 8 of each group of 16, then in each group of 8 the two pairs that
    // hold most of them, ranked by (count, larger magnitude, lower index): keys
    // count << 32 | bits of the magnitude (non-negative floats order as their bits)
    uint32_t m16;
    const uint32_t keep16 = unit_mask<PAT_816>(h, m16);
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const float* hg = h + 8 * g;
      float sp[4];
      uint64_t key[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        sp[q] = fmaxf(fabsf(hg[2 * q]), fabsf(hg[2 * q + 1]));
        const uint32_t cnt = __popc((keep16 >> (8 * g + 2 * q)) & 3u);
        key[q] = ((uint64_t)cnt << 32) | __float_as_uint(sp[q]);
      }
      // pair p is kept iff it wins at least two of its three comparisons
      // (against a lower pair on a strictly larger key, a higher pair on >=)
      uint32_t kk[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        int wins = 0;
#pragma unroll
        for (int o = 0; o < 4; o++)
          if (o != q) wins += (o < q) ? (key[q] > key[o]) : (key[q] >= key[o]);
        kk[q] = wins >= 2 ? 0xFFFFFFFFu : 0u;
      }
      // the backbone block amax is over the kept values (the group maximum may be dropped)
#pragma unroll
      for (int q = 0; q < 4; q++) bamax = fmaxf(bamax, __uint_as_float(__float_as_uint(sp[q]) & kk[q]));
      meta |= kept_nibble(kk) << (4 * g);
      keepw[g] = (kk[0] & 0x000000FFu) | (kk[1] & 0x0000FF00u) | (kk[2] & 0x00FF0000u) | (kk[3] & 0xFF000000u);
    }
  } else if constexpr (PAT == PAT_24) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
      uint32_t k8 = 0;
#pragma unroll
      for (int q = 0; q < 2; q++) {
        const float* hq = h + 8 * g + 4 * q;
        const float a0 = fabsf(hq[0]), a1 = fabsf(hq[1]), a2 = fabsf(hq[2]), a3 = fabsf(hq[3]);
        bamax = fmaxf(bamax, fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)));
        const uint32_t kg = top2of4(a0, a1, a2, a3);
        meta |= pair_nibble(kg) << (4 * (2 * g + q));
        k8 |= kg << (4 * q);
      }
      keepw[g] = nibble_mask8(k8);
    }
  } else {
    const uint32_t keep = unit_mask<PAT_816>(h, meta);
#pragma unroll
    for (int i = 0; i < 32; i++) bamax = fmaxf(bamax, fabsf(h[i]));
#pragma unroll
    for (int g = 0; g < 4; g++) keepw[g] = nibble_spread8((keep >> (8 * g)) & 0xFFu);
  }
  // the group maximum is always kept, so the backbone block amax is the window amax
  if constexpr (FMT == FMT_MX) bamax = fmaxf(bamax, __shfl_xor_sync(0xffffffffu, bamax, 1));
  float bmul, bsv;
  uint32_t bsh;
  bsc = block_scale<FMT>(bamax, g_enc, inv_tab, bmul, bsv, bsh);

  // backbone codes in expanded form; dropped positions -> +0
  uint32_t cw[4];
#pragma unroll
  for (int g = 0; g < 4; g++) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      q[i] = h[8 * g + i];
      q[i + 1] = h[8 * g + i + 1];
      mul2(q[i], q[i + 1], bmul, bmul);
    }
    cw[g] = (bmul == 0.0f ? 0u : cvt_e2m1x8(q)) & keepw[g];
  }
  // residual R = h - deq(backbone) (deq = +0 where dropped: R = h exactly)
#pragma unroll
  for (int g = 0; g < 4; g++) sub_deq8<FMT>(h + 8 * g, cw[g], bsh, bsv, g_dec);
  // compaction of the kept codes (K order) for storage
  if constexpr (pair_layout(PAT)) {
    uint32_t half[4];
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const uint32_t nib = (meta >> (4 * g)) & 15u;
      half[g] = compact_pairs(cw[g], nib & 3u, nib >> 2);
    }
    bc[0] = half[0] | (half[1] << 16);
    bc[1] = half[2] | (half[3] << 16);
    bc[2] = bc[3] = 0;
  } else if constexpr (PAT == PAT_24) {
    // per quad: two kept nibbles i0 < i1 -> one byte
    uint32_t byte8[8];
#pragma unroll
    for (int q = 0; q < 8; q++) {
      const uint32_t nib = (meta >> (4 * q)) & 15u;
      const uint32_t quad = (cw[q >> 1] >> (16 * (q & 1))) & 0xFFFFu;
      const uint32_t c0 = (quad >> (4 * (nib & 3u))) & 15u, c1 = (quad >> (4 * (nib >> 2))) & 15u;
      byte8[q] = c0 | (c1 << 4);
    }
    bc[0] = byte8[0] | (byte8[1] << 8) | (byte8[2] << 16) | (byte8[3] << 24);
    bc[1] = byte8[4] | (byte8[5] << 8) | (byte8[6] << 16) | (byte8[7] << 24);
    bc[2] = bc[3] = 0;
  } else {
#pragma unroll
    for (int g = 0; g < 4; g++) bc[g] = cw[g];
  }

  // residual quantization
  if constexpr (FMT == FMT_NV) {
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) a0 = fmaxf(a0, fabsf(h[i]));
#pragma unroll
    for (int i = 16; i < 32; i++) a1 = fmaxf(a1, fabsf(h[i]));
    float m0, m1, sv0, sv1;
    rsc0 = block_scale<FMT>(a0, g_enc, inv_tab, m0, sv0);
    rsc1 = block_scale<FMT>(a1, g_enc, inv_tab, m1, sv1);
#pragma unroll
    for (int w = 0; w < 4; w++) {
      const float mm = w < 2 ? m0 : m1;
      float q[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        q[i] = h[8 * w + i];
        q[i + 1] = h[8 * w + i + 1];
        mul2(q[i], q[i + 1], mm, mm);
      }
      rc[w] = mm == 0.0f ? 0u : cvt_e2m1x8(q);
    }
  } else {
    float a0 = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i++) a0 = fmaxf(a0, fabsf(h[i]));
    float m0, sv0;
    rsc0 = block_scale<FMT>(a0, g_enc, inv_tab, m0, sv0);
    rsc1 = 0;
#pragma unroll
    for (int w = 0; w < 4; w++) {
      float q[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        q[i] = h[8 * w + i];
        q[i + 1] = h[8 * w + i + 1];
        mul2(q[i], q[i + 1], m0, m0);
      }
      rc[w] = cvt_e2m1x8(q);
    }
  }
}

// Writes one unit's outputs (row r, unit u) in the documented layouts.
template <int FMT, int PAT>
__device__ __forceinline__ void store_unit(const PrepParams& p, int64_t r, int u, int64_t s_bb, int64_t s_res,
                                           uint32_t meta, const uint32_t (&bc)[4], uint32_t bsc,
                                           const uint32_t (&rc)[4], uint32_t rsc0, uint32_t rsc1) {
  const int64_t k = p.k;
  if constexpr (pair_layout(PAT)) {
    *reinterpret_cast<uint16_t*>(p.meta + r * (k / 16) + 2 * u) = (uint16_t)meta;
  } else {
    *reinterpret_cast<uint32_t*>(p.meta + r * (k / 8) + 4 * u) = meta;
  }
  if constexpr (PAT == PAT_816) {
    *reinterpret_cast<uint4*>(p.bb_codes + r * (k / 2) + 16 * u) = make_uint4(bc[0], bc[1], bc[2], bc[3]);
  } else {
    *reinterpret_cast<uint2*>(p.bb_codes + r * (k / 4) + 8 * u) = make_uint2(bc[0], bc[1]);
  }
  *reinterpret_cast<uint4*>(p.res_codes + r * (k / 2) + 16 * u) = make_uint4(rc[0], rc[1], rc[2], rc[3]);
  if constexpr (FMT == FMT_NV) {
    if constexpr (PAT == PAT_816) {
      *reinterpret_cast<uint16_t*>(p.bb_scales + tiled_sf_offset(r, 2 * u, s_bb)) = (uint16_t)(bsc | (bsc << 8));
    } else {
      p.bb_scales[tiled_sf_offset(r, u, s_bb)] = (uint8_t)bsc;
    }
    *reinterpret_cast<uint16_t*>(p.res_scales + tiled_sf_offset(r, 2 * u, s_res)) = (uint16_t)(rsc0 | (rsc1 << 8));
  } else {
    if constexpr (PAT == PAT_816) {
      p.bb_scales[tiled_sf_offset(r, u, s_bb)] = (uint8_t)bsc;
    } else {
      if ((u & 1) == 0) p.bb_scales[tiled_sf_offset(r, u >> 1, s_bb)] = (uint8_t)bsc;
    }
    p.res_scales[tiled_sf_offset(r, u, s_res)] = (uint8_t)rsc0;
  }
}

template <int FMT, int PAT, bool NORM, bool XBF16, bool ACT = false>
__global__ void __launch_bounds__(128, ACT ? 6 : 7) prep_kernel(PrepParams p) {
  static_assert(!(NORM && ACT), "the SwiGLU form has no RMSNorm");
  __shared__ float inv_tab[128];
  __shared__ float red[32 * 16];
  const int64_t k = p.k;
  const RowMap m = row_map(k, p.tpr);
  const int rpb = 128 / m.tpr;
  const int row_in_block = threadIdx.x >> m.lg, tt = threadIdx.x & (m.tpr - 1);
  grid_dep_wait();    // the amax pass (or whatever wrote x) has completed
  grid_dep_launch();  // the GEMM may be scheduled; it waits for this grid in turn
  float g_enc = 1.0f, g_dec = 1.0f;
  if constexpr (FMT == FMT_NV) {
    const float amax = p.act_amax > 0.0f ? p.act_amax : *reinterpret_cast<volatile const float*>(p.tensor);
    tensor_scales(amax, g_enc, g_dec);
    fill_inv_table(inv_tab, g_enc);
    __syncthreads();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      p.tensor[0] = amax;
      p.tensor[1] = g_enc;
      p.tensor[2] = g_dec;
    }
  } else if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.tensor[0] = 0.0f;
    p.tensor[1] = 1.0f;
    p.tensor[2] = 1.0f;
  }
  const int b = FMT == FMT_NV ? 16 : 32;
  const int64_t s_res = k / b;
  const int64_t s_bb = PAT == PAT_816 ? k / b : k / (2 * b);

  for (int64_t r0 = (int64_t)blockIdx.x * rpb; r0 < p.t_pad; r0 += (int64_t)gridDim.x * rpb) {
    const int64_t r = r0 + row_in_block;
    const bool in_pad = r < p.t_pad;
    const bool real = r < p.t;
    const int64_t off = r * k;
    float rs = 1.0f;
    if constexpr (NORM) {
      if (p.rstd) rs = real ? __ldg(p.rstd + r) : 1.0f;  // row statistics from the amax pass
      else rs = rstd_from_sumsq(row_sumsq<XBF16>(p.x, off, real, m, tt, row_in_block, red), k, p.eps);
    }

    for (int j = 0; j < m.nj; j++) {
      const int u = tt + m.tpr * j;
      const bool active = u < m.units;
      float h[32];
      if (real && active) {
        if constexpr (ACT) swiglu_unit<XBF16>(p.x, p.x2, off + (int64_t)u * 32, h);
        else load_unit<XBF16>(p.x, off + (int64_t)u * 32, h);
        if constexpr (NORM) {
          float g[32];
          load_unit<XBF16>(p.gamma, (int64_t)u * 32, g);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            mul2(h[i], h[i + 1], rs, rs);
            mul2(h[i], h[i + 1], g[i], g[i + 1]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; i++) h[i] = 0.0f;
      }
      uint32_t meta, bc[4], bsc, rc[4], rsc0, rsc1;
      quantize_unit<FMT, PAT>(h, g_enc, g_dec, inv_tab, meta, bc, bsc, rc, rsc0, rsc1);
      if (!active || !in_pad) continue;

      store_unit<FMT, PAT>(p, r, u, s_bb, s_res, meta, bc, bsc, rc, rsc0, rsc1);
    }
  }
}

// --------------------------------------------------------- row gather
// Prepared activations laid out again by row: destination row r takes source
// row rows[r] (r < t) -- metadata, backbone and residual codes as contiguous
// row segments (16-byte copies), the tiled scales as 32-bit words of four
// scales -- or, for rows[r] < 0 and for the padding rows t..t_pad-1, the
// encoding of an all-zero input row: no element beats another, so the mask
// keeps the first N of every group (nibble i0 | i1 << 2 = 4 for 2:4 and the
// 4:8 pair, mask 0x00FF for 8:16), and every code and scale is 0.
struct GatherParams {
  const uint8_t *s_meta, *s_bbc, *s_bbs, *s_rc, *s_rs;
  uint8_t *d_meta, *d_bbc, *d_bbs, *d_rc, *d_rs;
  const int32_t* rows;
  int64_t src_t, t, t_pad;
  int64_t meta_row, bbc_row, rc_row;  // bytes per row
  int64_t bbs_per_row, rs_per_row;    // scales per row (multiples of 4)
  uint32_t zero_meta;                 // 4 bytes of the zero row's metadata
};

__global__ void __launch_bounds__(256) gather_rows_kernel(const GatherParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  grid_dep_wait();
  grid_dep_launch();
  if (r >= p.t_pad) return;
  int64_t src = r < p.t ? (int64_t)__ldg(p.rows + r) : -1;
  if (src >= p.src_t) src = -1;  // out of range: treated as a zero row (the host checks nothing on the device data)
  auto seg = [&](const uint8_t* sb, uint8_t* db, int64_t row_bytes, uint32_t fill) {
    uint4* d = reinterpret_cast<uint4*>(db + r * row_bytes);
    const int64_t n = row_bytes / 16;
    if (src >= 0) {
      const uint4* s4 = reinterpret_cast<const uint4*>(sb + src * row_bytes);
      for (int64_t i = lane; i < n; i += 32) d[i] = __ldg(s4 + i);
    } else {
      for (int64_t i = lane; i < n; i += 32) d[i] = make_uint4(fill, fill, fill, fill);
    }
  };
  seg(p.s_meta, p.d_meta, p.meta_row, p.zero_meta);
  seg(p.s_bbc, p.d_bbc, p.bbc_row, 0u);
  seg(p.s_rc, p.d_rc, p.rc_row, 0u);
  auto scales = [&](const uint8_t* sb, uint8_t* db, int64_t per_row) {
    for (int64_t s4 = lane; s4 < per_row / 4; s4 += 32) {
      const uint32_t v = src >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(sb + tiled_sf_offset(src, 4 * s4, per_row))) : 0u;
      *reinterpret_cast<uint32_t*>(db + tiled_sf_offset(r, 4 * s4, per_row)) = v;
    }
  };
  scales(p.s_bbs, p.d_bbs, p.bbs_per_row);
  scales(p.s_rs, p.d_rs, p.rs_per_row);
}

// --------------------------------------------------------- weight kernel
// One thread quantizes 32 consecutive K values of a weight row; a scale block
// is 2b logical K (NVFP4: this unit; MXFP4: the unit and its neighbour lane).
struct WeightParams {
  const void* w;
  int64_t n, k, rows;  // rows = experts * n
  uint8_t* codes;
  uint8_t* sf_dense;
  uint8_t* sf_sparse;
  float* tensor;  // experts * 3, amax already folded into tensor[3e]
};

template <int FMT, bool XBF16>
__global__ void __launch_bounds__(256) weight_kernel(WeightParams p) {
  const int64_t units_per_row = p.k / 32;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t r = gid / units_per_row;
  const int64_t u = gid % units_per_row;
  const bool active = r < p.rows;
  const int64_t rr = active ? r : 0;
  const int64_t e = rr / p.n, rl = rr % p.n;
  float v[32];
  if (active) load_unit<XBF16>(p.w, rr * p.k + u * 32, v);
  else {
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = 0.0f;
  }
  float g_enc = 1.0f, g_dec = 1.0f;
  if constexpr (FMT == FMT_NV) tensor_scales(__ldg(p.tensor + 3 * e), g_enc, g_dec);
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
  if constexpr (FMT == FMT_MX) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  uint32_t codes[4];
  uint32_t sc;
  float mul;
  if constexpr (FMT == FMT_MX) {
    const int e = mx_exponent(amax);
    sc = (uint32_t)(e + 127);
    mul = pow2f(-e);
  } else {
    sc = cvt_e4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), g_enc));
    const float sv = e4m3_value(sc);
    mul = sv == 0.0f ? 0.0f : __fdiv_rn(g_enc, sv);
  }
#pragma unroll
  for (int w = 0; w < 4; w++) codes[w] = quant8(v + 8 * w, mul);
  if (!active) return;
  if (u == 0 && rl == 0) {
    p.tensor[3 * e + 1] = g_enc;
    p.tensor[3 * e + 2] = g_dec;
  }
  *reinterpret_cast<uint4*>(p.codes + rr * (p.k / 2) + 16 * u) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  const int b = (FMT == FMT_NV) ? 16 : 32;
  const int64_t Sd = p.k / b, Ss = p.k / (2 * b);
  uint8_t* sfd = p.sf_dense + e * tiled_sf_bytes(p.n, Sd);
  uint8_t* sfs = p.sf_sparse + e * tiled_sf_bytes(p.n, Ss);
  if constexpr (FMT == FMT_NV) {
    *reinterpret_cast<uint16_t*>(sfd + tiled_sf_offset(rl, 2 * u, Sd)) = (uint16_t)(sc | (sc << 8));
    sfs[tiled_sf_offset(rl, u, Ss)] = (uint8_t)sc;
  } else {
    sfd[tiled_sf_offset(rl, u, Sd)] = (uint8_t)sc;
    if ((u & 1) == 0) sfs[tiled_sf_offset(rl, u >> 1, Ss)] = (uint8_t)sc;
  }
}

// Per-expert amax of the weight: one block per (expert, slice of rows).
template <bool XBF16>
__global__ void __launch_bounds__(256) weight_amax_kernel(const void* w, int64_t n, int64_t k, float* tensor,
                                                          int blocks_per_expert) {
  const int64_t e = blockIdx.x / blocks_per_expert;
  const int64_t part = blockIdx.x % blocks_per_expert;
  const int64_t units = n * k / 32;
  float m = 0.0f;
  for (int64_t i = part * blockDim.x + threadIdx.x; i < units; i += (int64_t)blocks_per_expert * blockDim.x) {
    float v[32];
    load_unit<XBF16>(w, e * n * k + i * 32, v);
#pragma unroll
    for (int j = 0; j < 32; j++) m = fmaxf(m, fabsf(v[j]));
  }
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = 0.0f;
    for (int i = 0; i < (int)(blockDim.x / 32); i++) mm = fmaxf(mm, wm[i]);
    atomicMax(reinterpret_cast<unsigned int*>(tensor + 3 * e), __float_as_uint(mm));
  }
}

}  // namespace sharq
