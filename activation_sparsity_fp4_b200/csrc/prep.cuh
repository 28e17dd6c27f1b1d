// prep.cuh -- fused SharQ preprocessing and weight quantization for sm_100a.
//
// SharQ (arXiv 2606.26587) abstract / Section 1: per activation row, an online
// N:M mask extracts an outlier-dominated sparse backbone that is quantized to
// FP4; the dense residual is taken against the QUANTIZED backbone and quantized
// to FP4 as well; "a fused preprocessing kernel absorbs mask generation,
// residual construction and layer normalization into one operator".
//
// Work split: one thread owns 32 consecutive K elements of one row (one
// "unit"): 4 x 16-byte loads of bf16 (8 for fp32).  For NVFP4 a unit is exactly
// one backbone block (16 kept values) and two residual blocks; for MXFP4 a
// backbone block spans the two units of a lane pair (shuffle for its amax) and
// a residual block is one unit.  A row is handled by ceil(K/32) threads rounded
// up to whole warps; small K packs several rows into one block.  Every floating
// point step is an explicitly rounded fp32 op in a fixed order, so codes and
// scales are reproducible bit for bit.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace sharq {

enum { FMT_MX = 0, FMT_NV = 1 };
enum { PAT_24 = 0, PAT_48P = 1, PAT_816 = 2 };

// Byte offset of (row r, scale s) in the tiled scale layout with S scales per row.
__host__ __device__ __forceinline__ int64_t tiled_sf_offset(int64_t r, int64_t s, int64_t S) {
  const int64_t sblocks = (S + 3) >> 2;
  return ((r >> 7) * sblocks + (s >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (s & 3);
}
__host__ __device__ __forceinline__ int64_t tiled_sf_bytes(int64_t rows, int64_t S) {
  return ((rows + 127) / 128) * ((S + 3) / 4) * 512;
}

struct PrepParams {
  const void* x;
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

// Sum of squares of one row in the fixed order: 16-element chunk sums by
// sequential FMA, then a pairwise tree of adjacent chunks (levels 1..5 inside
// the warp by xor shuffles, the rest over the row's warps, zero padded).
// All threads of the block must call it.  red: per-block scratch [rows][32].
template <bool XBF16>
__device__ __forceinline__ float row_rstd(const float (&x)[32], bool active, float eps, int64_t k, float* red,
                                          int row_in_block, int warps_per_row) {
  float c0 = 0.0f, c1 = 0.0f;
  if (active) {
#pragma unroll
    for (int i = 0; i < 16; i++) c0 = __fmaf_rn(x[i], x[i], c0);
#pragma unroll
    for (int i = 16; i < 32; i++) c1 = __fmaf_rn(x[i], x[i], c1);
  }
  float s = __fadd_rn(c0, c1);
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, m));
  const int warp_in_row = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[row_in_block * 32 + warp_in_row] = s;
  __syncthreads();
  // adjacent-pair tree over the row's warp sums, zero padded to 16 leaves (a
  // larger zero padding than the minimal power of two adds only x + 0 = x)
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; i++) a[i] = (i < warps_per_row) ? red[row_in_block * 32 + i] : 0.0f;
#pragma unroll
  for (int w = 16; w > 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w / 2; i++) a[i] = __fadd_rn(a[2 * i], a[2 * i + 1]);
  const float mean = __fdiv_rn(a[0], (float)k);
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
}

// ------------------------------------------------------------------- mask
// keep bits (bit i = element i of the unit kept) and metadata for 32 values.
// Ranks: element i is kept iff fewer than N elements of its group beat it,
// where j beats i if |h_j| > |h_i|, or equal and j < i.
template <int PAT>
__device__ __forceinline__ uint32_t unit_mask(const float (&h)[32], uint32_t& meta) {
  uint32_t keep = 0;
  meta = 0;
  if constexpr (PAT == PAT_48P) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
      float sc[4];
#pragma unroll
      for (int p = 0; p < 4; p++) sc[p] = fmaxf(fabsf(h[8 * g + 2 * p]), fabsf(h[8 * g + 2 * p + 1]));
      uint32_t kp = 0;
#pragma unroll
      for (int p = 0; p < 4; p++) {
        int beat = 0;
#pragma unroll
        for (int q = 0; q < 4; q++) {
          if (q < p) beat += (sc[q] >= sc[p]) ? 1 : 0;
          if (q > p) beat += (sc[q] > sc[p]) ? 1 : 0;
        }
        kp |= (beat < 2 ? 1u : 0u) << p;
      }
      // kept pair indices p0 < p1
      const int p0 = __ffs(kp) - 1;
      const int p1 = 31 - __clz(kp);
      meta |= (uint32_t)(p0 | (p1 << 2)) << (4 * g);
      keep |= (3u << (8 * g + 2 * p0)) | (3u << (8 * g + 2 * p1));
    }
  } else if constexpr (PAT == PAT_24) {
#pragma unroll
    for (int g = 0; g < 8; g++) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = fabsf(h[4 * g + i]);
      uint32_t kg = 0;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        int beat = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
          if (j < i) beat += (a[j] >= a[i]) ? 1 : 0;
          if (j > i) beat += (a[j] > a[i]) ? 1 : 0;
        }
        kg |= (beat < 2 ? 1u : 0u) << i;
      }
      const int i0 = __ffs(kg) - 1;
      const int i1 = 31 - __clz(kg);
      meta |= (uint32_t)(i0 | (i1 << 2)) << (4 * g);
      keep |= kg << (4 * g);
    }
  } else {
#pragma unroll
    for (int g = 0; g < 2; g++) {
      uint32_t kg = 0;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        const float ai = fabsf(h[16 * g + i]);
        int beat = 0;
#pragma unroll
        for (int j = 0; j < 16; j++) {
          const float aj = fabsf(h[16 * g + j]);
          if (j < i) beat += (aj >= ai) ? 1 : 0;
          if (j > i) beat += (aj > ai) ? 1 : 0;
        }
        kg |= (beat < 8 ? 1u : 0u) << i;
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

// Quantize n (multiple of 8) values with one scale: writes packed codes
// (n/8 words) and the dequantized values (with g_dec); returns the scale code.
template <int FMT, int N>
__device__ __forceinline__ uint32_t quant_block(const float* v, float amax, float g_enc, float g_dec,
                                                uint32_t* codes, float* deq) {
  float q[N];
  uint32_t sc;
  if constexpr (FMT == FMT_MX) {
    const int e = mx_exponent(amax);
    sc = (uint32_t)(e + 127);
    const float mul = pow2f(-e);
    const float dsc = pow2f(e);
#pragma unroll
    for (int i = 0; i < N; i++) q[i] = __fmul_rn(v[i], mul);
#pragma unroll
    for (int w = 0; w < N / 8; w++) codes[w] = cvt_e2m1x8(q + 8 * w);
#pragma unroll
    for (int i = 0; i < N; i++) deq[i] = __fmul_rn(e2m1_value((codes[i / 8] >> (4 * (i % 8))) & 15), dsc);
  } else {
    const float s32 = __fmul_rn(__fdiv_rn(amax, 6.0f), g_enc);
    sc = cvt_e4m3(s32);
    const float sv = e4m3_value(sc);
    if (sv == 0.0f) {
#pragma unroll
      for (int w = 0; w < N / 8; w++) codes[w] = 0;
#pragma unroll
      for (int i = 0; i < N; i++) deq[i] = 0.0f;
    } else {
      const float inv = __fdiv_rn(g_enc, sv);
#pragma unroll
      for (int i = 0; i < N; i++) q[i] = __fmul_rn(v[i], inv);
#pragma unroll
      for (int w = 0; w < N / 8; w++) codes[w] = cvt_e2m1x8(q + 8 * w);
#pragma unroll
      for (int i = 0; i < N; i++)
        deq[i] = __fmul_rn(__fmul_rn(e2m1_value((codes[i / 8] >> (4 * (i % 8))) & 15), sv), g_dec);
    }
  }
  return sc;
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

// ------------------------------------------------------------ amax kernel
// max |h| over all rows, atomically folded into tensor[0] (zeroed beforehand).
// Grid-stride over row groups so that only one atomic per block is issued.
template <bool NORM, bool XBF16>
__global__ void __launch_bounds__(512) amax_kernel(const void* x, const void* gamma, float eps, int64_t t, int64_t k,
                                                   float* out, int rows_per_block, int threads_per_row) {
  __shared__ float red[16 * 32];
  __shared__ float bmax[16];
  const int row_in_block = threadIdx.y;
  const int u = threadIdx.x;
  const int units = (int)(k / 32);
  const bool in_row = u < units;
  const int warps_per_row = threads_per_row / 32;
  float my = 0.0f;
  for (int64_t r0 = (int64_t)blockIdx.x * rows_per_block; r0 < t; r0 += (int64_t)gridDim.x * rows_per_block) {
    const int64_t r = r0 + row_in_block;
    const bool active = in_row && r < t;
    float v[32];
    if (active) load_unit<XBF16>(x, r * k + (int64_t)u * 32, v);
    else {
#pragma unroll
      for (int i = 0; i < 32; i++) v[i] = 0.0f;
    }
    if constexpr (NORM) {
      const float rs = row_rstd<XBF16>(v, active, eps, k, red, row_in_block, warps_per_row);
      float g[32];
      if (active) load_unit<XBF16>(gamma, (int64_t)u * 32, g);
#pragma unroll
      for (int i = 0; i < 32; i++) v[i] = active ? __fmul_rn(__fmul_rn(v[i], rs), g[i]) : 0.0f;
      __syncthreads();  // red[] is reused by the next row group
    }
#pragma unroll
    for (int i = 0; i < 32; i++) my = fmaxf(my, fabsf(v[i]));
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, m));
  const int tid = threadIdx.y * blockDim.x + threadIdx.x;
  if ((tid & 31) == 0) bmax[tid >> 5] = my;
  __syncthreads();
  if (tid == 0) {
    float m = 0.0f;
    const int nw = (blockDim.x * blockDim.y) / 32;
    for (int i = 0; i < nw; i++) m = fmaxf(m, bmax[i]);
    atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(m));
  }
}

// ------------------------------------------------------------ prep kernel
template <int FMT, int PAT, bool NORM, bool XBF16>
__global__ void __launch_bounds__(512) prep_kernel(PrepParams p, int rows_per_block, int threads_per_row) {
  __shared__ float red[16 * 32];
  const int row_in_block = threadIdx.y;
  const int u = threadIdx.x;  // unit index in the row
  const int64_t k = p.k;
  const int units = (int)(k / 32);
  const int64_t r = (int64_t)blockIdx.x * rows_per_block + row_in_block;
  const bool in_row = u < units;
  const bool real = in_row && r < p.t;        // a row of the input
  const bool store = in_row && r < p.t_pad;   // padding rows are written as zero input

  float h[32];
  if (real) load_unit<XBF16>(p.x, r * k + (int64_t)u * 32, h);
  else {
#pragma unroll
    for (int i = 0; i < 32; i++) h[i] = 0.0f;
  }
  if constexpr (NORM) {
    const float rs = row_rstd<XBF16>(h, real, p.eps, k, red, row_in_block, threads_per_row / 32);
    float g[32];
    if (real) load_unit<XBF16>(p.gamma, (int64_t)u * 32, g);
#pragma unroll
    for (int i = 0; i < 32; i++) h[i] = real ? __fmul_rn(__fmul_rn(h[i], rs), g[i]) : 0.0f;
  }

  float g_enc = 1.0f, g_dec = 1.0f;
  if constexpr (FMT == FMT_NV) {
    const float amax = p.act_amax > 0.0f ? p.act_amax : *reinterpret_cast<volatile const float*>(p.tensor);
    tensor_scales(amax, g_enc, g_dec);
    if (blockIdx.x == 0 && threadIdx.x == 0 && threadIdx.y == 0) {
      p.tensor[0] = amax;
      p.tensor[1] = g_enc;
      p.tensor[2] = g_dec;
    }
  } else {
    if (blockIdx.x == 0 && threadIdx.x == 0 && threadIdx.y == 0) {
      p.tensor[0] = 0.0f;
      p.tensor[1] = 1.0f;
      p.tensor[2] = 1.0f;
    }
  }

  // ---- mask
  uint32_t meta;
  const uint32_t keep = unit_mask<PAT>(h, meta);

  // ---- backbone: the 16 kept values in K order
  float kv[16];
  if constexpr (PAT == PAT_816) {
    int n = 0;
#pragma unroll
    for (int i = 0; i < 32; i++) {
      // compaction by running count: kept element i goes to slot (popc of keep below i)
      const bool kp = (keep >> i) & 1u;
      const int slot = __popc(keep & ((1u << i) - 1u));
#pragma unroll
      for (int s = 0; s < 16; s++)
        if (kp && slot == s) kv[s] = h[i];
      n += kp;
    }
    (void)n;
  } else if constexpr (PAT == PAT_48P) {
    // group g keeps pairs p0 < p1 (from the metadata nibble)
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const int p0 = (meta >> (4 * g)) & 3, p1 = (meta >> (4 * g + 2)) & 3;
      const float* hg = h + 8 * g;
      kv[4 * g + 0] = (p0 == 0) ? hg[0] : (p0 == 1) ? hg[2] : hg[4];
      kv[4 * g + 1] = (p0 == 0) ? hg[1] : (p0 == 1) ? hg[3] : hg[5];
      kv[4 * g + 2] = (p1 == 1) ? hg[2] : (p1 == 2) ? hg[4] : hg[6];
      kv[4 * g + 3] = (p1 == 1) ? hg[3] : (p1 == 2) ? hg[5] : hg[7];
    }
  } else {
    // 2:4 keeps elements i0 < i1 of every quad
#pragma unroll
    for (int q = 0; q < 8; q++) {
      const int i0 = (meta >> (4 * q)) & 3, i1 = (meta >> (4 * q + 2)) & 3;
      const float* hq = h + 4 * q;
      kv[2 * q] = (i0 == 0) ? hq[0] : (i0 == 1) ? hq[1] : hq[2];
      kv[2 * q + 1] = (i1 == 1) ? hq[1] : (i1 == 2) ? hq[2] : hq[3];
    }
  }
  float bamax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; i++) bamax = fmaxf(bamax, fabsf(kv[i]));
  if constexpr (FMT == FMT_MX) bamax = fmaxf(bamax, __shfl_xor_sync(0xffffffffu, bamax, 1));
  uint32_t bcodes[2];
  float bdeq[16];
  const uint32_t bsc = quant_block<FMT, 16>(kv, bamax, g_enc, g_dec, bcodes, bdeq);

  // ---- residual against the quantized backbone
  float res[32];
  if constexpr (PAT == PAT_816) {
#pragma unroll
    for (int i = 0; i < 32; i++) {
      const bool kp = (keep >> i) & 1u;
      const int slot = __popc(keep & ((1u << i) - 1u));
      float d = 0.0f;
#pragma unroll
      for (int s = 0; s < 16; s++)
        if (slot == s) d = bdeq[s];
      res[i] = kp ? __fsub_rn(h[i], d) : h[i];
    }
  } else if constexpr (PAT == PAT_48P) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const int p0 = (meta >> (4 * g)) & 3, p1 = (meta >> (4 * g + 2)) & 3;
#pragma unroll
      for (int p = 0; p < 4; p++)
#pragma unroll
        for (int j = 0; j < 2; j++) {
          const float hv = h[8 * g + 2 * p + j];
          res[8 * g + 2 * p + j] = (p == p0)   ? __fsub_rn(hv, bdeq[4 * g + j])
                                   : (p == p1) ? __fsub_rn(hv, bdeq[4 * g + 2 + j])
                                               : hv;
        }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; q++) {
      const int i0 = (meta >> (4 * q)) & 3, i1 = (meta >> (4 * q + 2)) & 3;
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float hv = h[4 * q + j];
        res[4 * q + j] = (j == i0) ? __fsub_rn(hv, bdeq[2 * q]) : (j == i1) ? __fsub_rn(hv, bdeq[2 * q + 1]) : hv;
      }
    }
  }
  uint32_t rcodes[4];
  float rdeq[32];
  uint32_t rsc0, rsc1 = 0;
  if constexpr (FMT == FMT_NV) {
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) a0 = fmaxf(a0, fabsf(res[i]));
#pragma unroll
    for (int i = 16; i < 32; i++) a1 = fmaxf(a1, fabsf(res[i]));
    rsc0 = quant_block<FMT, 16>(res, a0, g_enc, g_dec, rcodes, rdeq);
    rsc1 = quant_block<FMT, 16>(res + 16, a1, g_enc, g_dec, rcodes + 2, rdeq + 16);
  } else {
    float a0 = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i++) a0 = fmaxf(a0, fabsf(res[i]));
    rsc0 = quant_block<FMT, 32>(res, a0, g_enc, g_dec, rcodes, rdeq);
  }

  if (!store) return;
  // ---- stores
  const int64_t K = k;
  if constexpr (PAT == PAT_48P) {
    *reinterpret_cast<uint16_t*>(p.meta + r * (K / 16) + 2 * u) = (uint16_t)meta;
  } else {
    *reinterpret_cast<uint32_t*>(p.meta + r * (K / 8) + 4 * u) = meta;
  }
  if constexpr (PAT == PAT_816) {
    // dense layout: code of kept element i at position i, 0 elsewhere
    uint32_t dense[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 32; i++) {
      const bool kp = (keep >> i) & 1u;
      const int slot = __popc(keep & ((1u << i) - 1u));
      const uint32_t c = (bcodes[slot >> 3] >> (4 * (slot & 7))) & 15u;
      dense[i >> 3] |= (kp ? c : 0u) << (4 * (i & 7));
    }
    *reinterpret_cast<uint4*>(p.bb_codes + r * (K / 2) + 16 * u) = make_uint4(dense[0], dense[1], dense[2], dense[3]);
  } else {
    *reinterpret_cast<uint2*>(p.bb_codes + r * (K / 4) + 8 * u) = make_uint2(bcodes[0], bcodes[1]);
  }
  *reinterpret_cast<uint4*>(p.res_codes + r * (K / 2) + 16 * u) = make_uint4(rcodes[0], rcodes[1], rcodes[2], rcodes[3]);

  if constexpr (FMT == FMT_NV) {
    // backbone: one scale per 16 kept values (32 logical); 8:16 stores the dense view twice
    if constexpr (PAT == PAT_816) {
      const int64_t S = K / 16;
      *reinterpret_cast<uint16_t*>(p.bb_scales + tiled_sf_offset(r, 2 * u, S)) = (uint16_t)(bsc | (bsc << 8));
    } else {
      p.bb_scales[tiled_sf_offset(r, u, K / 32)] = (uint8_t)bsc;
    }
    *reinterpret_cast<uint16_t*>(p.res_scales + tiled_sf_offset(r, 2 * u, K / 16)) = (uint16_t)(rsc0 | (rsc1 << 8));
  } else {
    if constexpr (PAT == PAT_816) {
      p.bb_scales[tiled_sf_offset(r, u, K / 32)] = (uint8_t)bsc;
    } else {
      if ((u & 1) == 0) p.bb_scales[tiled_sf_offset(r, u >> 1, K / 64)] = (uint8_t)bsc;
    }
    p.res_scales[tiled_sf_offset(r, u, K / 32)] = (uint8_t)rsc0;
  }
}

// Zero the tiled-scale padding that no thread writes (rows >= t_pad in the last
// 128-row block and scale columns beyond S in the last 4-column block).
__global__ void zero_bytes_kernel(uint8_t* p, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = 0;
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
  float deq[32];
  const uint32_t sc = quant_block<FMT, 32>(v, amax, g_enc, g_dec, codes, deq);
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
