// gemv.cuh -- the layer's two products for a handful of rows (decode).
//
// SharQ abstract and Section 1: y = g_dec(x) * g_dec(w) * sum_k (B + R)[t][k] * W[n][k],
// the sparse backbone product plus the dense residual product into one output,
// both reading the one FP4 weight.  With at most kGemvMaxRows rows the work is
// a weight stream (N*K/2 bytes of codes) with a few multiply-adds per byte, so
// it runs on the CUDA cores, bound by HBM: a 128-row tensor-core tile would be
// at least 97 % padding and its K loop latency bound.
//
// Each block first decodes the rows' backbone and residual (codes, metadata and
// block scales, without the tensor scale) for one K chunk into shared memory as
// fp32 B + R; then every warp streams four weight rows at a time along K (lane
// l takes 32-element units l, l+32, ...), multiplies the E2M1 values of a unit
// by the decoded rows, scales the unit's sum by its weight block scale and
// accumulates.  Lanes are summed by shuffles at the end.  The summation order
// differs from the tensor cores' (the tolerance of the GEMM applies).
#pragma once
#include <cuda_bf16.h>

#include "prep.cuh"

namespace sharq {

constexpr int kGemvMaxRows = 4;
constexpr int kGemvChunk = 2048;       // logical K per shared-memory chunk of decoded rows
constexpr int kGemvWarps = 4;          // warps per block
constexpr int kGemvRowsPerWarp = 2;    // weight rows a warp streams together

struct GemvParams {
  int64_t n, k;
  int paths;             // bit 0 backbone, bit 1 residual
  const uint8_t *meta, *bb_codes, *bb_scales, *res_codes, *res_scales;
  int64_t t_pad;         // rows of the prepared buffers (tiled scale layout)
  const float* tensor_x;
  const uint8_t* w_codes;   // [n][k / 2]
  const uint8_t* w_sf;      // weight scales, sparse view (one per 2b logical K), tiled
  const float* tensor_w;
  void* y;
  int y_bf16;
};

template <int FMT>
__device__ __forceinline__ float scale_value(uint32_t c) {
  if constexpr (FMT == FMT_MX) return c ? __uint_as_float(c << 23) : __uint_as_float(0x00400000u);
  else return e4m3_value(c);
}

// Decoded B + R (without tensor scale) of unit u (32 logical elements) of row r.
template <int FMT, int PAT>
__device__ __forceinline__ void gemv_decode_unit(const GemvParams& p, int r, int64_t u, float (&v)[32]) {
  constexpr int b = FMT == FMT_NV ? 16 : 32;
  const int64_t k = p.k;
#pragma unroll
  for (int i = 0; i < 32; i++) v[i] = 0.0f;
  if (p.paths & 2) {  // residual: 32 codes, scales per b
    const uint4 c4 = *reinterpret_cast<const uint4*>(p.res_codes + (int64_t)r * (k / 2) + 16 * u);
    const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
    const int64_t S = k / b;
    const float s0 = scale_value<FMT>(p.res_scales[tiled_sf_offset(r, FMT == FMT_NV ? 2 * u : u, S)]);
    const float s1 = FMT == FMT_NV ? scale_value<FMT>(p.res_scales[tiled_sf_offset(r, 2 * u + 1, S)]) : s0;
#pragma unroll
    for (int q = 0; q < 4; q++) {
      float d[8];
      e2m1x8_values(cw[q], d);
#pragma unroll
      for (int i = 0; i < 8; i++) v[8 * q + i] = __fmul_rn(d[i], q < 2 ? s0 : s1);
    }
  }
  if (p.paths & 1) {
    float bv[32];
    if constexpr (PAT == PAT_816) {  // dense backbone, dense-view scales per b
      const uint4 c4 = *reinterpret_cast<const uint4*>(p.bb_codes + (int64_t)r * (k / 2) + 16 * u);
      const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
      const int64_t S = k / b;
      const float s0 = scale_value<FMT>(p.bb_scales[tiled_sf_offset(r, FMT == FMT_NV ? 2 * u : u, S)]);
      const float s1 = FMT == FMT_NV ? scale_value<FMT>(p.bb_scales[tiled_sf_offset(r, 2 * u + 1, S)]) : s0;
#pragma unroll
      for (int q = 0; q < 4; q++) {
        float d[8];
        e2m1x8_values(cw[q], d);
#pragma unroll
        for (int i = 0; i < 8; i++) bv[8 * q + i] = __fmul_rn(d[i], q < 2 ? s0 : s1);
      }
    } else {  // 16 kept codes in K order, one sparse-view scale per 2b logical
      const uint2 c2 = *reinterpret_cast<const uint2*>(p.bb_codes + (int64_t)r * (k / 4) + 8 * u);
      const uint32_t cw[2] = {c2.x, c2.y};
      const int64_t S = k / (2 * b);
      const float s = scale_value<FMT>(p.bb_scales[tiled_sf_offset(r, FMT == FMT_NV ? u : u >> 1, S)]);
      float kv[16];  // the kept values in K order
      e2m1x8_values(cw[0], kv);
      e2m1x8_values(cw[1], kv + 8);
#pragma unroll
      for (int i = 0; i < 16; i++) kv[i] = __fmul_rn(kv[i], s);
      if constexpr (PAT == PAT_48P) {
        const uint32_t meta = *reinterpret_cast<const uint16_t*>(p.meta + (int64_t)r * (k / 16) + 2 * u);
#pragma unroll
        for (int g = 0; g < 4; g++) {  // kept pairs p0 < p1 of the group of 8: kept values 4g..4g+3
          const uint32_t nib = (meta >> (4 * g)) & 15u, p0 = nib & 3u, p1 = nib >> 2;
#pragma unroll
          for (int pr = 0; pr < 4; pr++) {
            const bool a = (uint32_t)pr == p0, c = (uint32_t)pr == p1;
            bv[8 * g + 2 * pr] = a ? kv[4 * g] : (c ? kv[4 * g + 2] : 0.0f);
            bv[8 * g + 2 * pr + 1] = a ? kv[4 * g + 1] : (c ? kv[4 * g + 3] : 0.0f);
          }
        }
      } else {  // 2:4: kept i0 < i1 of each group of 4: kept values 2g, 2g+1
        const uint32_t meta = *reinterpret_cast<const uint32_t*>(p.meta + (int64_t)r * (k / 8) + 4 * u);
#pragma unroll
        for (int g = 0; g < 8; g++) {
          const uint32_t nib = (meta >> (4 * g)) & 15u, i0 = nib & 3u, i1 = nib >> 2;
#pragma unroll
          for (int i = 0; i < 4; i++)
            bv[4 * g + i] = (uint32_t)i == i0 ? kv[2 * g] : ((uint32_t)i == i1 ? kv[2 * g + 1] : 0.0f);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __fadd_rn(v[i], bv[i]);
  }
}

// T: rows (1..kGemvMaxRows), a template parameter so that no multiply-add runs for absent rows.
template <int FMT, int PAT, int T>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const GemvParams p) {
  constexpr int b = FMT == FMT_NV ? 16 : 32;
  __shared__ __align__(16) float xs[T][kGemvChunk];
  grid_dep_wait();  // the prepared rows are complete
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = ((int64_t)blockIdx.x * kGemvWarps + warp) * kGemvRowsPerWarp;
  const int64_t ws = p.k / (2 * b);  // weight scales per row (sparse view)
  float acc[kGemvRowsPerWarp][T];
#pragma unroll
  for (int j = 0; j < kGemvRowsPerWarp; j++)
#pragma unroll
    for (int r = 0; r < T; r++) acc[j][r] = 0.0f;

  for (int64_t kc = 0; kc < p.k; kc += kGemvChunk) {
    const int units = (int)((p.k - kc < kGemvChunk ? p.k - kc : kGemvChunk) / 32);
    __syncthreads();  // the previous chunk has been consumed
    for (int w = threadIdx.x; w < T * units; w += blockDim.x) {
      const int r = w / units, uu = w % units;
      float v[32];
      gemv_decode_unit<FMT, PAT>(p, r, kc / 32 + uu, v);
      float4* d = reinterpret_cast<float4*>(&xs[r][32 * uu]);
#pragma unroll
      for (int i = 0; i < 8; i++)  // 16-byte groups XOR-swizzled by the unit: lanes on different units
        d[i ^ (uu & 7)] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);  // hit different banks
    }
    __syncthreads();
    if (n0 >= p.n) continue;
    for (int uu = lane; uu < units; uu += 32) {
      const int64_t u = kc / 32 + uu;
      uint4 wc[kGemvRowsPerWarp];
      float wsv[kGemvRowsPerWarp];
#pragma unroll
      for (int j = 0; j < kGemvRowsPerWarp; j++) {  // the weight stream: read once, bypassing L1
        const int64_t nr = n0 + j < p.n ? n0 + j : p.n - 1;
        wc[j] = __ldcs(reinterpret_cast<const uint4*>(p.w_codes + nr * (p.k / 2)) + u);
        wsv[j] = scale_value<FMT>(__ldg(p.w_sf + tiled_sf_offset(nr, FMT == FMT_NV ? u : u >> 1, ws)));
      }
      float part[kGemvRowsPerWarp][T];
#pragma unroll
      for (int j = 0; j < kGemvRowsPerWarp; j++)
#pragma unroll
        for (int r = 0; r < T; r++) part[j][r] = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; q++) {  // 8 elements at a time: one 32-bit word of codes per weight row
        float xv[T][8];
#pragma unroll
        for (int r = 0; r < T; r++) {
          const float4* xr = reinterpret_cast<const float4*>(&xs[r][32 * uu]);
          const float4 lo = xr[(2 * q) ^ (uu & 7)], hi = xr[(2 * q + 1) ^ (uu & 7)];
          xv[r][0] = lo.x; xv[r][1] = lo.y; xv[r][2] = lo.z; xv[r][3] = lo.w;
          xv[r][4] = hi.x; xv[r][5] = hi.y; xv[r][6] = hi.z; xv[r][7] = hi.w;
        }
#pragma unroll
        for (int j = 0; j < kGemvRowsPerWarp; j++) {
          const uint32_t word = q == 0 ? wc[j].x : q == 1 ? wc[j].y : q == 2 ? wc[j].z : wc[j].w;
          float wv[8];
          e2m1x8_values(word, wv);
#pragma unroll
          for (int e = 0; e < 8; e++)
#pragma unroll
            for (int r = 0; r < T; r++) part[j][r] = __fmaf_rn(xv[r][e], wv[e], part[j][r]);
        }
      }
#pragma unroll
      for (int j = 0; j < kGemvRowsPerWarp; j++)
#pragma unroll
        for (int r = 0; r < T; r++) acc[j][r] = __fmaf_rn(part[j][r], wsv[j], acc[j][r]);
    }
  }
  if (n0 >= p.n) return;
  const float alpha = __fmul_rn(__ldg(p.tensor_x + 2), __ldg(p.tensor_w + 2));
#pragma unroll
  for (int j = 0; j < kGemvRowsPerWarp; j++)
#pragma unroll
    for (int r = 0; r < T; r++) {
      float a = acc[j][r];
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, m));
      if (lane == 0 && n0 + j < p.n) {
        const float yv = __fmul_rn(a, alpha);
        if (p.y_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[r * p.n + n0 + j] = __float2bfloat16_rn(yv);
        else reinterpret_cast<float*>(p.y)[r * p.n + n0 + j] = yv;
      }
    }
}

}  // namespace sharq
