// gemv.cuh -- the layer's two products for a handful of rows (decode).
//
// SharQ abstract and Section 1: y = g_dec(x) * g_dec(w) * sum_k (B + R)[t][k] * W[n][k],
// the sparse backbone product plus the dense residual product into one output,
// both reading the one FP4 weight.  With at most kGemvMaxRows rows the work is
// a weight stream (N*K/2 bytes of codes) with a few multiply-adds per byte, so
// it runs on the CUDA cores: a 128-row tensor-core tile would be at least 97 %
// padding and its K loop latency bound.  Each weight element costs its E2M1 ->
// fp32 widening and half a packed FMA, so instruction issue, not HBM, is the
// limit at one row.
//
// Each block decodes the rows' backbone and residual (codes, metadata and block
// scales, without the tensor scale) one K chunk at a time into shared memory as
// fp32 B + R (two buffers); every warp streams two weight rows along K (lane l
// takes 32-element units l, l+32, ... of the chunk), multiplies the E2M1 values
// of a unit by the decoded rows, scales the unit's sum by its weight block scale
// and accumulates.  The next chunk's weight codes and stored row bytes are in
// flight while the current chunk's products run.  Lanes are summed by shuffles
// at the end.  The summation order differs from the tensor cores' (the
// tolerance of the GEMM applies).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "prep.cuh"

namespace sharq {

constexpr int kGemvMaxRows = 4;
constexpr int kGemvWarps = 8;          // warps per block
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

// acc += x * w on packed fp32 pairs (even element low, odd element high).
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t x, uint64_t w) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(x), "l"(w));
}

// Eight E2M1 codes of a word (element i in nibble i) -> four packed fp32 pairs
// (elements 2i, 2i + 1 in pair i): each byte through one cvt to f16x2, then
// both halves widened to fp32 (exact).
__device__ __forceinline__ void e2m1x8_pairs(uint32_t w, uint64_t (&o)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h;\n\t.reg .f16 l, u;\n\t.reg .f32 fl, fu;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 h, b0;\n\tmov.b32 {l, u}, h;\n\tcvt.f32.f16 fl, l;\n\tcvt.f32.f16 fu, u;\n\tmov.b64 %0, {fl, fu};\n\t"
      "cvt.rn.f16x2.e2m1x2 h, b1;\n\tmov.b32 {l, u}, h;\n\tcvt.f32.f16 fl, l;\n\tcvt.f32.f16 fu, u;\n\tmov.b64 %1, {fl, fu};\n\t"
      "cvt.rn.f16x2.e2m1x2 h, b2;\n\tmov.b32 {l, u}, h;\n\tcvt.f32.f16 fl, l;\n\tcvt.f32.f16 fu, u;\n\tmov.b64 %2, {fl, fu};\n\t"
      "cvt.rn.f16x2.e2m1x2 h, b3;\n\tmov.b32 {l, u}, h;\n\tcvt.f32.f16 fl, l;\n\tcvt.f32.f16 fu, u;\n\tmov.b64 %3, {fl, fu};\n\t}"
      : "=l"(o[0]), "=l"(o[1]), "=l"(o[2]), "=l"(o[3])
      : "r"(w));
}

template <int FMT>
__device__ __forceinline__ float scale_value(uint32_t c) {
  if constexpr (FMT == FMT_MX) return c ? __uint_as_float(c << 23) : __uint_as_float(0x00400000u);
  else return e4m3_value(c);
}

// The stored bytes of one quarter unit (8 logical elements, quarter q of unit
// u) of one prepared row: residual codes, backbone codes (4 kept codes, or 8
// for 8:16), the quarter's metadata and the two block scale codes (residual in
// byte 0, backbone in byte 1).  Loaded one chunk ahead and decoded after the
// current chunk's products; every thread of the block decodes a share.
struct GemvQuarterRaw {
  uint32_t rc, bc, meta, sc;
};

template <int FMT, int PAT>
__device__ __forceinline__ void gemv_load_quarter(const GemvParams& p, int r, int64_t u, int q, GemvQuarterRaw& x) {
  constexpr int b = FMT == FMT_NV ? 16 : 32;
  const int64_t k = p.k;
  // the dense-view scale index of the quarter (per b logical)
  const int64_t sd = FMT == FMT_NV ? 2 * u + (q >> 1) : u;
  x.rc = x.bc = x.meta = x.sc = 0;
  if (p.paths & 2) {
    x.rc = *reinterpret_cast<const uint32_t*>(p.res_codes + (int64_t)r * (k / 2) + 16 * u + 4 * q);
    x.sc = p.res_scales[tiled_sf_offset(r, sd, k / b)];
  }
  if (p.paths & 1) {
    if constexpr (PAT == PAT_816) {  // dense backbone, dense-view scales per b
      x.bc = *reinterpret_cast<const uint32_t*>(p.bb_codes + (int64_t)r * (k / 2) + 16 * u + 4 * q);
      x.sc |= (uint32_t)p.bb_scales[tiled_sf_offset(r, sd, k / b)] << 8;
    } else {  // 4 kept codes in K order, one sparse-view scale per 2b logical
      x.bc = *reinterpret_cast<const uint16_t*>(p.bb_codes + (int64_t)r * (k / 4) + 8 * u + 2 * q);
      x.sc |= (uint32_t)p.bb_scales[tiled_sf_offset(r, FMT == FMT_NV ? u : u >> 1, k / (2 * b))] << 8;
      if constexpr (PAT == PAT_48P)  // the group of 8 = the quarter: one nibble
        x.meta = (p.meta[(int64_t)r * (k / 16) + 2 * u + (q >> 1)] >> (4 * (q & 1))) & 15u;
      else  // two groups of 4: one byte
        x.meta = p.meta[(int64_t)r * (k / 8) + 4 * u + q];
    }
  }
}

// Decoded B + R (without tensor scale) of a loaded quarter unit.
template <int FMT, int PAT>
__device__ __forceinline__ void gemv_decode_quarter(const GemvParams& p, const GemvQuarterRaw& x, float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 8; i++) v[i] = 0.0f;
  if (p.paths & 2) {
    const float s = scale_value<FMT>(x.sc & 0xFFu);
    float d[8];
    e2m1x8_values(x.rc, d);
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = __fmul_rn(d[i], s);
  }
  if (p.paths & 1) {
    const float s = scale_value<FMT>((x.sc >> 8) & 0xFFu);
    float bv[8];
    if constexpr (PAT == PAT_816) {
      e2m1x8_values(x.bc, bv);
#pragma unroll
      for (int i = 0; i < 8; i++) bv[i] = __fmul_rn(bv[i], s);
    } else {
      float kv[8];  // kv[0..3]: the kept values in K order
      e2m1x8_values(x.bc, kv);
#pragma unroll
      for (int i = 0; i < 4; i++) kv[i] = __fmul_rn(kv[i], s);
      if constexpr (PAT == PAT_48P) {  // kept pairs p0 < p1
        const uint32_t p0 = x.meta & 3u, p1 = x.meta >> 2;
#pragma unroll
        for (int pr = 0; pr < 4; pr++) {
          const bool a = (uint32_t)pr == p0, c = (uint32_t)pr == p1;
          bv[2 * pr] = a ? kv[0] : (c ? kv[2] : 0.0f);
          bv[2 * pr + 1] = a ? kv[1] : (c ? kv[3] : 0.0f);
        }
      } else {  // 2:4: kept i0 < i1 of each group of 4
#pragma unroll
        for (int g = 0; g < 2; g++) {
          const uint32_t nib = (x.meta >> (4 * g)) & 15u, i0 = nib & 3u, i1 = nib >> 2;
#pragma unroll
          for (int i = 0; i < 4; i++)
            bv[4 * g + i] = (uint32_t)i == i0 ? kv[2 * g] : ((uint32_t)i == i1 ? kv[2 * g + 1] : 0.0f);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = __fadd_rn(v[i], bv[i]);
  }
}

// Logical K per chunk of decoded rows: at most two decoded quarter units per
// thread of the block, and two chunks of T rows in shared memory (double buffered).
template <int T>
__host__ __device__ constexpr int gemv_chunk() { return T <= 2 ? 2048 : 1024; }

// T: rows (1..kGemvMaxRows), a template parameter so that no multiply-add runs for absent rows.
//
// Pipeline per chunk c: the weight codes and scales of chunk c + 1 and the
// stored bytes of the prepared rows' chunk c + 1 are requested, the products of
// chunk c run on the registers and shared memory filled one step before, then
// chunk c + 1 is decoded into the other shared-memory buffer.  Before the wait
// for the prepared rows, each warp asks L2 for its whole weight rows, so the
// weight stream starts while the kernel before this one finishes.
template <int FMT, int PAT, int T>
__global__ void __launch_bounds__(kGemvWarps * 32, 2) gemv_kernel(const GemvParams p) {
  constexpr int b = FMT == FMT_NV ? 16 : 32;
  constexpr int kChunk = gemv_chunk<T>();
  constexpr int kUnits = kChunk / 32;  // units per chunk
  constexpr int kUpl = kUnits / 32;    // units per lane per chunk
  constexpr int R = kGemvRowsPerWarp;
  __shared__ __align__(16) float xs[2][T][kChunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = ((int64_t)blockIdx.x * kGemvWarps + warp) * R;
  const int64_t ws = p.k / (2 * b);  // weight scales per row (sparse view)
  const int64_t ku = p.k / 32;       // units per row
  const int64_t nchunks = (ku + kUnits - 1) / kUnits;
  int64_t nr[R];
#pragma unroll
  for (int j = 0; j < R; j++) nr[j] = n0 + j < p.n ? n0 + j : p.n - 1;
  const bool live = n0 < p.n;

  if (live && lane < R && n0 + lane < p.n) prefetch_l2(p.w_codes + (n0 + lane) * (p.k / 2), (uint32_t)(p.k / 2));
  if (live && lane == 0 && (n0 & 127) == 0) {  // the first row of a 128-row block: that block's scales
    const int64_t sblocks = (ws + 3) >> 2;
    prefetch_l2(p.w_sf + (n0 >> 7) * sblocks * 512, (uint32_t)(sblocks * 512));
  }
  grid_dep_wait();  // the prepared rows are complete

  // per weight row: its code row and the row part of its tiled scale offsets
  const int64_t sblocks = (ws + 3) >> 2;
  const uint4* wrow[R];
  int64_t srow[R];
#pragma unroll
  for (int j = 0; j < R; j++) {
    wrow[j] = reinterpret_cast<const uint4*>(p.w_codes + nr[j] * (p.k / 2));
    srow[j] = (nr[j] >> 7) * sblocks * 512 + (nr[j] & 31) * 16 + ((nr[j] >> 5) & 3) * 4;
  }
  auto load_w = [&](int64_t c, uint4 (&codes)[kUpl][R], uint32_t (&scl)[kUpl][R]) {
#pragma unroll
    for (int i = 0; i < kUpl; i++) {
      const int64_t u = c * kUnits + lane + 32 * i;
      const int64_t cs = FMT == FMT_NV ? u : u >> 1;  // sparse-view scale column
      const int64_t scol = (cs >> 2) * 512 + (cs & 3);
#pragma unroll
      for (int j = 0; j < R; j++) {
        if (live && u < ku) {  // the weight stream: read once, bypassing L1
          codes[i][j] = __ldcs(wrow[j] + u);
          scl[i][j] = __ldg(p.w_sf + srow[j] + scol);
        } else {
          codes[i][j] = make_uint4(0, 0, 0, 0);
          scl[i][j] = 0;
        }
      }
    }
  };
  // decode slots of a chunk: (row, unit, quarter), quarters of a unit on neighbouring threads
  constexpr int kSlotsTotal = T * kUnits * 4;
  constexpr int kSlots = (kSlotsTotal + kGemvWarps * 32 - 1) / (kGemvWarps * 32);
  int xrow[kSlots], xunit[kSlots], xq[kSlots];
  bool xon[kSlots];
#pragma unroll
  for (int sl = 0; sl < kSlots; sl++) {
    const int s = (int)threadIdx.x + sl * kGemvWarps * 32, rem = s % (kUnits * 4);
    xon[sl] = s < kSlotsTotal;
    xrow[sl] = s / (kUnits * 4);
    xunit[sl] = rem >> 2;
    xq[sl] = rem & 3;
  }
  auto load_x = [&](int64_t c, GemvQuarterRaw (&raw)[kSlots]) {
#pragma unroll
    for (int sl = 0; sl < kSlots; sl++)
      if (xon[sl] && c * kUnits + xunit[sl] < ku)
        gemv_load_quarter<FMT, PAT>(p, xrow[sl], c * kUnits + xunit[sl], xq[sl], raw[sl]);
  };
  auto store_x = [&](int64_t c, int buf, const GemvQuarterRaw (&raw)[kSlots]) {
#pragma unroll
    for (int sl = 0; sl < kSlots; sl++) {
      if (!(xon[sl] && c * kUnits + xunit[sl] < ku)) continue;
      const int uu = xunit[sl], q = xq[sl];
      float v[8];
      gemv_decode_quarter<FMT, PAT>(p, raw[sl], v);
      float4* d = reinterpret_cast<float4*>(&xs[buf][xrow[sl]][32 * uu]);
      // 16-byte groups XOR-swizzled by the unit: lanes on different units hit different banks
      d[(2 * q) ^ (uu & 7)] = make_float4(v[0], v[1], v[2], v[3]);
      d[(2 * q + 1) ^ (uu & 7)] = make_float4(v[4], v[5], v[6], v[7]);
    }
  };

  float acc[R][T];
#pragma unroll
  for (int j = 0; j < R; j++)
#pragma unroll
    for (int r = 0; r < T; r++) acc[j][r] = 0.0f;

  // one chunk: request chunk c + 1 (weights into nxt, activation bytes), products
  // of chunk c from cur and shared-memory buffer c & 1, then decode chunk c + 1
  auto step = [&](int64_t c, const uint4 (&cur)[kUpl][R], const uint32_t (&scur)[kUpl][R], uint4 (&nxt)[kUpl][R],
                  uint32_t (&snxt)[kUpl][R]) {
    const int buf = (int)(c & 1);
    const bool more = c + 1 < nchunks;
    GemvQuarterRaw raw[kSlots];
    if (more) {
      load_w(c + 1, nxt, snxt);
      load_x(c + 1, raw);
    }
    if (live) {
#pragma unroll
      for (int i = 0; i < kUpl; i++) {
        const int uu = lane + 32 * i;
        if (c * kUnits + uu >= ku) break;
        uint64_t part[R][T];  // packed (even, odd) element sums of the unit
#pragma unroll
        for (int j = 0; j < R; j++)
#pragma unroll
          for (int r = 0; r < T; r++) part[j][r] = 0;
#pragma unroll
        for (int w = 0; w < 4; w++) {  // 8 elements at a time: one 32-bit word of codes per weight row
          uint64_t xv[T][4];
#pragma unroll
          for (int r = 0; r < T; r++) {
            const ulonglong2* xp = reinterpret_cast<const ulonglong2*>(&xs[buf][r][32 * uu]);
            const ulonglong2 lo = xp[(2 * w) ^ (uu & 7)], hi = xp[(2 * w + 1) ^ (uu & 7)];
            xv[r][0] = lo.x; xv[r][1] = lo.y; xv[r][2] = hi.x; xv[r][3] = hi.y;
          }
#pragma unroll
          for (int j = 0; j < R; j++) {
            const uint32_t word = w == 0 ? cur[i][j].x : w == 1 ? cur[i][j].y : w == 2 ? cur[i][j].z : cur[i][j].w;
            uint64_t wv[4];
            e2m1x8_pairs(word, wv);
#pragma unroll
            for (int e = 0; e < 4; e++)
#pragma unroll
              for (int r = 0; r < T; r++) ffma2(part[j][r], xv[r][e], wv[e]);
          }
        }
#pragma unroll
        for (int j = 0; j < R; j++) {
          const float wsv = scale_value<FMT>(scur[i][j]);
#pragma unroll
          for (int r = 0; r < T; r++) {
            const float even = __uint_as_float((uint32_t)part[j][r]), odd = __uint_as_float((uint32_t)(part[j][r] >> 32));
            acc[j][r] = __fmaf_rn(__fadd_rn(even, odd), wsv, acc[j][r]);
          }
        }
      }
    }
    if (more) store_x(c + 1, buf ^ 1, raw);
    __syncthreads();  // chunk c + 1 decoded; chunk c's buffer free for chunk c + 2
  };

  uint4 wa[kUpl][R], wb[kUpl][R];  // weight codes of the current and the next chunk (ping-pong)
  uint32_t sa[kUpl][R], sb[kUpl][R];
  load_w(0, wa, sa);
  {
    GemvQuarterRaw raw[kSlots];
    load_x(0, raw);
    store_x(0, 0, raw);
  }
  __syncthreads();
  for (int64_t c = 0; c < nchunks; c += 2) {
    step(c, wa, sa, wb, sb);
    if (c + 1 < nchunks) step(c + 1, wb, sb, wa, sa);
  }
  if (!live) return;
  const float alpha = __fmul_rn(__ldg(p.tensor_x + 2), __ldg(p.tensor_w + 2));
#pragma unroll
  for (int j = 0; j < R; j++)
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
