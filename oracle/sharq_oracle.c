/*
 * sharq_oracle.c -- plain CPU oracle for the SharQ sparse-dense FP4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only tests/, the smoke check and the CPU-baseline leg of bench.py
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Method: SharQ, sparse-dense decomposition for FP4 inference (arXiv 2606.26587,
 * Meng, Luo, Zhao et al.), abstract and Section 1:
 *   - an input-adaptive N:M mask is built online from the current activation;
 *   - the masked, outlier-dominated sparse backbone is quantized to FP4;
 *   - the dense residual is defined against the QUANTIZED backbone;
 *   - the residual is quantized to FP4 and a dense FP4 GEMM accumulates it into
 *     the sparse output; both paths share one FP4 weight with path-specific
 *     scale views; the layer norm is absorbed into the preprocessing op.
 * The 4:8 "pair" pattern of NVFP4 is named in its Section 2.2; the OCP MX
 * (MXFP4) format in Section 2.3.  The 8:16 pattern and its metadata cost come
 * from the 2:4-to-8:16 sparsity-pattern paper (arXiv 2507.03052, abstract).
 * Top-k selection per group comes from the Huawei problem statement (Tea House
 * issue 137, problem 2, section 4).
 *
 * The pages give no equations.  Every step below is the plainest reading, with
 * fixed fp32 round-to-nearest-even operations so that a GPU implementation can
 * reproduce codes and scales bit for bit.  Compile with -ffp-contract=off and
 * without -ffast-math: every a*b and a+b here is a separately rounded IEEE op;
 * fused multiply-adds appear only where fmaf() is written.
 */
#include <math.h>
#include <float.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MXFP4 0
#define ORC_NVFP4 1
#define ORC_NM_2_4 0
#define ORC_NM_4_8_PAIR 1
#define ORC_NM_8_16 2
#define ORC_NM_8_16_PAIR 3 /* 8:16 selection re-packed into the 4:8 pair layout */

/* ------------------------------------------------------------------ E2M1 --
 * 4-bit float: sign | 2-bit exponent | 1-bit mantissa.  Magnitudes of codes
 * 0..7 are 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.                    */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
/* Midpoints between neighbouring magnitudes (exact in fp32). */
static const float E2M1_MID[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};

float orc_e2m1_decode(uint8_t c) {
  float m = E2M1_MAG[c & 7];
  return (c & 8) ? -m : m;
}

/* Round to the nearest grid magnitude; a tie goes to the even code; anything
 * above 5 (including values past 6) saturates to 6.  The sign bit follows the
 * sign of the input, so a negative value that rounds to zero gives code 8. */
uint8_t orc_e2m1_encode(float v) {
  uint8_t s = signbit(v) ? 8 : 0;
  float a = fabsf(v);
  int c = 0;
  for (int i = 0; i < 7; i++) {
    if (a > E2M1_MID[i]) {
      c = i + 1;
    } else if (a == E2M1_MID[i]) {
      c = ((i + 1) % 2 == 0) ? i + 1 : i;
      break;
    } else {
      break;
    }
  }
  return (uint8_t)(s | c);
}

/* ------------------------------------------------------------------ E4M3 --
 * OCP FP8 E4M3 ("FN"): bias 7, no infinities, 0x7F/0xFF are NaN, largest
 * finite 448, smallest subnormal 2^-9.                                        */
float orc_e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  float v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexpf((float)m, -9);
  else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -v : v;
}

/* Round to nearest with ties to the even code, saturating to +-448.  Written
 * as a search over the 127 non-negative finite codes in increasing order; the
 * midpoint of two neighbours is exact in fp32 (both have <= 4 significant
 * bits), so the comparisons are exact. */
uint8_t orc_e4m3_encode(float v) {
  uint8_t s = signbit(v) ? 0x80 : 0;
  float a = fabsf(v);
  int c = 0;
  for (int i = 0; i < 126; i++) {
    float lo = orc_e4m3_decode((uint8_t)i), hi = orc_e4m3_decode((uint8_t)(i + 1));
    float mid = (lo + hi) * 0.5f;
    if (a > mid) {
      c = i + 1;
    } else if (a == mid) {
      c = ((i + 1) % 2 == 0) ? i + 1 : i;
      break;
    } else {
      break;
    }
  }
  return (uint8_t)(s | c);
}

/* ------------------------------------------------------------------ E8M0 --
 * OCP MX shared scale: value 2^(c-127); code 255 (NaN) is never produced.    */
float orc_e8m0_decode(uint8_t c) { return ldexpf(1.0f, (int)c - 127); }

/* floor(log2(a)) for finite a > 0, exact (frexp is exact for subnormals too). */
int orc_floor_log2(float a) {
  int e;
  (void)frexpf(a, &e);
  return e - 1;
}

/* ------------------------------------------------------------- RMSNorm ----
 * rstd = 1 / sqrt(mean(x^2) + eps) in a fixed fp32 order:
 *   chunk sums s_j over 16 consecutive elements by sequential fmaf from 0;
 *   the chunk count is padded with zeros to a power of two and combined by a
 *   pairwise tree of adjacent entries (a[i] = a[2i] + a[2i+1] per level);
 *   mean = total / k, then add eps, sqrt and divide, each rounded once.
 * h_j = (x_j * rstd) * gamma_j, two rounded multiplies.                      */
float orc_rms_rstd(const float* x, int64_t k, float eps) {
  int64_t nchunk = k / 16, p = 1;
  while (p < nchunk) p *= 2;
  float* a = (float*)calloc((size_t)p, sizeof(float));
  for (int64_t j = 0; j < nchunk; j++) {
    float acc = 0.0f;
    for (int i = 0; i < 16; i++) acc = fmaf(x[16 * j + i], x[16 * j + i], acc);
    a[j] = acc;
  }
  for (int64_t w = p; w > 1; w /= 2)
    for (int64_t i = 0; i < w / 2; i++) a[i] = a[2 * i] + a[2 * i + 1];
  float total = a[0];
  free(a);
  float mean = total / (float)k;
  float r = 1.0f / sqrtf(mean + eps);
  return r;
}

/* -------------------------------------------------------------- SwiGLU ----
 * Gated activation feeding a down projection: h = SiLU(gate) * up, fused into
 * the preprocessing so that h never goes to memory (an extension of the SharQ
 * abstract's fusing of the layer norm into the preprocessing op; the pages
 * give no formula).  Fixed fp32 steps, each rounded once:
 *   SiLU(a) = a / (1 + E(-a)),   h = SiLU(a) * b,
 * with E the exponential below.
 *
 * E(x) = e^x by Cody and Waite's range reduction and a Taylor polynomial:
 *   x is clamped to [-104, 89] (outside, e^x is 0 or inf in fp32 anyway);
 *   n = rint(x * log2(e))                        (nearest integer, ties to even);
 *   r = fmaf(-n, LN2_HI, x), r = fmaf(-n, LN2_LO, r)   (|r| <= ln(2)/2 + tiny;
 *       LN2_HI = ln 2 to 15 significant bits, LN2_LO = ln 2 - LN2_HI rounded:
 *       ln 2 carried to about 39 bits across the two fused steps);
 *   p = sum_{i=0..7} r^i / i!  by Horner, p = fmaf(p, r, 1/i!) from i = 7 down;
 *   E = (p * 2^n1) * 2^n2 with n1 = n / 2, n2 = n - n1 (exact scalings while the
 *       result stays normal).
 * The truncation error of the degree-7 polynomial on |r| <= 0.35 is below
 * 1e-8 relative, so E is within a few ulp of e^x.                           */
static const float ORC_LOG2E = 1.44269502162933349609375f;     /* log2(e) rounded to fp32 */
static const float ORC_LN2_HI = 0.693145751953125f;            /* 0x3F317200 */
static const float ORC_LN2_LO = 1.428606765330187045037746429443359375e-06f;

static float pow2i(int e) { /* exact 2^e for -126 <= e <= 127 */
  uint32_t bits = (uint32_t)(e + 127) << 23;
  float f;
  memcpy(&f, &bits, sizeof(f));
  return f;
}

float orc_exp(float x) {
  x = fminf(fmaxf(x, -104.0f), 89.0f);
  float nf = rintf(x * ORC_LOG2E);
  int n = (int)nf;
  float r = fmaf(-nf, ORC_LN2_HI, x);
  r = fmaf(-nf, ORC_LN2_LO, r);
  float p = 1.0f / 5040.0f;
  p = fmaf(p, r, 1.0f / 720.0f);
  p = fmaf(p, r, 1.0f / 120.0f);
  p = fmaf(p, r, 1.0f / 24.0f);
  p = fmaf(p, r, 1.0f / 6.0f);
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int n1 = n / 2, n2 = n - n1;
  return (p * pow2i(n1)) * pow2i(n2);
}

float orc_silu(float a) { return a / (1.0f + orc_exp(-a)); }

void orc_swiglu(const float* gate, const float* up, int64_t n, float* h) {
  for (int64_t i = 0; i < n; i++) h[i] = orc_silu(gate[i]) * up[i];
}

/* ------------------------------------------------------------------ mask --
 * Top-N by magnitude per group of M consecutive K elements; ties go to the
 * lower index.  For the 4:8 pair pattern the unit is an adjacent pair (2p,
 * 2p+1) scored by the larger magnitude of the two, and the top 2 of 4 pairs
 * are kept (ties to the lower pair).
 * 8:16 re-packed into the 4:8 pair layout (the 8:16 selection run on the
 * sparse tensor cores, whose pattern is the 4:8 pair; what does not fit goes
 * to the residual): the top 8 of each group of 16 are found as for 8:16; then
 * in each aligned half of 8, pair p is ranked by (how many of those 8 it
 * holds, its larger magnitude, lower index first) and the top 2 of 4 are kept. */
static int pattern_m(int pat) { return pat == ORC_NM_2_4 ? 4 : (pat == ORC_NM_4_8_PAIR ? 8 : 16); }

static void mask_row_nm(const float* h, int64_t k, int m, int n, uint8_t* keep);

void orc_mask_row(const float* h, int64_t k, int pat, uint8_t* keep) {
  if (pat == ORC_NM_8_16_PAIR) {
    uint8_t* k16 = (uint8_t*)malloc((size_t)k);
    mask_row_nm(h, k, 16, 8, k16);
    for (int64_t g = 0; g < k; g += 8) {
      int cnt[4];
      float score[4];
      for (int p = 0; p < 4; p++) {
        cnt[p] = k16[g + 2 * p] + k16[g + 2 * p + 1];
        score[p] = fmaxf(fabsf(h[g + 2 * p]), fabsf(h[g + 2 * p + 1]));
      }
      for (int p = 0; p < 4; p++) {
        int beat = 0;
        for (int q = 0; q < 4; q++)
          if (cnt[q] > cnt[p] || (cnt[q] == cnt[p] && (score[q] > score[p] || (score[q] == score[p] && q < p))))
            beat++;
        keep[g + 2 * p] = keep[g + 2 * p + 1] = (uint8_t)(beat < 2);
      }
    }
    free(k16);
    return;
  }
  if (pat == ORC_NM_4_8_PAIR) {
    for (int64_t g = 0; g < k; g += 8) {
      float score[4];
      for (int p = 0; p < 4; p++) score[p] = fmaxf(fabsf(h[g + 2 * p]), fabsf(h[g + 2 * p + 1]));
      for (int p = 0; p < 4; p++) {
        int beat = 0;
        for (int q = 0; q < 4; q++)
          if (score[q] > score[p] || (score[q] == score[p] && q < p)) beat++;
        keep[g + 2 * p] = keep[g + 2 * p + 1] = (uint8_t)(beat < 2);
      }
    }
    return;
  }
  int m = pattern_m(pat);
  mask_row_nm(h, k, m, m / 2, keep);
}

static void mask_row_nm(const float* h, int64_t k, int m, int n, uint8_t* keep) {
  for (int64_t g = 0; g < k; g += m) {
    for (int i = 0; i < m; i++) {
      float ai = fabsf(h[g + i]);
      int beat = 0;
      for (int j = 0; j < m; j++) {
        float aj = fabsf(h[g + j]);
        if (aj > ai || (aj == ai && j < i)) beat++;
      }
      keep[g + i] = (uint8_t)(beat < n);
    }
  }
}

/* Metadata bytes for one row, in the layout the sparse tensor cores read:
 *   2:4      -- per group of 4, nibble = i0 | i1 << 2 (kept indices, ascending);
 *   4:8 pair -- per group of 8, nibble = p0 | p1 << 2 (kept pair indices);
 *   8:16     -- per group of 16, a 16-bit little-endian mask, bit j = kept.
 * Nibble g of a row sits in byte g/2, low nibble first.                       */
int64_t orc_meta_bytes_per_row(int64_t k, int pat) {
  return (pat == ORC_NM_4_8_PAIR || pat == ORC_NM_8_16_PAIR) ? k / 16 : k / 8;
}

void orc_meta_row(const uint8_t* keep, int64_t k, int pat, uint8_t* meta) {
  memset(meta, 0, (size_t)orc_meta_bytes_per_row(k, pat));
  if (pat == ORC_NM_8_16) {
    for (int64_t g = 0; g < k / 16; g++) {
      uint32_t mask = 0;
      for (int j = 0; j < 16; j++)
        if (keep[16 * g + j]) mask |= 1u << j;
      meta[2 * g] = (uint8_t)(mask & 0xFF);
      meta[2 * g + 1] = (uint8_t)(mask >> 8);
    }
    return;
  }
  int unit = (pat == ORC_NM_4_8_PAIR || pat == ORC_NM_8_16_PAIR) ? 2 : 1;
  int grp = 4 * unit;
  for (int64_t g = 0; g < k / grp; g++) {
    int idx[2], n = 0;
    for (int u = 0; u < 4; u++)
      if (keep[g * grp + u * unit] && n < 2) idx[n++] = u;
    uint8_t nib = (uint8_t)(idx[0] | (idx[1] << 2));
    meta[g / 2] |= (uint8_t)(nib << (4 * (g % 2)));
  }
}

/* --------------------------------------------------------- tensor scale --
 * NVFP4 second-level scale from the tensor amax A (6 * 448 = 2688):
 *   g_enc = 2688 / A, g_dec = A / 2688, both rounded once; A = 0 gives 1.
 * An A so small that 2688 / A overflows is clamped to FLT_MAX for g_enc.    */
void orc_tensor_scale(float amax, float* g_enc, float* g_dec) {
  if (!(amax > 0.0f)) {
    *g_enc = 1.0f;
    *g_dec = 1.0f;
    return;
  }
  float e = 2688.0f / amax;
  if (isinf(e)) e = FLT_MAX;
  *g_enc = e;
  *g_dec = amax / 2688.0f;
}

/* ---------------------------------------------------- block quantizer ----
 * Quantize n values that share one scale.  Writes n E2M1 codes, returns the
 * scale code.  MXFP4 (OCP MX rule): e = floor(log2 amax) - 2 clamped to
 * [-127, 127] (amax = 0 gives -127), code = e + 127, element = E2M1(v * 2^-e).
 * NVFP4: s = (amax / 6) * g_enc, each step rounded once: amax / 6 is the
 * block's decode scale (the largest E2M1 magnitude, 6, lands on the block
 * amax), and multiplying by g_enc expresses it in units of the tensor's decode
 * scale g_dec = 1 / g_enc, the form its E4M3 code stores.  S = E4M3(s); if S
 * is 0 every code is +0, else element = E2M1(v * (g_enc / S)).               */
uint8_t orc_quant_block(const float* v, int n, int fmt, float g_enc, uint8_t* codes) {
  float amax = 0.0f;
  for (int i = 0; i < n; i++) amax = fmaxf(amax, fabsf(v[i]));
  if (fmt == ORC_MXFP4) {
    int e = (amax > 0.0f) ? orc_floor_log2(amax) - 2 : -127;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    float mul = ldexpf(1.0f, -e);
    for (int i = 0; i < n; i++) codes[i] = orc_e2m1_encode(v[i] * mul);
    return (uint8_t)(e + 127);
  }
  float s32 = (amax / 6.0f) * g_enc;
  uint8_t sc = orc_e4m3_encode(s32);
  float sv = orc_e4m3_decode(sc);
  if (sv == 0.0f) {
    for (int i = 0; i < n; i++) codes[i] = 0;
    return sc;
  }
  float inv = g_enc / sv;
  for (int i = 0; i < n; i++) codes[i] = orc_e2m1_encode(v[i] * inv);
  return sc;
}

/* Value of one quantized element without the tensor scale: E2M1 * block
 * scale (exact in fp32: at most 2 x 4 significant bits). */
float orc_unscaled(uint8_t code, uint8_t scale, int fmt) {
  float sv = (fmt == ORC_MXFP4) ? orc_e8m0_decode(scale) : orc_e4m3_decode(scale);
  return orc_e2m1_decode(code) * sv;
}

/* Dequantized element as the residual sees it: unscaled * g_dec (NVFP4). */
float orc_dequant(uint8_t code, uint8_t scale, int fmt, float g_dec) {
  float u = orc_unscaled(code, scale, fmt);
  return (fmt == ORC_MXFP4) ? u : u * g_dec;
}

static int fmt_block(int fmt) { return fmt == ORC_MXFP4 ? 32 : 16; }

static void put_nibble(uint8_t* buf, int64_t idx, uint8_t code) {
  if (idx % 2 == 0) buf[idx / 2] = (uint8_t)((buf[idx / 2] & 0xF0) | (code & 15));
  else buf[idx / 2] = (uint8_t)((buf[idx / 2] & 0x0F) | ((code & 15) << 4));
}

/* ------------------------------------------------------------- prepare ----
 * Whole preprocessing of t rows of k activations (row-major fp32 input that
 * was exactly converted from the caller's dtype):
 *   1. optional RMSNorm (gamma != NULL);
 *   2. N:M mask per row;
 *   3. NVFP4 only: tensor scale from max |h| (or act_amax if > 0);
 *   4. backbone quantization: the kept values of a row, in K order, are cut
 *      into blocks of b (b = 32 MXFP4, 16 NVFP4) stored values -- i.e. 2b
 *      logical positions, since every pattern keeps exactly half of every
 *      aligned window of 16 -- each with one scale;
 *   5. residual R = h - dequant(backbone) at kept positions, R = h elsewhere;
 *   6. residual quantization in dense blocks of b logical positions.
 * Outputs (all row-major, codes packed two per byte, low nibble first):
 *   meta       t * meta_bytes_per_row
 *   bb_codes   2:4 and 4:8 pair: t * k/4 bytes (k/2 kept codes per row);
 *              8:16: t * k/2 bytes, dense layout with code 0 where dropped
 *   bb_scales  t * k/(2b)
 *   res_codes  t * k/2 bytes
 *   res_scales t * k/b
 *   tensor     [amax, g_enc, g_dec] (all 1 / amax for MXFP4)
 *   h_out, bdeq, rdeq: optional t*k fp32 (normalized input, dequantized
 *   backbone incl. g_dec at its logical positions, dequantized residual).
 * Returns 0, or -1 on an unsupported argument.                                */
int orc_prepare(const float* x, int64_t t, int64_t k, const float* gamma, float eps, int fmt, int pat,
                float act_amax, uint8_t* meta, uint8_t* bb_codes, uint8_t* bb_scales, uint8_t* res_codes,
                uint8_t* res_scales, float* tensor, float* h_out, float* bdeq, float* rdeq) {
  if (k <= 0 || k % 256 != 0 || t < 0) return -1;
  if (fmt != ORC_MXFP4 && fmt != ORC_NVFP4) return -1;
  if (pat < 0 || pat > 3) return -1;
  int b = fmt_block(fmt);
  float* h = (float*)malloc(sizeof(float) * (size_t)(t * k > 0 ? t * k : 1));
  for (int64_t r = 0; r < t; r++) {
    const float* xr = x + r * k;
    float* hr = h + r * k;
    if (gamma) {
      float rstd = orc_rms_rstd(xr, k, eps);
      for (int64_t j = 0; j < k; j++) hr[j] = (xr[j] * rstd) * gamma[j];
    } else {
      for (int64_t j = 0; j < k; j++) hr[j] = xr[j];
    }
  }
  float amax = 0.0f, g_enc = 1.0f, g_dec = 1.0f;
  if (fmt == ORC_NVFP4) {
    if (act_amax > 0.0f) {
      amax = act_amax;
    } else {
      for (int64_t i = 0; i < t * k; i++) amax = fmaxf(amax, fabsf(h[i]));
    }
    orc_tensor_scale(amax, &g_enc, &g_dec);
  }
  tensor[0] = amax;
  tensor[1] = g_enc;
  tensor[2] = g_dec;

  uint8_t* keep = (uint8_t*)malloc((size_t)k);
  float* bdq = (float*)malloc(sizeof(float) * (size_t)k);
  float* res = (float*)malloc(sizeof(float) * (size_t)k);
  float* kept = (float*)malloc(sizeof(float) * (size_t)k);
  int64_t* kpos = (int64_t*)malloc(sizeof(int64_t) * (size_t)k);
  uint8_t codes[64];
  int64_t mbytes = orc_meta_bytes_per_row(k, pat);
  int64_t bb_row_bytes = (pat == ORC_NM_8_16) ? k / 2 : k / 4;
  for (int64_t r = 0; r < t; r++) {
    const float* hr = h + r * k;
    orc_mask_row(hr, k, pat, keep);
    orc_meta_row(keep, k, pat, meta + r * mbytes);
    /* backbone: kept values in K order */
    int64_t nk = 0;
    for (int64_t j = 0; j < k; j++)
      if (keep[j]) {
        kept[nk] = hr[j];
        kpos[nk] = j;
        nk++;
      }
    uint8_t* bbc = bb_codes + r * bb_row_bytes;
    memset(bbc, 0, (size_t)bb_row_bytes);
    for (int64_t j = 0; j < k; j++) bdq[j] = 0.0f;
    for (int64_t blk = 0; blk < nk / b; blk++) {
      uint8_t sc = orc_quant_block(kept + blk * b, b, fmt, g_enc, codes);
      bb_scales[r * (k / (2 * b)) + blk] = sc;
      for (int i = 0; i < b; i++) {
        int64_t s = blk * b + i;
        int64_t pos = kpos[s];
        put_nibble(bbc, (pat == ORC_NM_8_16) ? pos : s, codes[i]);
        bdq[pos] = orc_dequant(codes[i], sc, fmt, g_dec);
      }
    }
    /* residual against the quantized backbone */
    for (int64_t j = 0; j < k; j++) res[j] = keep[j] ? hr[j] - bdq[j] : hr[j];
    uint8_t* rc = res_codes + r * (k / 2);
    memset(rc, 0, (size_t)(k / 2));
    for (int64_t blk = 0; blk < k / b; blk++) {
      uint8_t sc = orc_quant_block(res + blk * b, b, fmt, g_enc, codes);
      res_scales[r * (k / b) + blk] = sc;
      for (int i = 0; i < b; i++) {
        put_nibble(rc, blk * b + i, codes[i]);
        if (rdeq) rdeq[r * k + blk * b + i] = orc_dequant(codes[i], sc, fmt, g_dec);
      }
    }
    if (h_out) memcpy(h_out + r * k, hr, sizeof(float) * (size_t)k);
    if (bdeq) memcpy(bdeq + r * k, bdq, sizeof(float) * (size_t)k);
  }
  free(keep);
  free(bdq);
  free(res);
  free(kept);
  free(kpos);
  free(h);
  return 0;
}

/* ----------------------------------------------------- weight quantizer ----
 * The FP4 weight that both paths share.  The sparse tensor-core path applies
 * one scale per b stored backbone values, i.e. per 2b logical K, so a single
 * set of weight codes can only serve both paths if the weight's scale block
 * is 2b logical K; the dense path then views each scale twice.  Rows of W
 * (n x k, row-major) are quantized in blocks of 2b with the weight's own
 * tensor scale (NVFP4).  Outputs: codes n*k/2 bytes, scales n*k/(2b),
 * tensor [amax, g_enc, g_dec].                                               */
int orc_quantize_weight(const float* w, int64_t n, int64_t k, int fmt, uint8_t* codes, uint8_t* scales,
                        float* tensor) {
  if (k <= 0 || k % 256 != 0 || n <= 0) return -1;
  if (fmt != ORC_MXFP4 && fmt != ORC_NVFP4) return -1;
  int bw = 2 * fmt_block(fmt);
  float amax = 0.0f, g_enc = 1.0f, g_dec = 1.0f;
  if (fmt == ORC_NVFP4) {
    for (int64_t i = 0; i < n * k; i++) amax = fmaxf(amax, fabsf(w[i]));
    orc_tensor_scale(amax, &g_enc, &g_dec);
  }
  tensor[0] = amax;
  tensor[1] = g_enc;
  tensor[2] = g_dec;
  uint8_t c[64];
  for (int64_t r = 0; r < n; r++) {
    uint8_t* cr = codes + r * (k / 2);
    memset(cr, 0, (size_t)(k / 2));
    for (int64_t blk = 0; blk < k / bw; blk++) {
      uint8_t sc = orc_quant_block(w + r * k + blk * bw, bw, fmt, g_enc, c);
      scales[r * (k / bw) + blk] = sc;
      for (int i = 0; i < bw; i++) put_nibble(cr, blk * bw + i, c[i]);
    }
  }
  return 0;
}

/* ------------------------------------------------ operand decoders --------
 * Exact fp64 values of the operands the two GEMMs contract, without the
 * tensor scales (E2M1 * block scale is exact), for the fp64 reference GEMM:
 *   Y = g_dec_x * g_dec_w * (Bu + Ru) . Wu^T.                                 */
void orc_decode_prepared(const uint8_t* meta, const uint8_t* bb_codes, const uint8_t* bb_scales,
                         const uint8_t* res_codes, const uint8_t* res_scales, int64_t t, int64_t k, int fmt,
                         int pat, double* bu, double* ru) {
  int b = fmt_block(fmt);
  int64_t mbytes = orc_meta_bytes_per_row(k, pat);
  int64_t bb_row_bytes = (pat == ORC_NM_8_16) ? k / 2 : k / 4;
  uint8_t* keep = (uint8_t*)malloc((size_t)k);
  for (int64_t r = 0; r < t; r++) {
    const uint8_t* mr = meta + r * mbytes;
    memset(keep, 0, (size_t)k);
    if (pat == ORC_NM_8_16) {
      for (int64_t g = 0; g < k / 16; g++) {
        uint32_t mask = (uint32_t)mr[2 * g] | ((uint32_t)mr[2 * g + 1] << 8);
        for (int j = 0; j < 16; j++) keep[16 * g + j] = (uint8_t)((mask >> j) & 1);
      }
    } else {
      int unit = (pat == ORC_NM_4_8_PAIR || pat == ORC_NM_8_16_PAIR) ? 2 : 1, grp = 4 * unit;
      for (int64_t g = 0; g < k / grp; g++) {
        uint8_t nib = (uint8_t)((mr[g / 2] >> (4 * (g % 2))) & 15);
        int i0 = nib & 3, i1 = (nib >> 2) & 3;
        for (int u = 0; u < unit; u++) {
          keep[g * grp + i0 * unit + u] = 1;
          keep[g * grp + i1 * unit + u] = 1;
        }
      }
    }
    const uint8_t* bbc = bb_codes + r * bb_row_bytes;
    int64_t s = 0;
    for (int64_t j = 0; j < k; j++) {
      double v = 0.0;
      if (keep[j]) {
        int64_t ci = (pat == ORC_NM_8_16) ? j : s;
        uint8_t code = (uint8_t)((bbc[ci / 2] >> (4 * (ci % 2))) & 15);
        uint8_t sc = bb_scales[r * (k / (2 * b)) + s / b];
        v = (double)orc_unscaled(code, sc, fmt);
        s++;
      }
      bu[r * k + j] = v;
    }
    const uint8_t* rc = res_codes + r * (k / 2);
    for (int64_t j = 0; j < k; j++) {
      uint8_t code = (uint8_t)((rc[j / 2] >> (4 * (j % 2))) & 15);
      ru[r * k + j] = (double)orc_unscaled(code, res_scales[r * (k / b) + j / b], fmt);
    }
  }
  free(keep);
}

void orc_decode_weight(const uint8_t* codes, const uint8_t* scales, int64_t n, int64_t k, int fmt, double* wu) {
  int bw = 2 * fmt_block(fmt);
  for (int64_t r = 0; r < n; r++)
    for (int64_t j = 0; j < k; j++) {
      uint8_t code = (uint8_t)((codes[r * (k / 2) + j / 2] >> (4 * (j % 2))) & 15);
      wu[r * k + j] = (double)orc_unscaled(code, scales[r * (k / bw) + j / bw], fmt);
    }
}

/* ------------------------------------------------ array helpers -----------
 * Element-wise forms of the format functions and the row amax, so that
 * exhaustive checks and threaded drivers need one foreign call each.          */
void orc_e2m1_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_e2m1_encode(v[i]);
}
void orc_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_encode(v[i]);
}
/* Consecutive blocks of bs values, each quantized by orc_quant_block (codes one
 * per byte, one scale code per block). */
void orc_quant_blocks_n(const float* v, int64_t nblocks, int bs, int fmt, float g_enc, uint8_t* codes,
                        uint8_t* scales) {
  for (int64_t i = 0; i < nblocks; i++) scales[i] = orc_quant_block(v + i * bs, bs, fmt, g_enc, codes + i * bs);
}
void orc_floor_log2_n(const float* v, int64_t n, int32_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_floor_log2(v[i]);
}
void orc_mask_rows(const float* h, int64_t t, int64_t k, int pat, uint8_t* keep) {
  for (int64_t r = 0; r < t; r++) orc_mask_row(h + r * k, k, pat, keep + r * k);
}

/* max |h| over t rows (h = RMSNorm(x) when gamma != NULL, else x). */
float orc_rows_amax(const float* x, int64_t t, int64_t k, const float* gamma, float eps) {
  float amax = 0.0f;
  for (int64_t r = 0; r < t; r++) {
    const float* xr = x + r * k;
    if (gamma) {
      float rstd = orc_rms_rstd(xr, k, eps);
      for (int64_t j = 0; j < k; j++) amax = fmaxf(amax, fabsf((xr[j] * rstd) * gamma[j]));
    } else {
      for (int64_t j = 0; j < k; j++) amax = fmaxf(amax, fabsf(xr[j]));
    }
  }
  return amax;
}
