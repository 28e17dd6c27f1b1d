/*
 * sharq.h -- C ABI of the B200 (sm_100a) SharQ sparse-dense FP4 linear layer.
 *
 * The layer (SharQ, arXiv 2606.26587, abstract and Section 1) splits each
 * activation row online into an outlier-dominated N:M-sparse backbone, which
 * is quantized to FP4 and multiplied by a sparse FP4 GEMM, and a dense
 * residual taken against the QUANTIZED backbone, quantized to FP4 and
 * accumulated into the same output by a dense FP4 GEMM.  Both GEMMs read one
 * shared FP4 weight through path-specific scale views, and a fused
 * preprocessing op absorbs the layer norm, the mask and the residual.
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers on the current CUDA device,
 *    owned and allocated by the caller with the sizes the *_sizes queries
 *    return.  The library allocates no device memory and keeps no device
 *    state besides one error word per device and the static scratch of
 *    sharq_prepare_noalloc.
 *  - Calls are asynchronous on the given stream.  Argument errors are found
 *    on the host and returned before anything is launched.  A device-side
 *    wait that runs out of time sets the error word; sharq_sync_status()
 *    synchronizes the stream and reports it (SHARQ_ERR_TIMEOUT).
 *  - Shapes: k % 256 == 0; n % 256 == 0; t >= 1.  Row buffers of prepared
 *    activations hold t_pad = roundup(t, 128) rows; rows t..t_pad-1 are
 *    written as if their input were zero.
 *  - Byte layouts (little endian):
 *      codes      two E2M1 codes per byte, the lower K index in the low nibble;
 *      scales     "tiled scale layout": a tensor with R rows and S scales per
 *                 row is stored as ceil(R/128) x ceil(S/4) blocks of 512 bytes,
 *                 row-block major; inside a block, row r and scale s sit at
 *                 byte (r%32)*16 + ((r/32)%4)*4 + (s%4);
 *      meta       row-major, 2:4 and 4:8 pair (and 8:16 re-packed): one nibble per group of 4 (8)
 *                 K elements, nibble = i0 | i1 << 2 with the kept element
 *                 (pair) indices i0 < i1, group g in byte g/2, low nibble
 *                 first; 8:16: one little-endian uint16 mask per group of 16.
 *      tensor     3 floats: [amax, g_enc, g_dec] (NVFP4 second-level scale
 *                 g_enc = 2688/amax, g_dec = amax/2688; MXFP4: [0, 1, 1]).
 */
#ifndef SHARQ_H
#define SHARQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sharq_stream; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  SHARQ_OK = 0,
  SHARQ_ERR_INVALID = 1,     /* bad shape, pointer, alignment or enum value */
  SHARQ_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. NVFP4 with 2:4 in sharq_linear) */
  SHARQ_ERR_CUDA = 3,        /* a CUDA runtime call failed; see sharq_last_error() */
  SHARQ_ERR_TIMEOUT = 4,     /* a device-side wait ran out of time (error word) */
  SHARQ_ERR_WORKSPACE = 5    /* workspace missing or too small */
} sharq_status;

/* FP4 formats (SharQ abstract; Section 2.3 names OCP MX):
 *   MXFP4 -- E2M1 elements, one E8M0 scale per 32 elements, no tensor scale;
 *   NVFP4 -- E2M1 elements, one E4M3 scale per 16 elements, fp32 tensor scale. */
typedef enum { SHARQ_MXFP4 = 0, SHARQ_NVFP4 = 1 } sharq_format;

/* Online N:M activation masks: 2:4 (Huawei problem 137-2 asks for MXFP4/HiF4
 * combined with 2:4), the NVFP4 4:8 pair pattern (SharQ Section 2.2: two of four
 * adjacent pairs kept), and 8:16 (paper on 2:4-to-8:16 sparsity patterns, abstract).
 * SHARQ_NM_8_16_PAIR runs the 8:16 selection on the sparse tensor cores, whose
 * pattern is the 4:8 pair: the top 8 of each group of 16 are found as for 8:16,
 * then each group of 8 keeps the two adjacent pairs holding most of them (ties:
 * the larger magnitude, then the lower pair); the rest goes to the residual.  Its
 * buffers use the 4:8 pair layouts, and sharq_linear runs the 4:8 pair GEMM. */
typedef enum { SHARQ_NM_2_4 = 0, SHARQ_NM_4_8_PAIR = 1, SHARQ_NM_8_16 = 2, SHARQ_NM_8_16_PAIR = 3 } sharq_pattern;

typedef enum { SHARQ_F32 = 0, SHARQ_BF16 = 1 } sharq_dtype;

/* The FP4 weight shared by the sparse and the dense GEMM (SharQ abstract:
 * the two GEMM paths load the FP4 weight once and each reads it through its
 * own view of the scales).
 * The sparse tensor-core MMA applies one scale per b stored (2b logical) K
 * elements, so the weight is quantized in K blocks of 2b (b = 32 MXFP4, 16
 * NVFP4) and carries two views of the same scales:
 *   codes          experts * n * k/2 bytes, row-major per expert;
 *   scales_dense   per expert, tiled scale layout, n rows, k/b scales (each 2b
 *                  scale stored twice) -- the view of the dense residual GEMM
 *                  (the sparse-pattern GEMMs rebuild it on chip from
 *                  scales_sparse; the 8:16 dense-backbone GEMM reads it);
 *   scales_sparse  per expert, tiled scale layout, n rows, k/(2b) scales;
 *   tensor         experts * 3 floats. */
typedef struct {
  void* codes;
  void* scales_dense;
  void* scales_sparse;
  float* tensor;
  int64_t n, k;
  int32_t experts; /* 1 for a plain linear layer; stacked experts for sharq_linear_grouped */
  sharq_format fmt;
} sharq_weight;

/* Prepared activations (output of sharq_prepare):
 *   meta       t_pad * meta_row bytes (meta_row = k/8 for 2:4 and 8:16, k/16 for 4:8 pair)
 *   bb_codes   backbone codes: 2:4 and 4:8 pair -- t_pad * k/4 bytes, the k/2 kept values
 *              of a row in K order (the compressed sparse input of SharQ Section 1);
 *              8:16 -- t_pad * k/2 bytes, dense layout with code 0 at dropped positions
 *   bb_scales  tiled scale layout, t_pad rows: one scale per b kept values (k/(2b) per
 *              row); for 8:16 each is stored twice (k/b per row), the dense view
 *   res_codes  t_pad * k/2 bytes, dense residual codes
 *   res_scales tiled scale layout, t_pad rows, k/b scales per row
 *   tensor     3 floats shared by backbone and residual (NVFP4) */
typedef struct {
  void* meta;
  void* bb_codes;
  void* bb_scales;
  void* res_codes;
  void* res_scales;
  float* tensor;
  int64_t t, k;
  sharq_format fmt;
  sharq_pattern pat;
} sharq_prepared;

/* Byte sizes of the weight buffers for one expert (multiply by experts). */
sharq_status sharq_weight_sizes(int64_t n, int64_t k, sharq_format fmt, size_t* codes_bytes,
                                size_t* scales_dense_bytes, size_t* scales_sparse_bytes);

/* Byte sizes of the prepared-activation buffers for t rows and of the optional
 * workspace of sharq_prepare (t_pad floats: with RMSNorm and a device-computed
 * NVFP4 amax, the amax pass leaves each row's RMSNorm factor there for the
 * quantization pass, which then skips its own reduction). */
sharq_status sharq_prepared_sizes(int64_t t, int64_t k, sharq_format fmt, sharq_pattern pat, size_t* meta_bytes,
                                  size_t* bb_codes_bytes, size_t* bb_scales_bytes, size_t* res_codes_bytes,
                                  size_t* res_scales_bytes, size_t* workspace_bytes);

/* Offline weight quantization (W4 of W4A4, Huawei problem 137-2; the shared
 * weight of the SharQ abstract).  w: experts * n * k values (row-major, nn.Linear
 * out x in layout) of dtype w_dt.  Each expert gets its own tensor scale (NVFP4).
 * out->codes/scales/tensor must be set by the caller; n, k, experts, fmt too. */
sharq_status sharq_quantize_weight(const void* w, sharq_dtype w_dt, sharq_weight* out, sharq_stream stream);

/* Fused preprocessing (SharQ abstract: one fused operator does the mask, the
 * residual and the layer norm):
 *   h = RMSNorm(x) * gamma if gamma != NULL (fp32, eps added to the mean square), else x;
 *   N:M mask = top-N |h| per group of M, ties to the lower index (4:8 pair: top 2 of 4
 *   adjacent pairs by max |.|); backbone = kept values, FP4 in blocks of b kept values;
 *   R = h - dequant(backbone) where kept, h elsewhere; R to FP4 in blocks of b.
 * x: t * k row-major values of dtype x_dt; gamma: k values of dtype x_dt or NULL.
 * act_amax > 0 gives the NVFP4 tensor amax; <= 0 computes max |h| on the device
 * (one extra read of x).  out->pointers, t, k, fmt, pat must be set by the caller.
 * workspace: NULL, or >= t floats (16-byte aligned) of scratch; results are the same
 * either way.  Returns SHARQ_ERR_WORKSPACE for a non-NULL workspace that is too small. */
sharq_status sharq_prepare(const void* x, sharq_dtype x_dt, const void* gamma, float eps, float act_amax,
                           sharq_prepared* out, void* workspace, size_t workspace_bytes, sharq_stream stream);

/* Fused preprocessing of a down projection's input formed on the fly from a gated
 * MLP: h = SiLU(gate) * up, then the mask, backbone and residual of sharq_prepare (no
 * RMSNorm).  The SharQ abstract fuses the layer norm into the preprocessing op; this
 * extends the same fusion to the activation in front of the down projection, so h is
 * never written to or read from memory.  In fp32, each step rounded once:
 *   SiLU(a) = a / (1 + E(-a)),  h = SiLU(a) * b,
 * where E is the library's exponential: reduction by ln 2 in two fp32 steps (Cody and
 * Waite), the degree-7 Taylor polynomial by Horner with fused multiply-adds, exact
 * scaling by 2^n; inputs clamped to [-104, 89]; within one ulp of e^x.
 * gate, up: t * k row-major values of dtype dt (DEVICE).  act_amax as in sharq_prepare
 * (<= 0: the NVFP4 tensor amax of h is computed on the device).  out: as sharq_prepare. */
sharq_status sharq_prepare_swiglu(const void* gate, const void* up, sharq_dtype dt, float act_amax,
                                  sharq_prepared* out, sharq_stream stream);

/* Row gather of prepared activations, for a mixture-of-experts layer: prepare every token
 * once, then lay its prepared row out once per expert it is routed to (SharQ evaluates
 * Qwen3-30B-A3B; each token goes to several experts, so preparing the routed rows
 * repeats the per-row work for every copy).  dst row i is src row rows[i] for rows[i]
 * in [0, src->t), else (rows[i] < 0, and every padding row up to t_pad) the encoding of
 * an all-zero input row.  rows: DEVICE, dst->t int32 values.  src and dst share k, fmt
 * and pat; dst->tensor receives src->tensor.  The result equals preparing the gathered
 * rows directly whenever the NVFP4 tensor amax is the same (routed rows hold the tokens'
 * values and zeros).  Index values are not checked on the host: one at or beyond src->t
 * is treated as a zero row. */
sharq_status sharq_gather_prepared(const sharq_prepared* src, const int32_t* rows, sharq_prepared* dst,
                                   sharq_stream stream);

/* Largest t that sharq_prepare_noalloc accepts (its static scratch holds one float per row). */
#define SHARQ_NOALLOC_MAX_ROWS 65536

/* sharq_prepare without a caller workspace and without any allocation: the
 * per-row scratch (each row's RMSNorm factor, which the NVFP4 amax pass hands
 * to the quantization pass) is a static device array inside this library,
 * SHARQ_NOALLOC_MAX_ROWS floats (256 KiB) per device.  Arguments, outputs and
 * results are those of sharq_prepare with a workspace; the SharQ pages have no
 * counterpart of this call, which exists for callers that cannot allocate:
 *   - a host whose device memory is sized once at start-up and may not grow
 *     (a fixed pool, no allocator reachable from the calling code);
 *   - a plug-in or kernel interface with a fixed signature that has no room for a
 *     workspace pointer.
 * Such callers would otherwise lose the shortcut, and their NVFP4 + RMSNorm prepare
 * would recompute every row's statistics in the quantization pass.
 * Limits and rules:
 *   - t > SHARQ_NOALLOC_MAX_ROWS returns SHARQ_ERR_WORKSPACE before anything runs;
 *     use sharq_prepare with a workspace for larger t.
 *   - The first call on a device looks up the scratch's address with that device
 *     current (this may load the library's module there); make it before any
 *     stream capture.  Later calls do no set-up, unless the device's context was
 *     replaced in between (cudaDeviceReset, or a context rebuilt after an error):
 *     the call then notices the new context and looks the address up again, so
 *     the first call after a reset also has to come before any stream capture.
 *   - Nothing in the scratch needs to start at zero (every row read was written by
 *     the same call); the amax accumulator, out->tensor[0], is zeroed on the stream
 *     as in sharq_prepare.
 *   - One scratch per device: calls that overlap on one device (several streams or
 *     host threads) race on it.  Keep them in one stream order. */
sharq_status sharq_prepare_noalloc(const void* x, sharq_dtype x_dt, const void* gamma, float eps, float act_amax,
                                   sharq_prepared* out, sharq_stream stream);

/* The two GEMMs of the layer (SharQ abstract, Section 1): a sparse FP4 GEMM over
 * the compressed backbone and its metadata, and a dense FP4 GEMM over R that
 * accumulates into the same output, one weight load per K tile feeding both:
 *   y[t][n] = g_dec_x * g_dec_w * sum_k (B[t][k] + R[t][k]) * W[n][k]
 * y: t * n row-major, dtype y_dt.  Supported: MXFP4 with every pattern, NVFP4 with
 * 4:8 pair and 8:16 (NVFP4 2:4 returns SHARQ_ERR_UNSUPPORTED: no sparse tensor-core
 * kind takes E4M3 block-16 scales with element-wise 2:4 metadata).  With t = 1 the
 * product is a weight stream and runs on the CUDA cores (same operands and output,
 * fp32 sums in another order; SHARQ_GEMV=0 in the environment keeps the tensor
 * cores).  With 2 <= t <= 64 the weight is the 128-row MMA operand and the rows
 * (padded to 32 or 64) the other one (the backbone expanded to its dense form on
 * chip); each 128-row weight
 * tile's K loop is split over the CTAs of one thread-block cluster (up to 8, as many
 * as keep every cluster resident at once), whose first CTA adds the slices' fp32
 * sums in slice order through distributed shared memory, so the results repeat bit
 * for bit and no workspace is needed (SHARQ_SWAP=0 keeps the activation-as-A
 * kernels). */
sharq_status sharq_linear(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt,
                          sharq_stream stream);

/* sharq_linear with a stream-K workspace.  When the CTA-pair GEMM runs (the 4:8
 * pair kinds, t a multiple of 256 after padding, not grouped) and it has few
 * 256 x 256 output tiles with long K loops (at most half as many tiles as SM
 * pairs, at least 8 K tiles of 256 per pair), the K loops of all tiles are split
 * evenly over every pair: a pair whose share starts inside a tile leaves
 * its partial sums in its workspace slot, and the pair holding that tile's first
 * K tile adds them before writing y.  The single-CTA GEMM (the other shapes) with
 * few tiles and long K loops (at most half as many tiles as SMs, >= 32 K tiles of
 * 256, e.g. decode-size row counts of down_proj) splits each tile's K loop into
 * up to 4 slices on different SMs; each slice writes its raw sums to its own
 * workspace slot and the CTA that completes a tile's last slice adds the slots in
 * slice order and writes y.  Results equal sharq_linear's up to the order of the
 * fp32 partial sums, and repeat bit for bit.  Otherwise it is sharq_linear.
 * workspace: DEVICE, >= sharq_linear_workspace_size() bytes, 16-byte aligned,
 * zero-filled before its first use; every completed call leaves its counters as
 * it found them.  After SHARQ_ERR_TIMEOUT zero it again before reuse.  Calls that
 * overlap in time (several streams) need separate workspaces.
 * SHARQ_ERR_WORKSPACE: NULL, too small or misaligned (checked on the host). */
sharq_status sharq_linear_ws(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt,
                             void* workspace, size_t workspace_bytes, sharq_stream stream);

/* Bytes of sharq_linear_ws's workspace on the current device.  Layout: a fixed
 * counter region first (64 bytes of stream-K counters per pair of SMs, then one
 * 32-bit split-K counter per SM), then the partial sums from a 256-byte boundary
 * on (one 256 KiB stream-K slot per pair of SMs; split-K slices use the same
 * bytes).  No call's partial sums overlap any counter, so one workspace may
 * serve calls of every shape in turn. */
sharq_status sharq_linear_workspace_size(size_t* bytes);

/* Same, with a choice of paths for diagnosis: paths bit 0 = sparse backbone GEMM,
 * bit 1 = dense residual GEMM (3 = the layer). */
sharq_status sharq_linear_paths(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt,
                                int32_t paths, sharq_stream stream);

/* Mixture-of-experts form (SharQ evaluates Qwen3-30B-A3B): a holds the routed rows of
 * all experts, grouped by expert; group_offsets (DEVICE, experts+1 int32, non-decreasing,
 * each a multiple of 128, last = a->t rounded up to 128) delimits expert e's rows
 * [off[e], off[e+1]).  w holds w->experts stacked weights.  Rows of y outside every
 * group are left unwritten. */
sharq_status sharq_linear_grouped(const sharq_prepared* a, const sharq_weight* w, const int32_t* group_offsets,
                                  void* y, sharq_dtype y_dt, sharq_stream stream);

/* sharq_linear_grouped on rows gathered inside the GEMM (SharQ evaluates
 * Qwen3-30B-A3B; every token goes to several experts).  The routed operand is
 * never written out: routed row r (0 <= r < routed_rows) is row rows[r] of the
 * token-prepared buffers `tokens` (from sharq_prepare over the tokens), read
 * by index as each tile's operands are loaded; rows[r] < 0 or >= tokens->t
 * stands for an all-zero input row (the padding rows of an expert's segment).
 * The result equals sharq_gather_prepared(tokens, rows) followed by
 * sharq_linear_grouped, bit for bit.
 * rows: DEVICE, routed_rows int32 values; routed_rows a positive multiple of 128;
 * group_offsets as in sharq_linear_grouped, last = routed_rows; y: routed_rows * n.
 * Supported: NVFP4 with the 4:8 pair pattern (a padding row is encoded with zero
 * E4M3 scales); other formats and patterns return SHARQ_ERR_UNSUPPORTED.  Index
 * values are not checked on the host. */
sharq_status sharq_linear_grouped_gather(const sharq_prepared* tokens, const int32_t* rows, int64_t routed_rows,
                                         const sharq_weight* w, const int32_t* group_offsets, void* y,
                                         sharq_dtype y_dt, sharq_stream stream);

/* Synchronizes the stream, then reports and clears this device's error word. */
sharq_status sharq_sync_status(sharq_stream stream);

/* Test hook for the failure path: launches one block whose wait on a flag that
 * nothing sets gives up after timeout_ns, sets the error word and returns. */
sharq_status sharq_selftest_wait_timeout(uint64_t timeout_ns, sharq_stream stream);

/* Text of the last error on this host thread ("" if none). */
const char* sharq_last_error(void);

/* Number of kernel launches the calls above have made on this host thread since the
 * last reset (for launch accounting in benchmarks). */
uint64_t sharq_launch_count(int reset);

#ifdef __cplusplus
}
#endif
#endif /* SHARQ_H */
