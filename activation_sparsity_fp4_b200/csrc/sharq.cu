// sharq.cu -- C ABI of the SharQ sparse-dense FP4 linear layer for sm_100a.
// One translation unit: the kernels (prep.cuh, gemm.cuh) and the host code
// that validates arguments, encodes TMA descriptors and launches them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>

#include "../../include/sharq.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_swap.cuh"
#include "gemv.cuh"
#include "prep.cuh"

using namespace sharq;

namespace {

thread_local std::string g_last_error;
thread_local uint64_t g_launches = 0;

sharq_status fail(sharq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define SHARQ_CUDA(call)                                                                        \
  do {                                                                                          \
    cudaError_t e_ = (call);                                                                    \
    if (e_ != cudaSuccess) return fail(SHARQ_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

sharq_status launched() {
  g_launches++;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SHARQ_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return SHARQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

int fmt_block(sharq_format f) { return f == SHARQ_NVFP4 ? 16 : 32; }

int64_t meta_row_bytes(int64_t k, sharq_pattern p) {
  return (p == SHARQ_NM_4_8_PAIR || p == SHARQ_NM_8_16_PAIR) ? k / 16 : k / 8;
}

uint64_t wait_timeout_ns() {
  static uint64_t v = [] {
    const char* s = getenv("SHARQ_WAIT_TIMEOUT_NS");
    return s ? strtoull(s, nullptr, 10) : 2000000000ull;
  }();
  return v;
}

// SHARQ_GEMM_PAIRS=0 runs every GEMM on the single-CTA kernel (for comparison).
bool pair_enabled() {
  static const bool v = [] {
    const char* e = getenv("SHARQ_GEMM_PAIRS");
    return !(e && e[0] == '0');
  }();
  return v;
}

// SHARQ_STREAMK=0 keeps whole tiles even when a stream-K workspace is given (for comparison).
bool stream_k_enabled() {
  static const bool v = [] {
    const char* e = getenv("SHARQ_STREAMK");
    return !(e && e[0] == '0');
  }();
  return v;
}

// SHARQ_GEMV=0 runs even 1-4 row products on the tensor-core kernels (for comparison).
bool gemv_enabled() {
  static const bool v = [] {
    const char* e = getenv("SHARQ_GEMV");
    return !(e && e[0] == '0');
  }();
  return v;
}

// SHARQ_SWAP=0 keeps few-row products (2..64 rows) on the activation-as-A kernels (for comparison).
bool swap_enabled() {
  static const bool v = [] {
    const char* e = getenv("SHARQ_SWAP");
    return !(e && e[0] == '0');
  }();
  return v;
}

// SHARQ_PDL=0 launches every kernel with plain stream order (for comparison).
bool pdl_enabled() {
  static const bool v = [] {
    const char* e = getenv("SHARQ_PDL");
    return !(e && e[0] == '0');
  }();
  return v;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream still runs; it calls grid_dep_wait
// before touching global memory another kernel writes.  cluster > 1 also sets
// the cluster shape.
template <typename... KArgs, typename... Args>
sharq_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, unsigned cluster,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    n++;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    n++;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return fail(SHARQ_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return launched();
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Clusters of `csize` CTAs of this kernel that can be resident at once (0 on error).
template <typename Kern>
int max_active_clusters(Kern kern, int threads, size_t smem, int csize) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)csize);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D byte tensor [rows][row_bytes] with a (box_bytes x box_rows) box.
sharq_status make_map(CUtensorMap* map, const void* base, int64_t row_bytes, int64_t rows, int box_bytes, int box_rows,
                      CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SHARQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SHARQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SHARQ_OK;
}

// 2-D tensor of packed E2M1 codes [rows][elems] (two per byte) that TMA expands
// into 8-bit shared-memory containers (16 codes -> 16 bytes); box of 128 codes.
sharq_status make_map_u4(CUtensorMap* map, const void* base, int64_t elems, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SHARQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if (!aligned(base, 32) || (elems / 2) % 32 != 0 || elems % 128 != 0)
    return fail(SHARQ_ERR_INVALID, "unpacked FP4 operand needs 32-byte aligned rows of a multiple of 128 codes");
  cuuint64_t dims[2] = {(cuuint64_t)elems, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(elems / 2)};
  cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SHARQ_ERR_CUDA, "cuTensorMapEncodeTiled (16U4) failed (%d)", (int)r);
  return SHARQ_OK;
}

sharq_status check_shape(int64_t k, int64_t n_or_t, bool is_n) {
  if (k <= 0 || k % 256 != 0) return fail(SHARQ_ERR_INVALID, "k=%lld must be a positive multiple of 256", (long long)k);
  if (k > 16384) return fail(SHARQ_ERR_UNSUPPORTED, "k=%lld above 16384", (long long)k);
  if (is_n && (n_or_t <= 0 || n_or_t % 256 != 0))
    return fail(SHARQ_ERR_INVALID, "n=%lld must be a positive multiple of 256", (long long)n_or_t);
  if (!is_n && n_or_t <= 0) return fail(SHARQ_ERR_INVALID, "t=%lld must be positive", (long long)n_or_t);
  return SHARQ_OK;
}

// ---------------------------------------------------------------- launchers
// Blocks of 128 threads handle 128 / tpr rows at a time (tpr threads per row,
// see RowMap); as many resident blocks as the SMs hold, striding over rows.
struct RowLaunch {
  unsigned grid;
  int tpr;
};
// The occupancy is looked up once per kernel (a template argument, so that
// kernels of one signature keep separate figures).
template <auto Kern>
RowLaunch row_launch(int64_t rows, int64_t k) {
  static std::atomic<int> cached{0};
  int per_sm = cached.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, Kern, 128, 0) != cudaSuccess || per_sm < 1) {
      (void)cudaGetLastError();
      per_sm = 1;
    }
    cached.store(per_sm, std::memory_order_relaxed);
  }
  const int64_t cap = (int64_t)sm_count() * per_sm;
  const int tpr = rows_tpr(k / 32, rows, cap);
  const int64_t rpb = 128 / tpr;
  const int64_t groups = (rows + rpb - 1) / rpb;
  return RowLaunch{(unsigned)(groups < cap ? groups : cap), tpr};
}

template <int FMT, int PAT, bool NORM, bool XBF16>
sharq_status launch_prep(const PrepParams& pp, cudaStream_t s) {
  auto kern = prep_kernel<FMT, PAT, NORM, XBF16>;
  PrepParams q = pp;
  const RowLaunch rl = row_launch<prep_kernel<FMT, PAT, NORM, XBF16>>(pp.t_pad, pp.k);
  q.tpr = rl.tpr;
  return launch_ex(kern, dim3(rl.grid), dim3(128), 0, s, 1, q);
}

template <bool NORM, bool XBF16>
sharq_status launch_amax(const void* x, const void* gamma, float eps, int64_t t, int64_t k, float* out,
                         float* rstd_out, cudaStream_t s) {
  if (XBF16 && k <= 4096) {  // two warps per row, the row in registers, two rows per block
    amax_rows_kernel<NORM><<<(unsigned)((t + 1) / 2), 128, 0, s>>>(x, gamma, eps, t, k, out, rstd_out);
    return launched();
  }
  auto kern = amax_kernel<NORM, XBF16>;
  const RowLaunch rl = row_launch<amax_kernel<NORM, XBF16>>(t, k);
  kern<<<rl.grid, 128, 0, s>>>(x, gamma, eps, t, k, out, rstd_out, nullptr, rl.tpr);
  return launched();
}

template <int FMT, int PAT, bool NORM>
sharq_status prep_dispatch_x(const PrepParams& pp, bool xbf16, cudaStream_t s) {
  return xbf16 ? launch_prep<FMT, PAT, NORM, true>(pp, s) : launch_prep<FMT, PAT, NORM, false>(pp, s);
}
template <int FMT, int PAT>
sharq_status prep_dispatch_n(const PrepParams& pp, bool norm, bool xbf16, cudaStream_t s) {
  return norm ? prep_dispatch_x<FMT, PAT, true>(pp, xbf16, s) : prep_dispatch_x<FMT, PAT, false>(pp, xbf16, s);
}
template <int FMT>
sharq_status prep_dispatch_p(const PrepParams& pp, int pat, bool norm, bool xbf16, cudaStream_t s) {
  switch (pat) {
    case PAT_24: return prep_dispatch_n<FMT, PAT_24>(pp, norm, xbf16, s);
    case PAT_48P: return prep_dispatch_n<FMT, PAT_48P>(pp, norm, xbf16, s);
    case PAT_816P: return prep_dispatch_n<FMT, PAT_816P>(pp, norm, xbf16, s);
    default: return prep_dispatch_n<FMT, PAT_816>(pp, norm, xbf16, s);
  }
}

// SwiGLU form (no RMSNorm): h = SiLU(x) * x2 inside the prep and amax kernels.
template <int FMT, int PAT, bool XBF16>
sharq_status launch_prep_swiglu(const PrepParams& pp, cudaStream_t s) {
  auto kern = prep_kernel<FMT, PAT, false, XBF16, true>;
  const RowLaunch rl = row_launch<prep_kernel<FMT, PAT, false, XBF16, true>>(pp.t_pad, pp.k);
  PrepParams q = pp;
  q.tpr = rl.tpr;
  return launch_ex(kern, dim3(rl.grid), dim3(128), 0, s, 1, q);
}
template <int FMT, int PAT>
sharq_status swiglu_dispatch_x(const PrepParams& pp, bool xbf16, cudaStream_t s) {
  return xbf16 ? launch_prep_swiglu<FMT, PAT, true>(pp, s) : launch_prep_swiglu<FMT, PAT, false>(pp, s);
}
template <int FMT>
sharq_status swiglu_dispatch_p(const PrepParams& pp, int pat, bool xbf16, cudaStream_t s) {
  switch (pat) {
    case PAT_24: return swiglu_dispatch_x<FMT, PAT_24>(pp, xbf16, s);
    case PAT_48P: return swiglu_dispatch_x<FMT, PAT_48P>(pp, xbf16, s);
    case PAT_816P: return swiglu_dispatch_x<FMT, PAT_816P>(pp, xbf16, s);
    default: return swiglu_dispatch_x<FMT, PAT_816>(pp, xbf16, s);
  }
}
template <bool XBF16>
sharq_status launch_amax_swiglu(const void* gate, const void* up, int64_t t, int64_t k, float* out, cudaStream_t s) {
  auto kern = amax_kernel<false, XBF16, true>;
  const RowLaunch rl = row_launch<amax_kernel<false, XBF16, true>>(t, k);
  kern<<<rl.grid, 128, 0, s>>>(gate, nullptr, 0.0f, t, k, out, nullptr, up, rl.tpr);
  return launched();
}

// cudaFuncSetAttribute acts on the current device's context: a kernel's
// dynamic shared-memory limit is raised once per (kernel, device).
template <auto Kern>
sharq_status ensure_smem_limit(int bytes) {
  static std::atomic<uint64_t> done{0};  // bit d: set on device d
  int dev = 0;
  SHARQ_CUDA(cudaGetDevice(&dev));
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return SHARQ_OK;
  SHARQ_CUDA(cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (bit) done.fetch_or(bit, std::memory_order_release);
  return SHARQ_OK;
}

template <int KIND, bool SPARSE, bool SPLIT = false, bool GATHER = false>
sharq_status launch_gemm(const GemmMaps& maps, const GemmParams& gp, cudaStream_t s) {
  using C = GemmCfg<KIND, SPARSE>;
  sharq_status st = ensure_smem_limit<gemm_kernel<KIND, SPARSE, SPLIT, GATHER>>(C::kSmemBytes);
  if (st != SHARQ_OK) return st;
  const int items = (int)(gp.t_pad / C::BM) * (int)(gp.n / C::BN) * (SPLIT ? gp.split : 1);
  const int sms = sm_count();
  dim3 grid(items < sms ? items : sms);
  return launch_ex(gemm_kernel<KIND, SPARSE, SPLIT, GATHER>, grid, dim3(448), C::kSmemBytes, s, 1, maps, gp);
}

// Workspace of sharq_linear_ws.  Every counter sits in a fixed region at the
// start, so that no call's partial sums can land on another call's counters
// whatever the shapes of the calls that share the workspace:
//   [0, npairs * kSkFlagBytes)        stream-K counters (CTA-pair GEMM): one per
//                                     (pair, CTA, epilogue warp);
//   [.., + sms * 4)                   split-K counters (single-CTA GEMM): one per
//                                     tile (split-K runs at most sms / 2 tiles);
//   [ws_data_offset(), end)           partial sums: a stream-K slot of
//                                     kSkSlotBytes per pair, or the split-K
//                                     slices (one fp32 [t_pad][n] slot each).
constexpr size_t kSkSlotBytes = 2 * 8 * 32 * 128 * sizeof(float);
constexpr size_t kSkFlagBytes = 2 * 8 * sizeof(uint32_t);
size_t ws_split_cnt_offset() { return (size_t)(sm_count() / 2) * kSkFlagBytes; }
size_t ws_data_offset() { return (size_t)round_up((int64_t)(ws_split_cnt_offset() + sm_count() * sizeof(uint32_t)), 256); }
size_t sk_workspace_bytes() { return ws_data_offset() + (size_t)(sm_count() / 2) * kSkSlotBytes; }

// Split-K of the single-CTA GEMM for few tiles with long K loops: slices per
// tile so that the work items fill the SMs, each slice at least 4 K tiles, at
// most kMaxSplit slices.
// Returns 0 (no split) when it does not apply or the workspace is too small.
template <int KIND, bool SPARSE>
int split_for(const GemmParams& gp, size_t ws_bytes) {
  using C = GemmCfg<KIND, SPARSE>;
  const int64_t tiles = (gp.t_pad / C::BM) * (gp.n / C::BN);
  const int64_t k_tiles = gp.k / C::BK;
  const int sms = sm_count();
  // measured on B200: down_proj (k = 14336, 56 K tiles) at 1..256 rows 2.2-1.4x faster;
  // q_proj (16 K tiles) gains at 1-16 rows but loses at 64, so short K loops stay whole
  if (gp.experts > 1 || 2 * tiles > sms || k_tiles < 32) return 0;
  int64_t split = sms / tiles;
  if (split > k_tiles / 4) split = k_tiles / 4;
  if (split > kMaxSplit) split = kMaxSplit;
  const size_t slot = (size_t)gp.t_pad * gp.n * sizeof(float);
  while (split >= 2 && ws_data_offset() + (size_t)split * slot > ws_bytes) split--;  // one slot per slice must fit
  return split >= 2 ? (int)split : 0;
}

template <int KIND, bool SPARSE>
sharq_status launch_gemm_ws(const GemmMaps& maps, GemmParams gp, cudaStream_t s, void* ws, size_t ws_bytes) {
  const int split = ws ? split_for<KIND, SPARSE>(gp, ws_bytes) : 0;
  if (split < 2) return launch_gemm<KIND, SPARSE>(maps, gp, s);
  gp.split = split;
  gp.split_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ws_data_offset());
  gp.split_cnt = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + ws_split_cnt_offset());
  return launch_gemm<KIND, SPARSE, true>(maps, gp, s);
}

sharq_status check_prepared(const sharq_prepared* a) {
  if (!a) return fail(SHARQ_ERR_INVALID, "prepared activations: NULL");
  sharq_status st = check_shape(a->k, a->t, false);
  if (st != SHARQ_OK) return st;
  if (a->fmt != SHARQ_MXFP4 && a->fmt != SHARQ_NVFP4) return fail(SHARQ_ERR_INVALID, "bad format %d", (int)a->fmt);
  if (a->pat < SHARQ_NM_2_4 || a->pat > SHARQ_NM_8_16_PAIR) return fail(SHARQ_ERR_INVALID, "bad pattern %d", (int)a->pat);
  const void* ptrs[6] = {a->meta, a->bb_codes, a->bb_scales, a->res_codes, a->res_scales, a->tensor};
  for (int i = 0; i < 6; i++) {
    if (!ptrs[i]) return fail(SHARQ_ERR_INVALID, "prepared buffer %d is NULL", i);
    if (!aligned(ptrs[i], 16)) return fail(SHARQ_ERR_INVALID, "prepared buffer %d is not 16-byte aligned", i);
  }
  return SHARQ_OK;
}

sharq_status check_weight(const sharq_weight* w) {
  if (!w) return fail(SHARQ_ERR_INVALID, "weight: NULL");
  sharq_status st = check_shape(w->k, w->n, true);
  if (st != SHARQ_OK) return st;
  if (w->fmt != SHARQ_MXFP4 && w->fmt != SHARQ_NVFP4) return fail(SHARQ_ERR_INVALID, "bad format %d", (int)w->fmt);
  if (w->experts < 1) return fail(SHARQ_ERR_INVALID, "experts=%d", (int)w->experts);
  const void* ptrs[4] = {w->codes, w->scales_dense, w->scales_sparse, w->tensor};
  for (int i = 0; i < 4; i++) {
    if (!ptrs[i]) return fail(SHARQ_ERR_INVALID, "weight buffer %d is NULL", i);
    if (!aligned(ptrs[i], 16)) return fail(SHARQ_ERR_INVALID, "weight buffer %d is not 16-byte aligned", i);
  }
  return SHARQ_OK;
}

// Clusters of the CTA-pair GEMM that can be resident at once on this device (0 if unknown).
template <int KIND>
int pair_max_resident() {
  static int v = -1;
  if (v < 0) {
    using C = PairCfg<KIND>;
    if (ensure_smem_limit<gemm_pair_kernel<KIND, true>>(C::kSmemBytes) != SHARQ_OK) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sm_count() & ~1));
    cfg.blockDim = dim3(448);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<KIND, true>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    v = n;
  }
  return v;
}

// CTA-pair GEMM: clusters of 2 CTAs, one per SM, persistent over 256 x BN tiles.
template <int KIND>
sharq_status launch_pair(const GemmMaps& maps, const GemmParams& gp, cudaStream_t s) {
  using C = PairCfg<KIND>;
  sharq_status st = ensure_smem_limit<gemm_pair_kernel<KIND, false>>(C::kSmemBytes);
  if (st != SHARQ_OK) return st;
  st = ensure_smem_limit<gemm_pair_kernel<KIND, true>>(C::kSmemBytes);
  if (st != SHARQ_OK) return st;
  const int tiles = (int)(gp.t_pad / 256) * (int)(gp.n / C::BN);
  const int pairs = sm_count() / 2;
  int clusters = tiles < pairs ? tiles : pairs;
  if (gp.sk_part) {
    // stream-K: as many pairs as can be resident at once (a pair waits for the
    // partial sums of the pairs after it), and at least two K tiles per pair
    const int64_t units = (int64_t)tiles * (gp.k / C::BK);
    clusters = pair_max_resident<KIND>();
    if (clusters > pairs) clusters = pairs;
    if (units < 2 * (int64_t)clusters) clusters = (int)(units / 2);
  }
  if (gp.sk_part)
    return launch_ex(gemm_pair_kernel<KIND, true>, dim3((unsigned)(2 * clusters)), dim3(448), C::kSmemBytes, s, 2,
                     maps, gp);
  return launch_ex(gemm_pair_kernel<KIND, false>, dim3((unsigned)(2 * clusters)), dim3(448), C::kSmemBytes, s, 2,
                   maps, gp);
}

// The 1-4 row form on the CUDA cores (gemv.cuh).
template <int FMT, int PAT>
sharq_status launch_gemv(const GemvParams& gp, int64_t t, cudaStream_t s) {
  constexpr int rows_per_block = kGemvWarps * kGemvRowsPerWarp;
  const dim3 grid((unsigned)((gp.n + rows_per_block - 1) / rows_per_block)), block(kGemvWarps * 32);
  switch (t) {
    case 1: return launch_ex(gemv_kernel<FMT, PAT, 1>, grid, block, 0, s, 1, gp);
    case 2: return launch_ex(gemv_kernel<FMT, PAT, 2>, grid, block, 0, s, 1, gp);
    case 3: return launch_ex(gemv_kernel<FMT, PAT, 3>, grid, block, 0, s, 1, gp);
    default: return launch_ex(gemv_kernel<FMT, PAT, 4>, grid, block, 0, s, 1, gp);
  }
}

sharq_status run_gemv(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt, int32_t paths,
                      cudaStream_t s) {
  GemvParams gp;
  gp.n = w->n;
  gp.k = w->k;
  gp.paths = paths;
  gp.meta = static_cast<const uint8_t*>(a->meta);
  gp.bb_codes = static_cast<const uint8_t*>(a->bb_codes);
  gp.bb_scales = static_cast<const uint8_t*>(a->bb_scales);
  gp.res_codes = static_cast<const uint8_t*>(a->res_codes);
  gp.res_scales = static_cast<const uint8_t*>(a->res_scales);
  gp.t_pad = round_up(a->t, 128);
  gp.tensor_x = a->tensor;
  gp.w_codes = static_cast<const uint8_t*>(w->codes);
  gp.w_sf = static_cast<const uint8_t*>(w->scales_sparse);
  gp.tensor_w = w->tensor;
  gp.y = y;
  gp.y_bf16 = y_dt == SHARQ_BF16;
  const int64_t t = a->t;
  if (a->fmt == SHARQ_NVFP4)
    return a->pat == SHARQ_NM_8_16 ? launch_gemv<FMT_NV, PAT_816>(gp, t, s) : launch_gemv<FMT_NV, PAT_48P>(gp, t, s);
  switch (a->pat) {
    case SHARQ_NM_2_4: return launch_gemv<FMT_MX, PAT_24>(gp, t, s);
    case SHARQ_NM_4_8_PAIR:
    case SHARQ_NM_8_16_PAIR: return launch_gemv<FMT_MX, PAT_48P>(gp, t, s);  // the 4:8 pair layout
    default: return launch_gemv<FMT_MX, PAT_816>(gp, t, s);
  }
}

// Few rows: the weight as the 128-row MMA operand (gemm_swap.cuh), the K loop of
// each 128-row weight tile split over the CTAs of a cluster.  Measured on B200
// (GEMM alone, down_proj, back-to-back over rotating weights): 2 rows 16.2 us,
// 16 rows 16.9 us, 33-64 rows 22.0-22.6 us against 27.7-28.2 us for the
// activation-as-A split-K kernel; at 1 row the CUDA-core form is faster, so it
// serves 2..64 rows (activation tiles of 32 or 64 columns).
constexpr int64_t kSwapMinRows = 2, kSwapMaxRows = 64;
template <int KIND, int BL, int TN>
sharq_status launch_swap(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt, cudaStream_t s) {
  using C = SwapCfg<KIND, BL, TN>;
  sharq_status st0 = ensure_smem_limit<gemm_swap_kernel<KIND, BL, TN>>(C::kSmemBytes);
  if (st0 != SHARQ_OK) return st0;
  const int64_t t_pad = round_up(a->t, 128), k = w->k;
  SwapMaps maps;
  memset(&maps, 0, sizeof(maps));
  sharq_status st = make_map(&maps.w, w->codes, k / 2, w->n, 128, C::BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SHARQ_OK) return st;
  st = make_map(&maps.r, a->res_codes, k / 2, t_pad, 128, TN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SHARQ_OK) return st;
  if (BL == SW_DENSE) {
    st = make_map(&maps.c, a->bb_codes, k / 2, t_pad, 128, TN, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    st = make_map(&maps.c, a->bb_codes, k / 4, t_pad, C::kCRow, TN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != SHARQ_OK) return st;
    st = make_map(&maps.e, a->meta, meta_row_bytes(k, a->pat), t_pad, C::kMetaRow, TN, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (st != SHARQ_OK) return st;
  SwapParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.t = a->t;
  sp.n = w->n;
  sp.k = k;
  sp.k_tiles = k / C::BK;
  sp.w_codes = static_cast<const uint8_t*>(w->codes);
  sp.sf_w = static_cast<const uint8_t*>(w->scales_dense);
  sp.sf_res = static_cast<const uint8_t*>(a->res_scales);
  sp.sf_bb = static_cast<const uint8_t*>(a->bb_scales);
  sp.tensor_x = a->tensor;
  sp.tensor_w = w->tensor;
  sp.y = y;
  sp.y_bf16 = y_dt == SHARQ_BF16;
  sp.timeout_ns = wait_timeout_ns();
  const int64_t tiles = w->n / C::BM;
  const int sms = sm_count();
  // K slices per weight tile = CTAs per cluster: enough work items for every
  // SM, at least two K tiles each, at most 8 (the portable cluster size), and
  // only as many as let every cluster be resident at once
  int64_t split = 1;
  if (tiles <= sms) {
    split = sms / tiles;
    if (split > sp.k_tiles / 2) split = sp.k_tiles / 2;
    if (split > 8) split = 8;
    static int resident[9] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};  // clusters of each size (per device kind)
    auto fits = [&](int64_t cs) {
      if (resident[cs] < 0) resident[cs] = max_active_clusters(gemm_swap_kernel<KIND, BL, TN>, 192, C::kSmemBytes, (int)cs);
      return resident[cs] >= tiles;
    };
    while (split > 1 && !fits(split)) split--;
    if (split < 1) split = 1;
  }
  sp.split = (int32_t)split;
  return launch_ex(gemm_swap_kernel<KIND, BL, TN>, dim3((unsigned)(tiles * split)), dim3(192), C::kSmemBytes, s,
                   (unsigned)split, maps, sp);
}

template <int KIND, int BL>
sharq_status swap_rows(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt, cudaStream_t s) {
  static_assert(kSwapMaxRows <= 64, "activation tile widths 32 and 64");
  if (a->t > 32) return launch_swap<KIND, BL, 64>(a, w, y, y_dt, s);
  return launch_swap<KIND, BL, 32>(a, w, y, y_dt, s);
}

sharq_status run_swap(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt, cudaStream_t s) {
  const bool pair = a->pat == SHARQ_NM_4_8_PAIR || a->pat == SHARQ_NM_8_16_PAIR;
  if (a->fmt == SHARQ_NVFP4)
    return pair ? swap_rows<GK_NVF4, SW_PAIR>(a, w, y, y_dt, s) : swap_rows<GK_NVF4, SW_DENSE>(a, w, y, y_dt, s);
  if (pair) return swap_rows<GK_MXF4, SW_PAIR>(a, w, y, y_dt, s);
  return a->pat == SHARQ_NM_2_4 ? swap_rows<GK_MXF4, SW_24>(a, w, y, y_dt, s)
                                : swap_rows<GK_MXF4, SW_DENSE>(a, w, y, y_dt, s);
}

sharq_status run_linear(const sharq_prepared* a, const sharq_weight* w, const int32_t* offsets, void* y,
                        sharq_dtype y_dt, int32_t paths, cudaStream_t s, void* ws = nullptr, size_t ws_bytes = 0) {
  sharq_status st = check_prepared(a);
  if (st != SHARQ_OK) return st;
  st = check_weight(w);
  if (st != SHARQ_OK) return st;
  if (a->k != w->k) return fail(SHARQ_ERR_INVALID, "k mismatch: activations %lld, weight %lld", (long long)a->k,
                                (long long)w->k);
  if (a->fmt != w->fmt) return fail(SHARQ_ERR_INVALID, "format mismatch between activations and weight");
  if (!y || !aligned(y, 16)) return fail(SHARQ_ERR_INVALID, "y must be a 16-byte aligned device pointer");
  if (y_dt != SHARQ_F32 && y_dt != SHARQ_BF16) return fail(SHARQ_ERR_INVALID, "bad y dtype %d", (int)y_dt);
  if (paths < 1 || paths > 3) return fail(SHARQ_ERR_INVALID, "paths=%d", (int)paths);
  if (offsets == nullptr && w->experts != 1)
    return fail(SHARQ_ERR_INVALID, "a stacked weight needs sharq_linear_grouped");
  if (a->fmt == SHARQ_NVFP4 && a->pat == SHARQ_NM_2_4)
    return fail(SHARQ_ERR_UNSUPPORTED, "NVFP4 with element-wise 2:4 has no sparse tensor-core kind");
  const bool swap = offsets == nullptr && a->t >= kSwapMinRows && a->t <= kSwapMaxRows && paths == 3 && swap_enabled();
  if (offsets == nullptr && a->t <= kGemvMaxRows && gemv_enabled() && !swap) return run_gemv(a, w, y, y_dt, paths, s);
  if (swap) {
    if (ws && (ws_bytes < sk_workspace_bytes() || !aligned(ws, 16)))
      return fail(SHARQ_ERR_WORKSPACE, "workspace: %zu bytes, 16-byte aligned, needed", sk_workspace_bytes());
    return run_swap(a, w, y, y_dt, s);
  }

  const int64_t t_pad = round_up(a->t, 128);
  const bool sparse = a->pat != SHARQ_NM_8_16;
  const bool unpacked = a->fmt == SHARQ_MXFP4 && a->pat == SHARQ_NM_2_4;  // kind::mxf8f6f4
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (unpacked) {
    st = make_map_u4(&maps.w, w->codes, w->k, w->n * w->experts, GemmCfg<GK_MXF8, true>::BN);
    if (st != SHARQ_OK) return st;
    st = make_map_u4(&maps.r, a->res_codes, a->k, t_pad, 128);
    if (st != SHARQ_OK) return st;
    st = make_map_u4(&maps.b, a->bb_codes, a->k / 2, t_pad, 128);
    if (st != SHARQ_OK) return st;
    st = make_map(&maps.e, a->meta, meta_row_bytes(a->k, a->pat), t_pad, 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != SHARQ_OK) return st;
  } else {
    st = make_map(&maps.w, w->codes, w->k / 2, w->n * w->experts, 128, 256, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SHARQ_OK) return st;
    st = make_map(&maps.r, a->res_codes, a->k / 2, t_pad, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SHARQ_OK) return st;
    if (sparse) {
      st = make_map(&maps.b, a->bb_codes, a->k / 4, t_pad, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B);
      if (st != SHARQ_OK) return st;
      st = make_map(&maps.e, a->meta, meta_row_bytes(a->k, a->pat), t_pad, 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (st != SHARQ_OK) return st;
    } else {
      st = make_map(&maps.b, a->bb_codes, a->k / 2, t_pad, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
      if (st != SHARQ_OK) return st;
    }
  }
  const bool pairs = sparse && !unpacked && offsets == nullptr && t_pad % 256 == 0 && pair_enabled();
  if (y_dt == SHARQ_BF16) {
    // output tiles of 32 rows x 32 (CTA pairs) or 16 bf16 columns; rows t.. are outside the map
    st = make_map(&maps.y, y, w->n * 2, a->t, pairs ? 64 : 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != SHARQ_OK) return st;
  }
  GemmParams gp;
  gp.t = a->t;
  gp.t_pad = t_pad;
  gp.n = w->n;
  gp.k = w->k;
  gp.experts = w->experts;
  gp.group_offsets = offsets;
  gp.sf_res = static_cast<const uint8_t*>(a->res_scales);
  gp.sf_bb = static_cast<const uint8_t*>(a->bb_scales);
  gp.sf_w_dense = static_cast<const uint8_t*>(w->scales_dense);
  gp.sf_w_sparse = static_cast<const uint8_t*>(w->scales_sparse);
  gp.tensor_x = a->tensor;
  gp.tensor_w = w->tensor;
  gp.w_codes = w->codes;
  gp.y = y;
  gp.y_bf16 = y_dt == SHARQ_BF16;
  gp.paths = paths;
  gp.timeout_ns = wait_timeout_ns();
  gp.sk_part = nullptr;
  gp.sk_flag = nullptr;
  gp.split_acc = nullptr;
  gp.split_cnt = nullptr;
  gp.split = 0;
  gp.gather_rows = nullptr;
  gp.gather_src_t = gp.gather_src_tpad = 0;
  gp.g_res_codes = gp.g_bb_codes = gp.g_meta = nullptr;
  if (ws) {
    if (ws_bytes < sk_workspace_bytes() || !aligned(ws, 16))
      return fail(SHARQ_ERR_WORKSPACE, "stream-K workspace: %zu bytes, 16-byte aligned, needed",
                  sk_workspace_bytes());
  }
  if (pairs) {
    // CTA pairs: each SM loads half of every weight tile (boxes of BNh weight rows)
    constexpr int kPairBN = PairCfg<GK_NVF4>::BN, kPairBNh = PairCfg<GK_NVF4>::BNh;
    static_assert(kPairBN == PairCfg<GK_MXF4>::BN && kPairBNh == PairCfg<GK_MXF4>::BNh, "one pair tile shape");
    st = make_map(&maps.w, w->codes, w->k / 2, w->n, 128, kPairBNh, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SHARQ_OK) return st;
    const int64_t tiles = (t_pad / 256) * (w->n / kPairBN);
    const int npairs = sm_count() / 2;
    const int resident = a->fmt == SHARQ_NVFP4 ? pair_max_resident<GK_NVF4>() : pair_max_resident<GK_MXF4>();
    const int np = resident < npairs ? resident : npairs;
    const int64_t units = tiles * (w->k / 256);
    if (ws && stream_k_enabled() && np > 0 && 2 * tiles <= np && units >= 8 * (int64_t)np) {
      // few tiles with long K loops (most pairs would idle): split the K loops
      // of all tiles evenly over every pair (stream-K).  Measured on B200: at
      // 256 x 4096 x 16384 it takes 44 instead of 54 us; with more tiles or
      // shorter K the extra segment boundaries and the partial sums cost more
      // than the balance gains (2048 x 4096 x 4096: 41 instead of 35 us)
      gp.sk_part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ws_data_offset());
      gp.sk_flag = reinterpret_cast<uint32_t*>(ws);
    }
    return a->fmt == SHARQ_NVFP4 ? launch_pair<GK_NVF4>(maps, gp, s) : launch_pair<GK_MXF4>(maps, gp, s);
  }
  if (a->fmt == SHARQ_NVFP4)
    return sparse ? launch_gemm_ws<GK_NVF4, true>(maps, gp, s, ws, ws_bytes)
                  : launch_gemm_ws<GK_NVF4, false>(maps, gp, s, ws, ws_bytes);
  if (unpacked) return launch_gemm_ws<GK_MXF8, true>(maps, gp, s, ws, ws_bytes);
  return sparse ? launch_gemm_ws<GK_MXF4, true>(maps, gp, s, ws, ws_bytes)
                : launch_gemm_ws<GK_MXF4, false>(maps, gp, s, ws, ws_bytes);
}

}  // namespace

// Scratch of sharq_prepare_noalloc: one float (a row's RMSNorm factor) per row
// for at most SHARQ_NOALLOC_MAX_ROWS rows, 256 KiB per device.  It is part of
// the module image, so the driver places it when the module loads and no call
// allocates it.  No entry of it has to start at zero: the amax pass writes the
// factor of every row 0..t-1 before the quantization pass reads it, and rows
// from t up are never read.
static __device__ __align__(256) float g_noalloc_rstd[SHARQ_NOALLOC_MAX_ROWS];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocMaxDevices] = {};  // id of the context the address belongs to

// Unique id of the calling thread's current CUDA context (cuCtxGetId, through
// the runtime's driver entry points); 0 if it cannot be read.  A device reset
// destroys the primary context, and the one created after it has a new id.
unsigned long long current_ctx_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<GetCurrentFn>(p);
  }();
  static GetIdFn get_id = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<GetIdFn>(p);
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the current device's copy of g_noalloc_rstd, looked up
// with that device current and cached together with the id of the context it
// belongs to.  The lookup runs on the first call on a device and again after
// the device's context was replaced (cudaDeviceReset, or a context rebuilt
// after an error: the module is loaded afresh and the old address is gone).
// A lookup may load the module on that device, which is why the first call
// on a device (and the first one after a reset) has to come before any
// stream capture.
sharq_status noalloc_scratch(float** out) {
  int dev = -1;
  SHARQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(SHARQ_ERR_INVALID, "device %d is beyond the %d devices the static scratch tracks", dev,
                kNoAllocMaxDevices);
  // before the device's first runtime call there is no current context (id 0):
  // the lookup below creates it, and its id is read afterwards
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    SHARQ_CUDA(cudaGetSymbolAddress(&p, g_noalloc_rstd));
    g_noalloc_ptr[dev] = static_cast<float*>(p);
    g_noalloc_ctx[dev] = current_ctx_id();
  }
  *out = g_noalloc_ptr[dev];
  return SHARQ_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

sharq_status sharq_weight_sizes(int64_t n, int64_t k, sharq_format fmt, size_t* codes_bytes,
                                size_t* scales_dense_bytes, size_t* scales_sparse_bytes) {
  sharq_status st = check_shape(k, n, true);
  if (st != SHARQ_OK) return st;
  if (fmt != SHARQ_MXFP4 && fmt != SHARQ_NVFP4) return fail(SHARQ_ERR_INVALID, "bad format %d", (int)fmt);
  const int b = fmt_block(fmt);
  if (codes_bytes) *codes_bytes = (size_t)(n * k / 2);
  if (scales_dense_bytes) *scales_dense_bytes = (size_t)tiled_sf_bytes(n, k / b);
  if (scales_sparse_bytes) *scales_sparse_bytes = (size_t)tiled_sf_bytes(n, k / (2 * b));
  return SHARQ_OK;
}

sharq_status sharq_prepared_sizes(int64_t t, int64_t k, sharq_format fmt, sharq_pattern pat, size_t* meta_bytes,
                                  size_t* bb_codes_bytes, size_t* bb_scales_bytes, size_t* res_codes_bytes,
                                  size_t* res_scales_bytes, size_t* workspace_bytes) {
  sharq_status st = check_shape(k, t, false);
  if (st != SHARQ_OK) return st;
  if (fmt != SHARQ_MXFP4 && fmt != SHARQ_NVFP4) return fail(SHARQ_ERR_INVALID, "bad format %d", (int)fmt);
  if (pat < SHARQ_NM_2_4 || pat > SHARQ_NM_8_16_PAIR) return fail(SHARQ_ERR_INVALID, "bad pattern %d", (int)pat);
  const int64_t tp = round_up(t, 128);
  const int b = fmt_block(fmt);
  if (meta_bytes) *meta_bytes = (size_t)(tp * meta_row_bytes(k, pat));
  if (bb_codes_bytes) *bb_codes_bytes = (size_t)(pat == SHARQ_NM_8_16 ? tp * k / 2 : tp * k / 4);
  if (bb_scales_bytes) *bb_scales_bytes = (size_t)tiled_sf_bytes(tp, pat == SHARQ_NM_8_16 ? k / b : k / (2 * b));
  if (res_codes_bytes) *res_codes_bytes = (size_t)(tp * k / 2);
  if (res_scales_bytes) *res_scales_bytes = (size_t)tiled_sf_bytes(tp, k / b);
  if (workspace_bytes) *workspace_bytes = (size_t)(tp * sizeof(float));  // per-row RMSNorm factors
  return SHARQ_OK;
}

sharq_status sharq_quantize_weight(const void* w, sharq_dtype w_dt, sharq_weight* out, sharq_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!w || !aligned(w, 16)) return fail(SHARQ_ERR_INVALID, "w must be a 16-byte aligned device pointer");
  if (w_dt != SHARQ_F32 && w_dt != SHARQ_BF16) return fail(SHARQ_ERR_INVALID, "bad w dtype %d", (int)w_dt);
  sharq_status st = check_weight(out);
  if (st != SHARQ_OK) return st;
  const int64_t rows = out->n * out->experts;
  SHARQ_CUDA(cudaMemsetAsync(out->tensor, 0, sizeof(float) * 3 * out->experts, s));
  const bool bf16 = w_dt == SHARQ_BF16;
  if (out->fmt == SHARQ_NVFP4) {
    const int bpe = 64;
    dim3 grid((unsigned)(out->experts * bpe));
    if (bf16) weight_amax_kernel<true><<<grid, 256, 0, s>>>(w, out->n, out->k, out->tensor, bpe);
    else weight_amax_kernel<false><<<grid, 256, 0, s>>>(w, out->n, out->k, out->tensor, bpe);
    st = launched();
    if (st != SHARQ_OK) return st;
  }
  WeightParams wp;
  wp.w = w;
  wp.n = out->n;
  wp.k = out->k;
  wp.rows = rows;
  wp.codes = static_cast<uint8_t*>(out->codes);
  wp.sf_dense = static_cast<uint8_t*>(out->scales_dense);
  wp.sf_sparse = static_cast<uint8_t*>(out->scales_sparse);
  wp.tensor = out->tensor;
  const int64_t threads = rows * (out->k / 32);
  dim3 grid((unsigned)((threads + 255) / 256));
  if (out->fmt == SHARQ_NVFP4) {
    if (bf16) weight_kernel<FMT_NV, true><<<grid, 256, 0, s>>>(wp);
    else weight_kernel<FMT_NV, false><<<grid, 256, 0, s>>>(wp);
  } else {
    if (bf16) weight_kernel<FMT_MX, true><<<grid, 256, 0, s>>>(wp);
    else weight_kernel<FMT_MX, false><<<grid, 256, 0, s>>>(wp);
  }
  return launched();
}

sharq_status sharq_prepare(const void* x, sharq_dtype x_dt, const void* gamma, float eps, float act_amax,
                           sharq_prepared* out, void* workspace, size_t workspace_bytes, sharq_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sharq_status st = check_prepared(out);
  if (st != SHARQ_OK) return st;
  if (!x || !aligned(x, 16)) return fail(SHARQ_ERR_INVALID, "x must be a 16-byte aligned device pointer");
  if (gamma && !aligned(gamma, 16)) return fail(SHARQ_ERR_INVALID, "gamma must be 16-byte aligned");
  if (x_dt != SHARQ_F32 && x_dt != SHARQ_BF16) return fail(SHARQ_ERR_INVALID, "bad x dtype %d", (int)x_dt);
  if (!(eps >= 0.0f)) return fail(SHARQ_ERR_INVALID, "eps must be >= 0");
  const bool bf16 = x_dt == SHARQ_BF16, norm = gamma != nullptr;
  PrepParams pp;
  pp.x = x;
  pp.x2 = nullptr;
  pp.gamma = gamma;
  pp.eps = eps;
  pp.t = out->t;
  pp.t_pad = round_up(out->t, 128);
  pp.k = out->k;
  pp.meta = static_cast<uint8_t*>(out->meta);
  pp.bb_codes = static_cast<uint8_t*>(out->bb_codes);
  pp.bb_scales = static_cast<uint8_t*>(out->bb_scales);
  pp.res_codes = static_cast<uint8_t*>(out->res_codes);
  pp.res_scales = static_cast<uint8_t*>(out->res_scales);
  pp.tensor = out->tensor;
  pp.act_amax = act_amax > 0.0f ? act_amax : 0.0f;
  pp.rstd = nullptr;
  if (workspace && (workspace_bytes < (size_t)out->t * sizeof(float) || !aligned(workspace, 16)))
    return fail(SHARQ_ERR_WORKSPACE, "workspace must hold t floats, 16-byte aligned");
  if (out->fmt == SHARQ_NVFP4 && !(act_amax > 0.0f)) {
    // the amax pass already computes each row's RMSNorm factor: keep it for the prep pass
    float* rstd = (norm && workspace) ? static_cast<float*>(workspace) : nullptr;
    SHARQ_CUDA(cudaMemsetAsync(out->tensor, 0, sizeof(float), s));
    if (norm) st = bf16 ? launch_amax<true, true>(x, gamma, eps, out->t, out->k, out->tensor, rstd, s)
                        : launch_amax<true, false>(x, gamma, eps, out->t, out->k, out->tensor, rstd, s);
    else st = bf16 ? launch_amax<false, true>(x, gamma, eps, out->t, out->k, out->tensor, nullptr, s)
                   : launch_amax<false, false>(x, gamma, eps, out->t, out->k, out->tensor, nullptr, s);
    if (st != SHARQ_OK) return st;
    pp.rstd = rstd;
  }
  if (out->fmt == SHARQ_NVFP4) return prep_dispatch_p<FMT_NV>(pp, out->pat, norm, bf16, s);
  return prep_dispatch_p<FMT_MX>(pp, out->pat, norm, bf16, s);
}

sharq_status sharq_prepare_swiglu(const void* gate, const void* up, sharq_dtype dt, float act_amax,
                                  sharq_prepared* out, sharq_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sharq_status st = check_prepared(out);
  if (st != SHARQ_OK) return st;
  if (!gate || !aligned(gate, 16)) return fail(SHARQ_ERR_INVALID, "gate must be a 16-byte aligned device pointer");
  if (!up || !aligned(up, 16)) return fail(SHARQ_ERR_INVALID, "up must be a 16-byte aligned device pointer");
  if (dt != SHARQ_F32 && dt != SHARQ_BF16) return fail(SHARQ_ERR_INVALID, "bad dtype %d", (int)dt);
  const bool bf16 = dt == SHARQ_BF16;
  PrepParams pp;
  pp.x = gate;
  pp.x2 = up;
  pp.gamma = nullptr;
  pp.eps = 0.0f;
  pp.t = out->t;
  pp.t_pad = round_up(out->t, 128);
  pp.k = out->k;
  pp.meta = static_cast<uint8_t*>(out->meta);
  pp.bb_codes = static_cast<uint8_t*>(out->bb_codes);
  pp.bb_scales = static_cast<uint8_t*>(out->bb_scales);
  pp.res_codes = static_cast<uint8_t*>(out->res_codes);
  pp.res_scales = static_cast<uint8_t*>(out->res_scales);
  pp.tensor = out->tensor;
  pp.act_amax = act_amax > 0.0f ? act_amax : 0.0f;
  pp.rstd = nullptr;
  if (out->fmt == SHARQ_NVFP4 && !(act_amax > 0.0f)) {
    SHARQ_CUDA(cudaMemsetAsync(out->tensor, 0, sizeof(float), s));
    st = bf16 ? launch_amax_swiglu<true>(gate, up, out->t, out->k, out->tensor, s)
              : launch_amax_swiglu<false>(gate, up, out->t, out->k, out->tensor, s);
    if (st != SHARQ_OK) return st;
  }
  if (out->fmt == SHARQ_NVFP4) return swiglu_dispatch_p<FMT_NV>(pp, out->pat, bf16, s);
  return swiglu_dispatch_p<FMT_MX>(pp, out->pat, bf16, s);
}

sharq_status sharq_gather_prepared(const sharq_prepared* src, const int32_t* rows, sharq_prepared* dst,
                                   sharq_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sharq_status st = check_prepared(src);
  if (st != SHARQ_OK) return st;
  st = check_prepared(dst);
  if (st != SHARQ_OK) return st;
  if (src->k != dst->k || src->fmt != dst->fmt || src->pat != dst->pat)
    return fail(SHARQ_ERR_INVALID, "source and destination differ in k, format or pattern");
  if (dst->t > 0 && (!rows || !aligned(rows, 4))) return fail(SHARQ_ERR_INVALID, "rows must be a device int32 array");
  const int64_t k = dst->k;
  const int b = fmt_block(dst->fmt);
  const bool d816 = dst->pat == SHARQ_NM_8_16;
  GatherParams gp;
  gp.s_meta = static_cast<const uint8_t*>(src->meta);
  gp.s_bbc = static_cast<const uint8_t*>(src->bb_codes);
  gp.s_bbs = static_cast<const uint8_t*>(src->bb_scales);
  gp.s_rc = static_cast<const uint8_t*>(src->res_codes);
  gp.s_rs = static_cast<const uint8_t*>(src->res_scales);
  gp.d_meta = static_cast<uint8_t*>(dst->meta);
  gp.d_bbc = static_cast<uint8_t*>(dst->bb_codes);
  gp.d_bbs = static_cast<uint8_t*>(dst->bb_scales);
  gp.d_rc = static_cast<uint8_t*>(dst->res_codes);
  gp.d_rs = static_cast<uint8_t*>(dst->res_scales);
  gp.rows = rows;
  gp.src_t = src->t;
  gp.t = dst->t;
  gp.t_pad = round_up(dst->t, 128);
  gp.meta_row = meta_row_bytes(k, dst->pat);
  gp.bbc_row = d816 ? k / 2 : k / 4;
  gp.rc_row = k / 2;
  gp.bbs_per_row = d816 ? k / b : k / (2 * b);
  gp.rs_per_row = k / b;
  gp.zero_meta = d816 ? 0x00FF00FFu : 0x44444444u;
  st = launch_ex(gather_rows_kernel, dim3((unsigned)((gp.t_pad + 7) / 8)), dim3(256), 0, s, 1, gp);
  if (st != SHARQ_OK) return st;
  SHARQ_CUDA(cudaMemcpyAsync(dst->tensor, src->tensor, 3 * sizeof(float), cudaMemcpyDeviceToDevice, s));
  return SHARQ_OK;
}

sharq_status sharq_prepare_noalloc(const void* x, sharq_dtype x_dt, const void* gamma, float eps, float act_amax,
                                   sharq_prepared* out, sharq_stream stream) {
  if (!out) return fail(SHARQ_ERR_INVALID, "out is NULL");
  if (out->t > SHARQ_NOALLOC_MAX_ROWS)
    return fail(SHARQ_ERR_WORKSPACE,
                "sharq_prepare_noalloc: t = %lld rows exceeds its static scratch of %d rows; "
                "call sharq_prepare with a caller workspace instead",
                (long long)out->t, SHARQ_NOALLOC_MAX_ROWS);
  float* scratch = nullptr;
  sharq_status st = noalloc_scratch(&scratch);
  if (st != SHARQ_OK) return st;
  return sharq_prepare(x, x_dt, gamma, eps, act_amax, out, scratch, sizeof(float) * SHARQ_NOALLOC_MAX_ROWS, stream);
}

sharq_status sharq_linear(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt,
                          sharq_stream stream) {
  return run_linear(a, w, nullptr, y, y_dt, 3, reinterpret_cast<cudaStream_t>(stream));
}

sharq_status sharq_linear_workspace_size(size_t* bytes) {
  if (!bytes) return fail(SHARQ_ERR_INVALID, "bytes is NULL");
  *bytes = sk_workspace_bytes();
  return SHARQ_OK;
}
sharq_status sharq_linear_ws(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt,
                             void* workspace, size_t workspace_bytes, sharq_stream stream) {
  if (!workspace) return fail(SHARQ_ERR_WORKSPACE, "workspace is NULL");
  return run_linear(a, w, nullptr, y, y_dt, 3, reinterpret_cast<cudaStream_t>(stream), workspace, workspace_bytes);
}
sharq_status sharq_linear_paths(const sharq_prepared* a, const sharq_weight* w, void* y, sharq_dtype y_dt,
                                int32_t paths, sharq_stream stream) {
  return run_linear(a, w, nullptr, y, y_dt, paths, reinterpret_cast<cudaStream_t>(stream));
}

sharq_status sharq_linear_grouped(const sharq_prepared* a, const sharq_weight* w, const int32_t* group_offsets,
                                  void* y, sharq_dtype y_dt, sharq_stream stream) {
  if (!group_offsets) return fail(SHARQ_ERR_INVALID, "group_offsets is NULL");
  if (a && a->t % 128 != 0) return fail(SHARQ_ERR_INVALID, "grouped rows must be a multiple of 128");
  return run_linear(a, w, group_offsets, y, y_dt, 3, reinterpret_cast<cudaStream_t>(stream));
}

sharq_status sharq_linear_grouped_gather(const sharq_prepared* tokens, const int32_t* rows, int64_t routed_rows,
                                         const sharq_weight* w, const int32_t* group_offsets, void* y,
                                         sharq_dtype y_dt, sharq_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sharq_status st = check_prepared(tokens);
  if (st != SHARQ_OK) return st;
  st = check_weight(w);
  if (st != SHARQ_OK) return st;
  if (tokens->fmt != SHARQ_NVFP4 || tokens->pat != SHARQ_NM_4_8_PAIR)
    return fail(SHARQ_ERR_UNSUPPORTED, "gathered rows: NVFP4 with the 4:8 pair pattern only");
  if (w->fmt != tokens->fmt) return fail(SHARQ_ERR_INVALID, "format mismatch between activations and weight");
  if (tokens->k != w->k) return fail(SHARQ_ERR_INVALID, "k mismatch: activations %lld, weight %lld",
                                     (long long)tokens->k, (long long)w->k);
  if (routed_rows <= 0 || routed_rows % 128 != 0)
    return fail(SHARQ_ERR_INVALID, "routed_rows=%lld must be a positive multiple of 128", (long long)routed_rows);
  if (!rows || !aligned(rows, 4)) return fail(SHARQ_ERR_INVALID, "rows must be a device int32 array");
  if (!group_offsets) return fail(SHARQ_ERR_INVALID, "group_offsets is NULL");
  if (!y || !aligned(y, 16)) return fail(SHARQ_ERR_INVALID, "y must be a 16-byte aligned device pointer");
  if (y_dt != SHARQ_F32 && y_dt != SHARQ_BF16) return fail(SHARQ_ERR_INVALID, "bad y dtype %d", (int)y_dt);
  using C = GemmCfg<GK_NVF4, true>;
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  st = make_map(&maps.w, w->codes, w->k / 2, w->n * w->experts, 128, C::BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SHARQ_OK) return st;
  if (y_dt == SHARQ_BF16) {
    st = make_map(&maps.y, y, w->n * 2, routed_rows, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != SHARQ_OK) return st;
  }
  GemmParams gp;
  memset(&gp, 0, sizeof(gp));
  gp.t = routed_rows;
  gp.t_pad = routed_rows;
  gp.n = w->n;
  gp.k = w->k;
  gp.experts = w->experts;
  gp.group_offsets = group_offsets;
  gp.sf_res = static_cast<const uint8_t*>(tokens->res_scales);
  gp.sf_bb = static_cast<const uint8_t*>(tokens->bb_scales);
  gp.sf_w_dense = static_cast<const uint8_t*>(w->scales_dense);
  gp.sf_w_sparse = static_cast<const uint8_t*>(w->scales_sparse);
  gp.tensor_x = tokens->tensor;
  gp.tensor_w = w->tensor;
  gp.w_codes = w->codes;
  gp.y = y;
  gp.y_bf16 = y_dt == SHARQ_BF16;
  gp.paths = 3;
  gp.timeout_ns = wait_timeout_ns();
  gp.gather_rows = rows;
  gp.gather_src_t = tokens->t;
  gp.gather_src_tpad = round_up(tokens->t, 128);
  gp.g_res_codes = static_cast<const uint8_t*>(tokens->res_codes);
  gp.g_bb_codes = static_cast<const uint8_t*>(tokens->bb_codes);
  gp.g_meta = static_cast<const uint8_t*>(tokens->meta);
  return launch_gemm<GK_NVF4, true, false, true>(maps, gp, s);
}

sharq_status sharq_sync_status(sharq_stream stream) {
  SHARQ_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  unsigned int word = 0, zero = 0;
  SHARQ_CUDA(cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)));
  SHARQ_CUDA(cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)));
  if (word & kErrTimeout) return fail(SHARQ_ERR_TIMEOUT, "a device-side wait ran out of time");
  return SHARQ_OK;
}

sharq_status sharq_selftest_wait_timeout(uint64_t timeout_ns, sharq_stream stream) {
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return launched();
}

const char* sharq_last_error(void) { return g_last_error.c_str(); }

uint64_t sharq_launch_count(int reset) {
  uint64_t v = g_launches;
  if (reset) g_launches = 0;
  return v;
}

}  // extern "C"
