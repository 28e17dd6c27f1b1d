// gemm.cuh -- the two GEMMs of the SharQ layer in one persistent tcgen05 kernel.
//
// SharQ (arXiv 2606.26587), abstract and Section 1: a sparse FP4 GEMM runs over
// the compressed backbone and its N:M metadata, a dense FP4 GEMM runs over the
// residual and adds its result into the same output, and the two paths load
// the FP4 weight once, each reading it through its own scale view.  Here both MMAs of
// a K tile read the SAME shared-memory copy of the weight tile (one TMA load)
// and write the SAME tensor-memory accumulator; each path brings its own
// scale-factor view of the weight (one scale per 2b logical K for the sparse
// MMA, the same scales repeated per b for the dense MMA).
//
// Structure (one CTA per SM, 14 warps):
//   warp 0      TMA producer: weight, residual, backbone and metadata tiles by
//               cp.async.bulk.tensor, scale factors by 1-D cp.async.bulk;
//   warp 1      TMEM owner and MMA issuer (one thread): tcgen05.mma.sp over the
//               backbone, tcgen05.mma over the residual, tcgen05.commit to free
//               stages and to hand the accumulator to the epilogue;
//   warps 2-9   epilogue, two warps per 32-lane quadrant, half the columns
//               each: tcgen05.ld of the fp32 accumulator, times the tensor
//               scales g_dec(x) * g_dec(w); bf16 output is packed into
//               registers, the accumulator released, and the tile written by
//               TMA stores through shared memory; fp32 output is stored directly;
//   warps 10-13 scale factors and metadata of each K tile, shared memory ->
//               the stage's tensor-memory slot (tcgen05.st), one warp per quadrant.
// Tiles are 128 x 256 outputs; a stage is 256 logical K.  Every wait is
// bounded in time and reports through the device error word.
#pragma once
#include <cuda_bf16.h>

#include "prep.cuh"
#include "ptx.cuh"

namespace sharq {

enum { GK_NVF4 = 0, GK_MXF4 = 1, GK_MXF8 = 2 };

// Per-kind tile configuration.
//   GK_NVF4  NVFP4: kind::mxf4nvf4 (dense K=64, 4 E4M3 scales of 16) and its
//            4:8-pair sparse form (K=128 logical, 4 scales of 32 logical);
//   GK_MXF4  MXFP4 with the 4:8 pair: kind::mxf4 (2 E8M0 scales of 32) and
//            kind::mxf4.sp (2 scales of 64 logical);
//   GK_MXF8  MXFP4 with element-wise 2:4: the only sparse kind that takes it is
//            kind::mxf8f6f4.sp, with E2M1 held in 8-bit shared-memory containers
//            (TMA unpacks 16 packed codes into 16 bytes); the dense residual runs
//            as kind::mxf8f6f4 on the same unpacked weight tile.
// SPARSE = false is the 8:16 form: the backbone is stored dense and runs through
// the dense MMA like the residual.
template <int KIND, bool SPARSE>
struct GemmCfg {
  static constexpr bool kUnpacked = KIND == GK_MXF8;
  static constexpr int BM = 128, BN = kUnpacked ? 128 : 256, BK = 256;
  static constexpr int kNRB = BN / 128;                        // 128-row blocks of the weight tile
  static constexpr int kDenseMmaK = kUnpacked ? 32 : 64;       // logical K per dense MMA
  static constexpr int kSparseMmaK = kUnpacked ? 64 : 128;     // logical K per sparse MMA
  static constexpr int kVecDense = (KIND == GK_NVF4) ? 16 : 32;  // logical K per scale, dense MMA
  static constexpr int kVecSparse = 2 * kVecDense;                // logical K per scale, sparse MMA
  static constexpr int kBoxElems = kUnpacked ? 128 : 256;      // K elements per 128-byte smem row of a box
  static constexpr int kBoxesDense = BK / kBoxElems;           // boxes per stage of W and R
  static constexpr int kBoxR = BM * 128, kBoxW = BN * 128;     // bytes of one box
  static constexpr int kWBytes = kBoxesDense * kBoxW;
  static constexpr int kRBytes = kBoxesDense * kBoxR;
  static constexpr int kRowB = SPARSE ? (kUnpacked ? 128 : 64) : 128;  // smem bytes per backbone row per box
  static constexpr int kBoxesB = SPARSE ? 1 : kBoxesDense;
  static constexpr int kBBytes = kBoxesB * BM * kRowB;
  static constexpr int kMetaStage = SPARSE ? (kUnpacked ? BK / 8 : BK / 16) : 0;  // metadata bytes per row
  static constexpr int kEBoxes = kMetaStage / 16;              // 16-byte metadata boxes per stage
  static constexpr int kEBytes = kEBoxes * BM * 16;
  // TMA inner coordinate per stage (packed maps count bytes, unpacked maps elements)
  static constexpr int kXStage = kUnpacked ? BK : BK / 2;
  static constexpr int kXStageB = SPARSE ? (kUnpacked ? BK / 2 : BK / 4) : kXStage;
  static constexpr int kChunksR = BK / kVecDense / 4;                  // 512-byte scale chunks per stage
  static constexpr int kChunksB = SPARSE ? BK / kVecSparse / 4 : kChunksR;
  static constexpr int kSfaR = kChunksR * 512;
  // the sparse kinds load only the weight's sparse-view scales: its dense view is
  // each of them repeated (one weight scale per 2b logical K), written into
  // tensor memory by the staging warps; the dense-backbone form loads the dense view
  static_assert(!SPARSE || kChunksR == 2 * kChunksB, "dense view = each sparse-view scale twice");
  static constexpr int kSfbD = SPARSE ? 0 : kNRB * kChunksR * 512;
  static constexpr int kSfaB = kChunksB * 512;
  static constexpr int kSfbS = SPARSE ? kNRB * kChunksB * 512 : 0;
  // stage layout (offsets in bytes)
  static constexpr int oW = 0;
  static constexpr int oR = oW + kWBytes;
  static constexpr int oB = oR + kRBytes;
  static constexpr int oE = oB + kBBytes;
  static constexpr int oSfaR = oE + kEBytes;
  static constexpr int oSfbD = oSfaR + kSfaR;
  static constexpr int oSfaB = oSfbD + kSfbD;
  static constexpr int oSfbS = oSfaB + kSfaB;
  static constexpr int kStageBytes = ((oSfbS + kSfbS + 1023) / 1024) * 1024;
  static constexpr int kStages = kUnpacked ? 2 : 3;
  // transaction bytes: unpacking loads count the packed (global) size, half their smem footprint
  static constexpr uint32_t kTx = (kWBytes + kRBytes + kBBytes) / (kUnpacked ? 2 : 1) + kEBytes + kSfaR + kSfbD + kSfaB +
                                  kSfbS;
  // tensor memory columns: accumulator, then one slot of scales + metadata per stage
  static constexpr int cSfaR = 0;
  static constexpr int cSfbD = cSfaR + 4 * kChunksR;
  static constexpr int cSfaB = cSfbD + 4 * kNRB * kChunksR;
  static constexpr int cSfbS = cSfaB + 4 * kChunksB;
  static constexpr int cE = cSfbS + (SPARSE ? 4 * kNRB * kChunksB : 0);
  static constexpr int kSlotCols = cE + 4 * kEBoxes;
  static constexpr int kTmemCols = BN + kStages * kSlotCols <= 256 ? 256 : 512;
  static_assert(BN + kStages * kSlotCols <= kTmemCols, "tensor memory budget");
  static constexpr int kYCols = 16;                // bf16 output staged 32 rows x 16 columns at a time
  static constexpr int kYBuf = 8 * 32 * kYCols * 2;  // one chunk per epilogue warp
  static constexpr int kGatherIdx = BM * 4;  // gathered form: the tile's source row indices
  static constexpr int kSmemBytes = kStages * kStageBytes + kYBuf + 1024 /*align*/ + 256 /*barriers*/ + kGatherIdx;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // instruction descriptor (block-scaled kinds): E2M1 x E2M1, K-major, M=128, N=BN
  static constexpr uint32_t kFmt = kUnpacked ? 5u : 1u;
  static constexpr uint32_t kIdesc = (kFmt << 7) | (kFmt << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((KIND == GK_NVF4 ? 0u : 1u) << 23) | ((uint32_t)(BM >> 4) << 24);
  static constexpr uint32_t kIdescSp = kIdesc | (1u << 2);
  static constexpr int kBandTiles = 16;  // row tiles per raster band (2048 rows)
  // 16-byte-unit offset inside a stage of the dense operand slice for logical K index kk
  __host__ __device__ static constexpr uint32_t dense_off(int box_bytes, int kk) {
    return (uint32_t)((kk / kBoxElems) * (box_bytes / 16) + (kUnpacked ? (kk % kBoxElems) / 16 : (kk % kBoxElems) / 32));
  }
};

// Raster order of the output tiles: bands of up to gm row tiles; inside a band
// the row tile varies fastest, so the tiles in flight at one time share a few
// activation row blocks and weight column blocks, which stay in L2 (plain row-
// major order would sweep all activation rows once per weight column block).
struct TileXY {
  int mt, nt;    // row tile, column tile
  int lo, h;     // the band: row tiles lo .. lo + h - 1
};
__device__ __forceinline__ TileXY tile_xy(int t, int m_tiles, int n_tiles, int gm) {
  const int per_band = gm * n_tiles;
  const int b = t / per_band;
  TileXY x;
  x.lo = b * gm;
  x.h = m_tiles - x.lo < gm ? m_tiles - x.lo : gm;
  const int r = t - b * per_band;
  x.mt = x.lo + r % x.h;
  x.nt = r / x.h;
  return x;
}

constexpr int kMaxSplit = 4;  // K slices per tile in the split-K form of the single-CTA kernel

struct GemmParams {
  int64_t t;          // rows of y to store (rows >= t are computed but not stored)
  int64_t t_pad;      // rows of the prepared operands (multiple of 128)
  int64_t n, k;
  int32_t experts;    // 1 = plain; >1 grouped by group_offsets
  const int32_t* group_offsets;  // device, experts + 1 (grouped only)
  const uint8_t* sf_res;         // tiled, t_pad rows, k/b scales
  const uint8_t* sf_bb;          // tiled, t_pad rows, k/(2b) scales (dense backbone: k/b)
  const uint8_t* sf_w_dense;     // per expert tiled, n rows, k/b
  const uint8_t* sf_w_sparse;    // per expert tiled, n rows, k/(2b)
  const float* tensor_x;         // [amax, g_enc, g_dec]
  const float* tensor_w;         // experts * 3
  const void* w_codes;           // packed weight codes, row-major [experts * n][k / 2] (L2 warm-up only)
  void* y;
  int y_bf16;
  int paths;          // bit 0 sparse backbone, bit 1 dense residual
  uint64_t timeout_ns;
  // stream-K (CTA-pair kernel only; null = whole tiles): per pair a slot of
  // partial sums (2 CTAs x 8 epilogue warps x 32 x 128 fp32) and one counter
  // per (slot, CTA, epilogue warp), odd while a partial waits to be added
  float* sk_part;
  uint32_t* sk_flag;
  // split-K (single-CTA kernel only, split >= 2): one fp32 slot [t_pad][n] of
  // raw sums per K slice, then one counter per tile
  float* split_acc;
  uint32_t* split_cnt;
  int32_t split;
  // gathered activation rows (single-CTA kernel, GATHER): row r of the routed
  // operand is row gather_rows[r] of the token-prepared buffers below (an index
  // < 0 or >= gather_src_t stands for an all-zero input row); sf_res / sf_bb
  // then point at the tokens' scales (tiled, gather_src_tpad rows)
  const int32_t* gather_rows;
  int64_t gather_src_t, gather_src_tpad;
  const uint8_t* g_res_codes;
  const uint8_t* g_bb_codes;
  const uint8_t* g_meta;
};

struct GemmMaps {
  CUtensorMap w, r, b, e;
  CUtensorMap y;  // bf16 output, 32 x 32 boxes (CTA-pair kernel only)
};

// SPLIT: each tile's K loop is cut into p.split slices run by different CTAs
// (few tiles, long K: the weight stream then uses every SM).
// GATHER (NVFP4 4:8 pair, grouped): the activation rows of a tile are read by
// index from the token-prepared buffers (a mixture-of-experts layer prepares
// each token once; its routed copies are never written out).  The producer
// warp copies each row's residual, backbone and metadata bytes and its scale
// words with cp.async into the stage, placing them where a tensor load with
// the same swizzle would, and writes the all-zero row's encoding for padding
// rows; a stage is handed to the MMA once its copies have landed and been made
// visible to the tensor cores (fence.proxy.async), kGatherLag stages behind.
template <int KIND, bool SPARSE, bool SPLIT, bool GATHER = false>
__global__ void __launch_bounds__(448, 1) gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using C = GemmCfg<KIND, SPARSE>;
  static_assert(!GATHER || (KIND == GK_NVF4 && SPARSE && !SPLIT), "gathered rows: NVFP4 4:8 pair, whole tiles");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ybuf = smem + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ybuf + C::kYBuf);
  uint64_t* empty = full + C::kStages;
  uint64_t* acc_full = empty + C::kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* sf_ready = drain + 1;  // per stage: its scale slot is in tensor memory
  uint64_t* ep_done = sf_ready + C::kStages;  // split-K: the 8 epilogue warps wrote their slice
  uint64_t* ep_flag = ep_done + 1;            // split-K: split_last is set
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ep_flag + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile uint32_t* split_last = reinterpret_cast<volatile uint32_t*>(tmem_holder + 2);  // split-K: last slice?
  int32_t* gidx = reinterpret_cast<int32_t*>(smem_raw + C::kSmemBytes - C::kGatherIdx);  // gathered: source rows

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; s++) {
      // gathered form: the weight's tensor loads and, later, the landed row copies
      mbar_init(&full[s], GATHER ? 2 : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 4);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);  // 8 epilogue warps
    mbar_init(drain, 1);
    mbar_init(ep_done, 8);
    mbar_init(ep_flag, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&maps.w);
    if (!GATHER) {
      tma_prefetch(&maps.r);
      tma_prefetch(&maps.b);
      if (C::kEBoxes > 0) tma_prefetch(&maps.e);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int m_tiles = (int)(p.t_pad / C::BM);
  const int n_tiles = (int)(p.n / C::BN);
  const int num_tiles = m_tiles * n_tiles;
  const int k_tiles = (int)(p.k / C::BK);
  if (warp == 0 && lane == 0 && p.experts <= 1 && (int)blockIdx.x < num_tiles) {
    // while the kernel before this one finishes: warm L2 with this CTA's share
    // of the weight tile of its first tile, whole TMA boxes (the CTAs on one
    // column of tiles split its K tiles); the weight is not written by the
    // preparation kernels
    const TileXY x = tile_xy((int)blockIdx.x, m_tiles, n_tiles, C::kBandTiles);
    const int per = (k_tiles + x.h - 1) / x.h, i = x.mt - x.lo;
    const int32_t wrow = (int32_t)((int64_t)x.nt * C::BN);
    for (int kt = i * per; kt < (i + 1) * per && kt < k_tiles; kt++)
#pragma unroll
      for (int bx = 0; bx < C::kBoxesDense; bx++) tma_prefetch_l2_2d(&maps.w, kt * C::kXStage + 128 * bx, wrow);
  }
  grid_dep_wait();  // the prepared activations (and scales) are complete
  // work items: (tile, K slice) with SPLIT, else whole tiles
  const int n_split = SPLIT ? p.split : 1;
  const int items = num_tiles * n_split;
  auto k_lo = [&](int item) { return (int)((int64_t)(item % n_split) * k_tiles / n_split); };
  auto k_hi = [&](int item) { return (int)((int64_t)(item % n_split + 1) * k_tiles / n_split); };
  const int64_t sd_per_row = p.k / C::kVecDense;                    // dense-view scales per row
  const int64_t sb_per_row = SPARSE ? p.k / C::kVecSparse : sd_per_row;
  const int64_t wsd_bytes = tiled_sf_bytes(p.n, sd_per_row);
  const int64_t wss_bytes = tiled_sf_bytes(p.n, p.k / C::kVecSparse);
  const bool run_sparse = (p.paths & 1) != 0;
  const bool run_dense = (p.paths & 2) != 0;

  // expert of an m tile (grouped form); -1 = rows outside every group
  auto tile_expert = [&](int64_t m0) -> int {
    if (p.experts <= 1) return 0;
    int lo = 0, hi = p.experts;  // find e with off[e] <= m0 < off[e+1]
    if (m0 >= (int64_t)__ldg(p.group_offsets + p.experts)) return -1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if ((int64_t)__ldg(p.group_offsets + mid) <= m0) lo = mid;
      else hi = mid;
    }
    return lo;
  };

  if (warp == 0 && GATHER) {
    // ------------------------------------------- producer, gathered rows
    // all 32 lanes copy the tile's rows; lane 0 also issues the weight loads
    constexpr int kLag = C::kStages - 1;  // stages in flight before the oldest is handed over
    const uint32_t smem0 = smem_u32(smem), full0 = smem_u32(full);
    const int64_t sd_blocks = (sd_per_row + 3) / 4, sb_blocks = (sb_per_row + 3) / 4;
    const int64_t ss_blocks = (p.k / C::kVecSparse + 3) / 4;
    const int64_t rc_row = p.k / 2, bc_row = p.k / 4, me_row = p.k / 16;
    const uint32_t gidx_s = smem_u32(gidx);
    uint32_t g = 0;  // stages issued so far
    uint32_t issued = 0, issued_par = 0;  // per stage: ever issued / parity of the last batch
    auto hand_over = [&](uint32_t gg) {  // the copies of stage gg have landed in every lane
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[gg % C::kStages]);
    };
    int stage = 0;
    uint32_t phase = 0;
    for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
      const int tile = item / n_split, k0 = k_lo(item), k1 = k_hi(item);
      const TileXY xy = tile_xy(tile, m_tiles, n_tiles, C::kBandTiles);
      const int mt = xy.mt, nt = xy.nt;
      const int64_t m0 = (int64_t)mt * C::BM;
      const int e = tile_expert(m0);
      if (e < 0) continue;
      const int32_t wrow = (int32_t)(e * p.n + (int64_t)nt * C::BN);
      const int64_t nb = (int64_t)nt * C::kNRB;
      const uint8_t* g_sfb_s = p.sf_w_sparse + e * wss_bytes + nb * ss_blocks * 512 + (int64_t)k0 * C::kChunksB * 512;
      int32_t kx = k0 * C::kXStage;
      // source rows of this tile (the copies in flight took their addresses at issue)
      __syncwarp();
      for (int i = lane; i < C::BM; i += 32) {
        const int64_t r = m0 + i;
        int32_t src = r < p.t ? __ldg(p.gather_rows + r) : -1;
        if (src >= p.gather_src_t) src = -1;
        gidx[i] = src;
      }
      __syncwarp();
      for (int kt = k0; kt < k1; kt++) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { *abort_flag = 1; break; }
        const uint32_t sb = smem0 + (uint32_t)(stage * C::kStageBytes);
        if (lane == 0) {
          const uint32_t fb = full0 + (uint32_t)(stage * 8);
          mbar_arrive_expect_tx_u32(fb, (uint32_t)(C::kWBytes + C::kSfbS));
          tma_load_2d_u32(sb + C::oW, &maps.w, kx, wrow, fb);
#pragma unroll
          for (int rb = 0; rb < C::kNRB; rb++)
            bulk_load_u32(sb + C::oSfbS + rb * C::kChunksB * 512, g_sfb_s + rb * ss_blocks * 512, C::kChunksB * 512, fb);
        }
        // residual codes: 128 bytes of a row per stage, eight 16-byte pieces placed
        // as the 128-byte swizzle does (piece c of row r at (c ^ (r % 8)) * 16)
#pragma unroll 4
        for (int j = 0; j < C::BM / 4; j++) {
          const int r = 4 * j + (lane >> 3), c = lane & 7;
          int32_t src;
          asm volatile("ld.shared.s32 %0, [%1];" : "=r"(src) : "r"(gidx_s + 4 * r));
          const uint32_t dst = sb + C::oR + (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
          if (src >= 0) cp_async16(dst, p.g_res_codes + src * rc_row + (int64_t)kt * 128 + c * 16);
          else st_shared_v4(dst, 0u, 0u, 0u, 0u);
        }
        // backbone codes: 64 bytes of a row, 64-byte swizzle (piece c at (c ^ ((r / 2) % 4)) * 16)
#pragma unroll 4
        for (int j = 0; j < C::BM / 8; j++) {
          const int r = 8 * j + (lane >> 2), c = lane & 3;
          int32_t src;
          asm volatile("ld.shared.s32 %0, [%1];" : "=r"(src) : "r"(gidx_s + 4 * r));
          const uint32_t dst = sb + C::oB + (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
          if (src >= 0) cp_async16(dst, p.g_bb_codes + src * bc_row + (int64_t)kt * 64 + c * 16);
          else st_shared_v4(dst, 0u, 0u, 0u, 0u);
        }
        // metadata (16 bytes a row) and the row's scale words (4 scales of each
        // 512-byte chunk, at the row's place in the tiled layout)
#pragma unroll
        for (int j = 0; j < C::BM / 32; j++) {
          const int r = 32 * j + lane;
          int32_t src;
          asm volatile("ld.shared.s32 %0, [%1];" : "=r"(src) : "r"(gidx_s + 4 * r));
          const uint32_t dst_e = sb + C::oE + (uint32_t)(r * 16);
          const uint32_t rpos = (uint32_t)((r & 31) * 16 + ((r >> 5) & 3) * 4);
          if (src >= 0) {
            cp_async16(dst_e, p.g_meta + src * me_row + (int64_t)kt * 16);
            const uint8_t* sr = p.sf_res + ((int64_t)(src >> 7) * sd_blocks + (int64_t)kt * C::kChunksR) * 512 +
                                (src & 31) * 16 + ((src >> 5) & 3) * 4;
            const uint8_t* sbb = p.sf_bb + ((int64_t)(src >> 7) * sb_blocks + (int64_t)kt * C::kChunksB) * 512 +
                                 (src & 31) * 16 + ((src >> 5) & 3) * 4;
#pragma unroll
            for (int c = 0; c < C::kChunksR; c++) cp_async4(sb + C::oSfaR + c * 512 + rpos, sr + c * 512);
#pragma unroll
            for (int c = 0; c < C::kChunksB; c++) cp_async4(sb + C::oSfaB + c * 512 + rpos, sbb + c * 512);
          } else {
            // an all-zero input row: each group of 8 keeps pairs 0 and 1 (nibble 4), codes and scales 0
            st_shared_v4(dst_e, 0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
#pragma unroll
            for (int c = 0; c < C::kChunksR; c++) st_shared_u32(sb + C::oSfaR + c * 512 + rpos, 0u);
#pragma unroll
            for (int c = 0; c < C::kChunksB; c++) st_shared_u32(sb + C::oSfaB + c * 512 + rpos, 0u);
          }
        }
        cp_async_commit();
        if (g >= (uint32_t)kLag) {
          cp_async_wait_group<kLag>();
          hand_over(g - kLag);
        }
        g++;
        kx += C::kXStage;
        g_sfb_s += C::kChunksB * 512;
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
    // the last stages: every copy lands before they are handed over (also on abort,
    // so that no copy is still in flight when the block exits)
    cp_async_wait_group<0>();
    for (uint32_t gg = g > (uint32_t)kLag ? g - kLag : 0; gg < g; gg++) hand_over(gg);
    if (*abort_flag && lane == 0) {
      // let the weight loads already issued land before the block can exit
      for (int i = 0; i < C::kStages; i++)
        if ((issued >> i) & 1u) (void)mbar_wait(&full[i], (issued_par >> i) & 1u, 1000000000ull, nullptr, true);
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;  // per stage: ever issued / parity of the last batch
      const uint32_t smem0 = smem_u32(smem), full0 = smem_u32(full);
      const int64_t sd_blocks = (sd_per_row + 3) / 4, sb_blocks = (sb_per_row + 3) / 4;
      const int64_t ss_blocks = (p.k / C::kVecSparse + 3) / 4;
      for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
        const int tile = item / n_split, k0 = k_lo(item), k1 = k_hi(item);
        const TileXY xy = tile_xy(tile, m_tiles, n_tiles, C::kBandTiles);
        const int mt = xy.mt, nt = xy.nt;
        const int64_t m0 = (int64_t)mt * C::BM;
        const int e = tile_expert(m0);
        if (e < 0) continue;
        const int32_t wrow = (int32_t)(e * p.n + (int64_t)nt * C::BN);
        const int64_t nb = (int64_t)nt * C::kNRB;
        // scale chunks of this tile: contiguous per 128-row block, advanced per K tile
        const uint8_t* g_sfa_r = p.sf_res + (m0 / 128) * sd_blocks * 512 + (int64_t)k0 * C::kSfaR;
        const uint8_t* g_sfa_b = p.sf_bb + (m0 / 128) * sb_blocks * 512 + (int64_t)k0 * C::kSfaB;
        const uint8_t* g_sfb_d = p.sf_w_dense + e * wsd_bytes + nb * sd_blocks * 512 + (int64_t)k0 * C::kChunksR * 512;
        const uint8_t* g_sfb_s = p.sf_w_sparse + e * wss_bytes + nb * ss_blocks * 512 + (int64_t)k0 * C::kChunksB * 512;
        int32_t kx = k0 * C::kXStage, kx_b = k0 * C::kXStageB, kx_e = k0 * C::kMetaStage;
        for (int kt = k0; kt < k1; kt++) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
          const uint32_t sb = smem0 + (uint32_t)(stage * C::kStageBytes);
          const uint32_t fb = full0 + (uint32_t)(stage * 8);
          mbar_arrive_expect_tx_u32(fb, C::kTx);
#pragma unroll
          for (int bx = 0; bx < C::kBoxesDense; bx++) {
            tma_load_2d_u32(sb + C::oW + bx * C::kBoxW, &maps.w, kx + 128 * bx, wrow, fb);
            tma_load_2d_u32(sb + C::oR + bx * C::kBoxR, &maps.r, kx + 128 * bx, (int32_t)m0, fb);
          }
#pragma unroll
          for (int bx = 0; bx < C::kBoxesB; bx++)
            tma_load_2d_u32(sb + C::oB + bx * C::BM * C::kRowB, &maps.b, kx_b + 128 * bx, (int32_t)m0, fb);
#pragma unroll
          for (int bx = 0; bx < C::kEBoxes; bx++)
            tma_load_2d_u32(sb + C::oE + bx * C::BM * 16, &maps.e, kx_e + 16 * bx, (int32_t)m0, fb);
          bulk_load_u32(sb + C::oSfaR, g_sfa_r, C::kSfaR, fb);
          bulk_load_u32(sb + C::oSfaB, g_sfa_b, C::kSfaB, fb);
          if constexpr (!SPARSE) {
#pragma unroll
            for (int rb = 0; rb < C::kNRB; rb++)
              bulk_load_u32(sb + C::oSfbD + rb * C::kChunksR * 512, g_sfb_d + rb * sd_blocks * 512, C::kChunksR * 512,
                            fb);
          }
          if constexpr (SPARSE) {
#pragma unroll
            for (int rb = 0; rb < C::kNRB; rb++)
              bulk_load_u32(sb + C::oSfbS + rb * C::kChunksB * 512, g_sfb_s + rb * ss_blocks * 512,
                            C::kChunksB * 512, fb);
          }
          kx += C::kXStage;
          kx_b += C::kXStageB;
          kx_e += C::kMetaStage;
          g_sfa_r += C::kSfaR;
          g_sfa_b += C::kSfaB;
          g_sfb_d += C::kChunksR * 512;
          g_sfb_s += C::kChunksB * 512;
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag) {
        // let every load already issued land before the block can exit
        for (int i = 0; i < C::kStages; i++)
          if ((issued >> i) & 1u) (void)mbar_wait(&full[i], (issued_par >> i) & 1u, 1000000000ull, nullptr, true);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      const uint32_t acc = tmem_base;
      // descriptor halves: start addresses in 16-byte units (stage 0), constant high words
      constexpr uint32_t kHi128 = desc_hi(1024, 2), kHi64 = desc_hi(512, 4);
      constexpr uint32_t kHiB = (SPARSE && !C::kUnpacked) ? kHi64 : kHi128;  // backbone rows of 64 or 128 bytes
      constexpr uint32_t kLbo = 1u << 16;  // 16-byte leading offset (ignored by swizzled K-major layouts)
      const uint32_t lo0 = smem_u32(smem) >> 4;
      const uint32_t empty0 = smem_u32(empty);
      for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x, it++) {
        const int tile = item / n_split, k0 = k_lo(item), k1 = k_hi(item);
        const int mt = tile_xy(tile, m_tiles, n_tiles, C::kBandTiles).mt;
        if (tile_expert((int64_t)mt * C::BM) < 0) { it--; continue; }
        if (!mbar_wait(acc_empty, (it & 1) ^ 1, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
        tc_fence_after();
        uint32_t accumulate = 0;
        for (int kt = k0; kt < k1; kt++) {
          if (!mbar_wait(&full[stage], phase, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint32_t ls = lo0 + (uint32_t)(stage * (C::kStageBytes >> 4));  // stage base, 16-byte units
          // scale factors and metadata of this stage were written to its slot by the epilogue warps
          if (!mbar_wait(&sf_ready[stage], phase, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint32_t slot = tmem_base + C::BN + (uint32_t)(stage * C::kSlotCols);
          if (run_sparse) {
            if constexpr (SPARSE) {
              // backbone: sparse MMAs (32 bytes of compressed A, 64 bytes of W per MMA)
#pragma unroll
              for (int kb = 0; kb < C::BK / C::kSparseMmaK; kb++) {
                constexpr int kScales = C::kSparseMmaK / C::kVecSparse;
                const uint32_t chunk = (kb * kScales) / 4, byte = (kb * kScales) % 4;
                const uint32_t idesc = C::kIdescSp | (byte << 29) | (byte << 4);
                const uint64_t a = desc_lohi((ls + (C::oB >> 4) + 2 * kb) | kLbo, kHiB);
                const uint32_t wo = (uint32_t)((kb * 64) / 128 * (C::kBoxW / 16) + ((kb * 64) % 128) / 16);
                const uint64_t b = desc_lohi((ls + (C::oW >> 4) + wo) | kLbo, kHi128);
                const uint32_t sfa = (slot + C::cSfaB + 4 * chunk) | (byte << 30);
                const uint32_t sfb = (slot + C::cSfbS + 4 * C::kNRB * chunk) | (byte << 30);
                const uint32_t e = slot + C::cE + 2 * kb;
                if constexpr (KIND == GK_NVF4) mma_nvf4_sp(acc, a, b, e, idesc, sfa, sfb, accumulate);
                else if constexpr (KIND == GK_MXF4) mma_mxf4_sp(acc, a, b, e, idesc, sfa, sfb, accumulate);
                else mma_mxf8f6f4_sp(acc, a, b, e, idesc, sfa, sfb, accumulate);
                accumulate = 1;
              }
            } else {
              // dense backbone (8:16): same as the residual path over the expanded backbone
#pragma unroll
              for (int kb = 0; kb < C::BK / C::kDenseMmaK; kb++) {
                constexpr int kScales = C::kDenseMmaK / C::kVecDense;
                const uint32_t chunk = (kb * kScales) / 4, byte = (kb * kScales) % 4;
                const uint32_t idesc = C::kIdesc | (byte << 29) | (byte << 4);
                const uint64_t a = desc_lohi((ls + (C::oB >> 4) + C::dense_off(C::BM * 128, kb * C::kDenseMmaK)) | kLbo,
                                             kHi128);
                const uint64_t b = desc_lohi((ls + (C::oW >> 4) + C::dense_off(C::kBoxW, kb * C::kDenseMmaK)) | kLbo,
                                             kHi128);
                const uint32_t sfa = (slot + C::cSfaB + 4 * chunk) | (byte << 30);
                const uint32_t sfb = (slot + C::cSfbD + 4 * C::kNRB * chunk) | (byte << 30);
                if constexpr (KIND == GK_NVF4) mma_nvf4(acc, a, b, idesc, sfa, sfb, accumulate);
                else if constexpr (KIND == GK_MXF4) mma_mxf4(acc, a, b, idesc, sfa, sfb, accumulate);
                else mma_mxf8f6f4(acc, a, b, idesc, sfa, sfb, accumulate);
                accumulate = 1;
              }
            }
          }
          if (run_dense) {
            // residual: dense MMAs over the same W tile
#pragma unroll
            for (int kb = 0; kb < C::BK / C::kDenseMmaK; kb++) {
              constexpr int kScales = C::kDenseMmaK / C::kVecDense;
              const uint32_t chunk = (kb * kScales) / 4, byte = (kb * kScales) % 4;
              const uint32_t idesc = C::kIdesc | (byte << 29) | (byte << 4);
              const uint64_t a = desc_lohi((ls + (C::oR >> 4) + C::dense_off(C::kBoxR, kb * C::kDenseMmaK)) | kLbo,
                                           kHi128);
              const uint64_t b = desc_lohi((ls + (C::oW >> 4) + C::dense_off(C::kBoxW, kb * C::kDenseMmaK)) | kLbo,
                                           kHi128);
              const uint32_t sfa = (slot + C::cSfaR + 4 * chunk) | (byte << 30);
              const uint32_t sfb = (slot + C::cSfbD + 4 * C::kNRB * chunk) | (byte << 30);
              if constexpr (KIND == GK_NVF4) mma_nvf4(acc, a, b, idesc, sfa, sfb, accumulate);
              else if constexpr (KIND == GK_MXF4) mma_mxf4(acc, a, b, idesc, sfa, sfb, accumulate);
              else mma_mxf8f6f4(acc, a, b, idesc, sfa, sfb, accumulate);
              accumulate = 1;
            }
          }
          tc_commit_u32(empty0 + (uint32_t)(stage * 8));
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (*abort_flag) break;
        tc_commit(acc_full);
      }
      // every tcgen05 op of this thread is complete before tensor memory is freed
      tc_commit(drain);
      (void)mbar_wait(drain, 0, 1000000000ull, nullptr, true);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------- epilogue
    // accumulator lanes 32q..32q+31 (output rows), columns kCols*hcol ..
    constexpr int kCols = C::BN / 2;
    const int q = warp & 3, hcol = (warp - 2) >> 2;
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(kCols * hcol);
    uint8_t* yb = ybuf + (warp - 2) * (32 * C::kYCols * 2);
    int it = 0;
    for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x, it++) {
      const int tile = item / n_split;
      const TileXY xy = tile_xy(tile, m_tiles, n_tiles, C::kBandTiles);
      const int mt = xy.mt, nt = xy.nt;
      const int64_t m0 = (int64_t)mt * C::BM;
      const int e = tile_expert(m0);
      if (e < 0) { it--; continue; }
      if (!mbar_wait(acc_full, it & 1, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
      tc_fence_after();
      const float alpha = __fmul_rn(__ldg(p.tensor_x + 2), __ldg(p.tensor_w + 3 * e + 2));
      const int64_t row = m0 + 32 * q + lane;
      const bool st = row < p.t;
      const int64_t n0 = (int64_t)nt * C::BN + kCols * hcol;
      if constexpr (SPLIT) {
        // this K slice's raw sums into its own slot of the fp32 buffer (each
        // warp its rows); the CTA that completes the tile's last slice adds
        // the slots in slice order (the same bits on every call) with all 256
        // epilogue threads, coalesced along the rows, scales, writes y and
        // resets the tile's counter for the next call
        const int sidx = item % n_split;
        const int64_t slot_elems = p.t_pad * p.n;
        float4* mine = reinterpret_cast<float4*>(p.split_acc + sidx * slot_elems + row * p.n + n0);
#pragma unroll 1
        for (int c2 = 0; c2 < kCols / 32; c2 += 2) {
          uint32_t v[2][32];
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2), v[0]);
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2 + 32), v[1]);
          tmem_ld_wait();
          if (!st) continue;
#pragma unroll
          for (int h = 0; h < 2; h++)
#pragma unroll
            for (int j = 0; j < 8; j++)
              __stcg(mine + (c2 + h) * 8 + j,
                     make_float4(__uint_as_float(v[h][4 * j]), __uint_as_float(v[h][4 * j + 1]),
                                 __uint_as_float(v[h][4 * j + 2]), __uint_as_float(v[h][4 * j + 3])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        __threadfence();  // this slice's sums are visible before the counter moves
        __syncwarp();
        const int et = threadIdx.x - 64;  // 0..255 over the eight epilogue warps
        if (lane == 0) mbar_arrive(ep_done);
        if (et == 0) {
          if (!mbar_wait(ep_done, it & 1, p.timeout_ns, abort_flag)) *abort_flag = 1;
          else *split_last = atomicAdd(p.split_cnt + tile, 1u) == (uint32_t)(n_split - 1) ? 1u : 0u;
          mbar_arrive(ep_flag);
        }
        if (!mbar_wait(ep_flag, it & 1, p.timeout_ns, abort_flag) || *abort_flag) { *abort_flag = 1; break; }
        const bool last = *split_last != 0u;
        if (!last) continue;
        __threadfence();
        const int64_t rows = (p.t - m0) < C::BM ? (p.t - m0) : C::BM;
        const int c4n = C::BN / 4;  // float4 groups per row of the tile
        const int64_t tile_f4 = (m0 * p.n + (int64_t)nt * C::BN) / 4;
        const float4* acc4 = reinterpret_cast<const float4*>(p.split_acc) + tile_f4;
#pragma unroll 1
        for (int64_t idx0 = 0; idx0 < rows * c4n; idx0 += 4 * 256) {
          float4 b[kMaxSplit][4];  // four groups per thread, every slice: all loads in flight at once
#pragma unroll
          for (int sl = 0; sl < kMaxSplit; sl++)
#pragma unroll
            for (int u = 0; u < 4; u++) {
              const int64_t idx = idx0 + u * 256 + et;
              const int64_t off = (idx / c4n) * (p.n / 4) + idx % c4n;
              b[sl][u] = (sl < n_split && idx < rows * c4n) ? __ldcg(acc4 + sl * (slot_elems / 4) + off)
                                                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          float4 a[4];
#pragma unroll
          for (int u = 0; u < 4; u++) {
            a[u] = b[0][u];
#pragma unroll
            for (int sl = 1; sl < kMaxSplit; sl++)
              if (sl < n_split)
                a[u] = make_float4(__fadd_rn(a[u].x, b[sl][u].x), __fadd_rn(a[u].y, b[sl][u].y),
                                   __fadd_rn(a[u].z, b[sl][u].z), __fadd_rn(a[u].w, b[sl][u].w));
          }
#pragma unroll
          for (int u = 0; u < 4; u++) {
            const int64_t idx = idx0 + u * 256 + et;
            if (idx >= rows * c4n) continue;
            const int64_t r = m0 + idx / c4n, c = (int64_t)nt * C::BN + 4 * (idx % c4n);
            const float f0 = __fmul_rn(a[u].x, alpha), f1 = __fmul_rn(a[u].y, alpha);
            const float f2 = __fmul_rn(a[u].z, alpha), f3 = __fmul_rn(a[u].w, alpha);
            if (p.y_bf16) {
              __nv_bfloat162 lo = __floats2bfloat162_rn(f0, f1), hi = __floats2bfloat162_rn(f2, f3);
              *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.y) + r * p.n + c) =
                  make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
            } else {
              *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + r * p.n + c) = make_float4(f0, f1, f2, f3);
            }
          }
        }
        if (et == 0) p.split_cnt[tile] = 0u;
        continue;
      }
      if (p.y_bf16) {
        // this warp's columns into registers as bf16, release the accumulator
        // so the next tile's MMAs start, then 32 x 16 tiles through shared
        // memory with TMA stores (rows at or beyond t are outside the map)
        uint32_t pk[kCols / 2];
#pragma unroll
        for (int c2 = 0; c2 < kCols / 32; c2 += 2) {
          uint32_t v[2][32];  // two loads in flight per wait
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2), v[0]);
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2 + 32), v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; h++) {
#pragma unroll
            for (int j = 0; j < 16; j++) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[h][2 * j]), alpha),
                                                        __fmul_rn(__uint_as_float(v[h][2 * j + 1]), alpha));
              pk[16 * (c2 + h) + j] = *reinterpret_cast<uint32_t*>(&h2);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        const int32_t row0 = (int32_t)(m0 + 32 * q);
        if (row0 >= p.t) continue;  // padding rows only: nothing to write
#pragma unroll
        for (int c = 0; c < kCols / C::kYCols; c++) {
          constexpr int kW = C::kYCols / 2;  // packed words per row and chunk
          if (lane == 0) bulk_wait_group_read0();  // the previous store has read the buffer
          __syncwarp();
          uint4* d = reinterpret_cast<uint4*>(yb + C::kYCols * 2 * lane);
#pragma unroll
          for (int j = 0; j < kW / 4; j++)
            d[j] = make_uint4(pk[kW * c + 4 * j], pk[kW * c + 4 * j + 1], pk[kW * c + 4 * j + 2], pk[kW * c + 4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&maps.y, smem_u32(yb), (int32_t)(2 * (n0 + C::kYCols * c)), row0);  // x in bytes
            bulk_commit_group();
          }
        }
        continue;
      }
#pragma unroll 1
      for (int c2 = 0; c2 < kCols / 32; c2 += 2) {
        uint32_t vv[2][32];
        tmem_ld32_nowait(tq + (uint32_t)(32 * c2), vv[0]);
        tmem_ld32_nowait(tq + (uint32_t)(32 * c2 + 32), vv[1]);
        tmem_ld_wait();
        if (!st) continue;
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const uint32_t(&v)[32] = vv[h];
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + row * p.n + n0 + 32 * (c2 + h));
#pragma unroll
          for (int j = 0; j < 8; j++)
            dst[j] = make_float4(__fmul_rn(__uint_as_float(v[4 * j]), alpha),
                                 __fmul_rn(__uint_as_float(v[4 * j + 1]), alpha),
                                 __fmul_rn(__uint_as_float(v[4 * j + 2]), alpha),
                                 __fmul_rn(__uint_as_float(v[4 * j + 3]), alpha));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
    if (lane == 0) bulk_wait_group0();  // output stores complete
  } else {
    // ------------------------------------------------ scale-slot staging
    // warps 10-13, one per tensor-memory lane quadrant: scale factors and
    // metadata of each K tile, shared memory -> this warp's quadrant of the
    // stage's tensor-memory slot (the layout tcgen05.cp .32x128b.warpx4 and
    // .128x128b would produce), so that the tensor pipe runs MMAs only
    const int q = warp & 3;
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16);
    int stage = 0;
    uint32_t phase = 0;
    for (int item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
      const int tile = item / n_split, k0 = k_lo(item), k1 = k_hi(item);
      const int mt = tile_xy(tile, m_tiles, n_tiles, C::kBandTiles).mt;
      if (tile_expert((int64_t)mt * C::BM) < 0) continue;
      for (int kt = k0; kt < k1; kt++) {
        if (!mbar_wait(&full[stage], phase, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
        const uint8_t* sb = smem + stage * C::kStageBytes;
        const uint32_t slot = tq + C::BN + (uint32_t)(stage * C::kSlotCols);
#pragma unroll
        for (int c = 0; c < C::kChunksR; c++) {
          tmem_st4(slot + C::cSfaR + 4 * c, *reinterpret_cast<const uint4*>(sb + C::oSfaR + 512 * c + 16 * lane));
          if constexpr (!SPARSE) {
#pragma unroll
            for (int rb = 0; rb < C::kNRB; rb++)
              tmem_st4(slot + C::cSfbD + 4 * C::kNRB * c + 4 * rb,
                       *reinterpret_cast<const uint4*>(sb + C::oSfbD + rb * C::kChunksR * 512 + 512 * c + 16 * lane));
          }
        }
#pragma unroll
        for (int c = 0; c < C::kChunksB; c++) {
          tmem_st4(slot + C::cSfaB + 4 * c, *reinterpret_cast<const uint4*>(sb + C::oSfaB + 512 * c + 16 * lane));
          if constexpr (SPARSE) {
#pragma unroll
            for (int rb = 0; rb < C::kNRB; rb++) {
              const uint4 v =
                  *reinterpret_cast<const uint4*>(sb + C::oSfbS + rb * C::kChunksB * 512 + 512 * c + 16 * lane);
              tmem_st4(slot + C::cSfbS + 4 * C::kNRB * c + 4 * rb, v);
              // dense-view chunks 2c and 2c+1: scales (s0 s0 s1 s1) and (s2 s2 s3 s3) of each row
              tmem_st4(slot + C::cSfbD + 4 * C::kNRB * (2 * c) + 4 * rb, dup_lo_scales(v));
              tmem_st4(slot + C::cSfbD + 4 * C::kNRB * (2 * c + 1) + 4 * rb, dup_hi_scales(v));
            }
          }
        }
#pragma unroll
        for (int bx = 0; bx < C::kEBoxes; bx++)  // metadata: tile row 32q + lane
          tmem_st4(slot + C::cE + 4 * bx,
                   *reinterpret_cast<const uint4*>(sb + C::oE + bx * C::BM * 16 + 16 * (32 * q + lane)));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_ready[stage]);
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Wait on a flag that nothing sets: exercises the bounded-wait failure path.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    (void)mbar_wait(&bar, 0, timeout_ns);
  }
}

}  // namespace sharq
