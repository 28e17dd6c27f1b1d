// gemm_pair.cuh -- the sparse + dense FP4 GEMM pair of the SharQ layer on CTA
// pairs (tcgen05 cta_group::2).
//
// Same computation as gemm_kernel (SharQ abstract and Section 1: a sparse FP4
// GEMM over the compressed backbone and its metadata, plus a dense FP4 GEMM
// over the residual, both reading one shared FP4 weight tile and accumulating
// into one output), for the 4:8 pair kinds (kind::mxf4nvf4 / kind::mxf4 and
// their .sp forms) with unscattered rows.  Two CTAs on neighbouring SMs form a
// cluster and compute a 256 x 256 output tile: each CTA holds 128 activation
// rows and 128 of the 256 weight rows in its shared memory, and the leader CTA
// (cluster rank 0) issues one M = 256 MMA that reads the operands of both.
// Each SM therefore loads half a weight tile per stage instead of a whole one
// (51 KB per stage instead of 67 KB), which leaves room for a fourth stage.
//
// Per CTA (448 threads, one CTA per SM):
//   warp 0      TMA producer: weight half, residual and backbone tiles with the
//               pair form of the tensor load, whose completion is counted on
//               the leader's full[] barrier; metadata and scale factors on this
//               CTA's own sfull[] barrier;
//   warp 1      tensor-memory allocation for the pair; in the leader, the MMA
//               issuer (one thread), committing to empty[] and acc_full of both
//               CTAs;
//   warps 2-9   the accumulator drain of its 128 output rows, two warps per
//               32-lane quadrant, 128 columns each (bf16 output: the columns
//               into registers first, then the accumulator is released and
//               the stores drain under the next tile's MMAs);
//   warps 10-13 scale factors and metadata of this CTA -> its tensor-memory
//               slot (its own 128 activation rows, all 256 weight rows).
// Four shared-memory stages, three tensor-memory scale slots (a slot is
// rewritten once the MMAs of the K tile that used it have retired).  Every
// wait is bounded in time; the abort flag of both CTAs is set on any timeout.
#pragma once
#include "gemm.cuh"

namespace sharq {

template <int KIND>
struct PairCfg {
  static_assert(KIND == GK_NVF4 || KIND == GK_MXF4, "CTA pairs run the 4:8 pair sparse kinds");
  static constexpr int BM = 128;   // activation (and accumulator) rows per CTA
  static constexpr int BN = 256;   // output columns of a pair tile, all in each CTA's accumulator
  static constexpr int BNh = 128;  // weight rows each CTA loads
  static constexpr int BK = 256;   // logical K per stage
  static constexpr int kNRB = 2;   // 128-row blocks of weight scales, all of them in every CTA
  static constexpr int kVecDense = (KIND == GK_NVF4) ? 16 : 32;
  static constexpr int kVecSparse = 2 * kVecDense;
  static constexpr int kDenseMmaK = 64, kSparseMmaK = 128;
  static constexpr int kBoxR = BM * 128, kBoxW = BNh * 128, kBBytes = BM * 64, kEBytes = BM * 16;
  static constexpr int kMetaStage = BK / 16;                   // metadata bytes per row per stage
  static constexpr int kXStage = BK / 2, kXStageB = BK / 4;    // TMA inner coordinate steps (bytes)
  static constexpr int kChunksR = BK / kVecDense / 4;          // 512-byte scale chunks per stage
  static constexpr int kChunksB = BK / kVecSparse / 4;
  // the weight's dense-view scales are its sparse-view scales repeated (one weight
  // scale per 2b logical K): only the sparse view is loaded, the staging warps
  // write both views into tensor memory
  static_assert(kChunksR == 2 * kChunksB, "dense view = each sparse-view scale twice");
  static constexpr int kSfaR = kChunksR * 512, kSfbD = 0;
  static constexpr int kSfaB = kChunksB * 512, kSfbS = kNRB * kChunksB * 512;
  static constexpr int oW = 0, oR = oW + kBoxW, oB = oR + kBoxR, oE = oB + kBBytes;
  static constexpr int oSfaR = oE + kEBytes, oSfbD = oSfaR + kSfaR, oSfaB = oSfbD + kSfbD, oSfbS = oSfaB + kSfaB;
  static constexpr int kStageBytes = ((oSfbS + kSfbS + 1023) / 1024) * 1024;
  static constexpr int kStages = 4;  // shared-memory stages
  static constexpr int kSlots = 3;   // tensor-memory scale slots
  static constexpr uint32_t kTxPair = 2u * (kBoxW + kBoxR + kBBytes);  // both CTAs' tensor loads, leader's full[]
  static constexpr uint32_t kTxLocal = kEBytes + kSfaR + kSfbD + kSfaB + kSfbS;
  static constexpr int cSfaR = 0, cSfbD = cSfaR + 4 * kChunksR, cSfaB = cSfbD + 4 * kNRB * kChunksR;
  static constexpr int cSfbS = cSfaB + 4 * kChunksB, cE = cSfbS + 4 * kNRB * kChunksB;
  static constexpr int kSlotCols = cE + 4;
  static constexpr int kTmemCols = 512;
  static_assert(BN + kSlots * kSlotCols <= kTmemCols, "tensor memory budget");
  static constexpr int kYBuf = 8 * 2048;  // bf16 output staging: 32 rows x 32 columns per epilogue warp
  static constexpr int kSmemBytes = kStages * kStageBytes + kYBuf + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // E2M1 x E2M1, K-major, M = 256 (the pair), N = 256
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((KIND == GK_NVF4 ? 0u : 1u) << 23) | ((uint32_t)(256 >> 4) << 24);
  static constexpr uint32_t kIdescSp = kIdesc | (1u << 2);
  static constexpr int kBandTiles = 8;  // row-tile pairs per raster band (2048 rows)
};

__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// SK: the stream-K form (p.sk_part set); otherwise whole tiles only.
template <int KIND, bool SK>
__global__ void __launch_bounds__(448, 1) gemm_pair_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using C = PairCfg<KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ybuf = smem + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ybuf + C::kYBuf);  // leader: both CTAs' tiles
  uint64_t* empty = full + C::kStages;       // this CTA: the stage's MMAs have retired
  uint64_t* sfull = empty + C::kStages;      // this CTA: its metadata and scale factors have landed
  uint64_t* sf_ready = sfull + C::kStages;   // leader: both CTAs' scale slots are in tensor memory
  uint64_t* acc_full = sf_ready + C::kSlots; // this CTA: the tile's accumulator is complete
  uint64_t* acc_empty = acc_full + 1;        // leader: both CTAs have drained their accumulator
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the leader, which issues the MMAs
  const int cluster = (int)(blockIdx.x >> 1), nclusters = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfull[s], 1);
    }
    for (int j = 0; j < C::kSlots; j++) mbar_init(&sf_ready[j], 8);  // 4 staging warps x 2 CTAs
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 16);  // 8 epilogue warps x 2 CTAs
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, C::kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&maps.w);
    tma_prefetch(&maps.r);
    tma_prefetch(&maps.b);
    tma_prefetch(&maps.e);
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t abort_peer = mapa_u32(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  auto abort_both = [&]() {
    *abort_flag = 1;
    st_cluster_u32(abort_peer, 1u);
  };

  const int m_pairs = (int)(p.t_pad / 256);
  const int n_tiles = (int)(p.n / C::BN);
  const int num_tiles = m_pairs * n_tiles;
  const int k_tiles = (int)(p.k / C::BK);
  if (warp == 0 && lane == 0 && cluster < num_tiles) {
    // while the kernel before this one finishes: warm L2 with this CTA's share
    // of the weight tile of its first tile, whole TMA boxes (the pairs on one
    // column of tiles split its K tiles); the weight is not written by the
    // preparation kernels
    const TileXY x = tile_xy(cluster, m_pairs, n_tiles, C::kBandTiles);
    const int per = (k_tiles + x.h - 1) / x.h, i = x.mt - x.lo;
    const int32_t wrow = (int32_t)((int64_t)x.nt * C::BN + C::BNh * rank);
    for (int kt = i * per; kt < (i + 1) * per && kt < k_tiles; kt++)
      tma_prefetch_l2_2d(&maps.w, kt * C::kXStage, wrow);
  }
  grid_dep_wait();  // the prepared activations (and scales) are complete

  // Work of this pair.  Whole tiles cluster, cluster + nclusters, ... in raster
  // order; or, with a stream-K workspace, the contiguous run [u_lo, u_hi) of
  // an even split of all (tile, K tile) units over the pairs, cut at tile
  // boundaries into segments [ks, ke) of one tile.  A segment that starts inside
  // its tile (ks > 0, only a pair's first) leaves its partial sums in this
  // pair's workspace slot; the segment that holds the tile's K tile 0 but not
  // its last (only a pair's last) adds the partials of the pairs after it
  // before writing the output; every other segment is a whole tile.
  constexpr bool sk = SK;
  const int64_t units = (int64_t)num_tiles * k_tiles;
  auto unit_lo = [&](int64_t q) -> int64_t { return q * units / nclusters; };
  auto next_seg = [&](int64_t& st, int& tile, int& ks, int& ke) -> bool {
    if (sk) {
      const int64_t hi = unit_lo(cluster + 1);
      if (st >= hi) return false;
      tile = (int)(st / k_tiles);
      ks = (int)(st - (int64_t)tile * k_tiles);
      const int64_t tend = (int64_t)(tile + 1) * k_tiles;
      ke = (int)((tend < hi ? tend : hi) - (int64_t)tile * k_tiles);
      st = (int64_t)tile * k_tiles + ke;
      return true;
    }
    if (st >= num_tiles) return false;
    tile = (int)st;
    ks = 0;
    ke = k_tiles;
    st += nclusters;
    return true;
  };
  const int64_t seg0 = sk ? unit_lo(cluster) : (int64_t)cluster;
  const int64_t sd_blocks = (p.k / C::kVecDense + 3) / 4;   // 512-byte blocks per 128-row block, dense view
  const int64_t sb_blocks = (p.k / C::kVecSparse + 3) / 4;  // backbone / sparse view
  const bool run_sparse = (p.paths & 1) != 0;
  const bool run_dense = (p.paths & 2) != 0;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t g = 0, issued = 0, issued_par = 0;
      const uint32_t smem0 = smem_u32(smem);
      const uint32_t full_leader = mapa_u32(smem_u32(full), 0);
      int64_t st = seg0;
      int tile, ks, ke;
      while (!*abort_flag && next_seg(st, tile, ks, ke)) {
        const TileXY xy = tile_xy(tile, m_pairs, n_tiles, C::kBandTiles);
        const int mt = xy.mt, nt = xy.nt;
        const int64_t m0 = (int64_t)mt * 256 + 128 * (int64_t)rank;         // this CTA's activation rows
        const int32_t wrow = (int32_t)((int64_t)nt * C::BN + C::BNh * rank);  // this CTA's weight rows
        const uint8_t* g_sfa_r = p.sf_res + (m0 / 128) * sd_blocks * 512 + (int64_t)ks * C::kSfaR;
        const uint8_t* g_sfa_b = p.sf_bb + (m0 / 128) * sb_blocks * 512 + (int64_t)ks * C::kSfaB;
        const uint8_t* g_sfb_s =
            p.sf_w_sparse + (int64_t)nt * C::kNRB * sb_blocks * 512 + (int64_t)ks * C::kChunksB * 512;
        int32_t kx = ks * C::kXStage, kx_b = ks * C::kXStageB, kx_e = ks * C::kMetaStage;
        for (int kt = ks; kt < ke; kt++, g++) {
          const int stage = (int)(g % C::kStages);
          const uint32_t ph = (g / C::kStages) & 1u;
          if (!mbar_wait(&empty[stage], ph ^ 1u, p.timeout_ns, abort_flag)) { abort_both(); break; }
          const uint32_t sb = smem0 + (uint32_t)(stage * C::kStageBytes);
          const uint32_t fl = full_leader + (uint32_t)(stage * 8);
          const uint32_t sf = smem_u32(&sfull[stage]);
          if (rank == 0) mbar_arrive_expect_tx_u32(smem_u32(&full[stage]), C::kTxPair);
          tma_load_2d_pair(sb + C::oW, &maps.w, kx, wrow, fl);
          tma_load_2d_pair(sb + C::oR, &maps.r, kx, (int32_t)m0, fl);
          tma_load_2d_pair(sb + C::oB, &maps.b, kx_b, (int32_t)m0, fl);
          mbar_arrive_expect_tx_u32(sf, C::kTxLocal);
          tma_load_2d_u32(sb + C::oE, &maps.e, kx_e, (int32_t)m0, sf);
          bulk_load_u32(sb + C::oSfaR, g_sfa_r, C::kSfaR, sf);
          bulk_load_u32(sb + C::oSfaB, g_sfa_b, C::kSfaB, sf);
#pragma unroll
          for (int rb = 0; rb < C::kNRB; rb++)
            bulk_load_u32(sb + C::oSfbS + rb * C::kChunksB * 512, g_sfb_s + rb * sb_blocks * 512, C::kChunksB * 512,
                          sf);
          kx += C::kXStage;
          kx_b += C::kXStageB;
          kx_e += C::kMetaStage;
          g_sfa_r += C::kSfaR;
          g_sfa_b += C::kSfaB;
          g_sfb_s += C::kChunksB * 512;
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (ph << stage);
        }
      }
      if (*abort_flag) {
        // let every local load already issued land before the block can exit
        for (int i = 0; i < C::kStages; i++)
          if ((issued >> i) & 1u) (void)mbar_wait(&sfull[i], (issued_par >> i) & 1u, 1000000000ull, nullptr, true);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (rank == 0 && lane == 0) {
      uint32_t g = 0;
      int it = 0;
      const uint32_t acc = tmem_base;
      constexpr uint32_t kHi128 = desc_hi(1024, 2), kHi64 = desc_hi(512, 4);
      constexpr uint32_t kLbo = 1u << 16;
      const uint32_t lo0 = smem_u32(smem) >> 4;
      const uint32_t empty_own = smem_u32(empty), empty_peer = mapa_u32(empty_own, 1);
      const uint32_t accf_own = smem_u32(acc_full), accf_peer = mapa_u32(accf_own, 1);
      int64_t st = seg0;
      int tile, ks, ke;
      for (; !*abort_flag && next_seg(st, tile, ks, ke); it++) {
        if (!mbar_wait(acc_empty, (uint32_t)(it & 1) ^ 1u, p.timeout_ns, abort_flag)) { abort_both(); break; }
        tc_fence_after();
        uint32_t accumulate = 0;
        for (int kt = ks; kt < ke; kt++, g++) {
          const int stage = (int)(g % C::kStages), slot = (int)(g % C::kSlots);
          if (!mbar_wait(&full[stage], (g / C::kStages) & 1u, p.timeout_ns, abort_flag)) { abort_both(); break; }
          if (!mbar_wait(&sf_ready[slot], (g / C::kSlots) & 1u, p.timeout_ns, abort_flag)) { abort_both(); break; }
          tc_fence_after();
          const uint32_t ls = lo0 + (uint32_t)(stage * (C::kStageBytes >> 4));
          const uint32_t sl = tmem_base + C::BN + (uint32_t)(slot * C::kSlotCols);
          if (run_sparse) {
#pragma unroll
            for (int kb = 0; kb < C::BK / C::kSparseMmaK; kb++) {
              constexpr int kScales = C::kSparseMmaK / C::kVecSparse;
              const uint32_t chunk = (kb * kScales) / 4, byte = (kb * kScales) % 4;
              const uint32_t idesc = C::kIdescSp | (byte << 29) | (byte << 4);
              const uint64_t a = desc_lohi((ls + (C::oB >> 4) + 2 * kb) | kLbo, kHi64);
              const uint64_t b = desc_lohi((ls + (C::oW >> 4) + 4 * kb) | kLbo, kHi128);
              const uint32_t sfa = (sl + C::cSfaB + 4 * chunk) | (byte << 30);
              const uint32_t sfb = (sl + C::cSfbS + 4 * C::kNRB * chunk) | (byte << 30);
              const uint32_t e = sl + C::cE + 2 * kb;
              if constexpr (KIND == GK_NVF4) mma_nvf4_sp_pair(acc, a, b, e, idesc, sfa, sfb, accumulate);
              else mma_mxf4_sp_pair(acc, a, b, e, idesc, sfa, sfb, accumulate);
              accumulate = 1;
            }
          }
          if (run_dense) {
#pragma unroll
            for (int kb = 0; kb < C::BK / C::kDenseMmaK; kb++) {
              constexpr int kScales = C::kDenseMmaK / C::kVecDense;
              const uint32_t chunk = (kb * kScales) / 4, byte = (kb * kScales) % 4;
              const uint32_t idesc = C::kIdesc | (byte << 29) | (byte << 4);
              const uint64_t a = desc_lohi((ls + (C::oR >> 4) + 2 * kb) | kLbo, kHi128);
              const uint64_t b = desc_lohi((ls + (C::oW >> 4) + 2 * kb) | kLbo, kHi128);
              const uint32_t sfa = (sl + C::cSfaR + 4 * chunk) | (byte << 30);
              const uint32_t sfb = (sl + C::cSfbD + 4 * C::kNRB * chunk) | (byte << 30);
              if constexpr (KIND == GK_NVF4) mma_nvf4_pair(acc, a, b, idesc, sfa, sfb, accumulate);
              else mma_mxf4_pair(acc, a, b, idesc, sfa, sfb, accumulate);
              accumulate = 1;
            }
          }
          tc_commit_pair(empty_own + (uint32_t)(stage * 8));
          tc_commit_pair(empty_peer + (uint32_t)(stage * 8));
        }
        if (*abort_flag) break;
        tc_commit_pair(accf_own);
        tc_commit_pair(accf_peer);
      }
      // every MMA of the pair is complete before either CTA frees tensor memory or exits
      tc_commit_pair(smem_u32(drain));
      (void)mbar_wait(drain, 0, 1000000000ull, nullptr, true);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------- epilogue
    // accumulator lanes 32q..32q+31 (this CTA's output rows), columns
    // 128h..128h+127
    constexpr int kCols = C::BN / 2;
    const int q = warp & 3, hcol = (warp - 2) >> 2;
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(kCols * hcol);
    const uint32_t acc_empty_leader = mapa_u32(smem_u32(acc_empty), 0);
    const int w8 = warp - 2;  // this warp's share of a partial-sum slot
    // partial sums of pair q's slot for this CTA and warp: 32 x 128 fp32 as
    // float4 [column chunk c (32)][4-column group j (8)][lane]
    auto part_of = [&](int64_t q) {
      return reinterpret_cast<float4*>(p.sk_part) + ((q * 2 + rank) * 8 + w8) * (kCols / 4) * 32;
    };
    auto flag_of = [&](int64_t q) { return p.sk_flag + (q * 2 + rank) * 8 + w8; };
    int it = 0;
    int64_t st = seg0;
    int tile, ks, ke;
    for (; !*abort_flag && next_seg(st, tile, ks, ke); it++) {
      const TileXY xy = tile_xy(tile, m_pairs, n_tiles, C::kBandTiles);
      const int mt = xy.mt, nt = xy.nt;
      if (!mbar_wait(acc_full, (uint32_t)(it & 1), p.timeout_ns, abort_flag)) { abort_both(); break; }
      tc_fence_after();
      if (sk && ks > 0) {
        // stream-K, a segment that starts inside its tile: the raw sums go to
        // this pair's slot; the pair holding the tile's K tile 0 adds them
        float4* part = part_of(cluster);
#pragma unroll 1
        for (int c2 = 0; c2 < kCols / 32; c2 += 2) {
          uint32_t v[2][32];
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2), v[0]);
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2 + 32), v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; h++)
#pragma unroll
            for (int j = 0; j < 8; j++)
              __stcg(part + ((c2 + h) * 8 + j) * 32 + lane,
                     make_float4(__uint_as_float(v[h][4 * j]), __uint_as_float(v[h][4 * j + 1]),
                                 __uint_as_float(v[h][4 * j + 2]), __uint_as_float(v[h][4 * j + 3])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader);
        __threadfence();  // the partial is visible device-wide before its counter turns odd
        __syncwarp();
        if (lane == 0) atomicAdd(flag_of(cluster), 1u);
        continue;
      }
      // pairs after this one whose first segments complete this tile (stream-K)
      // (the host launches stream-K only with at least two units per pair, so
      // every pair's run is non-empty and starts after the previous one's)
      int q_end = cluster + 1;
      if (sk && ke < k_tiles) {
        const int64_t tend = (int64_t)(tile + 1) * k_tiles;
        while (q_end < nclusters && unit_lo(q_end) < tend) q_end++;
        bool ok = true;
        if (lane == 0)
          for (int q = cluster + 1; q < q_end && ok; q++) ok = wait_odd_acquire(flag_of(q), p.timeout_ns, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        __syncwarp();
        __threadfence();
        if (!ok) { abort_both(); break; }
      }
      const float alpha = __fmul_rn(__ldg(p.tensor_x + 2), __ldg(p.tensor_w + 2));
      const int64_t row = (int64_t)mt * 256 + 128 * (int64_t)rank + 32 * q + lane;
      const bool store = row < p.t;
      const int64_t n0 = (int64_t)nt * C::BN + kCols * hcol;
      // 32 columns of this warp's accumulator (+ the partial sums) as fp32
      auto drain = [&](const uint32_t (&v)[32], int c, float (&f)[32]) {
#pragma unroll
        for (int i = 0; i < 32; i++) f[i] = __uint_as_float(v[i]);
        for (int qq = cluster + 1; SK && qq < q_end; qq++) {
          const float4* part = part_of(qq);
#pragma unroll
          for (int j = 0; j < 8; j++) {
            const float4 a = __ldcg(part + (c * 8 + j) * 32 + lane);
            f[4 * j] = __fadd_rn(f[4 * j], a.x);
            f[4 * j + 1] = __fadd_rn(f[4 * j + 1], a.y);
            f[4 * j + 2] = __fadd_rn(f[4 * j + 2], a.z);
            f[4 * j + 3] = __fadd_rn(f[4 * j + 3], a.w);
          }
        }
      };
      auto release_partials = [&]() {  // the partials added here may be rewritten by the next call
        if (SK) {
          __syncwarp();
          if (lane == 0)
            for (int qq = cluster + 1; qq < q_end; qq++) atomicAdd(flag_of(qq), 1u);
        }
      };
      if (p.y_bf16) {
        // this warp's columns into registers as bf16, then release the
        // accumulator so the next tile's MMAs start while the stores drain
        uint32_t pk[kCols / 2];
#pragma unroll
        for (int c2 = 0; c2 < kCols / 32; c2 += 2) {
          uint32_t v[2][32];  // two loads in flight per wait
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2), v[0]);
          tmem_ld32_nowait(tq + (uint32_t)(32 * c2 + 32), v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; h++) {
            float f[32];
            drain(v[h], c2 + h, f);
#pragma unroll
            for (int j = 0; j < 16; j++) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__fmul_rn(f[2 * j], alpha), __fmul_rn(f[2 * j + 1], alpha));
              pk[16 * (c2 + h) + j] = *reinterpret_cast<uint32_t*>(&h2);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader);
        release_partials();
        // 32 rows x 32 columns at a time through shared memory, written by a
        // TMA store (whole lines; rows at or beyond t are clipped by the map)
        (void)store;
        uint8_t* yb = ybuf + (warp - 2) * 2048;
        const int32_t row0 = (int32_t)(row - lane);
        if (row0 >= p.t) continue;  // padding rows only: nothing to write
#pragma unroll
        for (int c = 0; c < kCols / 32; c++) {
          if (lane == 0) bulk_wait_group_read0();  // the previous store has read the buffer
          __syncwarp();
          uint4* d = reinterpret_cast<uint4*>(yb + 64 * lane);
#pragma unroll
          for (int j = 0; j < 4; j++)
            d[j] = make_uint4(pk[16 * c + 4 * j], pk[16 * c + 4 * j + 1], pk[16 * c + 4 * j + 2], pk[16 * c + 4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&maps.y, smem_u32(yb), (int32_t)(2 * (n0 + 32 * c)), row0);  // x in bytes
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
        if (!store) continue;
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const int c = c2 + h;
          float f[32];
          drain(vv[h], c, f);
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + row * p.n + n0 + 32 * c);
#pragma unroll
          for (int j = 0; j < 8; j++)
            dst[j] = make_float4(__fmul_rn(f[4 * j], alpha), __fmul_rn(f[4 * j + 1], alpha),
                                 __fmul_rn(f[4 * j + 2], alpha), __fmul_rn(f[4 * j + 3], alpha));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_leader);
      release_partials();
    }
  } else {
    // ------------------------------------------------ scale-slot staging
    // warps 10-13, one per tensor-memory lane quadrant
    const int q = warp & 3;
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16);
    const uint32_t sf_ready_leader = mapa_u32(smem_u32(sf_ready), 0);
    uint32_t g = 0;
    int64_t st = seg0;
    int tile, ks, ke;
    while (!*abort_flag && next_seg(st, tile, ks, ke)) {
      for (int kt = ks; kt < ke; kt++, g++) {
        const int stage = (int)(g % C::kStages), slot = (int)(g % C::kSlots);
        if (g >= (uint32_t)C::kSlots) {  // the slot's previous K tile has been consumed by its MMAs
          const uint32_t gp = g - C::kSlots;
          if (!mbar_wait(&empty[gp % C::kStages], (gp / C::kStages) & 1u, p.timeout_ns, abort_flag)) {
            abort_both();
            break;
          }
        }
        if (!mbar_wait(&sfull[stage], (g / C::kStages) & 1u, p.timeout_ns, abort_flag)) { abort_both(); break; }
        const uint8_t* sb = smem + stage * C::kStageBytes;
        const uint32_t st = tq + C::BN + (uint32_t)(slot * C::kSlotCols);
#pragma unroll
        for (int c = 0; c < C::kChunksR; c++)
          tmem_st4(st + C::cSfaR + 4 * c, *reinterpret_cast<const uint4*>(sb + C::oSfaR + 512 * c + 16 * lane));
#pragma unroll
        for (int c = 0; c < C::kChunksB; c++) {
          tmem_st4(st + C::cSfaB + 4 * c, *reinterpret_cast<const uint4*>(sb + C::oSfaB + 512 * c + 16 * lane));
#pragma unroll
          for (int rb = 0; rb < C::kNRB; rb++) {
            const uint4 v = *reinterpret_cast<const uint4*>(sb + C::oSfbS + rb * C::kChunksB * 512 + 512 * c + 16 * lane);
            tmem_st4(st + C::cSfbS + 4 * C::kNRB * c + 4 * rb, v);
            // dense-view chunks 2c and 2c+1: scales (s0 s0 s1 s1) and (s2 s2 s3 s3) of each row
            tmem_st4(st + C::cSfbD + 4 * C::kNRB * (2 * c) + 4 * rb, dup_lo_scales(v));
            tmem_st4(st + C::cSfbD + 4 * C::kNRB * (2 * c + 1) + 4 * rb, dup_hi_scales(v));
          }
        }
        tmem_st4(st + C::cE, *reinterpret_cast<const uint4*>(sb + C::oE + 16 * (32 * q + lane)));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(sf_ready_leader + (uint32_t)(slot * 8));
      }
    }
  }

  if (warp >= 2 && warp < 10 && lane == 0) bulk_wait_group0();  // output stores complete

  // the leader's MMAs read this CTA's shared memory and write its tensor
  // memory: neither CTA frees tensor memory or exits before both are done
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

}  // namespace sharq
