// gemm_swap.cuh -- the layer's two GEMMs for a few activation rows (decode),
// with the weight as the 128-row MMA operand.
//
// SharQ abstract and Section 1: y = g_dec(x) g_dec(w) sum_k (B + R)[t][k] W[n][k],
// a sparse backbone product plus a dense residual product into one output,
// both reading the one FP4 weight.  With t <= 64 rows a 128-row activation tile
// would be mostly padding and the layer is a weight stream, so this kernel
// turns the product around: D[n][t] = sum_k W[n][k] (B + R)[t][k], the weight
// tile (128 rows) is operand A and the t rows (padded to TN = 32 or 64) are
// operand B.  Structured sparsity applies to operand A only, so the backbone
// is expanded on chip to its dense form (dropped positions +0, its scales
// viewed per b) and both products run as dense block-scaled MMAs into one
// tensor-memory accumulator; at this size their cost is far below the weight
// stream's.  The K loop of each 128-row weight tile is split into slices on
// different SMs that form one thread-block cluster; the cluster's first CTA
// sums the slices in slice order through distributed shared memory.
//
// Per CTA (192 threads, one work item = one weight tile x one K slice):
//   warp 0      TMA producer: weight tile, residual rows, backbone rows (compressed,
//               or dense for 8:16), metadata, and the scale chunks of both;
//   warp 1      tensor-memory owner and MMA issuer (one thread);
//   warps 2-5   per stage: the backbone expanded into its swizzled dense tile,
//               the scale chunks into the stage's tensor-memory slot (one warp per
//               32-lane quadrant, warp % 4); at the end the accumulator drain (lane = weight
//               row, column = activation row) into y, or into shared memory for the
//               cluster's first CTA.
// Every wait is bounded in time and reports through the device error word.
#pragma once
#include <cuda_bf16.h>

#include "gemm.cuh"

namespace sharq {

enum { SW_PAIR = 0, SW_24 = 1, SW_DENSE = 2 };  // backbone layouts: 4:8 pair, 2:4, dense (8:16)

template <int KIND, int BL, int TN>
struct SwapCfg {
  static_assert(KIND == GK_NVF4 || KIND == GK_MXF4, "packed FP4 kinds");
  static_assert(TN == 32 || TN == 64, "activation rows per MMA");
  static constexpr int BM = 128, BK = 256;
  static constexpr int kVec = (KIND == GK_NVF4) ? 16 : 32;         // logical K per scale (dense view)
  static constexpr int kChunksR = BK / kVec / 4;                    // 512-byte scale chunks per stage, dense view
  static constexpr int kChunksB = BL == SW_DENSE ? kChunksR : kChunksR / 2;  // backbone scales as stored
  static constexpr int kMetaRow = BL == SW_PAIR ? BK / 16 : (BL == SW_24 ? BK / 8 : 0);  // metadata bytes / row
  static constexpr int kCRow = BL == SW_DENSE ? 0 : BK / 4;         // compressed backbone bytes per row
  // stage layout (bytes)
  static constexpr int oW = 0;                    // weight: 128 rows x 128 bytes, 128-byte swizzle
  static constexpr int oR = oW + BM * 128;        // residual rows: TN x 128, 128-byte swizzle
  static constexpr int oD = oR + TN * 128;        // dense backbone: TN x 128, 128-byte swizzle
  static constexpr int oC = oD + TN * 128;        // compressed backbone: TN x 64, plain
  static constexpr int oE = oC + TN * kCRow;      // metadata: TN x kMetaRow, plain
  static constexpr int oSA = oE + TN * kMetaRow;  // weight scales (dense view)
  static constexpr int oSR = oSA + kChunksR * 512;
  static constexpr int oSB = oSR + kChunksR * 512;
  static constexpr int kStageBytes = ((oSB + kChunksB * 512 + 1023) / 1024) * 1024;
  static constexpr int kStages = TN == 32 ? 6 : 5;
  static constexpr uint32_t kTx = BM * 128 + TN * 128 + (BL == SW_DENSE ? TN * 128 : TN * kCRow + TN * kMetaRow) +
                                  (2 * kChunksR + kChunksB) * 512;
  // tensor memory: accumulator (TN columns), then one scale slot per stage
  static constexpr int cSA = 0, cSR = 4 * kChunksR, cSD = 8 * kChunksR;
  static constexpr int kSlotCols = 12 * kChunksR;
  static constexpr int kTmemCols = 512;
  static_assert(TN + kStages * kSlotCols <= kTmemCols, "tensor memory budget");
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // E2M1 x E2M1, K-major, M = 128, N = TN
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(TN >> 3) << 17) |
                                     ((KIND == GK_NVF4 ? 0u : 1u) << 23) | ((uint32_t)(BM >> 4) << 24);
};

struct SwapParams {
  int64_t t, n, k;          // activation rows (<= TN), weight rows, K
  int64_t k_tiles;          // K tiles of 256
  int32_t split;            // K slices per weight tile = CTAs per cluster (1: no split)
  const uint8_t* w_codes;   // weight codes [n][k / 2] (L2 warm-up only)
  const uint8_t* sf_w;      // weight scales, dense view, tiled
  const uint8_t* sf_res;    // activation scales, tiled (rows of the first 128-row block)
  const uint8_t* sf_bb;
  const float* tensor_x;
  const float* tensor_w;
  void* y;
  int y_bf16;
  uint64_t timeout_ns;
};

struct SwapMaps {
  CUtensorMap w, r, c, e;   // c: compressed backbone (dense backbone for 8:16)
};

// Dense 16-byte piece (32 logical K) of a backbone row from its compressed codes
// and metadata.  PAIR: per group of 8, nibble p0 | p1 << 2 of the kept pairs and
// 2 bytes of codes -> bytes p0, p1 of the group's 4 bytes.  2:4: per group of 4,
// nibble i0 | i1 << 2 and one byte (2 codes) -> nibbles i0, i1 of the group's 2 bytes.
template <int BL>
__device__ __forceinline__ uint4 expand_piece(const uint8_t* comp, const uint8_t* meta) {
  uint32_t out[4];
  if constexpr (BL == SW_PAIR) {
    const uint16_t m = *reinterpret_cast<const uint16_t*>(meta);    // 4 groups of 8
    const uint2 cw = *reinterpret_cast<const uint2*>(comp);         // 8 bytes, 2 per group
#pragma unroll
    for (int g = 0; g < 4; g++) {
      const uint32_t nib = (m >> (4 * g)) & 15u;
      const uint32_t two = ((g < 2 ? cw.x : cw.y) >> (16 * (g & 1))) & 0xFFFFu;
      const uint32_t p0 = nib & 3u, p1 = nib >> 2;
      out[g] = ((two & 0xFFu) << (8 * p0)) | ((two >> 8) << (8 * p1));
    }
  } else {
    const uint32_t m = *reinterpret_cast<const uint32_t*>(meta);    // 8 groups of 4
    const uint2 cw = *reinterpret_cast<const uint2*>(comp);         // 8 bytes, 1 per group
#pragma unroll
    for (int w = 0; w < 4; w++) {
      uint32_t v = 0;
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int g = 2 * w + h;
        const uint32_t nib = (m >> (4 * g)) & 15u;
        const uint32_t byte = ((g < 4 ? cw.x : cw.y) >> (8 * (g & 3))) & 0xFFu;
        const uint32_t i0 = nib & 3u, i1 = nib >> 2;
        v |= (((byte & 15u) << (4 * i0)) | ((byte >> 4) << (4 * i1))) << (16 * h);
      }
      out[w] = v;
    }
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <int KIND, int BL, int TN>
__global__ void __launch_bounds__(192, 1) gemm_swap_kernel(const __grid_constant__ SwapMaps maps, const SwapParams p) {
  using C = SwapCfg<KIND, BL, TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* ready = empty + C::kStages;  // backbone expanded, scales in tensor memory
  uint64_t* acc_full = ready + C::kStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work item: weight tile blockIdx / split, K slice = rank in the cluster of split CTAs
  const int tile = (int)(blockIdx.x / p.split), slice = (int)(blockIdx.x % p.split);
  const int k0 = (int)((int64_t)slice * p.k_tiles / p.split), k1 = (int)((int64_t)(slice + 1) * p.k_tiles / p.split);
  const int64_t n0 = (int64_t)tile * C::BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 4);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch(&maps.w);
      tma_prefetch(&maps.r);
      tma_prefetch(&maps.c);
      if (BL != SW_DENSE) tma_prefetch(&maps.e);
    }
    // while the kernel before this one finishes: warm L2 with this slice of the
    // weight tile, one box (the stage's 128 rows x 128 bytes) per lane (the
    // weight is not written by the preparation kernels)
    for (int kt = k0 + lane; kt < k1; kt += 32) tma_prefetch_l2_2d(&maps.w, kt * 128, (int32_t)n0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  grid_dep_wait();  // the prepared rows are complete

  const int64_t sw_blocks = (p.k / C::kVec + 3) / 4;  // 512-byte chunks per 128-row block of the weight scales
  float f[TN];  // drain warps: this CTA's raw sums of its row (lane) for each activation row
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t smem0 = smem_u32(smem), full0 = smem_u32(full);
      const uint8_t* g_sa = p.sf_w + (n0 / 128) * sw_blocks * 512 + (int64_t)k0 * C::kChunksR * 512;
      const uint8_t* g_sr = p.sf_res + (int64_t)k0 * C::kChunksR * 512;
      const uint8_t* g_sb = p.sf_bb + (int64_t)k0 * C::kChunksB * 512;
      uint32_t issued = 0, issued_par = 0;
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = k0; kt < k1 && !*abort_flag; kt++) {
        if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
        const uint32_t sb = smem0 + (uint32_t)(stage * C::kStageBytes);
        const uint32_t fb = full0 + (uint32_t)(stage * 8);
        mbar_arrive_expect_tx_u32(fb, C::kTx);
        tma_load_2d_u32(sb + C::oW, &maps.w, kt * 128, (int32_t)n0, fb);
        tma_load_2d_u32(sb + C::oR, &maps.r, kt * 128, 0, fb);
        if constexpr (BL == SW_DENSE) {
          tma_load_2d_u32(sb + C::oD, &maps.c, kt * 128, 0, fb);
        } else {
          tma_load_2d_u32(sb + C::oC, &maps.c, kt * C::kCRow, 0, fb);
          tma_load_2d_u32(sb + C::oE, &maps.e, kt * C::kMetaRow, 0, fb);
        }
        bulk_load_u32(sb + C::oSA, g_sa, C::kChunksR * 512, fb);
        bulk_load_u32(sb + C::oSR, g_sr, C::kChunksR * 512, fb);
        bulk_load_u32(sb + C::oSB, g_sb, C::kChunksB * 512, fb);
        g_sa += C::kChunksR * 512;
        g_sr += C::kChunksR * 512;
        g_sb += C::kChunksB * 512;
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
      if (*abort_flag) {  // let every load already issued land before the block can exit
        for (int i = 0; i < C::kStages; i++)
          if ((issued >> i) & 1u) (void)mbar_wait(&full[i], (issued_par >> i) & 1u, 1000000000ull, nullptr, true);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t kHi128 = desc_hi(1024, 2);
      constexpr uint32_t kLbo = 1u << 16;
      const uint32_t lo0 = smem_u32(smem) >> 4, empty0 = smem_u32(empty);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t accumulate = 0;
      for (int kt = k0; kt < k1; kt++) {
        if (!mbar_wait(&full[stage], phase, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
        if (!mbar_wait(&ready[stage], phase, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t ls = lo0 + (uint32_t)(stage * (C::kStageBytes >> 4));
        const uint32_t slot = tmem_base + TN + (uint32_t)(stage * C::kSlotCols);
#pragma unroll
        for (int path = 0; path < 2; path++) {  // backbone (dense form), then residual
          const uint32_t ob = path == 0 ? C::oD : C::oR;
          const uint32_t cb = path == 0 ? C::cSD : C::cSR;
#pragma unroll
          for (int kb = 0; kb < C::BK / 64; kb++) {
            constexpr int kScales = 64 / C::kVec;
            const uint32_t chunk = (kb * kScales) / 4, byte = (kb * kScales) % 4;
            const uint32_t idesc = C::kIdesc | (byte << 29) | (byte << 4);
            const uint64_t a = desc_lohi((ls + (C::oW >> 4) + 2 * kb) | kLbo, kHi128);
            const uint64_t b = desc_lohi((ls + (ob >> 4) + 2 * kb) | kLbo, kHi128);
            const uint32_t sfa = (slot + C::cSA + 4 * chunk) | (byte << 30);
            const uint32_t sfb = (slot + cb + 4 * chunk) | (byte << 30);
            if constexpr (KIND == GK_NVF4) mma_nvf4(tmem_base, a, b, idesc, sfa, sfb, accumulate);
            else mma_mxf4(tmem_base, a, b, idesc, sfa, sfb, accumulate);
            accumulate = 1;
          }
        }
        tc_commit_u32(empty0 + (uint32_t)(stage * 8));
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
      tc_commit(acc_full);
      tc_commit(drain);
      (void)mbar_wait(drain, 0, 1000000000ull, nullptr, true);
    }
  } else {
    // ----------------------------------------- staging, then the drain (warps 2-5)
    const int q = warp & 3;  // a warp reaches the tensor-memory lanes of quadrant warp % 4
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16);
    int stage = 0;
    uint32_t phase = 0;
    for (int kt = k0; kt < k1; kt++) {
      if (!mbar_wait(&full[stage], phase, p.timeout_ns, abort_flag)) { *abort_flag = 1; break; }
      uint8_t* sb = smem + stage * C::kStageBytes;
      const uint32_t slot = tq + TN + (uint32_t)(stage * C::kSlotCols);
#pragma unroll
      for (int c = 0; c < C::kChunksR; c++) {
        tmem_st4(slot + C::cSA + 4 * c, *reinterpret_cast<const uint4*>(sb + C::oSA + 512 * c + 16 * lane));
        tmem_st4(slot + C::cSR + 4 * c, *reinterpret_cast<const uint4*>(sb + C::oSR + 512 * c + 16 * lane));
      }
#pragma unroll
      for (int c = 0; c < C::kChunksB; c++) {
        const uint4 v = *reinterpret_cast<const uint4*>(sb + C::oSB + 512 * c + 16 * lane);
        if constexpr (BL == SW_DENSE) {
          tmem_st4(slot + C::cSD + 4 * c, v);
        } else {  // the dense view: each stored backbone scale covers 2b logical K
          tmem_st4(slot + C::cSD + 4 * (2 * c), dup_lo_scales(v));
          tmem_st4(slot + C::cSD + 4 * (2 * c + 1), dup_hi_scales(v));
        }
      }
      if constexpr (BL != SW_DENSE) {
        // expand the compressed backbone rows into the swizzled dense tile:
        // piece j (0..7) of row r at r * 128 + ((j ^ (r % 8)) * 16)
        for (int i = q * 32 + lane; i < TN * 8; i += 128) {
          const int r = i >> 3, j = i & 7;
          const uint8_t* comp = sb + C::oC + r * C::kCRow + j * 8;
          const uint8_t* meta = sb + C::oE + r * C::kMetaRow + j * (BL == SW_PAIR ? 2 : 4);
          *reinterpret_cast<uint4*>(sb + C::oD + r * 128 + ((j ^ (r & 7)) << 4)) = expand_piece<BL>(comp, meta);
        }
        fence_proxy_async_smem();  // the dense tile is read by the tensor cores
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[stage]);
      if (++stage == C::kStages) { stage = 0; phase ^= 1; }
    }
    // drain: lane = weight row n0 + 32 q + lane, column = activation row
    if (!*abort_flag && !mbar_wait(acc_full, 0, p.timeout_ns, abort_flag)) *abort_flag = 1;
    if (!*abort_flag) {
      tc_fence_after();
      uint32_t v[TN];
      tmem_ld32_nowait(tq, *reinterpret_cast<uint32_t(*)[32]>(v));
      if constexpr (TN == 64) tmem_ld32_nowait(tq + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < TN; t++) f[t] = __uint_as_float(v[t]);
      if (p.split > 1 && slice != 0) {
        // this slice's raw sums for the cluster's first CTA: column-major
        // [TN][128] fp32 in the (now idle) stage buffers, consecutive lanes on
        // consecutive words
        float* part = reinterpret_cast<float*>(smem);
#pragma unroll
        for (int t = 0; t < TN; t++) part[t * C::BM + 32 * q + lane] = f[t];
      }
    }
  }

  // Split K: the K slices of a weight tile are the CTAs of one cluster.  After
  // the first cluster barrier every slice's raw sums are in its shared memory;
  // the first CTA adds them in slice order (a fixed order) through distributed
  // shared memory and stores y; the second barrier keeps the other CTAs (and
  // their shared memory) alive until it has read them.
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (p.split > 1) cluster_sync_all();
  if (warp >= 2 && (p.split <= 1 || slice == 0) && !*abort_flag) {
    const int q = warp & 3;
    const int64_t n = n0 + 32 * q + lane;
    if (p.split > 1) {
      const uint32_t part = smem_u32(smem) + (uint32_t)((32 * q + lane) * 4);
      for (int r = 1; r < p.split; r++) {
        const uint32_t peer = mapa_u32(part, (uint32_t)r);
#pragma unroll
        for (int t = 0; t < TN; t++) f[t] = __fadd_rn(f[t], ld_cluster_f32(peer + (uint32_t)(t * C::BM * 4)));
      }
    }
    const float alpha = __fmul_rn(__ldg(p.tensor_x + 2), __ldg(p.tensor_w + 2));
    if (n < p.n) {
#pragma unroll
      for (int t = 0; t < TN; t++) {  // lanes write consecutive n of row t
        if (t >= p.t) break;
        const float yv = __fmul_rn(f[t], alpha);
        if (p.y_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[t * p.n + n] = __float2bfloat16_rn(yv);
        else reinterpret_cast<float*>(p.y)[t * p.n + n] = yv;
      }
    }
  }
  __syncwarp();
  if (p.split > 1) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace sharq
