// tcgen05 GEMM for the MLA projections (bf16 in, fp32 TMEM accumulators).
//
// C = A B^T, A [M, K] and B [N, K] both K-major (nn.Linear [out, in] weights,
// MiniMind "Attention 前向传播" section 2), output columns split in up to two
// segments with their own B matrix (the fused q_a | kv_a down-projection of
// the CSDN DeepseekV3Attention forward shares the input x).
//
// Batched products (one per head, for the absorbed decode) index a third
// tensor-map dimension; a B stored [K, N] (the up_k slice of the kv
// up-projection) is loaded as four 64-column MN-major boxes per stage.
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0      TMA producer: 128x64 A box + 256x64 B box per stage,
//               128-byte swizzle, 4-stage ring of mbarriers
//   warp 1      TMEM allocator and MMA issuer: 4 x tcgen05.mma M128 N256 K16
//               per stage into one of two TMEM accumulators (2 x 256 columns)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = row), the
//               fused RMSNorm statistics / row scale / gain and RoPE of the
//               rope columns (see EpiSeg), bf16 stores.
// The two TMEM accumulators let the epilogue of tile i overlap the MMAs of
// tile i+1.  Every mbarrier wait is bounded (sm100::mbar_wait).
//
// Large non-batched products with K >= 1024 run on gemm_tc2_kernel instead:
// the same roles on 2-CTA clusters with 256 x 256 tiles and cta_group::2
// MMAs (see the comment above it), which halves each CTA's bytes per k-block
// and so fits six stages instead of four.
#include "sm100.cuh"
#include "tc.h"

namespace mla {
namespace {

using namespace sm100;

constexpr int BM = 128, BN = kTcTileN, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
// Output staging for TMA stores: per epilogue warp two 32-row x 64-column
// bf16 boxes (4 KB each), 128-byte swizzled.
constexpr int OUT_BOX = 32 * 64 * 2;
constexpr int NTHREADS = 192;
constexpr int BMN_BOX = 64 * BK * 2;       // one 64-column MN-major box of B
constexpr uint32_t TMEM_COLS = 2 * BN;

struct TcGemmParams {
  int M, K;
  int nseg;
  int tiles_m;
  int tiles_n[2];
  int per_batch;          // tiles of one batch entry
  int total_tiles;
  int a_batch_inner, b_mn;
  int64_t sOut;
  int tma_store;          // outputs written by TMA stores (non-batched bf16)
  int group_m;            // row blocks per raster group
  EpiSeg seg[2];
  uint32_t* status;
};

template <int TBN>
__device__ __forceinline__ void tile_coords(const TcGemmParams& p, int t, int& bi, int& s,
                                            int& m0, int& n0) {
  bi = t / p.per_batch;
  t -= bi * p.per_batch;
  const int first = p.tiles_m * p.tiles_n[0];
  s = (t >= first) ? 1 : 0;
  const int local = s ? t - first : t;
  // Groups of group_m row blocks: inside a group the row block changes
  // fastest, so a wave of CTAs shares fewer, fuller A and B panels in L2.
  const int tn = p.tiles_n[s], G = p.group_m;
  const int g = local / (G * tn);
  const int gm = min(G, p.tiles_m - g * G);               // rows of this group
  const int in = local - g * G * tn;
  m0 = (g * G + in % gm) * BM;
  n0 = (in / gm) * TBN;
}

// Epilogue of one 128 x TBN tile; this thread owns output row m0 + row.
// Columns go out in groups of 64 (a TMA store each); a last group narrower
// than 64 (TBN = 224) is stored directly so that no store reaches the next
// tile's columns.
template <int TBN = BN>
__device__ __forceinline__ void epilogue_tile(const TcGemmParams& p, const EpiSeg& e, int bi,
                                              int m0, int n0, int row, uint32_t taddr,
                                              const CUtensorMap* tmO, uint32_t stg, int& gidx) {
  const int m = m0 + row;
  const bool row_ok = m < p.M;
  float rs = 1.f;
  if (e.ssq_in && row_ok) {
    float ss = 0.f;
    for (int q = 0; q < e.ssq_parts; ++q) ss += e.ssq_in[q * e.ssq_ld + m];
    rs = rsqrtf(ss * e.rs_inv_dim + e.eps);
  }
  const int pos = row_ok ? (e.pos ? e.pos[m] : m % e.T + e.pos_offset) : 0;
  float ssq = 0.f;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(e.out) + (int64_t)bi * p.sOut;
  const __nv_bfloat16* gamma = reinterpret_cast<const __nv_bfloat16*>(e.gamma);
#pragma unroll 1
  for (int g = 0; g < (TBN + 63) / 64; ++g) {
    const int nl = n0 + g * 64;
    const int tw = min(64, TBN - g * 64);   // columns of this group inside the tile
    if (nl >= e.ncols) break;  // uniform over the warp
    uint32_t r0[32], r1[32];
    tmem_ld32(taddr + g * 64, r0);
    tmem_ld32(taddr + g * 64 + 32, r1);
    tmem_wait_ld();
    float v[64];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      v[i] = __uint_as_float(r0[i]);
      v[i + 32] = __uint_as_float(r1[i]);
    }
    if (e.ssq_out) {
      const int lim = e.norm_cols - nl;
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (i < lim) ssq = fmaf(v[i], v[i], ssq);
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] *= rs;
    if (e.cos && (nl % e.rope_period) == e.rope_start) {
      if (e.rope_interleave) {   // pairs (2i, 2i+1) -> rotate_half order (i, i + 32)
        float u[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) u[i] = v[i];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = u[2 * i];
          v[i + 32] = u[2 * i + 1];
        }
      }
      // rotate_half RoPE on a 64-wide rope segment: pairs (i, i + 32).
      const float4* cs = reinterpret_cast<const float4*>(e.cos + (int64_t)pos * 64);
      const float4* sn = reinterpret_cast<const float4*>(e.sin + (int64_t)pos * 64);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 c1 = __ldg(cs + j), s1 = __ldg(sn + j);
        const float4 c2 = __ldg(cs + j + 8), s2 = __ldg(sn + j + 8);
        const float cc1[4] = {c1.x, c1.y, c1.z, c1.w}, ss1[4] = {s1.x, s1.y, s1.z, s1.w};
        const float cc2[4] = {c2.x, c2.y, c2.z, c2.w}, ss2[4] = {s2.x, s2.y, s2.z, s2.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = 4 * j + k;
          const float x1 = v[i], x2 = v[i + 32];
          v[i] = x1 * cc1[k] - x2 * ss1[k];
          v[i + 32] = x2 * cc2[k] + x1 * ss2[k];
        }
      }
    }
    if (gamma && nl < e.norm_cols) {
      const int lim = e.norm_cols - nl;
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (i < lim) v[i] *= __bfloat162float(gamma[nl + i]);
    }
    if (p.tma_store && tw == 64) {
      // this warp's 32 rows x 64 columns through shared memory, one TMA store
      const int lane = row & 31;
      const uint32_t sb = stg + (gidx & 1) * OUT_BOX;
      if (gidx >= 2) {            // the store issued from this box two groups ago
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(sb + lane * 128 + ((c ^ (lane & 7)) << 4),
                     pack_bf16(v[8 * c], v[8 * c + 1]), pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                     pack_bf16(v[8 * c + 4], v[8 * c + 5]),
                     pack_bf16(v[8 * c + 6], v[8 * c + 7]));
      fence_proxy_async();
      __syncwarp();
      if (lane == 0 && m0 + (row & ~31) < p.M) {   // boxes wholly below M: nothing to write
        tma_store_2d(tmO, sb, nl, m0 + (row & ~31));
        bulk_commit_group();
      }
      ++gidx;
    } else if (row_ok) {
      __nv_bfloat16* dst = out + (int64_t)m * e.ldo + nl;
      const int lim = min(e.ncols - nl, tw);
#pragma unroll
      for (int c = 0; c < 64; c += 8) {
        if (c < lim)
          st_global_v4(dst + c, pack_bf16(v[c], v[c + 1]), pack_bf16(v[c + 2], v[c + 3]),
                       pack_bf16(v[c + 4], v[c + 5]), pack_bf16(v[c + 6], v[c + 7]));
      }
    }
  }
  if (e.ssq_out && row_ok && n0 < e.norm_cols) e.ssq_out[(n0 / TBN) * e.ssq_ld + m] = ssq;
}

// TBN: tile width (256 in general; 512 for one-wave batched products whose
// whole output row fits one tile, using all of TMEM for one accumulator; 128
// for batched products of at most 128 columns), TST: ring stages.
template <int TBN, int TST>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmO0,
                   const __grid_constant__ CUtensorMap tmO1,
                   const __grid_constant__ TcGemmParams p) {
  constexpr int kBBytes = TBN * BK * 2;
  constexpr int kStage = A_BYTES + kBBytes;
  constexpr int kOffOut = TST * kStage;
  constexpr int kNBuf = TBN == 512 ? 1 : 2;              // TMEM accumulators
  constexpr uint32_t kTmem = TBN == 512 ? 512u : 2u * TBN;
  constexpr int kNMma = TBN == 512 ? 2 : 1;              // MMAs of N = TBN / kNMma per K step
  constexpr uint32_t kIdesc = idesc_bf16(BM, TBN / kNMma);
  constexpr uint32_t kIdescMN = idesc_bf16(BM, TBN / kNMma, 0, 1);
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[TST], empty[TST], tfull[2], tempty[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB0);
    if (p.nseg > 1) tma_prefetch(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, kTmem);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  griddep_wait();               // the previous kernel's outputs (A, row scales) are ready
  griddep_launch_dependents();
  const uint32_t tbase = tmem_base;
  const int nk = (p.K + BK - 1) / BK;

  if (warp == 0) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
        int bi, s, m0, n0;
        tile_coords<TBN>(p, t, bi, s, m0, n0);
        const CUtensorMap* tmB = s ? &tmB1 : &tmB0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_v, p.status)) goto done;
          uint8_t* sa = smem + stage * kStage;
          mbar_arrive_expect_tx(&full[stage], kStage);
          if (p.a_batch_inner)
            tma_load_3d(sa, &tmA, kb * BK, bi, m0, &full[stage]);
          else
            tma_load_3d(sa, &tmA, kb * BK, m0, bi, &full[stage]);
          if (p.b_mn) {
            for (int q = 0; q < TBN / 64; ++q)
              tma_load_3d(sa + A_BYTES + q * BMN_BOX, tmB, n0 + 64 * q, kb * BK, bi, &full[stage]);
          } else {
            for (int q = 0; q < kNMma; ++q)    // boxes of at most 256 rows
              tma_load_3d(sa + A_BYTES + q * (kBBytes / kNMma), tmB, kb * BK,
                          n0 + q * (TBN / kNMma), bi, &full[stage]);
          }
          if (++stage == TST) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++local) {
        const int buf = local % kNBuf;
        const uint32_t tph = (local / kNBuf) & 1;
        if (!mbar_wait(&tempty[buf], tph ^ 1, abort_v, p.status)) goto done;
        tc_fence_after();
        const uint32_t d = tbase + buf * TBN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_v, p.status)) goto done;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStage);
          const uint32_t sb = sa + A_BYTES;
          if (p.b_mn) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
#pragma unroll
              for (int q = 0; q < kNMma; ++q)
                mma_bf16(d + q * (TBN / kNMma), desc_kmajor_sw128(sa + k * 32),
                         desc_mnmajor_sw128(sb + q * (kBBytes / kNMma) + k * 16 * 128, BMN_BOX),
                         kIdescMN, (kb | k) != 0);
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
#pragma unroll
              for (int q = 0; q < kNMma; ++q)
                mma_bf16(d + q * (TBN / kNMma), desc_kmajor_sw128(sa + k * 32),
                         desc_kmajor_sw128(sb + q * (kBBytes / kNMma) + k * 32), kIdesc,
                         (kb | k) != 0);
          }
          mma_commit(&empty[stage]);
          if (++stage == TST) {
            stage = 0;
            phase ^= 1;
          }
        }
        mma_commit(&tfull[buf]);
      }
    }
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t stg = smem_u32(smem + kOffOut + quad * 2 * OUT_BOX);
    int gidx = 0;
    int local = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++local) {
      const int buf = local % kNBuf;
      const uint32_t tph = (local / kNBuf) & 1;
      if (!warp_wait(&tfull[buf], tph, abort_v, p.status)) break;
      tc_fence_after();
      int bi, s, m0, n0;
      tile_coords<TBN>(p, t, bi, s, m0, n0);
      epilogue_tile<TBN>(p, p.seg[s], bi, m0, n0, row,
                         tbase + ((uint32_t)(quad * 32) << 16) + buf * TBN, s ? &tmO1 : &tmO0,
                         stg, gidx);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
    if (p.tma_store && lane == 0) bulk_wait_group<0>();   // stores done before exit
  }
done:
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmem);
  }
}

// ---------------------------------------------------------------------------
// Pair variant for large non-batched GEMMs: a 2-CTA cluster computes one
// 256 x 256 tile with cta_group::2 MMAs issued by the rank-0 CTA.  Each CTA
// loads its 128 rows of A and its 128 of the tile's 256 B rows (32 KB per
// k-block), so the same shared memory holds six stages instead of four and
// covers more load latency; each CTA's TMEM holds its 128 output rows x 256
// columns and its own epilogue warps write them.
//
// The tile is 256 x TBN2 with TBN2 = 256, or 224 where that leaves fewer
// idle CTA pairs in the last wave (o_proj at 4096 rows: 448 tiles of 256 on
// 74 pairs are 6.05 waves, 512 of 224 are 6.92); each CTA loads TBN2 / 2
// rows of B.
constexpr int BM2 = 256, STAGES2 = 6;
constexpr int HALF_BYTES = 128 * BK * 2;                  // 16 KB of A per CTA and stage
template <int TBN2>
constexpr int stage2_bytes() { return HALF_BYTES + TBN2 / 2 * BK * 2; }   // + B half
template <int TBN2>
constexpr int smem2_bytes() { return STAGES2 * stage2_bytes<TBN2>() + 4 * 2 * OUT_BOX + 1024; }
static_assert(smem2_bytes<256>() <= 227 * 1024, "shared memory");

template <int TBN2>
__device__ __forceinline__ void tile_coords2(const TcGemmParams& p, int t, int& s, int& m0,
                                             int& n0) {
  const int first = p.tiles_m * p.tiles_n[0];
  s = (t >= first) ? 1 : 0;
  const int local = s ? t - first : t;
  const int tn = p.tiles_n[s], G = p.group_m;
  const int g = local / (G * tn);
  const int gm = min(G, p.tiles_m - g * G);
  const int in = local - g * G * tn;
  m0 = (g * G + in % gm) * BM2;
  n0 = (in / gm) * TBN2;
}

template <int TBN2>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmO0,
                    const __grid_constant__ CUtensorMap tmO1,
                    const __grid_constant__ TcGemmParams p) {
  constexpr int kStage = stage2_bytes<TBN2>();
  constexpr int kOffOut = STAGES2 * kStage;
  constexpr uint32_t kIdesc = idesc_bf16(BM2, TBN2);
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[STAGES2], empty[STAGES2], tfull[2], tempty[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;
  const uint32_t rank = cluster_rank();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&full[s], 1);       // leader: its producer's arrive + both CTAs' bytes
      mbar_init(&empty[s], 1);      // the leader's MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);      // the leader's MMA commit
      mbar_init(&tempty[b], 8);     // leader: the epilogue warps of both CTAs
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB0);
    if (p.nseg > 1) tma_prefetch(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base, TMEM_COLS);
    tc_fence_before();
  }
  // both CTAs' barriers exist before either addresses the other's
  cluster_sync_all();
  tc_fence_after();
  griddep_wait();               // the previous kernel's outputs (A, row scales) are ready
  griddep_launch_dependents();
  const uint32_t tbase = tmem_base;
  const int nk = (p.K + BK - 1) / BK;
  const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);       // the leader's
  const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
  const uint32_t peer = rank ^ 1u;

  if (warp == 0) {
    // ---------------- producer (both CTAs): this CTA's halves of each stage
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      for (int t = cid; t < p.total_tiles; t += ncl) {
        int s, m0, n0;
        tile_coords2<TBN2>(p, t, s, m0, n0);
        const CUtensorMap* tmB = s ? &tmB1 : &tmB0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_v, p.status)) goto done;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kStage);
          uint8_t* sa = smem + stage * kStage;
          const uint32_t fb = full0 + stage * 8;
          tma_load_3d_pair(sa, &tmA, kb * BK, m0 + 128 * (int)rank, 0, fb);
          tma_load_3d_pair(sa + HALF_BYTES, tmB, kb * BK, n0 + TBN2 / 2 * (int)rank, 0, fb);
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (leader only) for both CTAs
    if (rank == 0 && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = cid; t < p.total_tiles; t += ncl, ++local) {
        const int buf = local & 1;
        const uint32_t tph = (local >> 1) & 1;
        if (!mbar_wait(&tempty[buf], tph ^ 1, abort_v, p.status)) goto done;
        tc_fence_after();
        const uint32_t d = tbase + buf * BN;     // accumulators 256 columns apart
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_v, p.status)) goto done;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStage);
          const uint32_t sb = sa + HALF_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_pair(d, desc_kmajor_sw128(sa + k * 32), desc_kmajor_sw128(sb + k * 32),
                          kIdesc, (kb | k) != 0);
          const uint32_t eb = smem_u32(&empty[stage]);
          mma_commit_pair(eb);
          mma_commit_pair(mapa_shared(eb, peer));
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1;
          }
        }
        const uint32_t tb = smem_u32(&tfull[buf]);
        mma_commit_pair(tb);
        mma_commit_pair(mapa_shared(tb, peer));
      }
    }
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows of each tile
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t stg = smem_u32(smem + kOffOut + quad * 2 * OUT_BOX);
    int gidx = 0;
    int local = 0;
    for (int t = cid; t < p.total_tiles; t += ncl, ++local) {
      const int buf = local & 1;
      const uint32_t tph = (local >> 1) & 1;
      if (!warp_wait(&tfull[buf], tph, abort_v, p.status)) break;
      tc_fence_after();
      int s, m0, n0;
      tile_coords2<TBN2>(p, t, s, m0, n0);
      epilogue_tile<TBN2>(p, p.seg[s], 0, m0 + 128 * (int)rank, n0, row,
                          tbase + ((uint32_t)(quad * 32) << 16) + buf * BN, s ? &tmO1 : &tmO0,
                          stg, gidx);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + buf * 8);
    }
    if (p.tma_store && lane == 0) bulk_wait_group<0>();   // stores done before exit
  }
done:
  __syncwarp();
  // no load, commit or arrive of either CTA addresses the other past here
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, TMEM_COLS);
  }
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool tc_gemm_supported(const GemmArgs& a, int dtype) {
  if (dtype != MLA_BF16 || a.M < 1 || a.K < 1 || a.batch < 1) return false;
  if (a.K % 8 || a.lda % 8 || a.sA % 8 || a.sB % 8 || !aligned16(a.A)) return false;
  if (a.batch > 1 && (a.nseg != 1 || a.seg[0].ssq_out || a.seg[0].ssq_in || a.seg[0].cos))
    return false;
  for (int s = 0; s < a.nseg; ++s) {
    const EpiSeg& e = a.seg[s];
    if (a.ldb[s] % 8 || !aligned16(a.Bm[s]) || !aligned16(e.out)) return false;
    if (e.ncols < 1 || e.ncols % 8 || e.ldo % 8) return false;
    if (a.b_mn && e.ncols % 64) return false;
    if (e.cos && (e.rope_dim != 64 || e.rope_start % 64 || e.rope_period % 64)) return false;
    if (e.ssq_in && e.ssq_parts < 1) return false;
  }
  return true;
}

namespace {
template <int TBN, int TST>
cudaError_t launch_single(int grid, const CUtensorMap& tmA, const CUtensorMap (&tmB)[2],
                          const CUtensorMap (&tmO)[2], const TcGemmParams& p, cudaStream_t st) {
  constexpr int smem = TST * (A_BYTES + TBN * BK * 2) + 4 * 2 * OUT_BOX + 1024;
  static_assert(smem <= 227 * 1024, "shared memory");
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t ea = set_dynamic_smem((const void*)gemm_tc_kernel<TBN, TST>, smem, smem_set);
  if (ea != cudaSuccess) return ea;
  const cudaError_t e = launch_pdl(gemm_tc_kernel<TBN, TST>, dim3(grid), dim3(NTHREADS), smem, st,
                                   tmA, tmB[0], tmB[1], tmO[0], tmO[1], p);
  count_launches();
  return e;
}

template <int TBN2>
cudaError_t launch_pair(int pairs, const CUtensorMap& tmA, const CUtensorMap (&tmB)[2],
                        const CUtensorMap (&tmO)[2], const TcGemmParams& p, cudaStream_t st) {
  constexpr int smem = smem2_bytes<TBN2>();
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t ea = set_dynamic_smem((const void*)gemm_tc2_kernel<TBN2>, smem, smem_set);
  if (ea != cudaSuccess) return ea;
  const cudaError_t e = launch_pdl(gemm_tc2_kernel<TBN2>, dim3(2 * pairs), dim3(NTHREADS), smem,
                                   st, tmA, tmB[0], tmB[1], tmO[0], tmO[1], p);
  count_launches();
  return e;
}
}  // namespace

cudaError_t tc_gemm(const GemmArgs& a, cudaStream_t st, uint32_t* status) {
  CUtensorMap tmA, tmB[2];
  const uint64_t nb = (uint64_t)a.batch;
  {
    // 3D map ordered so that strides grow: {K, rows, batch} or {K, batch, rows}
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    if (a.a_batch_inner) {
      dims[0] = a.K; dims[1] = nb; dims[2] = a.M;
      strides[0] = (uint64_t)a.sA * 2; strides[1] = (uint64_t)a.lda * 2;
      box[0] = BK; box[1] = 1; box[2] = BM;
    } else {
      dims[0] = a.K; dims[1] = a.M; dims[2] = nb;
      strides[0] = (uint64_t)a.lda * 2;
      strides[1] = a.batch > 1 ? (uint64_t)a.sA * 2 : (uint64_t)a.lda * 2 * a.M;
      box[0] = BK; box[1] = BM; box[2] = 1;
    }
    if (!encode_tmap(&tmA, a.A, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  // large non-batched K-major products run on CTA pairs (256-row tiles);
  // short K (the 512-deep kv up-projection: 8 k-blocks a tile) measured
  // faster on single CTAs
  const bool pair = a.batch == 1 && !a.b_mn && !a.a_batch_inner && a.M >= 512 && a.K >= 1024;
  const int bm = pair ? BM2 : BM;
  // Batched products whose rows fit one 128-row tile (the absorbed decode's
  // per-head products, M = the sequences): the whole output row of a batch
  // entry in one tile -- 512 columns in all of TMEM, or 128 -- so that one
  // wave of CTAs covers the batch and no B rows beyond the product are read.
  int tbn = BN;
  if (!pair && a.batch > 1 && a.M <= BM && a.nseg == 1) {
    const int n = a.seg[0].ncols;
    if (n <= 128) tbn = 128;
    else if (n > BN && n <= 512) tbn = 512;
  }
  // pair tile width: 224 instead of 256 where that cuts waves x width by at
  // least 5 % (fewer pairs idle in the last wave; o_proj at 4096 rows: 12 %
  // predicted, 0.663 -> 0.608 ms measured; at 16384 rows only 2 % predicted
  // and 224 measured 3 % slower), for outputs without RoPE or RMS partials
  // (both assume 256-column tiles)
  int tbn2 = BN;
  if (pair) {
    bool plain_epi = true;
    int64_t t256 = 0, t224 = 0;
    const int64_t tm = (a.M + BM2 - 1) / BM2, np = num_sms() / 2;
    for (int s = 0; s < a.nseg; ++s) {
      plain_epi = plain_epi && !a.seg[s].cos && !a.seg[s].ssq_out;
      t256 += tm * ((a.seg[s].ncols + 255) / 256);
      t224 += tm * ((a.seg[s].ncols + 223) / 224);
    }
    const int64_t w256 = (t256 + np - 1) / np, w224 = (t224 + np - 1) / np;
    if (plain_epi && w224 * 224 * 20 <= w256 * 256 * 19) tbn2 = 224;
    tbn = tbn2;
  }
  const int b_rows = pair ? tbn2 / 2 : (tbn < 256 ? tbn : 256);   // B rows per CTA and box
  TcGemmParams p{};
  p.M = a.M;
  p.K = a.K;
  p.nseg = a.nseg;
  p.tiles_m = (a.M + bm - 1) / bm;
  p.per_batch = 0;
  for (int s = 0; s < a.nseg; ++s) {
    const int64_t n = a.seg[s].ncols;
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    if (a.b_mn) {   // B stored [K, N]
      dims[0] = n; dims[1] = a.K; dims[2] = nb;
      strides[0] = (uint64_t)a.ldb[s] * 2;
      strides[1] = a.batch > 1 ? (uint64_t)a.sB * 2 : (uint64_t)a.ldb[s] * 2 * a.K;
      box[0] = 64; box[1] = BK; box[2] = 1;
    } else {        // B stored [N, K]
      dims[0] = a.K; dims[1] = n; dims[2] = nb;
      strides[0] = (uint64_t)a.ldb[s] * 2;
      strides[1] = a.batch > 1 ? (uint64_t)a.sB * 2 : (uint64_t)a.ldb[s] * 2 * n;
      box[0] = BK; box[1] = b_rows; box[2] = 1;
    }
    if (!encode_tmap(&tmB[s], a.Bm[s], 3, dims, strides, box)) return cudaErrorInvalidValue;
    p.seg[s] = a.seg[s];
    p.tiles_n[s] = (int)((n + tbn - 1) / tbn);
    p.per_batch += p.tiles_m * p.tiles_n[s];
  }
  if (a.nseg == 1) {
    tmB[1] = tmB[0];
    p.tiles_n[1] = 0;
  }
  // Outputs of a non-batched GEMM go out by TMA stores: boxes of 32 rows x
  // 64 columns, 128-byte swizzled, clipped at the tensor's edges.
  CUtensorMap tmO[2];
  p.tma_store = a.batch == 1;
  for (int s = 0; s < a.nseg && p.tma_store; ++s) {
    const EpiSeg& e = a.seg[s];
    if (!aligned16(e.out) || (e.ldo * 2) % 16 != 0) {
      p.tma_store = 0;
      break;
    }
    const uint64_t dims[2] = {(uint64_t)e.ncols, (uint64_t)a.M};
    const uint64_t strides[1] = {(uint64_t)e.ldo * 2};
    const uint32_t box[2] = {64, 32};
    if (!encode_tmap(&tmO[s], e.out, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  if (!p.tma_store || a.nseg == 1) tmO[1] = p.tma_store ? tmO[0] : tmA;
  if (!p.tma_store) tmO[0] = tmA;
  p.total_tiles = p.per_batch * a.batch;
  // long K: grouped raster (measured: o_proj, K = 16384, -0.8 %); short K keeps
  // the plain column-major order, which the 268 MB kv up-projection prefers
  p.group_m = a.K >= 4096 ? 2048 / bm : p.tiles_m;
  p.a_batch_inner = a.a_batch_inner;
  p.b_mn = a.b_mn;
  p.sOut = a.sOut;
  p.status = status;
  if (pair) {
    const int pairs = p.total_tiles < num_sms() / 2 ? p.total_tiles : num_sms() / 2;
    if (tbn2 == 224) return launch_pair<224>(pairs, tmA, tmB, tmO, p, st);
    return launch_pair<256>(pairs, tmA, tmB, tmO, p, st);
  }
  const int grid = p.total_tiles < num_sms() ? p.total_tiles : num_sms();
  if (tbn == 512) return launch_single<512, 2>(grid, tmA, tmB, tmO, p, st);
  if (tbn == 128) return launch_single<128, 6>(grid, tmA, tmB, tmO, p, st);
  return launch_single<BN, STAGES>(grid, tmA, tmB, tmO, p, st);
}

}  // namespace mla
