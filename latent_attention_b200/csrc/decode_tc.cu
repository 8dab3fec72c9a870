// Weight-absorbed MLA decode on sm_100a (bf16 in, fp32 softmax/accumulation).
//
// Megatron-LM MLA guide, 推理优化: each cached token keeps the compressed
// latent [kv_compressed | k_pos_emb]; decode folds up_k (rows [0, nope) of a
// head's block of the kv up-projection) into the query and applies up_v
// (rows [nope, nope+v)) after attention.  Three kernels:
//
//   D1 q_lat[b,h] = W_UK[h]^T q_nope[b,h]          batched tcgen05 GEMM (one
//                                                   product per head, W_UK read
//                                                   as an MN-major operand)
//   D2 latent_attn_kernel  split-KV attention of the 128 heads of a sequence
//                          over its [ctx, 576] cache, on tcgen05 (below)
//   D3 combine_kernel      log-sum-exp merge of the splits -> o_lat (bf16)
//   D4 o[b,h] = W_UV[h] o_lat[b,h]                  batched tcgen05 GEMM
//
// D2 design.  With 128 heads as the MMA M dimension the latent output
// O[128, 512] in fp32 fills all 512 TMEM columns, so a cluster of two CTAs
// shares one (sequence, split): CTA c accumulates latent columns
// [256c, 256c+256) of O (256 TMEM columns).  Each CTA computes the full
// scores S = Q C^T over all 576 cached dims itself -- the query's latent
// dims [0, 256) sit in TMEM (A operand from tensor memory, 128 columns), the
// rest (latent [256, 512) and rope) in shared memory -- so the two CTAs need
// no partial-score exchange and run the identical online softmax.  Each CTA
// TMA-loads every 64-token chunk in full (9 boxes of 64 dims): the pair reads
// the same rows at the same time, so the second read is served by L2 and
// every cache byte crosses HBM once.  The same chunk tile is the K-major B
// operand of S and, for the CTA's 256 latent dims, the MN-major B operand of
// O += P C.  P_j (bf16 pairs) is written over S_j's TMEM slot.
// A chunk's boxes form two groups with their own barriers: the 5 boxes only
// the scores read are released as soon as the first part of S_j has run and
// are refilled with chunk j+2 while softmax_j and PV_j are still to come; the
// 4 value boxes of this CTA's latent columns are released by PV_j and read
// last by S_{j+2}, so their load overlaps the first part of S_{j+2}.
// Warp roles (384 threads per CTA):
//   warp 0     TMA: query share once, score-only boxes of the chunk ring
//              (2 stages), L2 prefetch ahead
//   warp 1     TMEM allocation, MMA issue (S_j or PV, whichever is ready)
//   warp 2     TMA: the value boxes of the chunk ring
//   warps 4-7, 8-11  two softmax groups taking alternate chunks (thread =
//              head), P into TMEM; group 0 also loads the TMEM query part and
//              writes the epilogue
// All waits are bounded; a timeout sets the device status word.
#include <cfloat>

#include "sm100.cuh"
#include "tc.h"

namespace mla {
namespace {

using namespace sm100;

constexpr int R = 512, DR = 64, W = R + DR;      // latent, rope, cache row width
constexpr int NT = 64;                           // tokens per chunk
constexpr int QBOX = 128 * 64 * 2;               // 128 heads x 64 dims bf16
constexpr int CBOX = NT * 64 * 2;                // 64 tokens x 64 dims bf16
constexpr int QT_ATOMS = 4;                      // query dims [0, 256) in TMEM
constexpr int QS_ATOMS = 5;                      // query dims [256, 576) in shared memory
constexpr int C_ATOMS = 9;                       // a chunk's 576 dims
constexpr int NSTAGE = 2;                        // chunk ring
constexpr int NSLOT = 2;                         // score slots
constexpr int OFF_Q = 0;
constexpr int OFF_C = OFF_Q + QS_ATOMS * QBOX;           // 80 KB
constexpr int STAGE = C_ATOMS * CBOX;                    // 72 KB
constexpr int SMEM_BYTES = OFF_C + NSTAGE * STAGE + 1024;
constexpr int NTHREADS = 384;
constexpr int PREFETCH = 4;                              // chunks prefetched to L2
constexpr uint32_t IDESC_S = idesc_bf16(128, NT);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, 0, 1);
// TMEM: score slots [0, 128) (64 columns each; P_j over the first 32 of slot
// j % 2), O [128, 384), query dims [0, 256) as bf16 pairs [384, 512).
constexpr uint32_t TM_S = 0, TM_O = 128, TM_Q = 384;
constexpr float kRescaleLog2 = 8.f;
constexpr int SO_BOXES = 5, V_BOXES = 4;      // score-only / value boxes of a chunk

// Box i of the score-only group of the CTA with cluster rank `rank` (the
// latent half the CTA does not accumulate, then the rope box); the value
// group of rank c is boxes 4c .. 4c + 3.
__device__ __forceinline__ int score_only_box(uint32_t rank, int i) {
  return i < 4 ? (rank ? i : 4 + i) : 8;
}

struct DecTcParams {
  const int32_t* cu_ctx;
  const __nv_bfloat16* q_lat;  // [B, h, 512]
  int B, h, max_ctx;
  int split_tokens, max_splits;
  float scale_log2;
  float* part_o;      // [B, max_splits, h, R]
  float* part_lse;    // [B, max_splits, h]
  uint32_t* status;
};

__device__ __forceinline__ int seq_len(const int32_t* cu, int b, int max_ctx, uint32_t* status,
                                       int64_t* start) {
  const int64_t s = cu[b], e = cu[b + 1];
  int64_t n = e - s;
  if (n < 1 || n > max_ctx) {
    if (threadIdx.x == 0) atomicOr(status, kStatusBadCtx);
    n = n < 1 ? 0 : max_ctx;
  }
  *start = s;
  return (int)n;
}

// First token (relative to the sequence start) of the 64-row box that chunk j
// of a split starting at token t0 loads.  A box never reaches past the last
// token n - 1 of its sequence, so the load stays inside the caller's cache:
// the last chunk of a sequence is shifted back and its leading tokens, which
// the previous chunk already covered, are masked.  For n < 64 the box starts
// before the sequence (rows of earlier sequences, or negative rows that the
// tensor map fills with zeros); those columns are masked too.
__device__ __forceinline__ int chunk_base(int n, int t0, int j) {
  const int lt = t0 + j * NT;
  return n >= NT ? min(lt, n - NT) : n - NT;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    latent_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmQpe,
                       const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ DecTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, qt_full, ca_full[NSTAGE], ca_empty[NSTAGE],
      cb_full[NSTAGE], cb_empty[NSTAGE], s_full[NSLOT], p_full[NSLOT], pv_done[2], o_done, ref_ready[2], fin;
  __shared__ float m_hand[2][128];          // reference max after chunk j, slot j % 2
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;

  const uint32_t rank = cluster_rank();
  const int item = blockIdx.x >> 1;
  const int b = item / p.max_splits, sp = item % p.max_splits;
  const int h0 = blockIdx.z * 128;
  int64_t start;
  const int n = seq_len(p.cu_ctx, b, p.max_ctx, p.status, &start);
  const int t0 = sp * p.split_tokens;
  if (t0 >= n) {   // empty split (both CTAs of the pair take this branch)
    if (rank == 0 && threadIdx.x < 128 && h0 + threadIdx.x < p.h)
      p.part_lse[((int64_t)b * p.max_splits + sp) * p.h + h0 + threadIdx.x] = -INFINITY;
    return;
  }
  const int tcount = min(p.split_tokens, n - t0);
  const int nch = (tcount + NT - 1) / NT;
  const int dim0 = 256 * (int)rank;              // this CTA's latent columns of O

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&qt_full, 4);         // softmax group 0 stored the TMEM query part
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&ca_full[s], 1);
      mbar_init(&ca_empty[s], 1);
      mbar_init(&cb_full[s], 1);
      mbar_init(&cb_empty[s], 1);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);     // the chunk's softmax group wrote P_j
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&o_done, 1);
    mbar_init(&ref_ready[0], 4);    // a softmax group published chunk j's reference
    mbar_init(&ref_ready[1], 4);
    mbar_init(&fin, 4);             // softmax group 1 published its final sum
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 512);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  // softmax groups: warps 4..7 (group 0) and 8..11 (group 1)
  const int sm_wg = (warp >= 4 && warp < 8) ? 0 : (warp >= 8 ? 1 : -1);

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmQpe);
      tma_prefetch(&tmC);
      mbar_arrive_expect_tx(&q_full, QS_ATOMS * QBOX);
      for (int a = 0; a < 4; ++a)      // query latent dims [256, 512)
        tma_load_2d(smem + OFF_Q + a * QBOX, &tmQ, 256 + 64 * a, b * p.h + h0, &q_full);
      tma_load_2d(smem + OFF_Q + 4 * QBOX, &tmQpe, 0, b * p.h + h0, &q_full);
      for (int j = 0; j < PREFETCH && j < nch; ++j)
        for (int a = 0; a < C_ATOMS; ++a)
          tma_prefetch_l2_2d(&tmC, 64 * a, (int)start + chunk_base(n, t0, j));
      for (int j = 0; j < nch; ++j) {
        const int st = j % NSTAGE;
        if (j + PREFETCH < nch)
          for (int a = 0; a < C_ATOMS; ++a)
            tma_prefetch_l2_2d(&tmC, 64 * a, (int)start + chunk_base(n, t0, j + PREFETCH));
        if (!mbar_wait(&ca_empty[st], ((j / NSTAGE) & 1) ^ 1, abort_v, p.status)) break;
        uint8_t* sc = smem + OFF_C + st * STAGE;
        mbar_arrive_expect_tx(&ca_full[st], SO_BOXES * CBOX);
        const int y = (int)start + chunk_base(n, t0, j);
        for (int i = 0; i < SO_BOXES; ++i) {
          const int a = score_only_box(rank, i);
          tma_load_2d(sc + a * CBOX, &tmC, 64 * a, y, &ca_full[st]);
        }
      }
    }
  } else if (warp == 2) {
    if (elect_one()) {
      for (int j = 0; j < nch; ++j) {
        const int st = j % NSTAGE;
        if (!mbar_wait(&cb_empty[st], ((j / NSTAGE) & 1) ^ 1, abort_v, p.status)) break;
        uint8_t* sc = smem + OFF_C + st * STAGE;
        mbar_arrive_expect_tx(&cb_full[st], V_BOXES * CBOX);
        const int y = (int)start + chunk_base(n, t0, j);
        for (int i = 0; i < V_BOXES; ++i) {
          const int a = 4 * (int)rank + i;
          tma_load_2d(sc + a * CBOX, &tmC, 64 * a, y, &cb_full[st]);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint64_t dq = desc_kmajor_sw128(smem_u32(smem + OFF_Q));
      bool ok = mbar_wait(&q_full, 0, abort_v, p.status) &&
                mbar_wait(&qt_full, 0, abort_v, p.status);
      // S_j += Q box a . C_j box a^T (four MMAs of 16 dims): query dims
      // [0, 256) from TMEM, the rest from shared memory
      auto s_box = [&](uint32_t d, uint64_t dc, int a, bool first) {
        if (a < QT_ATOMS) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ts(d, tbase + TM_Q + a * 32 + k * 8,
                        dc + (uint64_t)((a * CBOX + k * 32) >> 4), IDESC_S, !(first && k == 0));
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16(d, dq + (uint64_t)(((a - QT_ATOMS) * QBOX + k * 32) >> 4),
                     dc + (uint64_t)((a * CBOX + k * 32) >> 4), IDESC_S, !(first && k == 0));
        }
      };
      // Issue S_js and O += P_jp C_jp in whichever order their inputs become
      // ready.  S_js reuses the slot of S/P_{js-2}, so it follows PV_{js-2} in
      // issue order (js < jp + 2), which is execution order; PV_jp follows S_jp.
      // S_js goes out in two parts: the score-only boxes, then the value boxes.
      int js = 0, jp = 0;
      bool s_part = false;                 // S_js's score-only part is issued
      const uint64_t t_start = globaltimer();
      uint32_t idle = 0;
      while (ok && jp < nch) {
        bool progress = false;
        if (js < nch && js < jp + NSLOT) {
          const int st = js % NSTAGE, sl = js % NSLOT;
          const uint32_t par = (js / NSTAGE) & 1;
          const uint32_t d = tbase + TM_S + sl * NT;
          const uint64_t dc = desc_kmajor_sw128(smem_u32(smem + OFF_C + st * STAGE));
          if (!s_part && mbar_test(&ca_full[st], par)) {
            tc_fence_after();
            for (int i = 0; i < SO_BOXES; ++i) s_box(d, dc, score_only_box(rank, i), i == 0);
            mma_commit(&ca_empty[st]);
            s_part = true;
            progress = true;
          }
          if (s_part && mbar_test(&cb_full[st], par)) {
            tc_fence_after();
            for (int i = 0; i < V_BOXES; ++i) s_box(d, dc, 4 * (int)rank + i, false);
            mma_commit(&s_full[sl]);
            s_part = false;
            ++js;
            progress = true;
          }
        }
        if (jp < js) {
          const int st = jp % NSTAGE, sl = jp % NSLOT;
          if (mbar_test(&p_full[sl], (jp / NSLOT) & 1)) {
            tc_fence_after();
            const uint64_t dv =
                desc_mnmajor_sw128(smem_u32(smem + OFF_C + st * STAGE + (dim0 / 64) * CBOX), CBOX);
#pragma unroll
            for (int k = 0; k < NT / 16; ++k)
              mma_bf16_ts(tbase + TM_O, tbase + TM_S + sl * NT + k * 8,
                          dv + (uint64_t)((k * 16 * 128) >> 4), IDESC_PV, (jp | k) != 0);
            mma_commit(&cb_empty[st]);
            mma_commit(&pv_done[jp & 1]);
            if (jp == nch - 1) mma_commit(&o_done);
            ++jp;
            progress = true;
          }
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 63u) == 0) {   // bounded like every other wait
          if (*abort_v) {
            ok = false;
          } else if (globaltimer() - t_start > kWaitNs) {
            *abort_v = 1;
            atomicOr(p.status, kStatusTimeout);
            ok = false;
          }
        }
      }
    }
  } else if (sm_wg >= 0) {
    // ---------------- softmax (thread = head): group g takes chunks g, g + 2,
    // ... (always score slot g).  The reference max of every row passes from
    // one group to the other through shared memory; each group keeps the row
    // sum of its own chunks, relative to its last reference.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int head = h0 + r;
    const bool head_ok = head < p.h;
    if (sm_wg == 0) {   // query latent dims [0, 256) of this head into TMEM (A operand)
      const uint4* src = reinterpret_cast<const uint4*>(p.q_lat + ((int64_t)b * p.h + head) * R);
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {
        uint32_t q[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = head_ok ? src[part * 8 + c] : make_uint4(0u, 0u, 0u, 0u);
          q[4 * c] = v.x;
          q[4 * c + 1] = v.y;
          q[4 * c + 2] = v.z;
          q[4 * c + 3] = v.w;
        }
        tmem_st32(tbase + lane_off + TM_Q + part * 32, q);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&qt_full);
    }
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = sm_wg; j < nch; j += 2) {
      const int sl = j % NSLOT, xs = j & 1;
      if (!warp_wait(&s_full[sl], (j / NSLOT) & 1, abort_v, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tbase + lane_off + TM_S + sl * NT, sr[0]);
      tmem_ld32(tbase + lane_off + TM_S + sl * NT + 32, sr[1]);
      tmem_wait_ld();
      float s[NT];
#pragma unroll
      for (int i = 0; i < NT; ++i) s[i] = __uint_as_float(sr[i >> 5][i & 31]);
      // column i holds token base + i; chunk j owns tokens [t0 + 64j, t0 + tcount)
      const int lo = j * NT - (chunk_base(n, t0, j) - t0);
      const int hi = tcount - (chunk_base(n, t0, j) - t0);
      // Raw scores; the (positive) scale is folded into the exp argument.
      if (lo > 0 || hi < NT) {       // first / last chunk of the split only
#pragma unroll
        for (int i = 0; i < NT; ++i)
          if (i < lo || i >= hi) s[i] = -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < NT; i += 2) mx4[(i >> 1) & 3] = max3f(mx4[(i >> 1) & 3], s[i], s[i + 1]);
      const float cmax = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * p.scale_log2;
      // reference of chunk j-1, left by the other group
      float m_prev = -INFINITY;
      if (j > 0) {
        if (!warp_wait(&ref_ready[xs ^ 1], ((j - 1) >> 1) & 1, abort_v, p.status)) {
          ok = false;
          break;
        }
        m_prev = m_hand[xs ^ 1][r];
      }
      // lazy rescaling: a new reference only when the max grew by > 2^8
      const bool grow = cmax > m_prev + kRescaleLog2;     // always at j = 0
      const float m_new = grow ? cmax : m_prev;
      m_hand[xs][r] = m_new;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ref_ready[xs]);
      if (m_new != m_ref) {          // this group's sum, moved to the new reference
        l *= ex2(m_ref - m_new);
        m_ref = m_new;
      }
      const float neg_m = -m_ref;
      float ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ls[k] = 0.f;
      uint32_t w[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float a0, a1;
        fma2(a0, a1, s[2 * e], s[2 * e + 1], p.scale_log2, p.scale_log2, neg_m, neg_m);
        const float p0 = ex2(a0);
        const float p1 = ex2(a1);
        add2(ls[2 * (e & 3)], ls[2 * (e & 3) + 1], p0, p1);
        w[e] = pack_bf16(p0, p1);
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      // O holds the sum through chunk j-1 at reference m_prev: rescale it
      // when this chunk moved the reference (PV_{j-1} must be complete).
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        const float alpha = ex2(m_prev - m_new);
        if (!warp_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_v, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_off + TM_O + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tbase + lane_off + TM_O + c * 32, o);
        }
      }
      // P_j over the first half of S_j's slot (S_j is in registers already)
      tmem_st32(tbase + lane_off + TM_S + sl * NT, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sl]);
    }
    // Row sum of the split: both groups' sums at the last chunk's reference
    // (references never decrease, so that is the larger of the two).  Group 1
    // hands over through m_hand[1] only once group 0 no longer reads it: the
    // final barrier below orders the two.
    if (sm_wg == 1) {
      named_barrier_sync(1, 256);              // group 0 has left its loop
      m_hand[1][r] = m_ref;
      m_hand[0][r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&fin);
    } else {
      named_barrier_sync(1, 256);
      if (ok && warp_wait(&fin, 0, abort_v, p.status) &&
          warp_wait(&o_done, 0, abort_v, p.status)) {
        const float m1 = m_hand[1][r], l1 = m_hand[0][r];
        const float m_last = fmaxf(m_ref, m1);
        const float l_tot = l * ex2(m_ref - m_last) + (l1 > 0.f ? l1 * ex2(m1 - m_last) : 0.f);
        tc_fence_after();
        const int64_t part = ((int64_t)b * p.max_splits + sp) * p.h + head;
        const float inv = 1.f / l_tot;
        float* dst = p.part_o + part * R + dim0;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_off + TM_O + c * 32, o);
          tmem_wait_ld();
          if (head_ok) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              st_global_v4(dst + c * 32 + i, __float_as_uint(__uint_as_float(o[i]) * inv),
                           __float_as_uint(__uint_as_float(o[i + 1]) * inv),
                           __float_as_uint(__uint_as_float(o[i + 2]) * inv),
                           __float_as_uint(__uint_as_float(o[i + 3]) * inv));
          }
        }
        if (rank == 0 && head_ok)
          p.part_lse[part] = (m_last + __log2f(l_tot)) * 0.6931471805599453f;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// D3: o_lat[b,h] = sum_s w_s part_o[b,s,h] with w_s = exp(lse_s - max) / sum,
// one block per (sequence, head), 4 latent columns per thread.
__global__ void __launch_bounds__(128)
    combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                   __nv_bfloat16* __restrict__ o_lat, int h, int max_splits) {
  const int b = blockIdx.x / h, hh = blockIdx.x % h;
  const int c = threadIdx.x * 4;
  const float* lse = part_lse + (int64_t)b * max_splits * h + hh;
  float mx = -INFINITY;
  for (int s = 0; s < max_splits; ++s) mx = fmaxf(mx, lse[(int64_t)s * h]);
  float den = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
  for (int s = 0; s < max_splits; ++s) {
    const float l = lse[(int64_t)s * h];
    if (l == -INFINITY) continue;
    const float w = __expf(l - mx);
    const float4 v = *reinterpret_cast<const float4*>(
        part_o + (((int64_t)b * max_splits + s) * h + hh) * R + c);
    den += w;
    a0 = fmaf(w, v.x, a0);
    a1 = fmaf(w, v.y, a1);
    a2 = fmaf(w, v.z, a2);
    a3 = fmaf(w, v.w, a3);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* dst = o_lat + ((int64_t)b * h + hh) * R + c;
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(a0 * inv, a1 * inv),
                                              pack_bf16(a2 * inv, a3 * inv));
}

}  // namespace

bool tc_decode_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.kv_lora_rank == R && c.qk_rope_head_dim == DR &&
         c.qk_nope_head_dim % 8 == 0 && c.v_head_dim % 8 == 0;
}

int tc_decode_split_tokens() { return 4096; }

cudaError_t tc_decode(const DecodeArgs& a, cudaStream_t st) {
  cudaError_t e;
  // D1: q_lat[b, h, :] = q_nope[b, h, :] W_UK[h]  (per head: [B, dn] x [dn, R])
  {
    GemmArgs g;
    g.A = a.q_nope; g.lda = (int64_t)a.h * a.dn; g.sA = a.dn; g.a_batch_inner = true;
    g.Bm[0] = a.w_kv_b; g.ldb[0] = R; g.sB = (int64_t)(a.dn + a.dv) * R; g.b_mn = true;
    g.M = a.B; g.K = a.dn; g.batch = a.h; g.nseg = 1;
    g.seg[0].out = a.q_lat; g.seg[0].ldo = (int64_t)a.h * R; g.seg[0].ncols = R;
    g.sOut = R;
    if (!tc_gemm_supported(g, MLA_BF16)) return cudaErrorNotSupported;
    e = tc_gemm(g, st, a.status);
    if (e != cudaSuccess) return e;
  }
  stage_event(1, st);
  // D2
  {
    CUtensorMap tmQ, tmQpe, tmC;
    const uint32_t qbox[2] = {64, 128}, cbox[2] = {64, NT};
    const uint64_t qdims[2] = {(uint64_t)R, (uint64_t)a.B * a.h};
    const uint64_t qstr[1] = {(uint64_t)R * 2};
    if (!encode_tmap(&tmQ, a.q_lat, 2, qdims, qstr, qbox)) return cudaErrorInvalidValue;
    const uint64_t pdims[2] = {(uint64_t)DR, (uint64_t)a.B * a.h};
    const uint64_t pstr[1] = {(uint64_t)DR * 2};
    if (!encode_tmap(&tmQpe, a.q_pe, 2, pdims, pstr, qbox)) return cudaErrorInvalidValue;
    // The cache holds sum(ctx) <= B * max_ctx rows; cu_ctx lives on the
    // device, so the map is declared with the bound and every box is clamped
    // inside its own sequence (chunk_base).
    const uint64_t cdims[2] = {(uint64_t)W, (uint64_t)a.B * (uint64_t)a.max_ctx};
    const uint64_t cstr[1] = {(uint64_t)W * 2};
    if (!encode_tmap(&tmC, a.cache, 2, cdims, cstr, cbox)) return cudaErrorInvalidValue;
    DecTcParams p{};
    p.cu_ctx = a.cu_ctx;
    p.q_lat = reinterpret_cast<const __nv_bfloat16*>(a.q_lat);
    p.B = a.B;
    p.h = a.h;
    p.max_ctx = a.max_ctx;
    p.split_tokens = a.split_tokens;
    p.max_splits = a.max_splits;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.part_o = a.part_o;
    p.part_lse = a.part_lse;
    p.status = a.status;
    static std::atomic<uint64_t> smem_set{0};
    {
      const cudaError_t ea = set_dynamic_smem((const void*)latent_attn_kernel, SMEM_BYTES, smem_set);
      if (ea != cudaSuccess) return ea;
    }
    dim3 grid(2 * a.B * a.max_splits, 1, (a.h + 127) / 128);
    latent_attn_kernel<<<grid, NTHREADS, SMEM_BYTES, st>>>(tmQ, tmQpe, tmC, p);
    count_launches();
  }
  stage_event(2, st);
  // D3
  combine_kernel<<<a.B * a.h, R / 4, 0, st>>>(a.part_o, a.part_lse, (__nv_bfloat16*)a.o_lat,
                                              a.h, a.max_splits);
  count_launches();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  stage_event(3, st);
  // D4: o[b, h, :] = o_lat[b, h, :] W_UV[h]^T  (per head: [B, R] x [R, dv])
  {
    GemmArgs g;
    g.A = a.o_lat; g.lda = (int64_t)a.h * R; g.sA = R; g.a_batch_inner = true;
    g.Bm[0] = reinterpret_cast<const __nv_bfloat16*>(a.w_kv_b) + (int64_t)a.dn * R;
    g.ldb[0] = R; g.sB = (int64_t)(a.dn + a.dv) * R;
    g.M = a.B; g.K = R; g.batch = a.h; g.nseg = 1;
    g.seg[0].out = a.o; g.seg[0].ldo = (int64_t)a.h * a.dv; g.seg[0].ncols = a.dv;
    g.sOut = a.dv;
    if (!tc_gemm_supported(g, MLA_BF16)) return cudaErrorNotSupported;
    e = tc_gemm(g, st, a.status);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace mla
