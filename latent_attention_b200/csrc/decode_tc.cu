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
// O[128, 512] in fp32 fills all 512 TMEM columns, leaving none for the
// scores.  A cluster of two CTAs therefore shares one (sequence, split):
// CTA c holds latent columns [256c, 256c+256) of O (256 TMEM columns) and
// contracts the scores over its share of the 576 cached dims -- CTA 0 over
// dims [0, 256), CTA 1 over [256, 576) (latent half + the 64 rope dims, whose
// query part sits in TMEM).  Each CTA TMA-loads only its own dims of every
// 64-token chunk, so every cache byte crosses HBM once; the same shared-memory
// tile is the K-major B operand of S = Q C^T and the MN-major B operand of
// O += P C.  The partial score tiles are exchanged through distributed shared
// memory as fp16; each CTA adds the peer's partial to its own fp32 one and runs
// the online softmax for all 128 heads.  The MMA warp issues the scores two
// chunks ahead of the PV product (three chunk stages, three score slots), so
// the exchange and softmax of chunk j overlap the tensor work of j+1 and j+2.
// P_j (bf16 pairs) is written over the first half of S_j's TMEM slot.
// Warp roles (448 threads per CTA):
//   warp 0     TMA: Q share once, chunk ring (3 stages), L2 prefetch ahead
//   warp 1     TMEM allocation, MMA issue (S_j, then O += P_{j-2} C_{j-2})
//   warps 2, 3, 8, 9  score exchange (fp16 partial to the peer)
//   warps 4-7, 10-13  two softmax groups taking alternate chunks (thread =
//              head), P into TMEM; group 0 also writes the epilogue
// All waits are bounded; a timeout sets the device status word.
#include <cfloat>
#include <cuda_fp16.h>

#include "sm100.cuh"
#include "tc.h"

namespace mla {
namespace {

using namespace sm100;

constexpr int R = 512, DR = 64, W = R + DR;      // latent, rope, cache row width
constexpr int NT = 64;                           // tokens per chunk
constexpr int QBOX = 128 * 64 * 2;               // 128 heads x 64 dims bf16
constexpr int CBOX = NT * 64 * 2;                // 64 tokens x 64 dims bf16
constexpr int QATOMS = 4;                        // latent dims of Q in shared memory
constexpr int MAX_ATOMS = 5;                     // cache atoms per chunk (CTA 1: + rope)
constexpr int NSTAGE = 3;                        // chunk ring / score slots
constexpr int OFF_Q = 0;
constexpr int OFF_C = OFF_Q + QATOMS * QBOX;             // 64 KB
constexpr int STAGE = MAX_ATOMS * CBOX;                  // 40 KB
constexpr int XBUF = 128 * NT * 2;                       // exchange: 128 x 64 fp16
constexpr int OFF_X = OFF_C + NSTAGE * STAGE;            // peer partials received (x2)
constexpr int SMEM_BYTES = OFF_X + 2 * XBUF + 1024;
constexpr int NTHREADS = 448;
constexpr int PREFETCH = 4;                              // chunks prefetched to L2
constexpr uint32_t IDESC_S = idesc_bf16(128, NT);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, 0, 1);
// TMEM: score slots [0, 192) (64 columns each; P_j over the first 32 of slot
// j % 3), rope part of Q on CTA 1 [192, 224), O [256, 512).
constexpr uint32_t TM_S = 0, TM_QPE = 192, TM_O = 256;
constexpr float kRescaleLog2 = 8.f;

struct DecTcParams {
  const int32_t* cu_ctx;
  const __nv_bfloat16* q_pe;   // [B, h, 64]
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

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  return __half22float2(*reinterpret_cast<__half2*>(&v));
}

// S_j = Q_share C_j^T over the ATOMS 64-dim atoms held in shared memory.
// Descriptors advance by their 16-byte address field only (shared-memory
// addresses stay below 2^18, so the field never carries).
template <int ATOMS>
__device__ __forceinline__ void issue_scores(uint32_t d_tmem, uint64_t dq, uint64_t dc) {
#pragma unroll
  for (int a = 0; a < ATOMS; ++a)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      mma_bf16(d_tmem, dq + (uint64_t)((a * QBOX + k * 32) >> 4),
               dc + (uint64_t)((a * CBOX + k * 32) >> 4), IDESC_S, (a | k) != 0);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    latent_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ DecTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, qpe_full, c_full[NSTAGE], c_empty[NSTAGE],
      s_full[NSTAGE], s_free[NSTAGE], p_full[NSTAGE], pv_done[2], o_done, x_full[2], x_empty[2],
      ref_ready[2], fin;
  __shared__ float m_hand[2][128];          // reference max after chunk j, slot j % 2
  __shared__ float m_fin[128], l_fin[128];  // softmax group 1's final reference and sum
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;

  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
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
  const bool rope = rank == 1;
  const int atoms = rope ? 5 : 4;
  const int dim0 = 256 * (int)rank;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&qpe_full, 4);        // softmax warps stored the rope query (CTA 1)
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);     // exchange warps have read S_j from TMEM
      mbar_init(&p_full[s], 4);     // softmax warps have written P_j
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&o_done, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&x_full[s], 1);    // one local arrive.expect_tx + the peer's st.async bytes
      mbar_init(&x_empty[s], 4);   // one arrive per softmax warp of the peer
      mbar_init(&ref_ready[s], 4); // a softmax group published chunk j's reference
    }
    mbar_init(&fin, 4);            // softmax group 1 published its final sum
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 512);
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync();          // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  // exchange warps 2, 3, 8, 9 and softmax warps 4..7 each cover TMEM lane
  // quarter (warp & 3), i.e. heads 32 * (warp & 3) .. + 31.
  const bool xwg = warp == 2 || warp == 3 || warp == 8 || warp == 9;
  // softmax groups: warps 4..7 (group 0) and 10..13 (group 1)
  const int sm_wg = (warp >= 4 && warp < 8) ? 0 : (warp >= 10 ? 1 : -1);

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmC);
      mbar_arrive_expect_tx(&q_full, QATOMS * QBOX);
      for (int a = 0; a < QATOMS; ++a)
        tma_load_2d(smem + OFF_Q + a * QBOX, &tmQ, dim0 + 64 * a, b * p.h + h0, &q_full);
      for (int j = 0; j < PREFETCH && j < nch; ++j)
        for (int a = 0; a < atoms; ++a)
          tma_prefetch_l2_2d(&tmC, dim0 + 64 * a, (int)start + chunk_base(n, t0, j));
      for (int j = 0; j < nch; ++j) {
        const int st = j % NSTAGE;
        if (j + PREFETCH < nch)
          for (int a = 0; a < atoms; ++a)
            tma_prefetch_l2_2d(&tmC, dim0 + 64 * a, (int)start + chunk_base(n, t0, j + PREFETCH));
        if (!mbar_wait(&c_empty[st], ((j / NSTAGE) & 1) ^ 1, abort_v, p.status)) break;
        uint8_t* sc = smem + OFF_C + st * STAGE;
        mbar_arrive_expect_tx(&c_full[st], atoms * CBOX);
        const int y = (int)start + chunk_base(n, t0, j);
        for (int a = 0; a < atoms; ++a)
          tma_load_2d(sc + a * CBOX, &tmC, dim0 + 64 * a, y, &c_full[st]);
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint64_t dq = desc_kmajor_sw128(smem_u32(smem + OFF_Q));
      bool ok = mbar_wait(&q_full, 0, abort_v, p.status);
      if (ok && rope) ok = mbar_wait(&qpe_full, 0, abort_v, p.status);
      // Issue S_js and O += P_jp C_jp in whichever order their inputs become
      // ready.  S_js reuses the slot of S_{js-3}/P_{js-3}, so it waits for
      // PV_{js-3} to be issued (js < jp + 3); PV_jp follows S_jp.
      int js = 0, jp = 0;
      const uint64_t t_start = globaltimer();
      uint32_t idle = 0;
      while (ok && jp < nch) {
        bool progress = false;
        if (js < nch && js < jp + NSTAGE) {
          const int st = js % NSTAGE;
          if (mbar_test(&c_full[st], (js / NSTAGE) & 1) &&
              (js < NSTAGE || mbar_test(&s_free[st], ((js - NSTAGE) / NSTAGE) & 1))) {
            tc_fence_after();
            const uint64_t dc = desc_kmajor_sw128(smem_u32(smem + OFF_C + st * STAGE));
            issue_scores<QATOMS>(tbase + TM_S + st * NT, dq, dc);
            if (rope) {
#pragma unroll
              for (int k = 0; k < 4; ++k)   // A = rope query from TMEM, 8 columns per K step
                mma_bf16_ts(tbase + TM_S + st * NT, tbase + TM_QPE + k * 8,
                            dc + (uint64_t)((QATOMS * CBOX + k * 32) >> 4), IDESC_S, 1);
            }
            mma_commit(&s_full[st]);
            ++js;
            progress = true;
          }
        }
        if (jp < js) {
          const int st = jp % NSTAGE;
          if (mbar_test(&p_full[st], (jp / NSTAGE) & 1)) {
            tc_fence_after();
            const uint64_t dv = desc_mnmajor_sw128(smem_u32(smem + OFF_C + st * STAGE), CBOX);
#pragma unroll
            for (int k = 0; k < NT / 16; ++k)
              mma_bf16_ts(tbase + TM_O, tbase + TM_S + st * NT + k * 8,
                          dv + (uint64_t)((k * 16 * 128) >> 4), IDESC_PV, (jp | k) != 0);
            mma_commit(&c_empty[st]);
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
  } else if (xwg) {
    // ---------------- score exchange: this CTA's partial S_j as fp16 pairs
    // into the peer's receive buffer j % 2 (rows of this warp's lane quarter).
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    for (int j = 0; j < nch; ++j) {
      const int st = j % NSTAGE, xs = j & 1;
      const uint32_t px = map_peer(smem_u32(smem + OFF_X + xs * XBUF), peer);
      const uint32_t px_full = map_peer(smem_u32(&x_full[xs]), peer);
      if (!warp_wait(&s_full[st], (j / NSTAGE) & 1, abort_v, p.status)) break;
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tbase + lane_off + TM_S + st * NT, sr[0]);
      tmem_ld32(tbase + lane_off + TM_S + st * NT + 32, sr[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[st]);
      uint32_t h[32];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        h[i] = pack_half2(__uint_as_float(sr[i >> 4][(2 * i) & 31]),
                          __uint_as_float(sr[i >> 4][(2 * i + 1) & 31]));
      // the peer's receive buffer j % 2 is free once its softmax consumed j - 2
      if (!warp_wait_cluster(&x_empty[xs], ((j >> 1) & 1) ^ 1, abort_v, p.status)) break;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_async_v4(px + r * 128 + ((c ^ (r & 7)) << 4), h[4 * c], h[4 * c + 1], h[4 * c + 2],
                    h[4 * c + 3], px_full);
    }
  } else if (sm_wg >= 0) {
    // ---------------- softmax (thread = head): warpgroup g takes chunks
    // g, g + 2, ...  The reference max of every row passes from one group to
    // the other through shared memory (chunk j needs chunk j-1's); each group
    // keeps the row sum of its own chunks, relative to its last reference.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int head = h0 + r;
    const bool head_ok = head < p.h;
    if (rope && sm_wg == 0) {   // rope part of this head's query into TMEM (A operand layout)
      uint32_t q[32];
      const uint4* src = reinterpret_cast<const uint4*>(p.q_pe + ((int64_t)b * p.h + head) * DR);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = head_ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        q[4 * c] = v.x;
        q[4 * c + 1] = v.y;
        q[4 * c + 2] = v.z;
        q[4 * c + 3] = v.w;
      }
      tmem_st32(tbase + lane_off + TM_QPE, q);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&qpe_full);
    }
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = sm_wg; j < nch; j += 2) {
      const int st = j % NSTAGE, xs = j & 1;
      if (!warp_wait(&s_full[st], (j / NSTAGE) & 1, abort_v, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tbase + lane_off + TM_S + st * NT, sr[0]);
      tmem_ld32(tbase + lane_off + TM_S + st * NT + 32, sr[1]);
      if (r == 0) mbar_arrive_expect_tx(&x_full[xs], XBUF);
      if (!warp_wait_cluster(&x_full[xs], (j >> 1) & 1, abort_v, p.status)) { ok = false; break; }
      tmem_wait_ld();
      // S_j = own fp32 partial + the peer's fp16 partial
      const uint32_t sx = smem_u32(smem + OFF_X + xs * XBUF);
      float s[NT];
      uint32_t dep = 0;               // depends on every word loaded below
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t t[4];
        ld_shared_v4u(sx + r * 128 + ((c ^ (r & 7)) << 4), t[0], t[1], t[2], t[3]);
        dep ^= (t[0] ^ t[1]) ^ (t[2] ^ t[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 8 * c + 2 * e;
          const float2 theirs = unpack_half2(t[e]);
          float s0 = __uint_as_float(sr[i >> 5][i & 31]);
          float s1 = __uint_as_float(sr[(i + 1) >> 5][(i + 1) & 31]);
          add2(s0, s1, theirs.x, theirs.y);
          s[i] = s0;
          s[i + 1] = s1;
        }
      }
      // The receive buffer of chunk j may be refilled by the peer: the loads
      // from it have completed, since `dep` (an input below) needs them all.
      asm volatile("" ::"r"(dep));
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(map_peer(smem_u32(&x_empty[xs]), peer));
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
      // P_j goes over S_j: this CTA's exchange warps must have read S_j.
      if (!warp_wait(&s_free[st], (j / NSTAGE) & 1, abort_v, p.status)) { ok = false; break; }
      tc_fence_after();
      tmem_st32(tbase + lane_off + TM_S + st * NT, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
    }
    // Row sum of the split: both groups' sums at the last chunk's reference
    // (references never decrease, so that is the larger of the two).
    if (sm_wg == 1) {
      m_fin[r] = m_ref;
      l_fin[r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&fin);
    } else if (ok && warp_wait(&fin, 0, abort_v, p.status) &&
               warp_wait(&o_done, 0, abort_v, p.status)) {
      const float m1 = m_fin[r], l1 = l_fin[r];
      const float m_last = fmaxf(m_ref, m1);
      const float l_tot = l * ex2(m_ref - m_last) + (l1 > 0.f ? l1 * ex2(m1 - m_last) : 0.f);
      m_ref = m_last;
      l = l_tot;
      tc_fence_after();
      const int64_t part = ((int64_t)b * p.max_splits + sp) * p.h + head;
      const float inv = 1.f / l;
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
      if (rank == 0 && head_ok) p.part_lse[part] = (m_ref + __log2f(l)) * 0.6931471805599453f;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // the peer no longer touches this CTA's shared memory
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
    CUtensorMap tmQ, tmC;
    const uint32_t qbox[2] = {64, 128}, cbox[2] = {64, NT};
    const uint64_t qdims[2] = {(uint64_t)R, (uint64_t)a.B * a.h};
    const uint64_t qstr[1] = {(uint64_t)R * 2};
    if (!encode_tmap(&tmQ, a.q_lat, 2, qdims, qstr, qbox)) return cudaErrorInvalidValue;
    // The cache holds sum(ctx) <= B * max_ctx rows; cu_ctx lives on the
    // device, so the map is declared with the bound and every box is clamped
    // inside its own sequence (chunk_base).
    const uint64_t cdims[2] = {(uint64_t)W, (uint64_t)a.B * (uint64_t)a.max_ctx};
    const uint64_t cstr[1] = {(uint64_t)W * 2};
    if (!encode_tmap(&tmC, a.cache, 2, cdims, cstr, cbox)) return cudaErrorInvalidValue;
    DecTcParams p{};
    p.cu_ctx = a.cu_ctx;
    p.q_pe = reinterpret_cast<const __nv_bfloat16*>(a.q_pe);
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
    latent_attn_kernel<<<grid, NTHREADS, SMEM_BYTES, st>>>(tmQ, tmC, p);
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
