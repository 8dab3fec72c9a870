// Weight-absorbed MLA decode on sm_100a (bf16 in, fp32 softmax/accumulation).
//
// Megatron-LM MLA guide, 推理优化: each cached token keeps the compressed
// latent [kv_compressed | k_pos_emb]; decode folds up_k (rows [0, nope) of a
// head's block of the kv up-projection) into the query and applies up_v
// (rows [nope, nope+v)) after attention.  Four kernels:
//
//   D1 q_lat[b,h] = W_UK[h]^T q_nope[b,h]          batched tcgen05 GEMM (one
//                                                   product per head, W_UK read
//                                                   as an MN-major operand)
//   D2 latent_attn_kernel  attention of the 128 heads of a sequence over its
//                          [ctx, 576] cache, on tcgen05 (below)
//   D3 combine_kernel      log-sum-exp merge of the partial results of the
//                          sequences D2 split -> o_lat (bf16)
//   D4 o[b,h] = W_UV[h] o_lat[b,h]                  batched tcgen05 GEMM
//
// D2 schedule.  The tokens of all sequences, concatenated in cu_ctx order,
// are cut into equal slices, one per CTA pair ("unit", one pair per two
// SMs, a single wave), each sequence charged a fixed number of extra
// positions for the cost of starting it (kSeqCost), so every unit has about
// the same work whatever the length mix.  A unit walks the segments of its
// slice (the parts of the sequences inside it) with one continuous chunk
// pipeline; a segment covering a whole sequence writes o_lat itself, the
// first and last segment of a slice leave a partial (o, lse) for D3.
//
// D2 design.  With 128 heads as the MMA M dimension the latent output
// O[128, 512] in fp32 fills all 512 TMEM columns, so the two CTAs of a unit
// split the latent dims: CTA c owns dims [256c, 256c + 256) and the rope
// dims [32c, 32c + 32).  Per 64-token chunk it loads only its own half of
// every cache row (four 64-dim latent boxes and a 32-dim rope box with
// 64-byte swizzle, 36 KB), computes the partial scores Q_c C_c^T over its own
// dims (the query's latent half from TMEM, its rope half from shared memory)
// and accumulates O[:, own dims] += P C[:, own dims] from the same tiles (the
// K-major B operand of the scores is the MN-major B operand of P C).  The two partial score tiles (128 heads
// x 64 tokens) are exchanged through distributed shared memory as fp16 (16
// KB each way per chunk; about 19.5 B/clk per SM of DSMEM bandwidth on B200
// would make an fp32 exchange, 32 KB, the limit of the chunk period) and both
// CTAs add fp16(s_0) + fp16(s_1) in fp32, the same values in the same order,
// so the two run bit-identical online softmaxes and never exchange anything
// else.  A group frees the chunk's TMEM score slot as soon as it has loaded
// the partial scores, so the tensor core can compute S_{g+2} while the
// exchange and the softmax of chunk g run; P_g (bf16) goes to shared memory
// as the A operand of P C.
// Between segments the query changes: the next segment's first S waits for
// its query (both parts are reloaded once the previous segment's last S has
// completed), and its first PV for the previous O to have been read out.  The
// epilogue stages its TMA stores in the latent boxes of the segment's last
// chunk, which the producer refills only after the epilogue.
// Warp roles (384 threads per CTA):
//   warp 0     TMA: the chunk ring (5 stages of 36 KB), L2 prefetch ahead
//              (into the next segment)
//   warp 1     TMEM allocation, MMA issue (S_g or PV, whichever is ready)
//   warp 3     TMA: each segment's rope query (this CTA's half)
//   warps 4-7, 8-11  two softmax groups taking alternate chunks (thread =
//              head): score exchange, softmax, P into shared memory; group 1 also
//              stores each segment's TMEM query part, group 0 writes each
//              segment's result
// All waits are bounded; a timeout sets the device status word.  The pair
// passes a cluster barrier after its barriers are initialised and before it
// exits, so no remote store or arrive reaches a CTA that is not running.
#include <cfloat>

#include "decode_slices.cuh"
#include "sm100.cuh"
#include "tc.h"

namespace mla {
namespace {

using namespace sm100;
using namespace slices;   // NT (tokens per chunk), the slice schedule

constexpr int R = 512, DR = 64, W = R + DR;      // latent, rope, cache row width
constexpr int QPE_BOX = 128 * 32 * 2;            // 128 heads x this CTA's 32 rope dims
constexpr int CBOX = NT * 64 * 2;                // 64 tokens x 64 dims bf16
constexpr int RBOX = NT * 32 * 2;                // 64 tokens x this CTA's 32 rope dims
constexpr int NSTAGE = 4;                        // chunk ring
constexpr int NSLOT = 2;                         // score slots (TMEM)
constexpr int NGRP = 2;                          // softmax groups, taking chunks in turn
constexpr int NSB = NGRP % 2 ? 2 * NGRP : NGRP;  // score barriers: chunk g uses g % NSB
constexpr int XBUF = 128 * NT * 2;               // one chunk's fp16 partial scores, 16 KB
constexpr int PBUF = 128 * NT * 2;               // one chunk's P (bf16), 16 KB
constexpr int OFF_QPE = 0;                               // rope query half, 8 KB
constexpr int OFF_X = OFF_QPE + QPE_BOX;                 // exchange buffers, one per group
constexpr int OFF_P = OFF_X + NGRP * XBUF;               // P buffers, one per group
constexpr int OFF_C = OFF_P + NGRP * PBUF;               // 72 KB
constexpr int STAGE = 4 * CBOX + RBOX;                   // 36 KB
constexpr int SMEM_BYTES = OFF_C + NSTAGE * STAGE + 1024;
constexpr int NTHREADS = 128 + 128 * NGRP;
constexpr int PREFETCH = 4;                              // chunks prefetched to L2
constexpr uint32_t IDESC_S = idesc_bf16(128, NT);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, 0, 1);
// TMEM: score slots [0, 128) (64 columns each), O [128, 384), the query's
// latent dims [256c, 256c + 256) of CTA c as bf16 pairs [384, 512).
constexpr uint32_t TM_S = 0, TM_O = 128, TM_Q = 384;
constexpr float kRescaleLog2 = 8.f;
constexpr int EPI_BOX = 32 * 128;             // epilogue staging: 32 rows of 128 bytes

struct DecTcParams {
  const int32_t* cu_ctx;
  const uint8_t* cache;        // [sum ctx, 576] bf16 rows (for L2 prefetch)
  const __nv_bfloat16* q_lat;  // [B, h, 512]
  int B, h, max_ctx;
  int n_units, min_len;        // CTA pairs; shortest slice of the token stream
  float scale_log2;
  float* part_o;               // [2 n_units, h, R]
  float* part_lse;             // [2 n_units, h]
  __nv_bfloat16* o_lat;        // [B, h, R]
  uint32_t* status;
};

// Bounded wait until a shared counter reaches `target` (same limit and abort
// protocol as the barrier waits).
__device__ __forceinline__ bool wait_count(const int* counter, int target,
                                           volatile int* abort_flag, uint32_t* status) {
  const volatile int* c = counter;
  if (*c >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (*c >= target) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitNs) {
        *abort_flag = 1;
        if (status) atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
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
                       const __grid_constant__ CUtensorMap tmCr,
                       const __grid_constant__ CUtensorMap tmPO,
                       const __grid_constant__ CUtensorMap tmOL,
                       const __grid_constant__ DecTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, qt_full, q_free, c_full[NSTAGE], c_empty[NSTAGE],
      s_full[NSB], s_free[NSB], x_full[NGRP], x_empty[NGRP], p_full[NGRP], pv_done[NGRP],
      o_done, o_free, ref_ready[NGRP];
  __shared__ int epi_count;                    // epilogue warps done, all segments
  __shared__ float m_hand[128];                // reference max after the last chunk
  __shared__ float fin_m[NGRP - 1][128], fin_l[NGRP - 1][128];  // groups 1.. at a segment's end
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag, seq_lo, seq_hi;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;
  griddep_wait();
  griddep_launch_dependents();

  const uint32_t rank = cluster_rank();
  const int u = blockIdx.x >> 1;
  const int h0 = blockIdx.z * 128;
  const int32_t* cu = p.cu_ctx;
  const Slice sl = unit_slice(cu, p.B, p.max_ctx, u, p.n_units, p.min_len);
  if (sl.r0 >= sl.r1) return;                    // past the end of the stream (both CTAs)
  const int dim0 = 256 * (int)rank;              // this CTA's latent columns

  if (threadIdx.x == 0) {
    seq_lo = seq_at(cu, p.B, sl.r0);
    seq_hi = seq_at(cu, p.B, sl.r1 - 1) + 1;
    mbar_init(&q_full, 1);
    mbar_init(&qt_full, 4);         // the last softmax group stored the TMEM query part
    mbar_init(&q_free, 1);          // the last S of a segment completed
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 1);
    }
    for (int s = 0; s < NSB; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);     // the chunk's softmax group loaded S_g
    }
    // Chunk g uses the exchange buffer, the P buffer and the barriers of
    // its group x = g % NGRP (phase g / NGRP; the score barriers likewise by
    // g % NSB), so that every barrier is waited on by one party, in order,
    // and no waiter ever looks for a phase two ahead of the current one (a
    // parity wait would take the older phase for it).  x_full[x] counts the
    // bytes of the peer's partial scores of a chunk (armed for the first
    // NGRP chunks here, then for chunk g + NGRP by the group that has seen
    // chunk g arrive); x_empty[x] completes when the peer's group has read
    // this CTA's partial scores of the buffer; p_full[x] when P_g is written;
    // pv_done[x] when PV_g has run.
    for (int x = 0; x < NGRP; ++x) {
      mbar_init(&x_full[x], 1);
      mbar_arrive_expect_tx(&x_full[x], XBUF);
      mbar_init(&x_empty[x], 4);
      mbar_init(&p_full[x], 4);
      mbar_init(&pv_done[x], 1);
    }
    epi_count = 0;
    mbar_init(&o_done, 1);          // the last PV of a segment completed
    mbar_init(&o_free, 4);          // softmax group 0 has read O out of TMEM
    for (int x = 0; x < NGRP; ++x)
      mbar_init(&ref_ready[x], 4);  // a softmax group published chunk g's reference
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 512);
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync_all();               // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  const int b0 = seq_lo, b1 = seq_hi;
  // softmax groups: warps 4 + 4x .. 7 + 4x (group x)
  const int sm_wg = warp >= 4 ? (warp - 4) >> 2 : -1;

  if (warp == 0) {
    // ---------------- the chunk ring, L2 prefetch
    if (elect_one()) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmC);
      tma_prefetch(&tmCr);
      // chunk j of segment s into L2: its rows are contiguous in the cache
      // (the rows its boxes read, less any before row 0); this CTA takes
      // half of the bytes
      auto prefetch = [&](const Seg& s, int j) {
        const int y = (int)s.start + chunk_base(s.n, s.t0, j);
        const int y0 = max(y, 0);
        const uint32_t half = (uint32_t)(y + NT - y0) * (W * 2 / 2);   // 576 bytes per row
        bulk_prefetch_l2(p.cache + (uint64_t)y0 * (W * 2) + rank * half, half);
      };
      // this CTA's latent half of a segment's query rows into L2
      auto prefetch_q = [&](const Seg& s) {
        for (int a = 0; a < 4; ++a) tma_prefetch_l2_2d(&tmQ, dim0 + 64 * a, s.b * p.h + h0);
      };
      SegCursor c, nx;
      c.start(cu, b0, b1, p.max_ctx, sl, u);
      int prev_nch = 0;
      // a stage whose last chunk ended a segment also holds that segment's
      // epilogue staging: segment ordinal, or -1
      int staged[NSTAGE];
      for (int s = 0; s < NSTAGE; ++s) staged[s] = -1;
      for (int g = 0; !c.done; ++g) {
        const Seg& s = c.s;
        if (c.j == 0) {
          if (prev_nch < PREFETCH)         // not prefetched by the previous segment
            for (int j = 0; j < PREFETCH && j < s.nch; ++j) prefetch(s, j);
          prev_nch = s.nch;
          nx = c;                          // the next segment, prefetched near this one's end
          nx.next_seg(cu, b0, b1, p.max_ctx, sl, u);
        }
        if (c.j + PREFETCH < s.nch) {
          prefetch(s, c.j + PREFETCH);
        } else if (!nx.done) {
          const int jn = c.j + PREFETCH - s.nch;
          if (jn == 0) prefetch_q(nx.s);
          if (jn < nx.s.nch) prefetch(nx.s, jn);
        }
        const int st = g % NSTAGE;
        if (!mbar_wait(&c_empty[st], ((g / NSTAGE) & 1) ^ 1, abort_v, p.status)) break;
        // (a count, not a barrier phase: this wait may lag several segments)
        if (staged[st] >= 0 &&
            !wait_count(&epi_count, 4 * (staged[st] + 1), abort_v, p.status))
          break;
        staged[st] = c.j == s.nch - 1 ? c.kk : -1;
        uint8_t* sc = smem + OFF_C + st * STAGE;
        mbar_arrive_expect_tx(&c_full[st], STAGE);
        const int y = (int)s.start + chunk_base(s.n, s.t0, c.j);
        for (int a = 0; a < 4; ++a) tma_load_2d(sc + a * CBOX, &tmC, dim0 + 64 * a, y, &c_full[st]);
        tma_load_2d(sc + 4 * CBOX, &tmCr, R + 32 * (int)rank, y, &c_full[st]);
        c.next(cu, b0, b1, p.max_ctx, sl, u);
      }
    }
  } else if (warp == 3) {
    // ---------------- each segment's rope query (shared memory A operand)
    if (elect_one()) {
      tma_prefetch(&tmQpe);
      SegCursor c;
      c.start(cu, b0, b1, p.max_ctx, sl, u);
      for (; !c.done; c.next_seg(cu, b0, b1, p.max_ctx, sl, u)) {
        // the previous segment's scores no longer read the buffer
        if (c.kk > 0 && !mbar_wait(&q_free, (c.kk - 1) & 1, abort_v, p.status)) break;
        mbar_arrive_expect_tx(&q_full, QPE_BOX);
        tma_load_2d(smem + OFF_QPE, &tmQpe, 32 * (int)rank, c.s.b * p.h + h0, &q_full);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue
    if (elect_one()) {
      const uint64_t dq = desc_kmajor_sw64(smem_u32(smem + OFF_QPE));
      // Issue S_gs and O += P_gp C_gp in whichever order their inputs become
      // ready, across segments.  S_gs reuses the slot of S_{gs-2} once that
      // chunk's softmax group has loaded it; PV_gp follows S_gp.  A
      // segment's first S waits for its query (shared memory and TMEM
      // parts), its first PV for the previous segment's O to have been read
      // out.
      SegCursor cs, cp;
      cs.start(cu, b0, b1, p.max_ctx, sl, u);
      cp.start(cu, b0, b1, p.max_ctx, sl, u);
      int gs = 0, gp = 0;
      bool ok = true;
      uint64_t t_stall = 0;
      uint32_t idle = 0;
      while (ok && !cp.done) {
        bool progress = false;
        // PV first: its completion frees the chunk's stage
        if (gp < gs) {
          const int st = gp % NSTAGE;
          if (mbar_test(&p_full[gp % NGRP], (gp / NGRP) & 1) &&
              (cp.j != 0 || cp.kk == 0 || mbar_test(&o_free, (cp.kk - 1) & 1))) {
            tc_fence_after();
            const uint64_t dv = desc_mnmajor_sw128(smem_u32(smem + OFF_C + st * STAGE), CBOX);
            const uint64_t dp = desc_kmajor_sw128(smem_u32(smem + OFF_P + (gp % NGRP) * PBUF));
#pragma unroll
            for (int k = 0; k < NT / 16; ++k)
              mma_bf16(tbase + TM_O, dp + (uint64_t)((k * 32) >> 4),
                       dv + (uint64_t)((k * 16 * 128) >> 4), IDESC_PV, (cp.j | k) != 0);
            mma_commit(&c_empty[st]);
            mma_commit(&pv_done[gp % NGRP]);
            if (cp.j == cp.s.nch - 1) mma_commit(&o_done);
            ++gp;
            cp.next(cu, b0, b1, p.max_ctx, sl, u);
            progress = true;
          }
        }
        if (!cs.done) {
          const int st = gs % NSTAGE, sls = gs % NSLOT;
          const int sb = gs % NSB, sbf = (gs - NSLOT + NSB) % NSB;   // S_gs, S_{gs-2} barriers
          const uint32_t d = tbase + TM_S + sls * NT;
          const uint64_t dc = desc_kmajor_sw128(smem_u32(smem + OFF_C + st * STAGE));
          if ((cs.j != 0 || (mbar_test(&q_full, cs.kk & 1) && mbar_test(&qt_full, cs.kk & 1))) &&
              (gs < NSLOT || mbar_test(&s_free[sbf], ((gs - NSLOT) / NSB) & 1)) &&
              mbar_test(&c_full[st], (gs / NSTAGE) & 1)) {
            tc_fence_after();
            // partial S_gs over this CTA's dims: its latent half (query in
            // TMEM) and its half of the rope dims (query in shared memory)
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_bf16_ts(d, tbase + TM_Q + a * 32 + k * 8,
                            dc + (uint64_t)((a * CBOX + k * 32) >> 4), IDESC_S, (a | k) != 0);
            const uint64_t dr = desc_kmajor_sw64(smem_u32(smem + OFF_C + st * STAGE + 4 * CBOX));
#pragma unroll
            for (int k = 0; k < 2; ++k)
              mma_bf16(d, dq + (uint64_t)((k * 32) >> 4), dr + (uint64_t)((k * 32) >> 4), IDESC_S, 1);
            mma_commit(&s_full[sb]);
            if (cs.j == cs.s.nch - 1) mma_commit(&q_free);
            ++gs;
            cs.next(cu, b0, b1, p.max_ctx, sl, u);
            progress = true;
          }
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 63u) == 0) {   // bounded like every other wait
          const uint64_t now = globaltimer();
          if (idle == 64) t_stall = now;     // this stall began
          if (*abort_v) {
            ok = false;
          } else if (now - t_stall > kWaitNs) {
            *abort_v = 1;
            atomicOr(p.status, kStatusTimeout);
            ok = false;
          }
        }
      }
    }
  } else if (sm_wg >= 0) {
    // ---------------- softmax (thread = head): group g takes the chunks of
    // its parity in the unit's chunk sequence (score slot and exchange
    // buffer g).  The reference max of every row passes from one group to the
    // other through shared memory; each group keeps the row sum of its own
    // chunks, relative to its last reference.  Per segment, group 1 first
    // stores the query's TMEM part, group 0 finally merges both groups' sums
    // and writes the result.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int head = h0 + r;
    const bool head_ok = head < p.h;
    // this head's 16-byte column of the exchange buffer (16-byte piece k of
    // row r at k * 2048 + 16 r, so a warp's stores are 512 contiguous bytes),
    // here and in the peer; its 128-byte row of the P buffer (the 128-byte
    // swizzled K-major layout of an MMA operand)
    const uint32_t x_mine = smem_u32(smem + OFF_X) + r * 16;
    const uint32_t x_peer = mapa_shared(x_mine, rank ^ 1u);
    const uint32_t p_row = smem_u32(smem + OFF_P) + r * 128;
    // the peer's x_full / x_empty barriers (those of group x 8x bytes further)
    const uint32_t peer_x_full = mapa_shared(smem_u32(&x_full[0]), rank ^ 1u);
    const uint32_t peer_x_empty = mapa_shared(smem_u32(&x_empty[0]), rank ^ 1u);
    bool ok = true;
    SegCursor c;
    c.start(cu, b0, b1, p.max_ctx, sl, u);
    for (int g0 = 0; !c.done; c.next_seg(cu, b0, b1, p.max_ctx, sl, u)) {
      const Seg s = c.s;
      const int kk = c.kk;
      if (sm_wg == NGRP - 1 && ok) {   // this CTA's latent half of the head's query into TMEM
        // two rounds of 16 loads (the first issued before the wait for the
        // previous segment's last S), each stored as 64 TMEM columns
        const uint4* src =
            reinterpret_cast<const uint4*>(p.q_lat + ((int64_t)s.b * p.h + head) * R + dim0);
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = head_ok ? src[i] : make_uint4(0u, 0u, 0u, 0u);
        if (kk > 0 && !warp_wait(&q_free, (kk - 1) & 1, abort_v, p.status)) ok = false;
        if (ok) {
#pragma unroll
          for (int round = 0; round < 2; ++round) {
            if (round == 1) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                v[i] = head_ok ? src[16 + i] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t q[32];
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                q[4 * cc] = v[half * 8 + cc].x;
                q[4 * cc + 1] = v[half * 8 + cc].y;
                q[4 * cc + 2] = v[half * 8 + cc].z;
                q[4 * cc + 3] = v[half * 8 + cc].w;
              }
              tmem_st32(tbase + lane_off + TM_Q + round * 64 + half * 32, q);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&qt_full);
        }
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; ok && j < s.nch; ++j) {
        const int g = g0 + j;
        if (g % NGRP != sm_wg) continue;
        // score slot and barrier; this group and the previous chunk's group
        const int sls = g % NSLOT, sb = g % NSB, xs = sm_wg, xp = (g + NGRP - 1) % NGRP;
        const uint32_t ph = (g / NGRP) & 1, php = ((g - 1) / NGRP) & 1;   // their phases
        if (!warp_wait(&s_full[sb], (g / NSB) & 1, abort_v, p.status)) { ok = false; break; }
        tc_fence_after();
        // this CTA's partial scores as fp16 pairs
        uint32_t hx[32];
        {
          uint32_t sr[2][32];
          tmem_ld32(tbase + lane_off + TM_S + sls * NT, sr[0]);
          tmem_ld32(tbase + lane_off + TM_S + sls * NT + 32, sr[1]);
          tmem_wait_ld();
          tc_fence_before();      // the slot may take S_{g+2}
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[sb]);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            hx[e] = pack_f16_sat(__uint_as_float(sr[e >> 4][(2 * e) & 31]),
                                 __uint_as_float(sr[e >> 4][(2 * e + 1) & 31]));
        }
        // into the peer's exchange buffer xs, once the peer has read chunk
        // g - NGRP there: asynchronous stores that count their bytes on its
        // x_full[xs]
        if (g >= NGRP && !warp_wait(&x_empty[xs], ph ^ 1, abort_v, p.status)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_async_v4(x_peer + xs * XBUF + k * 2048, peer_x_full + 8 * xs, hx[4 * k], hx[4 * k + 1],
                      hx[4 * k + 2], hx[4 * k + 3]);
        // the peer's partial scores of chunk g; then x_full[xs] is armed for
        // chunk g + NGRP, whose bytes the peer sends only after chunk
        // g + NGRP - 1 has been read here, which follows this group's reading
        // of chunk g
        if (!warp_wait_cluster(&x_full[xs], ph, abort_v, p.status)) {
          ok = false;
          break;
        }
        if (quad == 0 && lane == 0) mbar_arrive_expect_tx(&x_full[xs], XBUF);
        float sv[NT];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 v = ld_shared_v4(x_mine + xs * XBUF + k * 2048);
          const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float a0, a1, b0, b1;
            unpack_f16(hx[4 * k + i], a0, a1);
            unpack_f16(pv[i], b0, b1);
            sv[8 * k + 2 * i] = a0 + b0;          // the same sum on both CTAs
            sv[8 * k + 2 * i + 1] = a1 + b1;
          }
        }
        __syncwarp();   // the values are summed: the buffer may take chunk g + NGRP
        if (lane == 0) mbar_arrive_cluster_relaxed(peer_x_empty + 8 * xs);
        // column i holds token base + i; chunk j owns tokens [t0 + 64j, t0 + tcount)
        const int base = chunk_base(s.n, s.t0, j) - s.t0;
        const int lo = j * NT - base, hi = s.tcount - base;
        // Raw scores; the (positive) scale is folded into the exp argument.
        if (lo > 0 || hi < NT) {       // first / last chunk of the segment only
#pragma unroll
          for (int i = 0; i < NT; ++i)
            if (i < lo || i >= hi) sv[i] = -INFINITY;
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < NT; i += 2)
          mx4[(i >> 1) & 3] = max3f(mx4[(i >> 1) & 3], sv[i], sv[i + 1]);
        const float cmax = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * p.scale_log2;
        // reference of chunk g-1, left by the other group (each thread reads
        // its row before it overwrites it).  The wait also keeps the hand-over
        // in order across segments, where the reference itself starts afresh.
        float m_prev = -INFINITY;
        if (g > 0) {
          if (!warp_wait(&ref_ready[xp], php, abort_v, p.status)) {
            ok = false;
            break;
          }
          if (j > 0) m_prev = m_hand[r];
        }
        // lazy rescaling: a new reference only when the max grew by > 2^8
        const bool grow = cmax > m_prev + kRescaleLog2;     // always at j = 0
        const float m_new = grow ? cmax : m_prev;
        m_hand[r] = m_new;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ref_ready[xs]);
        if (m_new != m_ref) {          // this group's sum, moved to the new reference
          l = l > 0.f ? l * ex2(m_ref - m_new) : 0.f;
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
          fma2(a0, a1, sv[2 * e], sv[2 * e + 1], p.scale_log2, p.scale_log2, neg_m, neg_m);
          const float p0 = ex2(a0);
          const float p1 = ex2(a1);
          add2(ls[2 * (e & 3)], ls[2 * (e & 3) + 1], p0, p1);
          w[e] = pack_bf16(p0, p1);
        }
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        // PV_{g-NGRP} has run: this group's P buffer is free (this wait, on
        // every chunk and in order, also completes PV_{g-NGRP-1}, so the one
        // below never sees a barrier two phases behind).
        if (g >= NGRP && !warp_wait(&pv_done[xs], ph ^ 1, abort_v, p.status)) {
          ok = false;
          break;
        }
        // O holds the segment's sum through chunk j-1 at reference m_prev:
        // rescale it when this chunk moved the reference (PV_{g-1} must have
        // run).
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          const float alpha = ex2(m_prev - m_new);
          if (!warp_wait(&pv_done[xp], php, abort_v, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t o[32];
            tmem_ld32(tbase + lane_off + TM_O + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tbase + lane_off + TM_O + cc * 32, o);
          }
          tmem_wait_st();
        }
        // P_g into this group's P buffer
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_shared_v4(p_row + xs * PBUF + ((k ^ (r & 7)) << 4), w[4 * k], w[4 * k + 1],
                       w[4 * k + 2], w[4 * k + 3]);
        fence_proxy_async();
        tc_fence_before();        // the O rescale above happens before PV_g
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[xs]);
      }
      g0 += s.nch;
      // Segment end.  Every group's sum at its last chunk's reference
      // (references never decrease, so the largest is the row's).  The other
      // groups hand over through fin_*; every softmax thread passes the two
      // barriers (after the writes, after group 0's reads) on every path.
      if (sm_wg > 0) {
        fin_m[sm_wg - 1][r] = m_ref;
        fin_l[sm_wg - 1][r] = l;
      }
      named_barrier_sync(1, 128 * NGRP);
      float m_last = m_ref, l_tot = 0.f;
      if (sm_wg == 0) {
#pragma unroll
        for (int x = 0; x < NGRP - 1; ++x) m_last = fmaxf(m_last, fin_m[x][r]);
        l_tot = l > 0.f ? l * ex2(m_ref - m_last) : 0.f;
#pragma unroll
        for (int x = 0; x < NGRP - 1; ++x) {
          const float lx = fin_l[x][r];
          l_tot += lx > 0.f ? lx * ex2(fin_m[x][r] - m_last) : 0.f;
        }
      }
      named_barrier_sync(1, 128 * NGRP);
      if (sm_wg == 0) {
        if (ok && !warp_wait(&o_done, kk & 1, abort_v, p.status)) ok = false;
        if (ok) {
          const float inv = 1.f / l_tot;
          tc_fence_after();
          // This warp's 32 rows go out through the latent boxes of the
          // segment's last chunk (free: its PV has completed; warp 0 refills
          // them only after o_free) and TMA stores, 32 x 64 bf16 or
          // 32 x 32 fp32 per box; a warp whose rows straddle the head count
          // stores directly.
          const int row0 = h0 + quad * 32;
          const bool tma_rows = row0 + 32 <= p.h;
          const int g_last = g0 - 1;
          const uint32_t stg =
              smem_u32(smem + OFF_C + (g_last % NSTAGE) * STAGE) + quad * 2 * EPI_BOX;
          auto stage = [&](int i, const uint32_t (&v)[32]) -> uint32_t {
            const uint32_t sb = stg + (i & 1) * EPI_BOX;
            if (i >= 2) {             // the store issued from this box two boxes ago
              if (lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
              st_shared_v4(sb + lane * 128 + ((k ^ (lane & 7)) << 4), v[4 * k], v[4 * k + 1],
                           v[4 * k + 2], v[4 * k + 3]);
            fence_proxy_async();
            __syncwarp();
            return sb;
          };
          if (s.whole) {           // the sequence's attention output, final
            __nv_bfloat16* dst = p.o_lat + ((int64_t)s.b * p.h + head) * R + dim0;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t w[32];
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                uint32_t o[32];
                tmem_ld32(tbase + lane_off + TM_O + cc * 64 + half * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  w[half * 16 + i] = pack_bf16(__uint_as_float(o[2 * i]) * inv,
                                               __uint_as_float(o[2 * i + 1]) * inv);
              }
              if (tma_rows) {
                const uint32_t sb = stage(cc, w);
                if (lane == 0) {
                  tma_store_2d(&tmOL, sb, dim0 + cc * 64, s.b * p.h + row0);
                  bulk_commit_group();
                }
              } else if (head_ok) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                  st_global_v4(dst + cc * 64 + 2 * i, w[i], w[i + 1], w[i + 2], w[i + 3]);
              }
            }
          } else {                 // a partial (o, lse) for the combine kernel
            const int64_t part = (int64_t)s.slot * p.h + head;
            float* dst = p.part_o + part * R + dim0;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
              uint32_t o[32];
              tmem_ld32(tbase + lane_off + TM_O + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * inv);
              if (tma_rows) {
                const uint32_t sb = stage(cc, o);
                if (lane == 0) {       // fp32 columns as bf16 pairs
                  tma_store_2d(&tmPO, sb, 2 * (dim0 + cc * 32), s.slot * p.h + row0);
                  bulk_commit_group();
                }
              } else if (head_ok) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                  st_global_v4(dst + cc * 32 + i, o[i], o[i + 1], o[i + 2], o[i + 3]);
              }
            }
            if (rank == 0 && head_ok)
              p.part_lse[part] = (m_last + __log2f(l_tot)) * 0.6931471805599453f;
          }
          // the staging boxes are read out before warp 0 refills them
          if (lane == 0) {
            bulk_wait_group_read<0>();
            atomicAdd(&epi_count, 1);
          }
          __syncwarp();
          // O may be overwritten by the next segment's first PV
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_free);
        }
      }
    }
  }
  if (sm_wg == 0 && lane == 0) bulk_wait_group<0>();   // epilogue stores done before exit
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // both CTAs are done with each other's shared memory
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// D3: o_lat[b,h] = sum_s w_s part_o[s,h] over the partial slots of sequence b
// (w_s = exp(lse_s - max) / sum), one warp per (sequence, head), HPB heads
// per block, 16 latent columns per thread.  A sequence inside one unit's
// slice was written by D2 itself; an invalid one (length outside [1,
// max_ctx]) is reported and zeroed.
template <int HPB>
__global__ void __launch_bounds__(32 * HPB)
    combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                   __nv_bfloat16* __restrict__ o_lat, const int32_t* __restrict__ cu, int B,
                   int max_ctx, int h, int n_units, int min_len, uint32_t* status) {
  griddep_wait();
  griddep_launch_dependents();
  const int hg = (h + HPB - 1) / HPB;
  const int b = blockIdx.x / hg;
  const int hh = (blockIdx.x % hg) * HPB + threadIdx.x / 32;
  if (hh >= h) return;
  const int c = (threadIdx.x % 32) * 16;
  uint4* dst = reinterpret_cast<uint4*>(o_lat + ((int64_t)b * h + hh) * R + c);
  const SeqUnits su = seq_units(cu, b, B, max_ctx, n_units, min_len);
  if (!su.valid) {
    if (hh == 0 && threadIdx.x == 0) atomicOr(status, kStatusBadCtx);
    dst[0] = make_uint4(0u, 0u, 0u, 0u);
    dst[1] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int u0 = su.u0, u1 = su.u1;
  if (u0 == u1) return;   // one unit covered the sequence and wrote o_lat
  float mx = -INFINITY;
  for (int uu = u0; uu <= u1; ++uu)
    mx = fmaxf(mx, part_lse[(int64_t)seq_slot(su, uu) * h + hh]);
  float den = 0.f, a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = 0.f;
  for (int uu = u0; uu <= u1; ++uu) {
    const int slot = seq_slot(su, uu);
    const float l = part_lse[(int64_t)slot * h + hh];
    if (l == -INFINITY) continue;
    const float w = __expf(l - mx);
    const float4* src = reinterpret_cast<const float4*>(part_o + ((int64_t)slot * h + hh) * R + c);
    den += w;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = src[q];
      a[4 * q] = fmaf(w, v.x, a[4 * q]);
      a[4 * q + 1] = fmaf(w, v.y, a[4 * q + 1]);
      a[4 * q + 2] = fmaf(w, v.z, a[4 * q + 2]);
      a[4 * q + 3] = fmaf(w, v.w, a[4 * q + 3]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int q = 0; q < 2; ++q)
    dst[q] = make_uint4(pack_bf16(a[8 * q] * inv, a[8 * q + 1] * inv),
                        pack_bf16(a[8 * q + 2] * inv, a[8 * q + 3] * inv),
                        pack_bf16(a[8 * q + 4] * inv, a[8 * q + 5] * inv),
                        pack_bf16(a[8 * q + 6] * inv, a[8 * q + 7] * inv));
}

}  // namespace

bool tc_decode_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.kv_lora_rank == R && c.qk_rope_head_dim == DR &&
         c.qk_nope_head_dim % 8 == 0 && c.v_head_dim % 8 == 0;
}

int tc_decode_min_slice() { return 512; }

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
    CUtensorMap tmQ, tmQpe, tmC, tmCr;
    const uint32_t qbox[2] = {64, 128}, cbox[2] = {64, NT};
    const uint32_t qpebox[2] = {32, 128}, rbox[2] = {32, NT};   // a CTA's rope half
    const uint64_t qdims[2] = {(uint64_t)R, (uint64_t)a.B * a.h};
    const uint64_t qstr[1] = {(uint64_t)R * 2};
    if (!encode_tmap(&tmQ, a.q_lat, 2, qdims, qstr, qbox)) return cudaErrorInvalidValue;
    const uint64_t pdims[2] = {(uint64_t)DR, (uint64_t)a.B * a.h};
    const uint64_t pstr[1] = {(uint64_t)DR * 2};
    if (!encode_tmap(&tmQpe, a.q_pe, 2, pdims, pstr, qpebox, 64)) return cudaErrorInvalidValue;
    // The cache holds sum(ctx) <= B * max_ctx rows; cu_ctx lives on the
    // device, so the map is declared with the bound and every box is clamped
    // inside its own sequence (chunk_base).
    const uint64_t cdims[2] = {(uint64_t)W, (uint64_t)a.B * (uint64_t)a.max_ctx};
    const uint64_t cstr[1] = {(uint64_t)W * 2};
    if (!encode_tmap(&tmC, a.cache, 2, cdims, cstr, cbox)) return cudaErrorInvalidValue;
    if (!encode_tmap(&tmCr, a.cache, 2, cdims, cstr, rbox, 64)) return cudaErrorInvalidValue;
    // epilogue stores: fp32 partials (as bf16 pairs) and the bf16 latent output,
    // 32 rows x 128 bytes per box
    CUtensorMap tmPO, tmOL;
    const uint32_t obox[2] = {64, 32};
    const uint64_t podims[2] = {(uint64_t)2 * R, (uint64_t)2 * a.n_units * a.h};
    const uint64_t postr[1] = {(uint64_t)R * 4};
    if (!encode_tmap(&tmPO, a.part_o, 2, podims, postr, obox)) return cudaErrorInvalidValue;
    const uint64_t oldims[2] = {(uint64_t)R, (uint64_t)a.B * a.h};
    const uint64_t olstr[1] = {(uint64_t)R * 2};
    if (!encode_tmap(&tmOL, a.o_lat, 2, oldims, olstr, obox)) return cudaErrorInvalidValue;
    DecTcParams p{};
    p.cu_ctx = a.cu_ctx;
    p.cache = reinterpret_cast<const uint8_t*>(a.cache);
    p.q_lat = reinterpret_cast<const __nv_bfloat16*>(a.q_lat);
    p.B = a.B;
    p.h = a.h;
    p.max_ctx = a.max_ctx;
    p.n_units = a.n_units;
    p.min_len = a.min_len;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.part_o = a.part_o;
    p.part_lse = a.part_lse;
    p.o_lat = reinterpret_cast<__nv_bfloat16*>(a.o_lat);
    p.status = a.status;
    static std::atomic<uint64_t> smem_set{0};
    {
      const cudaError_t ea = set_dynamic_smem((const void*)latent_attn_kernel, SMEM_BYTES, smem_set);
      if (ea != cudaSuccess) return ea;
    }
    dim3 grid(2 * a.n_units, 1, (a.h + 127) / 128);
    e = launch_pdl(latent_attn_kernel, grid, dim3(NTHREADS), SMEM_BYTES, st, tmQ, tmQpe, tmC,
                   tmCr, tmPO, tmOL, p);
    count_launches();
    if (e != cudaSuccess) return e;
  }
  stage_event(2, st);
  // D3
  // eight heads per block when the (sequence, head) pairs fill the GPU many
  // times over (fewer, fuller blocks); one otherwise (few sequences, many
  // partial slots each, spread over as many SMs as possible)
  if ((int64_t)a.B * a.h >= 16LL * (2 * a.n_units)) {
    e = launch_pdl(combine_kernel<8>, dim3(a.B * ((a.h + 7) / 8)), dim3(32 * 8), 0, st,
                   (const float*)a.part_o, (const float*)a.part_lse, (__nv_bfloat16*)a.o_lat,
                   a.cu_ctx, a.B, a.max_ctx, a.h, a.n_units, a.min_len, a.status);
  } else {
    e = launch_pdl(combine_kernel<1>, dim3(a.B * a.h), dim3(32), 0, st, (const float*)a.part_o,
                   (const float*)a.part_lse, (__nv_bfloat16*)a.o_lat, a.cu_ctx, a.B,
                   a.max_ctx, a.h, a.n_units, a.min_len, a.status);
  }
  count_launches();
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
