// tcgen05 causal flash attention for the MLA prefill (bf16 in, fp32 softmax).
//
// Per head h and query i: s_j = scale (q_nope_h . k_nope_h[j] + q_pe_h . k_pe[j])
// over keys j <= i (causal triu(1) mask, MiniMind "Attention 前向传播" section
// 5), softmax in fp32, O_i = sum_j p_j V_h[j] with V of width v_head_dim.
// Q_h = [q_nope_h | q_pe_h] and K_h = [k_nope_h | k_pe] are the concatenations
// of the CSDN DeepseekV3Attention forward; here they are never materialised:
// the QK^T contraction runs over three 64-wide K-major operand boxes, two
// from the per-head k_nope and one from the single shared k_pe head (read
// straight from the latent buffer, so it is not expanded per head).  V keeps
// its own width (128) as an MN-major operand: no zero padding to the query
// head dim and no trimming (the FA2 constraint the verl kimi_vl page works
// around does not apply).
//
// One CTA = (batch, head, two 128-query tiles A and B); every K/V block it
// loads serves both tiles.  The CTAs of eight (sequence, head) pairs at a
// time run together, longest first, so a head's keys and values leave HBM
// once and the grid ends on short CTAs.  Warp roles
// (384 threads):
//   warp 0       TMA: Q of both tiles (once), K (one stage of 3 boxes)
//   warp 2       TMA: V ring (2 stages of 2 boxes of 64 value columns)
//   warp 1       TMEM allocation and MMA issue, in the order
//                  PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)
//                so that the tensor core works on one tile while the other
//                tile's softmax runs; S_X(j+1) follows PV_X(j) in issue order,
//                which is execution order (P_X(j) lives in S_X's columns).
//   warps 4-7    softmax of tile A, warps 8-11 of tile B (thread = query
//                row, all 128 keys of a block in one thread, so no exchange
//                between threads; 12 warps leave each thread 168 registers):
//                S from TMEM, causal mask on the diagonal block,
//                running max with lazy rescaling (O and l rescaled only when
//                the max grows by more than 2^8), P as bf16 pairs written
//                over the first 64 columns of S (the A operand of PV, read
//                from tensor memory), final O / l to global.
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).  Every wait
// is bounded.
#include "sm100.cuh"
#include "tc.h"

namespace mla {
namespace {

using namespace sm100;

constexpr int BQ = 128, BKV = 128;
constexpr int DN = 128, DR = 64, DV = 128, DQ = DN + DR;
constexpr int BOX = 128 * 64 * 2;                // one 64-column box of 128 rows
constexpr int Q_BYTES = 3 * BOX;                 // 48 KB per tile
constexpr int K_BYTES = 3 * BOX;                 // 48 KB per stage
constexpr int V_BYTES = 2 * BOX;                 // 32 KB
constexpr int OFF_Q = 0, OFF_K = 2 * Q_BYTES, OFF_V = OFF_K + K_BYTES;
constexpr int SMEM_BYTES = OFF_V + 2 * V_BYTES + 1024;
constexpr int NTHREADS = 384;
constexpr uint32_t IDESC_S = idesc_bf16(128, BKV);
constexpr uint32_t IDESC_PV = idesc_bf16(128, DV, 0, 1);   // V is MN-major
constexpr uint32_t TM_S = 0, TM_O = 256;                   // + 128 * tile
constexpr float kRescaleLog2 = 8.f;
constexpr int kHeadGroup = 8;      // (sequence, head) pairs whose CTAs are ordered together

struct AttnTcParams {
  int B, T, h;           // T queries per sequence
  int Tk, q_off;         // keys per sequence, position of query 0
  float scale_log2;      // softmax scale * log2(e)
  int n_pairs;           // CTAs per head: ceil(T / 256)
  const int32_t* cu;     // packed sequences (or null): rows cu[b] .. cu[b+1]-1
  int total;             // packed row count
  __nv_bfloat16* o;      // [N, h, DV]
  uint32_t* status;
};

__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmKV,
                   const __grid_constant__ CUtensorMap tmKpe,
                   const __grid_constant__ AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, k_full, k_empty, v_full[2], v_empty[2], s_full[2],
      p_full[2], pv_done[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;
  griddep_wait();
  griddep_launch_dependents();

  // Launch order: groups of kHeadGroup (sequence, head) pairs, and inside a
  // group all its CTAs longest first (pair c has about 2c + 2 key blocks).
  // A group's keys and values stay in L2 while its CTAs run; longest first
  // keeps the last CTAs of the grid short.
  const int nbh = p.B * p.h;
  const int grp = blockIdx.x / (p.n_pairs * kHeadGroup);
  const int gh = min(kHeadGroup, nbh - grp * kHeadGroup);          // pairs in this group
  const int rem = blockIdx.x - grp * p.n_pairs * kHeadGroup;
  const int bh = grp * kHeadGroup + rem % gh;
  const int hh = bh % p.h;
  const int b = bh / p.h;
  const int c = p.n_pairs - 1 - rem / gh;
  int row0, krow0, Tq, Tk, q_off;                    // this sequence's rows and lengths
  if (p.cu) {   // packed: bounds clamped to [0, total) so no store leaves the buffer
    const int s0 = min(max(p.cu[b], 0), p.total);
    const int s1 = min(max(p.cu[b + 1], s0), p.total);
    row0 = krow0 = s0;
    Tq = Tk = min(s1 - s0, p.T);
    q_off = 0;
  } else {
    row0 = b * p.T;
    krow0 = b * p.Tk;
    Tq = p.T;
    Tk = p.Tk;
    q_off = p.q_off;
  }
  // tile X covers queries [q0X, q0X + 128) (positions + q_off) and key
  // blocks [0, nkvX)
  const int q0A = 256 * c, q0B = 256 * c + BQ;
  if (q0A >= Tq) return;   // a shorter packed sequence: nothing for this CTA
  const int nkvA = q0A < Tq ? min(q_off + q0A + BQ - 1, Tk - 1) / BKV + 1 : 0;
  const int nkvB = q0B < Tq ? min(q_off + q0B + BQ - 1, Tk - 1) / BKV + 1 : 0;
  const int nkv = max(nkvA, nkvB);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);          // the tile's softmax warps
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(&k_full, 1);
    mbar_init(&k_empty, 1);
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

  if (warp == 0) {
    // ---------------- Q and K producer
    if (elect_one()) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmKV);
      tma_prefetch(&tmKpe);
      mbar_arrive_expect_tx(&q_full, (nkvB > 0 ? 2 : 1) * Q_BYTES);
      for (int a = 0; a < 3; ++a) {
        tma_load_2d(smem + OFF_Q + a * BOX, &tmQ, hh * DQ + a * 64, row0 + q0A, &q_full);
        if (nkvB > 0)
          tma_load_2d(smem + OFF_Q + Q_BYTES + a * BOX, &tmQ, hh * DQ + a * 64, row0 + q0B,
                      &q_full);
      }
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(&k_empty, (j & 1) ^ 1, abort_v, p.status)) break;
        uint8_t* sk = smem + OFF_K;
        mbar_arrive_expect_tx(&k_full, K_BYTES);
        const int kr = krow0 + j * BKV;
        tma_load_2d(sk, &tmKV, hh * (DN + DV), kr, &k_full);
        tma_load_2d(sk + BOX, &tmKV, hh * (DN + DV) + 64, kr, &k_full);
        tma_load_2d(sk + 2 * BOX, &tmKpe, 0, kr, &k_full);
      }
    }
  } else if (warp == 2) {
    // ---------------- V producer
    if (elect_one()) {
      for (int j = 0; j < nkv; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(&v_empty[slot], ((j >> 1) & 1) ^ 1, abort_v, p.status)) break;
        uint8_t* sv = smem + OFF_V + slot * V_BYTES;
        mbar_arrive_expect_tx(&v_full[slot], V_BYTES);
        const int kr = krow0 + j * BKV;
        tma_load_2d(sv, &tmKV, hh * (DN + DV) + DN, kr, &v_full[slot]);
        tma_load_2d(sv + BOX, &tmKV, hh * (DN + DV) + DN + 64, kr, &v_full[slot]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      const uint32_t sq = smem_u32(smem + OFF_Q);
      const int nkvX[2] = {nkvA, nkvB};
      // S_X(j) = Q_X K_j^T into TMEM S_X (K_j in the single K stage)
      auto issue_s = [&](int x, int j) {
        const uint32_t sk = smem_u32(smem + OFF_K);
        const uint32_t qx = sq + x * Q_BYTES;
#pragma unroll
        for (int k = 0; k < DQ / 16; ++k) {
          const uint32_t off = (k >> 2) * BOX + (k & 3) * 32;
          mma_bf16(tbase + TM_S + x * 128, desc_kmajor_sw128(qx + off),
                   desc_kmajor_sw128(sk + off), IDESC_S, k != 0);
        }
        mma_commit(&s_full[x]);
      };
      // O_X += P_X(j) V_j, P_X(j) from TMEM (16 keys = 8 packed columns per step)
      auto issue_pv = [&](int x, int j) {
        const uint32_t sv = smem_u32(smem + OFF_V + (j & 1) * V_BYTES);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          mma_bf16_ts(tbase + TM_O + x * 128, tbase + TM_S + x * 128 + k * 8,
                      desc_mnmajor_sw128(sv + k * 16 * 128, BOX), IDESC_PV, (j | k) != 0);
        mma_commit(&pv_done[x]);
      };
      bool ok = mbar_wait(&q_full, 0, abort_v, p.status) &&
                mbar_wait(&k_full, 0, abort_v, p.status);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (nkvX[x] > 0) issue_s(x, 0);
        mma_commit(&k_empty);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const bool more = j + 1 < nkv;
        bool k_ready = false;
        if (!mbar_wait(&v_full[j & 1], (j >> 1) & 1, abort_v, p.status)) break;
        for (int x = 0; x < 2 && ok; ++x) {
          if (j < nkvX[x]) {
            if (!mbar_wait(&p_full[x], j & 1, abort_v, p.status)) { ok = false; break; }
            tc_fence_after();
            issue_pv(x, j);
          }
          if (j + 1 < nkvX[x]) {
            if (!k_ready) {       // K_{j+1} is waited for only where it is needed
              if (!mbar_wait(&k_full, (j + 1) & 1, abort_v, p.status)) { ok = false; break; }
              k_ready = true;
            }
            // S_X(j+1) overwrites the columns P_X(j) occupies; tcgen05.mma
            // operations of one thread execute in issue order, so PV_X(j),
            // issued just before, has read them first
            issue_s(x, j + 1);
          }
        }
        if (!ok) break;
        mma_commit(&v_empty[j & 1]);
        if (more) mma_commit(&k_empty);
      }
    }
  } else if (warp >= 4) {
    // ---------------- softmax: one warpgroup per tile (warps 4-7 tile A, 8-11
    // tile B), thread = query row, all 128 keys of a block in one thread (no
    // exchange between threads)
    const int x = (warp - 4) >> 2;                   // tile
    const int quad = warp & 3;
    const int r = quad * 32 + lane;                  // query row within the tile
    const int qi = (x ? q0B : q0A) + r;              // query position
    const int my_nkv = x ? nkvB : nkvA;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tbase + lane_off + TM_S + x * 128;
    const uint32_t tO = tbase + lane_off + TM_O + x * 128;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < my_nkv; ++j) {
      // S_X(j) completion also implies PV_X(j-1) completion (in-order MMAs,
      // and S_X(j) was issued after PV_X(j-1) completed)
      if (!warp_wait(&s_full[x], j & 1, abort_v, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + cc * 32, sr[cc]);
      tmem_wait_ld();
      // Raw scores; the scale is folded into the exp argument below (scale > 0).
      const int kmax = min(q_off + qi, Tk - 1) - j * BKV;   // last visible key here
      if (kmax < BKV - 1) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (cc * 32 + i > kmax) sr[cc][i] = __float_as_uint(-INFINITY);
      }
      float mx4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mx4[k] = __uint_as_float(sr[0][k]);
#pragma unroll
      for (int i = 4; i < 128; i += 2)
        mx4[(i >> 1) & 3] = max3f(mx4[(i >> 1) & 3], __uint_as_float(sr[i >> 5][i & 31]),
                                  __uint_as_float(sr[(i + 1) >> 5][(i + 1) & 31]));
      const float mx =
          fmaxf(m_ref, p.scale_log2 * max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])));
      const bool grow = mx > m_ref + kRescaleLog2;    // also true for the first block
      const float alpha = grow ? ex2(m_ref - mx) : 1.f;
      if (grow) {
        l *= alpha;
        m_ref = mx;
      }
      // P = 2^(scale * s - m_ref) as bf16 pairs over the first 64 columns of S,
      // 16 columns (32 keys) at a time: P of keys [32q, 32q + 32) goes over
      // the scores of keys [16q, 16q + 16), which are already used
      float ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ls[k] = 0.f;
      const float sc = p.scale_log2;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t wv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(fmaf(__uint_as_float(sr[q][2 * e]), sc, -m_ref));
          const float p1 = ex2(fmaf(__uint_as_float(sr[q][2 * e + 1]), sc, -m_ref));
          ls[e & 7] += p0 + p1;
          wv[e] = pack_bf16(p0, p1);
        }
        tmem_st16(tS + q * 16, wv);
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O_X holds the sum through block j-1 (complete, see above)
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x]);
    }
    if (ok && my_nkv > 0 && warp_wait(&pv_done[x], (my_nkv - 1) & 1, abort_v, p.status)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const bool row_ok = qi < Tq;
      __nv_bfloat16* dst = p.o + ((int64_t)(row0 + qi) * p.h + hh) * DV;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            st_global_v4(dst + cc * 32 + i,
                         pack_bf16(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv),
                         pack_bf16(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv),
                         pack_bf16(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv),
                         pack_bf16(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv));
        }
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

}  // namespace

bool tc_attention_supported(const mla_config& c) {
  return c.dtype == MLA_BF16 && c.qk_nope_head_dim == DN && c.qk_rope_head_dim == DR &&
         c.v_head_dim == DV && c.kv_lora_rank % 64 == 0;
}

cudaError_t tc_attention(const AttnArgs& a, cudaStream_t st) {
  const int Tk = a.Tk > 0 ? a.Tk : a.T;
  // query and key rows of the maps (packed: all sequences' rows)
  const int64_t N = a.cu_seqlens ? (int64_t)a.total : (int64_t)a.B * a.T;
  const int64_t Nk = a.cu_seqlens ? (int64_t)a.total : (int64_t)a.B * Tk;
  CUtensorMap tmQ, tmKV, tmKpe;
  const uint32_t box[2] = {64, 128};
  {
    const uint64_t dims[2] = {(uint64_t)a.h * DQ, (uint64_t)N};
    const uint64_t strides[1] = {(uint64_t)a.h * DQ * 2};
    if (!encode_tmap(&tmQ, a.q, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)a.h * (DN + DV), (uint64_t)Nk};
    const uint64_t strides[1] = {(uint64_t)a.h * (DN + DV) * 2};
    if (!encode_tmap(&tmKV, a.kv, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // k_pe columns [r_kv, r_kv + 64) of the latent buffer [N, r_kv + 64]
    const uint64_t dims[2] = {(uint64_t)DR, (uint64_t)Nk};
    const uint64_t strides[1] = {(uint64_t)(a.r_kv + a.dr) * 2};
    const __nv_bfloat16* kpe = reinterpret_cast<const __nv_bfloat16*>(a.ckv) + a.r_kv;
    if (!encode_tmap(&tmKpe, kpe, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  AttnTcParams p{};
  p.B = a.B;
  p.T = a.T;
  p.h = a.h;
  p.Tk = Tk;
  p.q_off = a.q_off;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.n_pairs = (a.T + 2 * BQ - 1) / (2 * BQ);
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.status = a.status;
  p.cu = a.cu_seqlens;
  p.total = a.total;
  static std::atomic<uint64_t> smem_set{0};
  {
    const cudaError_t ea = set_dynamic_smem((const void*)attn_tc_kernel, SMEM_BYTES, smem_set);
    if (ea != cudaSuccess) return ea;
  }
  dim3 grid(p.n_pairs * a.h * a.B);
  const cudaError_t e = launch_pdl(attn_tc_kernel, grid, dim3(NTHREADS), SMEM_BYTES, st, tmQ,
                                   tmKV, tmKpe, p);
  count_launches();
  return e;
}

}  // namespace mla
