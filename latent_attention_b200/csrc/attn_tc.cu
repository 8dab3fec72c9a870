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
// One CTA = (batch, head, 128-query block); heaviest causal blocks launch
// first.  Warp roles (256 threads):
//   warp 0     TMA: Q (once) and the K ring (2 stages of 3 boxes)
//   warp 1     TMEM allocation and MMA issue: S_j = Q K_j^T (12 x M128 N128
//              K16) into one of two TMEM S buffers, then O += P_{j-1} V_{j-1}
//   warp 2     TMA: V (2 stages, 2 boxes of 64 value columns)
//   warps 4-7  softmax, thread = query row: S row from TMEM, mask, running
//              max with lazy rescaling (O and l rescaled only when the max
//              grows by more than 2^8), P as bf16 into TMEM (the A operand of
//              the PV MMA is read from tensor memory), final O / l to global.
// TMEM: S0 [0,128), S1 [128,256), O [256,384), P [384,448).  All waits are
// bounded.
#include "sm100.cuh"
#include "tc.h"

namespace mla {
namespace {

using namespace sm100;

constexpr int BQ = 128, BKV = 128;
constexpr int DN = 128, DR = 64, DV = 128, DQ = DN + DR;
constexpr int BOX = 128 * 64 * 2;                // one 64-column box of 128 rows
constexpr int Q_BYTES = 3 * BOX;                 // 48 KB
constexpr int K_BYTES = 3 * BOX;                 // 48 KB per stage
constexpr int V_BYTES = 2 * BOX;                 // 32 KB per stage
constexpr int OFF_Q = 0, OFF_K = Q_BYTES, OFF_V = OFF_K + 2 * K_BYTES;
constexpr int SMEM_BYTES = OFF_V + 2 * V_BYTES + 1024;
constexpr int NTHREADS = 256;
constexpr uint32_t IDESC_S = idesc_bf16(128, BKV);
constexpr uint32_t IDESC_PV = idesc_bf16(128, DV, 0, 1);   // V is MN-major
constexpr uint32_t TM_S = 0, TM_O = 256, TM_P = 384;   // P: 2 slots of 64 columns
constexpr float kRescaleLog2 = 8.f;

struct AttnTcParams {
  int B, T, h;
  float scale_log2;      // softmax scale * log2(e)
  int n_qblk;
  __nv_bfloat16* o;      // [N, h, DV]
  uint32_t* status;
};

__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmKV,
                   const __grid_constant__ CUtensorMap tmKpe,
                   const __grid_constant__ AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2],
      s_full[2], s_free[2], p_full, pv_done[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_v = &abort_flag;

  // All query blocks of one head run together (heaviest first), so that the
  // head's keys and values come from HBM once and from L2 for the others.
  const int hh = blockIdx.y % p.h;
  const int b = blockIdx.y / p.h;
  const int qb = p.n_qblk - 1 - blockIdx.x;
  const int q0 = qb * BQ;
  const int row0 = b * p.T;                          // first token of the sequence
  const int nkv = qb + 1;                            // causal: key blocks 0..qb

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&p_full, 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
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
      uint8_t* sq = smem + OFF_Q;
      mbar_arrive_expect_tx(&q_full, Q_BYTES);
      for (int a = 0; a < 3; ++a)
        tma_load_2d(sq + a * BOX, &tmQ, hh * DQ + a * 64, row0 + q0, &q_full);
      for (int j = 0; j < nkv; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(&k_empty[slot], ((j >> 1) & 1) ^ 1, abort_v, p.status)) break;
        uint8_t* sk = smem + OFF_K + slot * K_BYTES;
        mbar_arrive_expect_tx(&k_full[slot], K_BYTES);
        const int kr = row0 + j * BKV;
        tma_load_2d(sk, &tmKV, hh * (DN + DV), kr, &k_full[slot]);
        tma_load_2d(sk + BOX, &tmKV, hh * (DN + DV) + 64, kr, &k_full[slot]);
        tma_load_2d(sk + 2 * BOX, &tmKpe, 0, kr, &k_full[slot]);
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
        const int kr = row0 + j * BKV;
        tma_load_2d(sv, &tmKV, hh * (DN + DV) + DN, kr, &v_full[slot]);
        tma_load_2d(sv + BOX, &tmKV, hh * (DN + DV) + DN + 64, kr, &v_full[slot]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      const uint32_t sq = smem_u32(smem + OFF_Q);
      bool ok = mbar_wait(&q_full, 0, abort_v, p.status);
      auto issue_pv = [&](int j) -> bool {
        const int vs = j & 1;
        if (!mbar_wait(&p_full, j & 1, abort_v, p.status)) return false;
        if (!mbar_wait(&v_full[vs], (j >> 1) & 1, abort_v, p.status)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + OFF_V + vs * V_BYTES);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          // A = P_j from TMEM slot j % 2: 16 keys = 8 packed columns per step
          const uint64_t bv = desc_mnmajor_sw128(sv + k * 16 * 128, BOX);
          mma_bf16_ts(tbase + TM_O, tbase + TM_P + (j & 1) * 64 + k * 8, bv, IDESC_PV,
                      (j | k) != 0);
        }
        mma_commit(&v_empty[vs]);
        mma_commit(&pv_done[j & 1]);
        return true;
      };
      for (int j = 0; ok && j < nkv; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(&k_full[slot], (j >> 1) & 1, abort_v, p.status)) break;
        if (!mbar_wait(&s_free[slot], ((j >> 1) & 1) ^ 1, abort_v, p.status)) break;
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + OFF_K + slot * K_BYTES);
#pragma unroll
        for (int k = 0; k < DQ / 16; ++k) {
          const uint32_t off = (k >> 2) * BOX + (k & 3) * 32;
          mma_bf16(tbase + TM_S + slot * BKV, desc_kmajor_sw128(sq + off),
                   desc_kmajor_sw128(sk + off), IDESC_S, k != 0);
        }
        mma_commit(&k_empty[slot]);
        mma_commit(&s_full[slot]);
        if (j > 0 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_pv(nkv - 1);
    }
  } else if (warp >= 4) {
    // ---------------- softmax warpgroup
    const int quad = warp & 3;
    const int r = quad * 32 + lane;                  // query row within the block
    const int qi = q0 + r;                           // query position
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int slot = j & 1;
      if (!warp_wait(&s_full[slot], (j >> 1) & 1, abort_v, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tbase + lane_off + TM_S + slot * BKV + c * 32, sr[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[slot]);

      // Raw scores; the scale is folded into the exp argument below (scale > 0,
      // so the row max commutes with it).  The causal compare is needed only on
      // the diagonal block and on the ragged tail.
      float s[128];
      const int k0 = j * BKV;
      const int kmax = min(qi, p.T - 1) - k0;         // last visible key in this block
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(sr[c][i]);
      if (kmax < 127) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > kmax) s[i] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = s[k];
#pragma unroll
      for (int i = 8; i < 128; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
      const float mx = fmaxf(m_ref, p.scale_log2 * fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]),
                                                                fmaxf(mx8[2], mx8[3])),
                                                          fmaxf(fmaxf(mx8[4], mx8[5]),
                                                                fmaxf(mx8[6], mx8[7]))));
      const bool grow = mx > m_ref + kRescaleLog2;    // also true for the first block
      const float alpha = grow ? ex2(m_ref - mx) : 1.f;
      if (grow) {
        l *= alpha;
        m_ref = mx;
      }
      // P = 2^(scale * s - m_ref) as packed bf16 pairs (computed before any wait)
      float ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ls[k] = 0.f;
      const float sc = p.scale_log2;
      uint32_t w[2][32];
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int i = half * 64 + 2 * e;
          const float p0 = ex2(fmaf(s[i], sc, -m_ref));
          const float p1 = ex2(fmaf(s[i + 1], sc, -m_ref));
          ls[e & 7] += p0 + p1;
          w[half][e] = pack_bf16(p0, p1);
        }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      // A rescale of O needs every earlier PV finished (PV_{j-1} is the last);
      // otherwise only the PV that read this P slot two blocks ago must be done.
      const bool rescale = j > 0 && __any_sync(0xffffffffu, grow);
      if (rescale) {
        if (!warp_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_v, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_off + TM_O + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tbase + lane_off + TM_O + c * 32, o);
        }
      } else if (j > 1) {
        if (!warp_wait(&pv_done[j & 1], ((j - 2) >> 1) & 1, abort_v, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st32(tbase + lane_off + TM_P + (j & 1) * 64, w[0]);
      tmem_st32(tbase + lane_off + TM_P + (j & 1) * 64 + 32, w[1]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full);
    }
    if (ok && warp_wait(&pv_done[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1, abort_v, p.status)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const bool row_ok = qi < p.T;
      __nv_bfloat16* dst = p.o + ((int64_t)(row0 + qi) * p.h + hh) * DV;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tbase + lane_off + TM_O + c * 32, o);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            st_global_v4(dst + c * 32 + i,
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
  const int64_t N = (int64_t)a.B * a.T;
  CUtensorMap tmQ, tmKV, tmKpe;
  const uint32_t box[2] = {64, 128};
  {
    const uint64_t dims[2] = {(uint64_t)a.h * DQ, (uint64_t)N};
    const uint64_t strides[1] = {(uint64_t)a.h * DQ * 2};
    if (!encode_tmap(&tmQ, a.q, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)a.h * (DN + DV), (uint64_t)N};
    const uint64_t strides[1] = {(uint64_t)a.h * (DN + DV) * 2};
    if (!encode_tmap(&tmKV, a.kv, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // k_pe columns [r_kv, r_kv + 64) of the latent buffer [N, r_kv + 64]
    const uint64_t dims[2] = {(uint64_t)DR, (uint64_t)N};
    const uint64_t strides[1] = {(uint64_t)(a.r_kv + a.dr) * 2};
    const __nv_bfloat16* kpe = reinterpret_cast<const __nv_bfloat16*>(a.ckv) + a.r_kv;
    if (!encode_tmap(&tmKpe, kpe, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  AttnTcParams p{};
  p.B = a.B;
  p.T = a.T;
  p.h = a.h;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.n_qblk = (a.T + BQ - 1) / BQ;
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.status = a.status;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(p.n_qblk, a.h * a.B);
  attn_tc_kernel<<<grid, NTHREADS, SMEM_BYTES, st>>>(tmQ, tmKV, tmKpe, p);
  count_launches();
  return cudaGetLastError();
}

}  // namespace mla
