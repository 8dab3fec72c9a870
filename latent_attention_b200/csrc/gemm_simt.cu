// CUDA-core GEMM with the MLA projection epilogues (fp32 FFMA).
//
// C = A B^T, A [M, K] row-major (stride lda), B [N, K] (nn.Linear [out, in],
// MiniMind "Attention 前向传播" section 2).  This is the fp32 configuration's
// path only (a tf32 tensor-core product cannot hold a 1e-5 relative
// tolerance); bf16 runs on the tensor-core GEMM.  The epilogue (see EpiSeg) fuses the RMSNorm row statistics and row scale, the
// RoPE rotation of the rope columns and the RMSNorm gain.
#include "internal.h"

namespace mla {
namespace {

constexpr int BM = 64, BN = kSimtTileN, BK = 16, NT = 256;

template <typename T>
__device__ __forceinline__ float ld(const void* p, int64_t i) {
  return Elem<T>::load(reinterpret_cast<const T*>(p) + i);
}

template <typename T>
__global__ void __launch_bounds__(NT) gemm_simt_kernel(GemmArgs a) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Cs[BM][BN + 1];

  // Which segment and which column tile inside it.
  int tile_n = blockIdx.x;
  const int tiles0 = (a.seg[0].ncols + BN - 1) / BN;
  const int s = (a.nseg > 1 && tile_n >= tiles0) ? 1 : 0;
  if (s == 1) tile_n -= tiles0;
  const EpiSeg& e = a.seg[s];
  const void* Bm = a.Bm[s];
  const int64_t ldb = a.ldb[s];
  const int n0 = tile_n * BN;
  const int m0 = blockIdx.y * BM;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;

  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += BK) {
#pragma unroll
    for (int i = 0; i < (BM * BK) / NT; ++i) {
      const int idx = tid + i * NT;
      const int r = idx / BK, kk = idx % BK;
      const int gm = m0 + r, gk = k0 + kk;
      As[kk][r] = (gm < a.M && gk < a.K) ? ld<T>(a.A, (int64_t)gm * a.lda + gk) : 0.f;
      const int gn = n0 + r;
      Bs[kk][r] = (gn < e.ncols && gk < a.K) ? ld<T>(Bm, (int64_t)gn * ldb + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) Cs[ty + 16 * i][tx + 16 * j] = acc[i][j];
  __syncthreads();

  // Epilogue: 4 threads per row, 16 columns each.
  const int r = tid / 4;
  const int cq = (tid % 4) * 16;
  const int m = m0 + r;
  if (m >= a.M) return;
  float rs = 1.f;
  if (e.ssq_in) {
    float ss = 0.f;
    for (int p = 0; p < e.ssq_parts; ++p) ss += e.ssq_in[p * e.ssq_ld + m];
    rs = rsqrtf(ss * e.rs_inv_dim + e.eps);
  }
  float ssq = 0.f;
  const int pos = e.pos ? e.pos[m] : m % e.T + e.pos_offset;
  T* out = reinterpret_cast<T*>(e.out);
  for (int c = cq; c < cq + 16; ++c) {
    const int n = n0 + c;
    if (n >= e.ncols) break;
    float v = Cs[r][c];
    if (n < e.norm_cols) ssq += v * v;
    v *= rs;
    if (e.cos) {
      const int p = n % e.rope_period;
      if (p >= e.rope_start && p < e.rope_start + e.rope_dim) {
        // pair (x1, x2) = columns (j, j + half) of the segment, or (2j, 2j+1)
        // for interleaved weights; output column i is x1' (i < half) or x2'.
        const int i = p - e.rope_start;
        const int half = e.rope_dim / 2;
        const int j = i < half ? i : i - half;
        const int cb = c - i;                              // segment start in the tile
        const float x1 = Cs[r][e.rope_interleave ? cb + 2 * j : cb + j] * rs;
        const float x2 = Cs[r][e.rope_interleave ? cb + 2 * j + 1 : cb + j + half] * rs;
        const float cs = e.cos[(int64_t)pos * e.rope_dim + i];
        const float sn = e.sin[(int64_t)pos * e.rope_dim + i];
        v = i < half ? x1 * cs - x2 * sn : x2 * cs + x1 * sn;
      }
    }
    if (e.gamma && n < e.norm_cols) v *= ld<T>(e.gamma, n);
    Elem<T>::store(out + (int64_t)m * e.ldo + n, v);
  }
  if (e.ssq_out) {
    ssq += __shfl_xor_sync(0xffffffffu, ssq, 1);
    ssq += __shfl_xor_sync(0xffffffffu, ssq, 2);
    if ((tid % 4) == 0 && n0 < e.norm_cols) e.ssq_out[tile_n * e.ssq_ld + m] = ssq;
  }
}

}  // namespace

cudaError_t launch_gemm_simt(int dtype, const GemmArgs& a, cudaStream_t st) {
  int tiles = (a.seg[0].ncols + BN - 1) / BN;
  if (a.nseg > 1) tiles += (a.seg[1].ncols + BN - 1) / BN;
  dim3 grid(tiles, (a.M + BM - 1) / BM);
  if (dtype != MLA_F32) return cudaErrorNotSupported;
  count_launches();
  gemm_simt_kernel<float><<<grid, NT, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
