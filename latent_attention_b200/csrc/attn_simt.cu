// CUDA-core causal MLA attention (fp32 math), online softmax.
//
// For head h and query position i: s_j = scale * (q_nope_h . k_nope_h[j] +
// q_pe_h . k_pe[j]) for keys j <= i (triu(1) mask, MiniMind "Attention 前向传播"
// section 5), softmax over j, O = sum_j p_j V_h[j] with V of width v_head_dim
// (no zero padding).  The single k_pe head is read once per key from the
// latent buffer and shared by all heads (CSDN DeepseekV3Attention forward:
// k_rot.expand over heads).  The fp32 configuration's path only; bf16 runs on
// the tensor-core attention kernel.
#include <cfloat>

#include "internal.h"

namespace mla {
namespace {

constexpr int BQ = 16, BKEY = 32, NT = 128;

template <typename T>
__global__ void __launch_bounds__(NT) attn_simt_kernel(AttnArgs a_in) {
  AttnArgs a = a_in;
  extern __shared__ float sm[];
  const int dq = a.dn + a.dr;
  float* Qs = sm;                       // [BQ][dq]
  float* Ks = Qs + BQ * dq;             // [BKEY][dq]
  float* Vs = Ks + BKEY * dq;           // [BKEY][dv]
  float* Ss = Vs + BKEY * a.dv;         // [BQ][BKEY]
  float* Os = Ss + BQ * BKEY;           // [BQ][dv]
  float* Ms = Os + BQ * a.dv;           // [BQ] running max
  float* Ls = Ms + BQ;                  // [BQ] running sum
  float* Al = Ls + BQ;                  // [BQ] rescale factor

  const int hh = blockIdx.y, b = blockIdx.z;
  const int q0 = blockIdx.x * BQ;
  const int tid = threadIdx.x;
  const T* q = reinterpret_cast<const T*>(a.q);
  const T* kv = reinterpret_cast<const T*>(a.kv);
  const T* ckv = reinterpret_cast<const T*>(a.ckv);
  const int64_t qstride = (int64_t)a.h * dq;
  const int64_t kvstride = (int64_t)a.h * (a.dn + a.dv);
  const int64_t cstride = a.r_kv + a.dr;
  int64_t base = (int64_t)b * a.T;              // first query row of the sequence
  int64_t kbase = (int64_t)b * a.Tk;            // first key row of the sequence
  if (a.cu_seqlens) {   // packed: bounds clamped to [0, total)
    const int s0 = min(max(a.cu_seqlens[b], 0), a.total);
    const int s1 = min(max(a.cu_seqlens[b + 1], s0), a.total);
    base = kbase = s0;
    a.T = a.Tk = min(s1 - s0, a.T);
    a.q_off = 0;
  }
  if (q0 >= a.T) return;

  for (int idx = tid; idx < BQ * dq; idx += NT) {
    const int i = idx / dq, d = idx % dq;
    const int t = q0 + i;
    Qs[idx] = t < a.T ? Elem<T>::load(q + (base + t) * qstride + (int64_t)hh * dq + d) : 0.f;
  }
  for (int idx = tid; idx < BQ * a.dv; idx += NT) Os[idx] = 0.f;
  if (tid < BQ) { Ms[tid] = -FLT_MAX; Ls[tid] = 0.f; }
  __syncthreads();

  const int q_last = min(q0 + BQ, a.T) - 1;
  const int k_last = min(a.q_off + q_last, a.Tk - 1);
  for (int k0 = 0; k0 <= k_last; k0 += BKEY) {
    for (int idx = tid; idx < BKEY * dq; idx += NT) {
      const int j = idx / dq, d = idx % dq;
      const int t = k0 + j;
      float v = 0.f;
      if (t < a.Tk) {
        v = d < a.dn ? Elem<T>::load(kv + (kbase + t) * kvstride + (int64_t)hh * (a.dn + a.dv) + d)
                     : Elem<T>::load(ckv + (kbase + t) * cstride + a.r_kv + (d - a.dn));
      }
      Ks[idx] = v;
    }
    for (int idx = tid; idx < BKEY * a.dv; idx += NT) {
      const int j = idx / a.dv, d = idx % a.dv;
      const int t = k0 + j;
      Vs[idx] = t < a.Tk ? Elem<T>::load(kv + (kbase + t) * kvstride +
                                         (int64_t)hh * (a.dn + a.dv) + a.dn + d)
                         : 0.f;
    }
    __syncthreads();
    for (int idx = tid; idx < BQ * BKEY; idx += NT) {
      const int i = idx / BKEY, j = idx % BKEY;
      float s = 0.f;
      for (int d = 0; d < dq; ++d) s = fmaf(Qs[i * dq + d], Ks[j * dq + d], s);
      const bool masked = (k0 + j > a.q_off + q0 + i) || (k0 + j >= a.Tk);
      Ss[idx] = masked ? -INFINITY : s * a.scale;
    }
    __syncthreads();
    if (tid < BQ) {
      const int i = tid;
      float mx = Ms[i];
      for (int j = 0; j < BKEY; ++j) mx = fmaxf(mx, Ss[i * BKEY + j]);
      const float alpha = __expf(Ms[i] - mx);
      float l = Ls[i] * alpha;
      for (int j = 0; j < BKEY; ++j) {
        const float p = __expf(Ss[i * BKEY + j] - mx);
        Ss[i * BKEY + j] = p;
        l += p;
      }
      Ms[i] = mx;
      Ls[i] = l;
      Al[i] = alpha;
    }
    __syncthreads();
    for (int idx = tid; idx < BQ * a.dv; idx += NT) {
      const int i = idx / a.dv, d = idx % a.dv;
      float o = Os[idx] * Al[i];
      for (int j = 0; j < BKEY; ++j) o = fmaf(Ss[i * BKEY + j], Vs[j * a.dv + d], o);
      Os[idx] = o;
    }
    __syncthreads();
  }
  T* o = reinterpret_cast<T*>(a.o);
  for (int idx = tid; idx < BQ * a.dv; idx += NT) {
    const int i = idx / a.dv, d = idx % a.dv;
    const int t = q0 + i;
    if (t < a.T)
      Elem<T>::store(o + (base + t) * (int64_t)a.h * a.dv + (int64_t)hh * a.dv + d,
                     Os[idx] / Ls[i]);
  }
}

}  // namespace

cudaError_t launch_attn_simt(int dtype, const AttnArgs& a_in, cudaStream_t st) {
  AttnArgs a = a_in;
  if (a.Tk <= 0) a.Tk = a.T;
  const int dq = a.dn + a.dr;
  const size_t smem = sizeof(float) *
      (BQ * dq + BKEY * dq + BKEY * a.dv + BQ * BKEY + BQ * a.dv + 3 * BQ);
  dim3 grid((a.T + BQ - 1) / BQ, a.h, a.B);
  if (dtype != MLA_F32) return cudaErrorNotSupported;
  cudaError_t err = cudaFuncSetAttribute(attn_simt_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  attn_simt_kernel<float><<<grid, NT, smem, st>>>(a);
  count_launches();
  return cudaGetLastError();
}

}  // namespace mla
