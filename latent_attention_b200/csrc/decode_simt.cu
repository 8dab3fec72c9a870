// CUDA-core weight-absorbed MLA decode (the fp32 configuration) and the
// latent-cache finalisation used by prefill (both element types).
//
// Megatron-LM MLA guide, 推理优化: the cache keeps [kv_compressed | k_pos_emb]
// per token; decode folds up_k (rows [0, nope) of each head block of the kv
// up-projection) into the query and applies up_v (rows [nope, nope+v)) after
// attention.  Steps:
//   D1 q_lat[b,h] = W_UK[h]^T q_nope[b,h]              (qlat kernel)
//   D2 split-KV latent attention, partial (o, lse)      (split kernel)
//   D3 log-sum-exp merge of the splits                  (combine kernel)
//   D4 o[b,h] = W_UV[h] o_lat[b,h]                      (vup kernel)
#include <cfloat>

#include "internal.h"

namespace mla {
namespace {

template <typename T>
__global__ void latent_finalize_kernel(const T* __restrict__ ckv,
                                       const float* __restrict__ ssq, int parts, int N,
                                       int r, int dr, float eps,
                                       T* __restrict__ cache, int Tsrc, int dst_T, int dst_off) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int w = r + dr;
  if (idx >= (int64_t)N * w) return;
  const int64_t m = idx / w;
  const int c = (int)(idx % w);
  const int64_t drow = (m / Tsrc) * dst_T + dst_off + (m % Tsrc);
  float v = Elem<T>::load(ckv + idx);
  if (c < r) {
    float ss = 0.f;
    for (int p = 0; p < parts; ++p) ss += ssq[(int64_t)p * N + m];
    v *= rsqrtf(ss * (1.0f / r) + eps);
  }
  Elem<T>::store(cache + drow * w + c, v);
}

// D1: one block per (b, h); q_lat row = [W_UK^T q_nope | q_pe] in fp32 math.
template <typename T>
__global__ void qlat_kernel(DecodeArgs a) {
  const int b = blockIdx.x, hh = blockIdx.y;
  extern __shared__ float qn[];
  const T* qnope = reinterpret_cast<const T*>(a.q_nope) + ((int64_t)b * a.h + hh) * a.dn;
  for (int d = threadIdx.x; d < a.dn; d += blockDim.x) qn[d] = Elem<T>::load(qnope + d);
  __syncthreads();
  const T* W = reinterpret_cast<const T*>(a.w_kv_b) + (int64_t)hh * (a.dn + a.dv) * a.r;
  T* out = reinterpret_cast<T*>(a.q_lat) + ((int64_t)b * a.h + hh) * (a.r + a.dr);
  for (int c = threadIdx.x; c < a.r; c += blockDim.x) {
    float s = 0.f;
    for (int d = 0; d < a.dn; ++d) s = fmaf(qn[d], Elem<T>::load(W + (int64_t)d * a.r + c), s);
    Elem<T>::store(out + c, s);
  }
  const T* qpe = reinterpret_cast<const T*>(a.q_pe) + ((int64_t)b * a.h + hh) * a.dr;
  for (int c = threadIdx.x; c < a.dr; c += blockDim.x) out[a.r + c] = qpe[c];
}

__device__ __forceinline__ int ctx_of(const DecodeArgs& a, int b, int64_t* start) {
  const int64_t s = a.cu_ctx[b], e = a.cu_ctx[b + 1];
  int64_t n = e - s;
  if (n < 1 || n > a.max_ctx) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusBadCtx);
    n = n < 1 ? 0 : a.max_ctx;
  }
  *start = s;
  return (int)n;
}

// D2: one block per (b, h, split).  Scores by one warp per token.
template <typename T>
__global__ void split_kernel(DecodeArgs a) {
  const int b = blockIdx.x, hh = blockIdx.y, sp = blockIdx.z;
  int64_t start;
  const int n = ctx_of(a, b, &start);
  const int t0 = sp * a.split_tokens;
  const int64_t part = ((int64_t)b * a.max_splits + sp) * a.h + hh;
  if (t0 >= n) {   // empty split: neutral partial
    for (int c = threadIdx.x; c < a.r; c += blockDim.x) a.part_o[part * a.r + c] = 0.f;
    if (threadIdx.x == 0) a.part_lse[part] = -INFINITY;
    return;
  }
  const int t1 = min(n, t0 + a.split_tokens);
  const int w = a.r + a.dr;
  extern __shared__ float sm[];
  float* q = sm;              // [w]
  float* s = q + w;           // [split_tokens]
  __shared__ float red[32];
  const T* ql = reinterpret_cast<const T*>(a.q_lat) + ((int64_t)b * a.h + hh) * w;
  for (int c = threadIdx.x; c < w; c += blockDim.x) q[c] = Elem<T>::load(ql + c);
  __syncthreads();
  const T* C = reinterpret_cast<const T*>(a.cache) + start * w;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  for (int t = t0 + warp; t < t1; t += nw) {
    float acc = 0.f;
    for (int c = lane; c < w; c += 32) acc = fmaf(q[c], Elem<T>::load(C + (int64_t)t * w + c), acc);
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s[t - t0] = acc * a.scale;
  }
  __syncthreads();
  float mx = -FLT_MAX;
  for (int t = threadIdx.x; t < t1 - t0; t += blockDim.x) mx = fmaxf(mx, s[t]);
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = -FLT_MAX;
  for (int i = 0; i < nw; ++i) mx = fmaxf(mx, red[i]);
  __syncthreads();
  float l = 0.f;
  for (int t = threadIdx.x; t < t1 - t0; t += blockDim.x) {
    const float p = __expf(s[t] - mx);
    s[t] = p;
    l += p;
  }
  for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  l = 0.f;
  for (int i = 0; i < nw; ++i) l += red[i];
  for (int c = threadIdx.x; c < a.r; c += blockDim.x) {
    float o = 0.f;
    for (int t = t0; t < t1; ++t) o = fmaf(s[t - t0], Elem<T>::load(C + (int64_t)t * w + c), o);
    a.part_o[part * a.r + c] = o / l;
  }
  if (threadIdx.x == 0) a.part_lse[part] = mx + logf(l);
}

// D3: merge the splits of (b, h) by their log-sum-exp weights.
template <typename T>
__global__ void combine_kernel(DecodeArgs a) {
  const int b = blockIdx.x, hh = blockIdx.y;
  float mx = -INFINITY;
  for (int sp = 0; sp < a.max_splits; ++sp)
    mx = fmaxf(mx, a.part_lse[((int64_t)b * a.max_splits + sp) * a.h + hh]);
  float den = 0.f;
  for (int sp = 0; sp < a.max_splits; ++sp) {
    const float l = a.part_lse[((int64_t)b * a.max_splits + sp) * a.h + hh];
    den += l == -INFINITY ? 0.f : __expf(l - mx);
  }
  T* out = reinterpret_cast<T*>(a.o_lat) + ((int64_t)b * a.h + hh) * a.r;
  for (int c = threadIdx.x; c < a.r; c += blockDim.x) {
    float o = 0.f;
    for (int sp = 0; sp < a.max_splits; ++sp) {
      const int64_t part = ((int64_t)b * a.max_splits + sp) * a.h + hh;
      const float l = a.part_lse[part];
      if (l != -INFINITY) o = fmaf(__expf(l - mx), a.part_o[part * a.r + c], o);
    }
    Elem<T>::store(out + c, den > 0.f ? o / den : 0.f);
  }
}

// D4: o[b,h,v] = W_UV[h][v] . o_lat[b,h]; one warp per output element.
template <typename T>
__global__ void vup_kernel(DecodeArgs a) {
  const int b = blockIdx.x, hh = blockIdx.y;
  const T* ol = reinterpret_cast<const T*>(a.o_lat) + ((int64_t)b * a.h + hh) * a.r;
  const T* W = reinterpret_cast<const T*>(a.w_kv_b) +
               ((int64_t)hh * (a.dn + a.dv) + a.dn) * a.r;
  T* o = reinterpret_cast<T*>(a.o) + ((int64_t)b * a.h + hh) * a.dv;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  for (int v = warp; v < a.dv; v += nw) {
    float acc = 0.f;
    for (int c = lane; c < a.r; c += 32)
      acc = fmaf(Elem<T>::load(W + (int64_t)v * a.r + c), Elem<T>::load(ol + c), acc);
    for (int s = 16; s; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) Elem<T>::store(o + v, acc);
  }
}

template <typename T>
cudaError_t run_decode(const DecodeArgs& a, cudaStream_t st) {
  dim3 bh(a.B, a.h);
  qlat_kernel<T><<<bh, 256, a.dn * sizeof(float), st>>>(a);
  stage_event(1, st);
  size_t smem = sizeof(float) * (a.r + a.dr + a.split_tokens);
  cudaError_t err = cudaFuncSetAttribute(split_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  split_kernel<T><<<dim3(a.B, a.h, a.max_splits), 256, smem, st>>>(a);
  stage_event(2, st);
  combine_kernel<T><<<bh, 256, 0, st>>>(a);
  stage_event(3, st);
  vup_kernel<T><<<bh, 256, 0, st>>>(a);
  count_launches(4);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_latent_finalize(int dtype, const void* ckv, const float* ssq_kv,
                                   int ssq_parts, int N, int r_kv, int dr, float eps, void* cache,
                                   cudaStream_t st, int T, int dst_T, int dst_off) {
  const int64_t total = (int64_t)N * (r_kv + dr);
  const unsigned blocks = (unsigned)((total + 255) / 256);
  count_launches();
  if (dtype == MLA_F32)
    latent_finalize_kernel<float><<<blocks, 256, 0, st>>>(
        (const float*)ckv, ssq_kv, ssq_parts, N, r_kv, dr, eps, (float*)cache, T, dst_T,
        dst_off);
  else
    latent_finalize_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        (const __nv_bfloat16*)ckv, ssq_kv, ssq_parts, N, r_kv, dr, eps, (__nv_bfloat16*)cache,
        T, dst_T, dst_off);
  return cudaGetLastError();
}

// The fp32 configuration's decode; bf16 runs on the tensor-core kernels.
cudaError_t launch_decode_simt(int dtype, const DecodeArgs& a, cudaStream_t st) {
  return dtype == MLA_F32 ? run_decode<float>(a, st) : cudaErrorNotSupported;
}

}  // namespace mla
