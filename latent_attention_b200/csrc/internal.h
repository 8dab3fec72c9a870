// Internal declarations shared by the host API and the kernel launchers.
#pragma once

#include <cstdint>
#include <atomic>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "mla.h"

namespace mla {

// Device status word bits (first 4 bytes of every workspace).
enum : uint32_t {
  kStatusTimeout = 1u << 0,   // a bounded wait ran out
  kStatusBadCtx = 1u << 1,    // a cu_ctx / cu_seqlens length outside its bounds
};

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
  }
};

// One column segment of a GEMM output and the epilogue applied to it.
// Order of operations on an fp32 accumulator value v of row m, local col n:
//   ssq_out[tile * ssq_ld + m] = sum v^2 over the tile's cols < norm_cols
//                                   (pre-gain partial, one per column tile)
//   v *= rsqrt(sum_p ssq_in[p * ssq_ld + m] * rs_inv_dim + eps)   if ssq_in
//                                   (RMS row scale; partials summed in order)
//   RoPE on cols with (n % rope_period) in [rope_start, rope_start+rope_dim)
//        position = m % T + pos_offset, pairs (i, i + rope_dim/2)  if cos
//   v *= gamma[n]                   for n < norm_cols           if gamma
//   out[m * ldo + n] = v (rounded to the element type)
struct EpiSeg {
  void* out = nullptr;
  int64_t ldo = 0;
  int ncols = 0;
  const void* gamma = nullptr;
  int norm_cols = 0;
  float* ssq_out = nullptr;
  const float* ssq_in = nullptr;
  int ssq_parts = 0;        // partial count to sum for ssq_in
  int64_t ssq_ld = 0;       // row count of the partial buffer (M)
  float rs_inv_dim = 0.f;
  float eps = 0.f;
  const float* cos = nullptr;
  const float* sin = nullptr;
  int rope_period = 0, rope_start = 0, rope_dim = 0, T = 1;
  int pos_offset = 0;       // RoPE position = (row % T) + pos_offset
  const int32_t* pos = nullptr;  // or, when set, the position of every row
  bool rope_interleave = false;  // rope columns arrive as pairs (2i, 2i+1)
};

// C = A B^T with A [M, K] (row stride lda) and the output columns split in up
// to two segments: columns of segment s come from rows of Bs [ncols_s, K].
//
// Batched products (one per attention head in decode): batch i reads
// A + i*sA, B + i*sB and writes out + i*sOut (elements).  a_batch_inner marks
// an A whose batch stride is smaller than its row stride ([rows, batch, K]
// storage).  b_mn marks a B stored [K, N] (N contiguous, row stride ldb)
// instead of nn.Linear's [N, K].
struct GemmArgs {
  const void* A = nullptr;
  int64_t lda = 0;
  const void* Bm[2] = {nullptr, nullptr};
  int64_t ldb[2] = {0, 0};
  int M = 0, K = 0;
  int nseg = 1;
  EpiSeg seg[2];
  int batch = 1;
  int64_t sA = 0, sB = 0, sOut = 0;
  bool a_batch_inner = false;
  bool b_mn = false;
};

// Causal attention of B sequences: T queries per sequence at positions
// q_off .. q_off + T - 1 against Tk keys per sequence at positions 0 .. Tk - 1
// (key j visible to query i iff j <= q_off + i).  Plain prefill: Tk = T,
// q_off = 0; prefill against a cache of T_past tokens: Tk = T_past + T,
// q_off = T_past.
struct AttnArgs {
  const void* q;        // [B*T, h, dq]
  const void* kv;       // [B*Tk, h, dn+dv]
  const void* ckv;      // [B*Tk, r_kv+dr]  (k_pe at column r_kv)
  void* o;              // [B*T, h, dv]
  int B, T, h, dn, dr, dv, r_kv;
  float scale;
  uint32_t* status;
  int Tk = 0, q_off = 0;
  // Packed (THD) prefill: sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1
  // of `total` rows; B is the sequence count and T the longest sequence.
  const int32_t* cu_seqlens = nullptr;
  int total = 0;
};

struct DecodeArgs {
  const void* q_nope;   // [B, h, dn]
  const void* q_pe;     // [B, h, dr]
  const void* w_kv_b;   // [h*(dn+dv), r]
  const void* cache;    // [sum ctx, r + dr]
  const int32_t* cu_ctx;
  int B, max_ctx, h, dn, dr, dv, r;
  float scale;
  int split_tokens, max_splits;   // SIMT path: tokens per split, splits per sequence
  int n_units, min_len;           // tensor-core path: CTA pairs, shortest slice
  void* q_lat;          // [B, h, r + dr]
  float* part_o;        // SIMT [B, max_splits, h, r]; tensor cores [2 n_units, h, r]
  float* part_lse;      // SIMT [B, max_splits, h];    tensor cores [2 n_units, h]
  void* o_lat;          // [B, h, r]
  void* o;              // [B, h, dv]
  uint32_t* status;
};

// cudaFuncSetAttribute applies to the current device only: set a kernel's
// dynamic shared-memory limit once per device (devices 0..63).
inline cudaError_t set_dynamic_smem(const void* kernel, int bytes,
                                    std::atomic<uint64_t>& done_devices) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done_devices.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done_devices.fetch_or(bit, std::memory_order_release);
  return e;
}

// Launches a kernel with programmatic stream serialization: it may start
// (prologue: barriers, TMEM, descriptor prefetch) while the previous kernel
// of the stream finishes.  Only for kernels that call griddep_wait() first
// (see sm100.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch accounting and stage events (defined in api.cu).
void count_launches(int n = 1);
// Sets the text mla_last_error_detail() returns on this host thread.
void set_error_detail(const char* msg);
// Records registered stage event i (if any) on stream st.
void stage_event(int i, cudaStream_t st);

// Launchers (return the launch error).
cudaError_t launch_rope_tables(const mla_config& cfg, int max_pos, float* cos,
                               float* sin, cudaStream_t st);
cudaError_t launch_gemm_simt(int dtype, const GemmArgs& a, cudaStream_t st);
// Column tile width of the CUDA-core GEMM (RMS partial count = ceil(cols/64)).
constexpr int kSimtTileN = 64;
cudaError_t launch_attn_simt(int dtype, const AttnArgs& a, cudaStream_t st);
// Normalised latent rows [RMSNorm(c) | k_pe] from the gain-scaled latent
// buffer: source row m (of N = B*T) goes to destination row
// (m / T) * dst_T + dst_off + (m % T).
// Packed prefill: pos[m] = m - cu_seqlens[b(m)] for the `total` packed rows;
// malformed cu_seqlens raise kStatusBadCtx (positions stay in [0, max_len)).
cudaError_t launch_packed_positions(const int32_t* cu_seqlens, int n_seq, int total, int max_len,
                                    int32_t* pos, uint32_t* status, cudaStream_t st);

cudaError_t launch_latent_finalize(int dtype, const void* ckv,
                                   const float* ssq_kv, int ssq_parts, int N, int r_kv,
                                   int dr, float eps, void* cache,
                                   cudaStream_t st, int T = 1, int dst_T = 1, int dst_off = 0);
cudaError_t launch_decode_simt(int dtype, const DecodeArgs& a, cudaStream_t st);
// Smallest workspace mla_decode_absorbed runs with (one SM pair on tensor cores).
size_t decode_min_workspace(const mla_config& c, int B, int max_ctx);

}  // namespace mla
