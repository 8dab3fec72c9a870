// Host side of the C ABI: argument validation, workspace layout and the
// launch sequence of each entry point.  No allocation, no synchronisation
// (except mla_check_device_status).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <string>

#include "internal.h"
#include "tc.h"

namespace {

thread_local std::string g_detail;
thread_local cudaEvent_t g_events[8];
thread_local int g_n_events = 0;
std::atomic<int64_t> g_launches{0};

mla_status fail(mla_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
mla_status fail(mla_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_detail = buf;
  return s;
}

mla_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

double yarn_m(double s, double a) { return s <= 1.0 ? 1.0 : 0.1 * a * std::log(s) + 1.0; }

// Softmax scale of the CSDN DeepseekV3Attention __init__ (and Megatron's
// mscale*mscale/sqrt(q_head_dim)); Kimi uses the plain q_head_dim^-0.5.
double softmax_scale(const mla_config& c) {
  if (c.softmax_scale > 0.0) return c.softmax_scale;
  double s = 1.0 / std::sqrt((double)(c.qk_nope_head_dim + c.qk_rope_head_dim));
  if (c.rope_type == MLA_ROPE_YARN && c.rope_mscale_all_dim != 0.0) {
    const double m = yarn_m(c.rope_factor, c.rope_mscale_all_dim);
    s *= m * m;
  }
  return s;
}

int elem_size(const mla_config& c) { return c.dtype == MLA_F32 ? 4 : 2; }

mla_status check_config(const mla_config* c) {
  if (!c) return fail(MLA_ERR_NULL, "cfg is NULL");
  if (c->dtype != MLA_F32 && c->dtype != MLA_BF16)
    return fail(MLA_ERR_DTYPE, "cfg->dtype=%d is not MLA_F32 or MLA_BF16", c->dtype);
  if (c->rope_interleave != 0 && c->rope_interleave != 1)
    return fail(MLA_ERR_SHAPE, "rope_interleave=%d is not 0 or 1", c->rope_interleave);
  const int lim = 1 << 20;
  if (c->hidden_size < 1 || c->hidden_size > lim) return fail(MLA_ERR_SHAPE, "hidden_size=%d", c->hidden_size);
  if (c->num_heads < 1 || c->num_heads > 4096) return fail(MLA_ERR_SHAPE, "num_heads=%d", c->num_heads);
  if (c->q_lora_rank < 0 || c->q_lora_rank > lim) return fail(MLA_ERR_SHAPE, "q_lora_rank=%d", c->q_lora_rank);
  if (c->kv_lora_rank < 1 || c->kv_lora_rank > lim) return fail(MLA_ERR_SHAPE, "kv_lora_rank=%d", c->kv_lora_rank);
  if (c->qk_nope_head_dim < 1 || c->qk_nope_head_dim > 1024)
    return fail(MLA_ERR_SHAPE, "qk_nope_head_dim=%d", c->qk_nope_head_dim);
  if (c->qk_rope_head_dim < 2 || c->qk_rope_head_dim > 1024 || (c->qk_rope_head_dim & 1))
    return fail(MLA_ERR_SHAPE, "qk_rope_head_dim=%d must be even and >= 2", c->qk_rope_head_dim);
  if (c->v_head_dim < 1 || c->v_head_dim > 1024) return fail(MLA_ERR_SHAPE, "v_head_dim=%d", c->v_head_dim);
  if (c->rope_type < MLA_ROPE_NONE || c->rope_type > MLA_ROPE_YARN)
    return fail(MLA_ERR_SHAPE, "rope_type=%d", c->rope_type);
  if (c->rope_type != MLA_ROPE_NONE && !(c->rope_theta > 1.0))
    return fail(MLA_ERR_SHAPE, "rope_theta=%g must be > 1", c->rope_theta);
  if (c->rope_type == MLA_ROPE_YARN) {
    if (!(c->rope_factor > 0.0)) return fail(MLA_ERR_SHAPE, "rope_factor=%g", c->rope_factor);
    if (c->original_max_position_embeddings < 1)
      return fail(MLA_ERR_SHAPE, "original_max_position_embeddings=%d", c->original_max_position_embeddings);
    if (!(c->beta_fast > 0.0) || !(c->beta_slow > 0.0))
      return fail(MLA_ERR_SHAPE, "beta_fast=%g beta_slow=%g", c->beta_fast, c->beta_slow);
  }
  if (!(c->rms_eps >= 0.0)) return fail(MLA_ERR_SHAPE, "rms_eps=%g", c->rms_eps);
  return MLA_OK;
}

// The CUDA-core GEMM keeps each rope pair inside one 64-column tile.
bool rope_fits_simt_tiles(int period, int start, int dr, int count) {
  for (int i = 0; i < count; ++i) {
    const int p0 = i * period + start;
    if ((p0 % 64) + dr > 64) return false;
  }
  return true;
}

struct PrefillPlan {
  mla_prefill_layout L;
  int N;
};

// Prefill workspace for B sequences of T new tokens after T_past cached ones
// (T_past = 0: plain prefill).  Buffers over the new tokens are N = B*T rows;
// with a cache, the full latent rows and kv cover B*(T_past + T) rows.
void prefill_layout(const mla_config& c, int B, int T, int T_past, mla_prefill_layout* L,
                    bool packed = false) {
  const int64_t N = (int64_t)B * T, Na = (int64_t)B * (T + T_past), es = elem_size(c);
  const int dq = c.qk_nope_head_dim + c.qk_rope_head_dim;
  const int w = c.kv_lora_rank + c.qk_rope_head_dim;
  int64_t off = 0;
  auto take = [&](int64_t bytes) { int64_t o = off; off = align256(off + bytes); return o; };
  L->status = take(256);
  // RMS statistics: one partial sum per 64-column tile (the narrowest
  // producer tile) and row.
  L->ssq_q = c.q_lora_rank > 0 ? take(N * 4 * ((c.q_lora_rank + 63) / 64)) : -1;
  L->ssq_kv = take(N * 4 * ((c.kv_lora_rank + 63) / 64));
  L->q_a = c.q_lora_rank > 0 ? take(N * c.q_lora_rank * es) : -1;
  L->ckv = take(N * w * es);
  L->latent = T_past > 0 ? take(Na * w * es) : -1;
  L->q = take(N * c.num_heads * dq * es);
  L->kv = take(Na * c.num_heads * (c.qk_nope_head_dim + c.v_head_dim) * es);
  L->attn = take(N * c.num_heads * c.v_head_dim * es);
  L->pos = packed ? take(N * 4) : -1;
  L->total_bytes = off;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  return n;
}

// Decode partitions.  Tensor cores: one CTA pair per two SMs, each taking an
// equal slice (at least tc_decode_min_slice() tokens) of all sequences'
// tokens; a sequence that crosses a slice boundary leaves one partial per
// slice in one of 2 slots per pair (split_tokens = the shortest slice,
// max_splits = the slot count).  SIMT: 1024-token splits of every sequence
// (max_splits per sequence).
// `units` > 0 asks for that many SM pairs (tensor cores) instead of one per
// two SMs of the current device.
void decode_layout(const mla_config& c, int B, int max_ctx, mla_decode_layout* L, int units = 0) {
  const int64_t es = elem_size(c);
  int64_t parts;
  if (mla::tc_decode_supported(c)) {
    L->split_tokens = mla::tc_decode_min_slice();
    L->max_splits = 2 * (units > 0 ? units : std::max(1, device_sms() / 2));
    parts = L->max_splits;
  } else {
    L->split_tokens = 1024;
    L->max_splits = (max_ctx + 1023) / 1024;
    parts = (int64_t)B * L->max_splits;
  }
  int64_t off = 0;
  auto take = [&](int64_t bytes) { int64_t o = off; off = align256(off + bytes); return o; };
  L->status = take(256);
  L->q_lat = take((int64_t)B * c.num_heads * (c.kv_lora_rank + c.qk_rope_head_dim) * es);
  L->part_o = take(parts * c.num_heads * c.kv_lora_rank * 4);
  L->part_lse = take(parts * c.num_heads * 4);
  L->o_lat = take((int64_t)B * c.num_heads * c.kv_lora_rank * es);
  L->o = take((int64_t)B * c.num_heads * c.v_head_dim * es);
  L->total_bytes = off;
}

}  // namespace

namespace mla {
size_t decode_min_workspace(const mla_config& c, int B, int max_ctx) {
  mla_decode_layout L;
  decode_layout(c, B, max_ctx, &L, mla::tc_decode_supported(c) ? 1 : 0);
  return (size_t)L.total_bytes;
}
}  // namespace mla

namespace {

char* at(void* ws, int64_t off) { return off < 0 ? nullptr : static_cast<char*>(ws) + off; }

}  // namespace

namespace {
// Packed (THD) sequences: cu_seqlens[0..n_seq] on the device, the longest
// sequence max_len.
struct Packed {
  const int32_t* cu;
  int n_seq, max_len;
};

// Prefill of B sequences of T new tokens after T_past tokens whose latent
// rows are in past_cache ([B, T_past, r_kv + rope]; T_past = 0: plain).
// Packed: B = 1, T = all packed rows, T_past = 0 and `pk` describes them.
mla_status run_prefill(const mla_config* cfg, const mla_weights* w, const void* x, int32_t B,
                       int32_t T, const void* past_cache, int32_t T_past,
                       const float* rope_cos, const float* rope_sin, void* out,
                       void* latent_cache_out, void* workspace, size_t workspace_bytes,
                       void* stream, const Packed* pk = nullptr) {
  mla_status s = check_config(cfg);
  if (s != MLA_OK) return s;
  const mla_config& c = *cfg;
  if (!w) return fail(MLA_ERR_NULL, "weights is NULL");
  if (!x || !out || !workspace) return fail(MLA_ERR_NULL, "x/out/workspace is NULL");
  const bool lora = c.q_lora_rank > 0;
  if (lora && (!w->w_q_a || !w->w_q_b)) return fail(MLA_ERR_NULL, "w_q_a/w_q_b is NULL (q_lora_rank > 0)");
  if (!lora && !w->w_q) return fail(MLA_ERR_NULL, "w_q is NULL (q_lora_rank == 0)");
  if (!w->w_kv_a || !w->w_kv_b || !w->w_o) return fail(MLA_ERR_NULL, "w_kv_a/w_kv_b/w_o is NULL");
  const bool rope = c.rope_type != MLA_ROPE_NONE;
  if (rope && (!rope_cos || !rope_sin)) return fail(MLA_ERR_NULL, "rope_cos/rope_sin is NULL");
  if (B < 1 || T < 1 || T_past < 0 || (int64_t)B * ((int64_t)T + T_past) >= (1ll << 31))
    return fail(MLA_ERR_SHAPE, "B=%d T=%d T_past=%d", B, T, T_past);
  const void* ptrs[] = {x, out, latent_cache_out, w->w_q_a, w->g_q_a, w->w_q_b, w->w_q,
                        w->w_kv_a, w->g_kv_a, w->w_kv_b, w->w_o, rope_cos, rope_sin, past_cache};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(MLA_ERR_ALIGN, "pointer %p is not 16-byte aligned", p);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(MLA_ERR_ALIGN, "workspace is not 256-byte aligned");
  mla_prefill_layout L;
  prefill_layout(c, B, T, T_past, &L, pk != nullptr);
  if ((int64_t)workspace_bytes < L.total_bytes)
    return fail(MLA_ERR_WORKSPACE, "workspace %zu < %lld bytes", workspace_bytes,
                (long long)L.total_bytes);

  const int N = B * T;
  const int Ta = T + T_past;                    // keys per sequence
  const int h = c.num_heads, dn = c.qk_nope_head_dim, dr = c.qk_rope_head_dim, dv = c.v_head_dim;
  const int dq = dn + dr, r_kv = c.kv_lora_rank, H = c.hidden_size;
  const float eps = (float)c.rms_eps;
  const bool tc_attn = mla::tc_attention_supported(c);
  // bf16 runs on the tensor-core kernels only
  if (c.dtype == MLA_BF16 && (!tc_attn || H % 8 || c.q_lora_rank % 8))
    return fail(MLA_ERR_UNSUPPORTED,
                "bf16 prefill takes qk_nope_head_dim 128, qk_rope_head_dim 64, v_head_dim 128, "
                "kv_lora_rank a multiple of 64, hidden_size and q_lora_rank multiples of 8 "
                "(got %d/%d/%d, %d, %d, %d)", dn, dr, dv, r_kv, H, c.q_lora_rank);
  if (rope && (!rope_fits_simt_tiles(dq, dn, dr, h) ||
               !rope_fits_simt_tiles(r_kv + dr, r_kv, dr, 1)) && c.dtype == MLA_F32)
    return fail(MLA_ERR_UNSUPPORTED, "rope columns straddle a 64-column tile");
  if (!tc_attn &&
      sizeof(float) * (16 * dq + 32 * dq + 32 * dv + 16 * 32 + 16 * dv + 48) > 227 * 1024)
    return fail(MLA_ERR_UNSUPPORTED, "head dims too large for the CUDA-core attention");
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = static_cast<char*>(workspace);
  float* ssq_q = (float*)at(ws, L.ssq_q);
  float* ssq_kv = (float*)at(ws, L.ssq_kv);
  void* q_a = at(ws, L.q_a);
  void* ckv = at(ws, L.ckv);
  void* q = at(ws, L.q);
  void* kv = at(ws, L.kv);
  void* attn = at(ws, L.attn);
  void* latent = at(ws, L.latent);
  uint32_t* status = (uint32_t*)at(ws, L.status);
  int32_t* pos = (int32_t*)at(ws, L.pos);

  // The status word starts at zero; every other buffer is fully written.
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  mla::stage_event(0, st);
  if (pk) {       // per-row positions of the packed sequences (RoPE)
    e = mla::launch_packed_positions(pk->cu, pk->n_seq, N, pk->max_len, pos, status, st);
    if (e != cudaSuccess) return cuda_fail(e, "packed positions");
  }

  // S1: fused down-projection [x W_qa^T | x W_kva^T]; epilogue: RMS row
  // statistics, gains, RoPE on k_pe.
  mla::GemmArgs g;
  g.A = x; g.lda = H; g.M = N; g.K = H;
  int si = 0;
  if (lora) {
    mla::EpiSeg& e0 = g.seg[si];
    g.Bm[si] = w->w_q_a; g.ldb[si] = H;
    e0.out = q_a; e0.ldo = c.q_lora_rank; e0.ncols = c.q_lora_rank;
    e0.gamma = w->g_q_a; e0.norm_cols = c.q_lora_rank; e0.ssq_out = ssq_q; e0.ssq_ld = N;
    ++si;
  }
  {
    mla::EpiSeg& e1 = g.seg[si];
    g.Bm[si] = w->w_kv_a; g.ldb[si] = H;
    e1.out = ckv; e1.ldo = r_kv + dr; e1.ncols = r_kv + dr;
    e1.gamma = w->g_kv_a; e1.norm_cols = r_kv; e1.ssq_out = ssq_kv; e1.ssq_ld = N;
    if (rope) {
      e1.cos = rope_cos; e1.sin = rope_sin; e1.rope_period = r_kv + dr;
      e1.rope_start = r_kv; e1.rope_dim = dr; e1.T = T; e1.pos_offset = T_past; e1.pos = pos;
      e1.rope_interleave = c.rope_interleave != 0;
    }
    ++si;
  }
  g.nseg = si;
  // Each projection runs on the tensor-core GEMM when it takes the shape;
  // the column tile of the down-projection fixes the RMS partial count.
  auto run_gemm = [&](const mla::GemmArgs& ga) {
    if (mla::tc_gemm_supported(ga, c.dtype)) return mla::tc_gemm(ga, st, status);
    if (c.dtype != MLA_F32) return cudaErrorNotSupported;   // excluded above
    if (ga.seg[0].cos && !rope_fits_simt_tiles(ga.seg[0].rope_period, ga.seg[0].rope_start,
                                               ga.seg[0].rope_dim,
                                               ga.seg[0].ncols / ga.seg[0].rope_period))
      return cudaErrorNotSupported;
    return mla::launch_gemm_simt(c.dtype, ga, st);
  };
  const int tile_n = mla::tc_gemm_supported(g, c.dtype) ? mla::kTcTileN : mla::kSimtTileN;
  e = run_gemm(g);
  if (e != cudaSuccess) return cuda_fail(e, "down-projection");
  mla::stage_event(1, st);

  // S2+S3: q up-projection (RMS row scale) or direct q_proj; RoPE on q_pe.
  mla::GemmArgs gq;
  gq.M = N; gq.nseg = 1;
  mla::EpiSeg& eq = gq.seg[0];
  if (lora) {
    gq.A = q_a; gq.lda = c.q_lora_rank; gq.K = c.q_lora_rank;
    gq.Bm[0] = w->w_q_b; gq.ldb[0] = c.q_lora_rank;
    eq.ssq_in = ssq_q; eq.rs_inv_dim = 1.0f / c.q_lora_rank; eq.eps = eps;
    eq.ssq_parts = (c.q_lora_rank + tile_n - 1) / tile_n; eq.ssq_ld = N;
  } else {
    gq.A = x; gq.lda = H; gq.K = H;
    gq.Bm[0] = w->w_q; gq.ldb[0] = H;
  }
  eq.out = q; eq.ldo = (int64_t)h * dq; eq.ncols = h * dq;
  if (rope) {
    eq.cos = rope_cos; eq.sin = rope_sin; eq.rope_period = dq; eq.rope_start = dn;
    eq.rope_dim = dr; eq.T = T; eq.pos_offset = T_past; eq.pos = pos;
    eq.rope_interleave = c.rope_interleave != 0;
  }
  e = run_gemm(gq);
  if (e != cudaSuccess) return cuda_fail(e, "q projection");
  mla::stage_event(2, st);

  // S2+S4: kv up-projection.  Plain prefill: straight from the gain-scaled
  // latent with the kv RMS row scale in the epilogue.  With a cache: over the
  // full latent rows [past | RMSNorm(c_new) | k_pe] (the uncompress step),
  // which are normalised already.
  const void* kv_src = ckv;
  if (T_past > 0) {
    const size_t row = (size_t)(r_kv + dr) * elem_size(c);
    e = cudaMemcpy2DAsync(latent, (size_t)Ta * row, past_cache, (size_t)T_past * row,
                          (size_t)T_past * row, (size_t)B, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "latent history copy");
    e = mla::launch_latent_finalize(c.dtype, ckv, ssq_kv, (r_kv + tile_n - 1) / tile_n, N, r_kv,
                                    dr, eps, latent, st, T, Ta, T_past);
    if (e != cudaSuccess) return cuda_fail(e, "latent assembly");
    kv_src = latent;
  }
  mla::GemmArgs gk;
  gk.A = kv_src; gk.lda = r_kv + dr; gk.M = B * Ta; gk.K = r_kv; gk.nseg = 1;
  gk.Bm[0] = w->w_kv_b; gk.ldb[0] = r_kv;
  mla::EpiSeg& ek = gk.seg[0];
  ek.out = kv; ek.ldo = (int64_t)h * (dn + dv); ek.ncols = h * (dn + dv);
  if (T_past == 0) {
    ek.ssq_in = ssq_kv; ek.rs_inv_dim = 1.0f / r_kv; ek.eps = eps;
    ek.ssq_parts = (r_kv + tile_n - 1) / tile_n; ek.ssq_ld = N;
  }
  e = run_gemm(gk);
  if (e != cudaSuccess) return cuda_fail(e, "kv up-projection");
  mla::stage_event(3, st);

  // S7: causal attention (new queries at positions T_past .. T_past + T - 1).
  mla::AttnArgs aa{q, kv, kv_src, attn, B, T, h, dn, dr, dv, r_kv, (float)softmax_scale(c), status};
  aa.Tk = Ta;
  aa.q_off = T_past;
  if (pk) {       // causal within each packed sequence
    aa.B = pk->n_seq;
    aa.T = aa.Tk = pk->max_len;
    aa.cu_seqlens = pk->cu;
    aa.total = N;
  }
  if ((int64_t)aa.B * h > 65535) return fail(MLA_ERR_UNSUPPORTED, "sequences x heads > 65535");
  e = tc_attn ? mla::tc_attention(aa, st) : mla::launch_attn_simt(c.dtype, aa, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention");
  mla::stage_event(4, st);

  // S8: o_proj.
  mla::GemmArgs go;
  go.A = attn; go.lda = (int64_t)h * dv; go.M = N; go.K = h * dv; go.nseg = 1;
  go.Bm[0] = w->w_o; go.ldb[0] = (int64_t)h * dv;
  go.seg[0].out = out; go.seg[0].ldo = H; go.seg[0].ncols = H;
  e = run_gemm(go);
  if (e != cudaSuccess) return cuda_fail(e, "o_proj");
  mla::stage_event(5, st);

  if (latent_cache_out) {
    e = mla::launch_latent_finalize(c.dtype, ckv, ssq_kv, (r_kv + tile_n - 1) / tile_n, N, r_kv,
                                    dr, eps, latent_cache_out, st);
    if (e != cudaSuccess) return cuda_fail(e, "latent cache");
  }
  g_detail.clear();
  return MLA_OK;
}


}  // namespace

namespace mla {
void set_error_detail(const char* msg) { g_detail = msg; }
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
void stage_event(int i, cudaStream_t st) {
  if (i < g_n_events && g_events[i]) cudaEventRecord(g_events[i], st);
}
}  // namespace mla

extern "C" {

mla_status mla_set_stage_events(void* const* events, int32_t n) {
  if (n < 0 || n > 8) return fail(MLA_ERR_SHAPE, "n=%d outside [0, 8]", n);
  if (!events) n = 0;
  for (int i = 0; i < 8; ++i) g_events[i] = i < n ? (cudaEvent_t)events[i] : nullptr;
  g_n_events = n;
  return MLA_OK;
}

int64_t mla_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }


int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_NULL: return "MLA_ERR_NULL";
    case MLA_ERR_SHAPE: return "MLA_ERR_SHAPE";
    case MLA_ERR_ALIGN: return "MLA_ERR_ALIGN";
    case MLA_ERR_DTYPE: return "MLA_ERR_DTYPE";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
  }
  return "MLA_ERR_<unknown>";
}

const char* mla_last_error_detail(void) { return g_detail.c_str(); }

mla_status mla_build_rope_tables(const mla_config* cfg, int32_t max_pos, float* cos_out,
                                 float* sin_out, void* stream) {
  mla_status s = check_config(cfg);
  if (s != MLA_OK) return s;
  if (!cos_out || !sin_out) return fail(MLA_ERR_NULL, "cos_out/sin_out is NULL");
  if (!aligned16(cos_out) || !aligned16(sin_out)) return fail(MLA_ERR_ALIGN, "cos_out/sin_out");
  if (max_pos < 1 || max_pos > (1 << 24)) return fail(MLA_ERR_SHAPE, "max_pos=%d", max_pos);
  cudaError_t e = mla::launch_rope_tables(*cfg, max_pos, cos_out, sin_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "rope tables");
  g_detail.clear();
  return MLA_OK;
}

size_t mla_prefill_workspace_size(const mla_config* cfg, int32_t B, int32_t T,
                                  mla_prefill_layout* layout) {
  if (check_config(cfg) != MLA_OK || B < 1 || T < 1 || (int64_t)B * T >= (1ll << 31)) return 0;
  mla_prefill_layout L;
  prefill_layout(*cfg, B, T, 0, &L);
  if (layout) *layout = L;
  return (size_t)L.total_bytes;
}

mla_status mla_prefill_forward(const mla_config* cfg, const mla_weights* w, const void* x,
                               int32_t B, int32_t T, const float* rope_cos,
                               const float* rope_sin, void* out, void* latent_cache_out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return run_prefill(cfg, w, x, B, T, nullptr, 0, rope_cos, rope_sin, out, latent_cache_out,
                     workspace, workspace_bytes, stream);
}

size_t mla_prefill_chunked_workspace_size(const mla_config* cfg, int32_t B, int32_t T_new,
                                          int32_t T_past, mla_prefill_layout* layout) {
  if (check_config(cfg) != MLA_OK || B < 1 || T_new < 1 || T_past < 0 ||
      (int64_t)B * ((int64_t)T_new + T_past) >= (1ll << 31))
    return 0;
  mla_prefill_layout L;
  prefill_layout(*cfg, B, T_new, T_past, &L);
  if (layout) *layout = L;
  return (size_t)L.total_bytes;
}

mla_status mla_prefill_chunked(const mla_config* cfg, const mla_weights* w, const void* x,
                               int32_t B, int32_t T_new, const void* past_cache,
                               int32_t T_past, const float* rope_cos, const float* rope_sin,
                               void* out, void* latent_cache_out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (T_past < 0) return fail(MLA_ERR_SHAPE, "T_past=%d", T_past);
  if (T_past > 0 && !past_cache) return fail(MLA_ERR_NULL, "past_cache is NULL (T_past > 0)");
  return run_prefill(cfg, w, x, B, T_new, past_cache, T_past, rope_cos, rope_sin, out,
                     latent_cache_out, workspace, workspace_bytes, stream);
}

size_t mla_prefill_varlen_workspace_size(const mla_config* cfg, int32_t n_seq, int32_t total,
                                         int32_t max_seqlen, mla_prefill_layout* layout) {
  if (check_config(cfg) != MLA_OK || n_seq < 1 || total < 1 || max_seqlen < 1 ||
      max_seqlen > total)
    return 0;
  mla_prefill_layout L;
  prefill_layout(*cfg, 1, total, 0, &L, true);
  if (layout) *layout = L;
  return (size_t)L.total_bytes;
}

mla_status mla_prefill_varlen(const mla_config* cfg, const mla_weights* w, const void* x,
                              const int32_t* cu_seqlens, int32_t n_seq, int32_t total,
                              int32_t max_seqlen, const float* rope_cos, const float* rope_sin,
                              void* out, void* latent_cache_out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!cu_seqlens) return fail(MLA_ERR_NULL, "cu_seqlens is NULL");
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
    return fail(MLA_ERR_ALIGN, "cu_seqlens is not 4-byte aligned");
  if (n_seq < 1 || total < 1 || max_seqlen < 1 || max_seqlen > total)
    return fail(MLA_ERR_SHAPE, "n_seq=%d total=%d max_seqlen=%d", n_seq, total, max_seqlen);
  const Packed pk{cu_seqlens, n_seq, max_seqlen};
  return run_prefill(cfg, w, x, 1, total, nullptr, 0, rope_cos, rope_sin, out, latent_cache_out,
                     workspace, workspace_bytes, stream, &pk);
}

size_t mla_decode_workspace_size(const mla_config* cfg, int32_t B, int32_t max_ctx,
                                 mla_decode_layout* layout) {
  if (check_config(cfg) != MLA_OK || B < 1 || max_ctx < 1) return 0;
  mla_decode_layout L;
  decode_layout(*cfg, B, max_ctx, &L);
  if (layout) *layout = L;
  return (size_t)L.total_bytes;
}

mla_status mla_decode_absorbed(const mla_config* cfg, const void* q_nope, const void* q_pe,
                               const void* w_kv_b, const void* latent_cache,
                               const int32_t* cu_ctx, int32_t B, int32_t max_ctx,
                               const void* w_o, void* out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  mla_status s = check_config(cfg);
  if (s != MLA_OK) return s;
  const mla_config& c = *cfg;
  if (!q_nope || !q_pe || !w_kv_b || !latent_cache || !cu_ctx || !out || !workspace)
    return fail(MLA_ERR_NULL, "a required decode pointer is NULL");
  if (B < 1 || B > (1 << 20) || max_ctx < 1) return fail(MLA_ERR_SHAPE, "B=%d max_ctx=%d", B, max_ctx);
  // bf16 runs on the tensor-core kernels only
  if (c.dtype == MLA_BF16 && (!mla::tc_decode_supported(c) || (w_o && c.hidden_size % 8)))
    return fail(MLA_ERR_UNSUPPORTED,
                "bf16 decode takes kv_lora_rank 512, qk_rope_head_dim 64, qk_nope_head_dim and "
                "v_head_dim multiples of 8, hidden_size a multiple of 8 with o_proj "
                "(got %d, %d, %d, %d, %d)", c.kv_lora_rank, c.qk_rope_head_dim,
                c.qk_nope_head_dim, c.v_head_dim, c.hidden_size);
  const void* ptrs[] = {q_nope, q_pe, w_kv_b, latent_cache, cu_ctx, w_o, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(MLA_ERR_ALIGN, "pointer %p is not 16-byte aligned", p);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(MLA_ERR_ALIGN, "workspace is not 256-byte aligned");
  mla_decode_layout L;
  decode_layout(c, B, max_ctx, &L);
  if ((int64_t)workspace_bytes < L.total_bytes && mla::tc_decode_supported(c)) {
    // a smaller workspace runs on as many SM pairs as its partial slots allow
    for (int u = L.max_splits / 2 - 1; u >= 1; --u) {
      decode_layout(c, B, max_ctx, &L, u);
      if ((int64_t)workspace_bytes >= L.total_bytes) break;
    }
  }
  if ((int64_t)workspace_bytes < L.total_bytes)
    return fail(MLA_ERR_WORKSPACE, "workspace %zu < %lld bytes", workspace_bytes,
                (long long)L.total_bytes);
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = static_cast<char*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  mla::stage_event(0, st);
  mla::DecodeArgs a{};
  a.q_nope = q_nope; a.q_pe = q_pe; a.w_kv_b = w_kv_b; a.cache = latent_cache; a.cu_ctx = cu_ctx;
  a.B = B; a.max_ctx = max_ctx; a.h = c.num_heads; a.dn = c.qk_nope_head_dim;
  a.dr = c.qk_rope_head_dim; a.dv = c.v_head_dim; a.r = c.kv_lora_rank;
  a.scale = (float)softmax_scale(c);
  a.split_tokens = L.split_tokens; a.max_splits = L.max_splits;
  a.n_units = L.max_splits / 2; a.min_len = L.split_tokens;
  a.q_lat = at(ws, L.q_lat); a.part_o = (float*)at(ws, L.part_o);
  a.part_lse = (float*)at(ws, L.part_lse); a.o_lat = at(ws, L.o_lat);
  a.o = w_o ? at(ws, L.o) : out;
  a.status = (uint32_t*)at(ws, L.status);
  e = mla::tc_decode_supported(c) ? mla::tc_decode(a, st) : mla::launch_decode_simt(c.dtype, a, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode");
  mla::stage_event(4, st);
  if (w_o) {
    mla::GemmArgs go;
    go.A = a.o; go.lda = (int64_t)a.h * a.dv; go.M = B; go.K = a.h * a.dv; go.nseg = 1;
    go.Bm[0] = w_o; go.ldb[0] = (int64_t)a.h * a.dv;
    go.seg[0].out = out; go.seg[0].ldo = c.hidden_size; go.seg[0].ncols = c.hidden_size;
    e = mla::tc_gemm_supported(go, c.dtype) ? mla::tc_gemm(go, st, a.status)
                                           : mla::launch_gemm_simt(c.dtype, go, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode o_proj");
  }
  mla::stage_event(5, st);
  g_detail.clear();
  return MLA_OK;
}

mla_status mla_check_device_status(void* workspace, void* stream) {
  if (!workspace) return fail(MLA_ERR_NULL, "workspace is NULL");
  uint32_t word = 0;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, 4, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word & mla::kStatusTimeout) return fail(MLA_ERR_DEVICE_TIMEOUT, "status word 0x%x", word);
  if (word & mla::kStatusBadCtx) return fail(MLA_ERR_SHAPE, "cu_ctx / cu_seqlens out of range (0x%x)", word);
  g_detail.clear();
  return MLA_OK;
}

}  // extern "C"
