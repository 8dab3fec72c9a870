/*
 * mla.h -- C ABI of the B200 (sm_100a) Multi-Latent Attention library.
 *
 * The library computes the MLA forward of the DeepSeek-V3 / Kimi attention
 * layer on one GPU: prefill over whole sequences and one-token decode over a
 * compressed latent cache with the projection weights absorbed.
 *
 * Sources (page titles and sections of the reference pages):
 *   [DSV3]     CSDN walkthrough of HF DeepseekV3Attention, section
 *              "代码+流程图": __init__ (layer shapes, YaRN softmax scale) and
 *              forward (q path, kv_a split, kv_b split, RoPE on the rot parts,
 *              shared k_rot broadcast, concat, FA2 V pad/trim, o_proj).
 *   [VERL]     verl docs "kimi_vl.py — KimiVL (DeepSeek-V3 架构) 注意力适配",
 *              sections "Q 投影和 KV 压缩", "拼接最终的 Q 和 K".
 *   [MEGATRON] "Megatron-LM 多潜在注意力MLA实战指南", sections 源码架构,
 *              MLA 专属参数详解, 配置自检约束, 推理优化.
 *   [MINIMIND] MiniMind "Attention 前向传播", sections 2 (nn.Linear [out,in],
 *              x W^T), 3 (RMSNorm, rotate_half RoPE), 5 (causal mask, softmax).
 *   [KIMI]     Kimi-K3 atlas "Gated MLA › Key and value heads": mla-init,
 *              mla-forward (no rotary), rmsnorm.
 *
 * Conventions that hold for every entry point:
 *   - All tensor arguments are DEVICE pointers unless stated otherwise, dense
 *     and row-major, 16-byte aligned (MLA_ERR_ALIGN otherwise).  The caller
 *     owns every buffer; the library never allocates, frees or synchronises
 *     (except mla_check_device_status, which synchronises by design).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Inputs are only read; outputs are overwritten.
 *   - Element type of activations/weights/outputs is cfg->dtype: MLA_BF16
 *     (bf16 storage, fp32 accumulation, bf16 intermediates at HBM boundaries;
 *     tensor-core kernels only) or MLA_F32 (fp32 throughout, CUDA-core FFMA
 *     path).  RoPE tables are always fp32; cu_ctx is int32.
 *   - MLA_BF16 shapes the tensor-core kernels take: prefill needs
 *     qk_nope_head_dim 128, qk_rope_head_dim 64, v_head_dim 128, kv_lora_rank
 *     a multiple of 64, hidden_size and q_lora_rank multiples of 8; decode
 *     needs kv_lora_rank 512, qk_rope_head_dim 64, qk_nope_head_dim and
 *     v_head_dim multiples of 8 (and hidden_size a multiple of 8 with o_proj).
 *     Any other bf16 shape returns MLA_ERR_UNSUPPORTED before any launch.
 *   - Weights use the nn.Linear layout [out_features, in_features] and the
 *     forward computes x W^T ([MINIMIND] section 2).  There are no biases:
 *     attention_bias is False in the DeepSeek-V3 and Kimi layers ([KIMI]
 *     mla-init builds every projection with bias=False).
 *   - Argument validation happens before any launch and mirrors the config
 *     self-checks of [MEGATRON] 配置自检约束: an invalid call returns an error
 *     status and enqueues nothing.  Nothing aborts or throws across the ABI.
 *     mla_last_error_detail() names the offending argument.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 4

/* Exported symbols keep default visibility even when the library is built
 * with -fvisibility=hidden. */
#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_NULL = 1,           /* a required pointer is NULL                    */
  MLA_ERR_SHAPE = 2,          /* a size is out of range or inconsistent        */
  MLA_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned              */
  MLA_ERR_DTYPE = 4,          /* cfg->dtype is not an mla_dtype                */
  MLA_ERR_WORKSPACE = 5,      /* workspace smaller than the *_workspace_size   */
  MLA_ERR_UNSUPPORTED = 6,    /* valid MLA shape the library does not implement */
  MLA_ERR_CUDA = 7,           /* a CUDA runtime call or launch failed          */
  MLA_ERR_DEVICE_TIMEOUT = 8  /* a bounded on-device wait gave up (reported by
                                 mla_check_device_status)                      */
} mla_status;

typedef enum mla_dtype { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Rotary variants: none (Kimi no-rotary MLA, [KIMI] mla-forward leaves k_pe
 * and q_pe unrotated), plain RoPE, YaRN-scaled RoPE ([MEGATRON] MLA 专属参数详解:
 * rope_type rope | yarn). */
typedef enum mla_rope_type {
  MLA_ROPE_NONE = 0,
  MLA_ROPE_PLAIN = 1,
  MLA_ROPE_YARN = 2
} mla_rope_type;

/* Layer configuration.  Field names follow [DSV3] __init__ and the YaRN
 * parameters of [MEGATRON] MLA 专属参数详解.  No field has a default: set all. */
typedef struct mla_config {
  int32_t hidden_size;
  int32_t num_heads;                /* num_attention_heads                      */
  int32_t q_lora_rank;              /* 0 means None: a direct q_proj            */
  int32_t kv_lora_rank;
  int32_t qk_nope_head_dim;
  int32_t qk_rope_head_dim;         /* even; the single shared k_pe head width  */
  int32_t v_head_dim;               /* may differ from nope+rope (handled natively) */
  int32_t rope_type;                /* mla_rope_type                            */
  double rope_theta;                /* rotary base                              */
  double rope_factor;               /* YaRN scaling factor s                    */
  double rope_mscale;               /* YaRN mscale                              */
  double rope_mscale_all_dim;       /* YaRN mscale_all_dim                      */
  double beta_fast;                 /* YaRN beta_fast                           */
  double beta_slow;                 /* YaRN beta_slow                           */
  int32_t original_max_position_embeddings; /* YaRN original context length L */
  int32_t dtype;                    /* mla_dtype                                */
  double rms_eps;                   /* RMSNorm epsilon ([KIMI] rmsnorm: 1e-6)   */
  double softmax_scale;             /* > 0: used as is; <= 0: derived:
                                       (nope+rope)^-0.5, times m(s,a)^2 under
                                       YaRN when mscale_all_dim != 0, with
                                       m(s,a) = 0.1 a ln s + 1 for s > 1
                                       ([DSV3] __init__; [MEGATRON] 源码架构) */
  int32_t rope_interleave;          /* 1: the projections emit each head's rope
                                       columns as adjacent pairs (2i, 2i+1)
                                       ("interleaved weights", [DSV3] forward);
                                       they are de-interleaved to rotate_half
                                       order [x0 x2 .. | x1 x3 ..] before RoPE,
                                       so q_pe, k_pe and the latent cache come
                                       out exactly as with the permuted weights.
                                       0: rotate_half order already. */
} mla_config;

/* Layer weights, all [out, in] row-major in cfg->dtype. */
typedef struct mla_weights {
  const void* w_q_a;   /* [q_lora_rank, hidden]            (q_lora_rank > 0)  */
  const void* g_q_a;   /* [q_lora_rank] q_a_layernorm gain; NULL = all ones    */
  const void* w_q_b;   /* [heads*(nope+rope), q_lora_rank] (q_lora_rank > 0)  */
  const void* w_q;     /* [heads*(nope+rope), hidden]      (q_lora_rank == 0) */
  const void* w_kv_a;  /* [kv_lora_rank+rope, hidden]  kv_a_proj_with_mqa     */
  const void* g_kv_a;  /* [kv_lora_rank] kv_a_layernorm gain; NULL = all ones  */
  const void* w_kv_b;  /* [heads*(nope+v), kv_lora_rank]                       */
  const void* w_o;     /* [hidden, heads*v]                                    */
} mla_weights;

/* Byte offsets of the prefill intermediates inside the workspace (for
 * inspection and tests; all rows are token-major, N = B*T):
 *   q      [N, heads, nope+rope]  queries, RoPE applied to the rope part
 *   kv     [N, heads, nope+v]     per-head k_nope | V
 *   ckv    [N, kv_lora+rope]      gain-scaled latent before the RMS row
 *                                 scale | roped k_pe
 *   attn   [N, heads, v]          attention output before o_proj
 *   latent [B*(T_past+T), kv_lora+rope]  (mla_prefill_chunked only) the
 *                                 normalised latent rows of history and new
 *                                 tokens; kv then covers these rows
 *   pos    [total] int32          (mla_prefill_varlen only) position of every
 *                                 packed row within its sequence
 * Offsets are -1 for buffers a configuration does not use. */
typedef struct mla_prefill_layout {
  int64_t status, ssq_q, ssq_kv, q_a, ckv, q, kv, attn, total_bytes, latent, pos;
} mla_prefill_layout;

/* Byte offsets of the decode intermediates inside the workspace:
 *   q_lat  [B, heads, kv_lora+rope] absorbed query (W_UK^T q_nope | q_pe)
 *   o_lat  [B, heads, kv_lora]      attention output in latent space
 *   part_o / part_lse               partial results of split sequences
 *                                   ([max_splits, heads, ...] on tensor
 *                                   cores, [B, max_splits, heads, ...] else)
 *   o      [B, heads, v]            output before the optional o_proj */
typedef struct mla_decode_layout {
  int64_t status, q_lat, part_o, part_lse, o_lat, o, total_bytes;
  int32_t split_tokens, max_splits;
} mla_decode_layout;

/* ABI version of the loaded library (MLA_ABI_VERSION at build time). */
MLA_API int32_t mla_abi_version(void);

/* Human-readable name of a status code.  Static storage; never NULL. */
MLA_API const char* mla_status_string(mla_status s);

/* Detail of the last error returned on the calling host thread (which
 * argument, which CUDA error).  Thread-local static storage; never NULL. */
MLA_API const char* mla_last_error_detail(void);

/*
 * mla_build_rope_tables -- RoPE / YaRN cos and sin tables.
 *
 * Computes, for t in [0, max_pos) and i in [0, rope/2):
 *   cos[t, i] = cos[t, i + rope/2] = mag * cos(t * theta'_i)
 *   sin[t, i] = sin[t, i + rope/2] = mag * sin(t * theta'_i)
 * the rotate_half layout of [MINIMIND] section 3 (cos/sin are [T, d_h] and
 * element i pairs with i + d/2).  Plain: theta'_i = base^(-2i/rope), mag = 1.
 * YaRN ([MEGATRON] MLA 专属参数详解 lists rotary_base, rotary_scaling_factor,
 * original_max_position_embeddings, beta_fast, beta_slow, mscale,
 * mscale_all_dim; the construction is the NTK-by-parts reading):
 *   corr(b) = rope * ln(L / (2 pi b)) / (2 ln base)
 *   lo = max(floor(corr(beta_fast)), 0), hi = min(ceil(corr(beta_slow)), rope-1)
 *   ramp_i = clamp((i - lo) / (hi - lo), 0, 1)   (hi += 0.001 if lo == hi)
 *   theta'_i = (1 - ramp_i) theta_i + ramp_i theta_i / s
 *   mag = m(s, mscale) / m(s, mscale_all_dim)
 * MLA_ROPE_NONE gives the identity tables (cos 1, sin 0).  Angles are
 * formed in fp64; the outputs are rounded once to fp32.
 *
 *   cfg       host pointer; uses rope fields, qk_rope_head_dim, dtype ignored
 *   max_pos   number of positions (rows), 1 .. 2^24
 *   cos_out, sin_out  device fp32 [max_pos, qk_rope_head_dim], written whole
 */
MLA_API mla_status mla_build_rope_tables(const mla_config* cfg, int32_t max_pos,
                                 float* cos_out, float* sin_out, void* stream);

/* Workspace bytes mla_prefill_forward needs for (cfg, B, T); 0 if the
 * arguments are invalid.  Fills *layout when it is not NULL. */
MLA_API size_t mla_prefill_workspace_size(const mla_config* cfg, int32_t B, int32_t T,
                                  mla_prefill_layout* layout);

/*
 * mla_prefill_forward -- causal MLA forward over B sequences of T tokens.
 *
 * For every token (position t = 0..T-1 within its sequence), in the order of
 * [DSV3] forward (same flow in [VERL] and [KIMI] mla-forward):
 *   q       = q_b_proj(RMSNorm_q(q_a_proj(x)))   or q_proj(x) if q_lora_rank==0
 *   [c|kpe] = kv_a_proj_with_mqa(x)              (kv_lora_rank | rope)
 *   [k_nope_h | V_h] = kv_b_proj(RMSNorm_kv(c))  per head
 *   q_pe, kpe rotated with cos/sin at position t (not for MLA_ROPE_NONE)
 *   Q_h = [q_nope_h | q_pe_h], K_h = [k_nope_h | kpe] (kpe shared by heads)
 *   O_h = softmax(scale Q_h K_h^T, keys j <= t) V_h  (V width v_head_dim;
 *         no zero padding of V)
 *   out = o_proj(concat_h O_h)
 * RMSNorm(v) = g * v / sqrt(mean(v^2) + rms_eps) ([KIMI] rmsnorm).
 *
 *   cfg, w     host pointers to the configuration and the device weights
 *   x          [B, T, hidden]
 *   B, T       >= 1, B*T < 2^31
 *   rope_cos, rope_sin  fp32 [>= T, rope] from mla_build_rope_tables; may be
 *              NULL for MLA_ROPE_NONE
 *   out        [B, T, hidden]
 *   latent_cache_out  NULL, or [B*T, kv_lora_rank + rope]: receives
 *              [RMSNorm_kv(c) | roped kpe] per token -- the compressed cache
 *              of [MEGATRON] 推理优化 that mla_decode_absorbed consumes.
 *   workspace  >= mla_prefill_workspace_size bytes, 256-byte aligned
 */
MLA_API mla_status mla_prefill_forward(const mla_config* cfg, const mla_weights* w,
                               const void* x, int32_t B, int32_t T,
                               const float* rope_cos, const float* rope_sin,
                               void* out, void* latent_cache_out,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* Workspace bytes mla_prefill_chunked needs; 0 if the arguments are invalid. */
MLA_API size_t mla_prefill_chunked_workspace_size(const mla_config* cfg, int32_t B,
                                                  int32_t T_new, int32_t T_past,
                                                  mla_prefill_layout* layout);

/*
 * mla_prefill_chunked -- prefill of T_new new tokens per sequence after T_past
 * tokens that are already in the compressed latent cache.
 *
 * [MEGATRON] 推理优化: with cache_mla_latents the cache keeps per token
 * [kv_compressed | k_pos_emb], and prefill against cached latents
 * uncompresses them through the kv up-projection (uncompress_kv_from_cache).
 * [MINIMIND] section 5: with a cache every history key is visible and only
 * the new T_q x T_q block is causally masked.  So new token i (position
 * T_past + i) attends to keys 0 .. T_past + i, whose k_nope / V are
 * kv_b_proj of the latent rows [past_cache | RMSNorm_kv(c_new)] and whose
 * shared rope key is the cached / newly roped k_pe.  Everything else is
 * mla_prefill_forward's computation (RoPE of the new tokens at positions
 * T_past + i).  T_past = 0 is exactly mla_prefill_forward.
 *
 *   x            [B, T_new, hidden] (new tokens)
 *   past_cache   [B, T_past, kv_lora_rank + rope] (NULL when T_past = 0),
 *                rows as written by latent_cache_out of an earlier call
 *   rope_cos/sin fp32 [>= T_past + T_new, rope]
 *   out          [B, T_new, hidden]
 *   latent_cache_out  NULL or [B*T_new, kv_lora_rank + rope]: the new tokens'
 *                cache rows (append them to the history for the next chunk)
 *   workspace    >= mla_prefill_chunked_workspace_size bytes, 256-aligned
 */
MLA_API mla_status mla_prefill_chunked(const mla_config* cfg, const mla_weights* w,
                                       const void* x, int32_t B, int32_t T_new,
                                       const void* past_cache, int32_t T_past,
                                       const float* rope_cos, const float* rope_sin,
                                       void* out, void* latent_cache_out, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Workspace bytes mla_prefill_varlen needs; 0 if the arguments are invalid. */
MLA_API size_t mla_prefill_varlen_workspace_size(const mla_config* cfg, int32_t n_seq,
                                                 int32_t total, int32_t max_seqlen,
                                                 mla_prefill_layout* layout);

/*
 * mla_prefill_varlen -- prefill of n_seq variable-length sequences packed back
 * to back (THD layout).
 *
 * Megatron-LM MLA guide, 训练支持与并行策略: packed sequences are described by
 * cumulative lengths.  Sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1;
 * its tokens sit at positions 0, 1, ... (RoPE restarts in every sequence) and
 * attend causally within their own sequence only.  Every other step is
 * mla_prefill_forward's computation, row by row.
 *
 *   x            [total, hidden] packed tokens
 *   cu_seqlens   DEVICE int32 [n_seq + 1], cu[0] = 0, non-decreasing,
 *                cu[n_seq] = total, every length <= max_seqlen.  It is read on
 *                the device only: a malformed array sets the device status word,
 *                which mla_check_device_status reports as MLA_ERR_SHAPE; all
 *                accesses stay clamped inside [0, total) rows.
 *   max_seqlen   longest sequence (sizes the launch; 1 <= max_seqlen <= total)
 *   rope_cos/sin fp32 [>= max_seqlen, rope]
 *   out          [total, hidden]
 *   latent_cache_out  NULL or [total, kv_lora_rank + rope], packed like x
 *   workspace    >= mla_prefill_varlen_workspace_size bytes, 256-aligned
 * Errors: MLA_ERR_NULL / SHAPE / ALIGN / DTYPE / WORKSPACE before any launch;
 * MLA_ERR_UNSUPPORTED when n_seq x heads exceeds 65535 (launch grid).
 */
MLA_API mla_status mla_prefill_varlen(const mla_config* cfg, const mla_weights* w, const void* x,
                                      const int32_t* cu_seqlens, int32_t n_seq, int32_t total,
                                      int32_t max_seqlen, const float* rope_cos,
                                      const float* rope_sin, void* out, void* latent_cache_out,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes mla_decode_absorbed needs for (cfg, B, max_ctx); 0 if the
 * arguments are invalid.  Fills *layout when it is not NULL.
 * Tensor-core configurations (bf16, kv_lora_rank 512, rope 64): the tokens of
 * all sequences, concatenated, are cut into equal slices of at least
 * layout->split_tokens tokens, one per pair of SMs; a sequence that crosses
 * a slice boundary leaves one partial result per slice, in one of
 * layout->max_splits slots (two per SM pair).  The result depends on the
 * current device's SM count.  Other configurations: split_tokens-token
 * splits of every sequence, max_splits of them per sequence. */
MLA_API size_t mla_decode_workspace_size(const mla_config* cfg, int32_t B,
                                 int32_t max_ctx, mla_decode_layout* layout);

/*
 * mla_decode_absorbed -- one query token per sequence against its latent
 * cache, with the kv up-projection absorbed ([MEGATRON] 推理优化: the kv
 * up-projection is split into up_k and up_v; up_k is folded into the query,
 * up_v recovers v_head_dim after attention):
 *   W_UK[h] = rows h*(nope+v) + [0, nope)      of w_kv_b
 *   W_UV[h] = rows h*(nope+v) + [nope, nope+v) of w_kv_b
 *   q_lat[b,h] = W_UK[h]^T q_nope[b,h]                       (kv_lora_rank)
 *   s_j = scale (q_lat[b,h] . c_j + q_pe[b,h] . kpe_j),  j < ctx_b
 *   o_lat[b,h] = sum_j softmax(s)_j c_j
 *   o[b,h] = W_UV[h] o_lat[b,h];   out = o_proj(o) if w_o != NULL
 * Every cached token is visible (a one-token query's causal block is empty,
 * [MINIMIND] section 5); ctx_b counts the current token.
 *
 *   q_nope        [B, heads, nope]
 *   q_pe          [B, heads, rope], already rotated at the query position
 *   w_kv_b        [heads*(nope+v), kv_lora_rank]
 *   latent_cache  [sum_b ctx_b, kv_lora_rank + rope]: row cu_ctx[b] + j holds
 *                 [RMSNorm_kv(c_j) | roped kpe_j] of sequence b
 *   cu_ctx        DEVICE int32 [B+1], cu_ctx[0] = 0, non-decreasing; each
 *                 ctx_b = cu_ctx[b+1]-cu_ctx[b] must lie in [1, max_ctx]
 *                 (the kernels clamp out-of-range lengths and flag
 *                 MLA_ERR_SHAPE in the device status word)
 *   max_ctx       host bound on every ctx_b, >= 1
 *   w_o           NULL, or [hidden, heads*v]
 *   out           [B, heads*v] when w_o is NULL, else [B, hidden]
 *   workspace     mla_decode_workspace_size bytes, 256-byte aligned; on
 *                 tensor cores a smaller one runs on as many SM pairs as its
 *                 partial slots allow (MLA_ERR_WORKSPACE below one pair)
 */
MLA_API mla_status mla_decode_absorbed(const mla_config* cfg, const void* q_nope,
                               const void* q_pe, const void* w_kv_b,
                               const void* latent_cache, const int32_t* cu_ctx,
                               int32_t B, int32_t max_ctx, const void* w_o,
                               void* out, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * mla_check_device_status -- synchronise `stream`, read the status word that
 * the last prefill/decode call on this workspace left at its start, and clear
 * it.  Returns MLA_OK, MLA_ERR_DEVICE_TIMEOUT (a bounded mbarrier or flag
 * wait in a kernel ran out and the kernel returned early; its outputs are
 * invalid) or MLA_ERR_SHAPE (decode saw a cu_ctx entry out of range).
 * workspace is a device pointer; this call blocks the host.
 */
MLA_API mla_status mla_check_device_status(void* workspace, void* stream);

/*
 * Benchmarking aids (no counterpart in the pages).
 *
 * mla_set_stage_events -- register up to 8 caller-created cudaEvent_t that
 * the following forward calls on this host thread record on their stream at
 * stage boundaries, so that per-kernel durations can be read with
 * cudaEventElapsedTime while the calls run back to back:
 *   prefill: [0] before S1 down-projection, [1] after it, [2] after the q
 *            projection, [3] after the kv up-projection, [4] after attention,
 *            [5] after o_proj (6 events)
 *   decode:  [0] before D1, [1] after D1 q absorption, [2] after D2 latent
 *            attention, [3] after D3 combine, [4] after D4 V up-projection,
 *            [5] after o_proj (6 events; [5] = [4] without o_proj)
 * n = 0 (or events NULL) switches recording off.  Returns MLA_ERR_SHAPE for
 * n outside [0, 8].
 *
 * mla_kernel_launches -- number of CUDA kernels this library has launched in
 * this process (all threads), for counting launches in a timed region.
 */
/*
 * mla_selftest_wait_timeout -- failure-detection self-test (no counterpart in
 * the pages).  Enqueues one small kernel whose single mbarrier wait can never
 * be satisfied; the wait gives up after the library's bounded-wait limit
 * (about 2 s), records MLA_ERR_DEVICE_TIMEOUT in the status word at the start
 * of `workspace` (>= 256 bytes, 256-byte aligned) and returns, leaving the
 * context usable.  The status is read with mla_check_device_status.  Nothing
 * traps, faults or hangs.
 */
MLA_API mla_status mla_selftest_wait_timeout(void* workspace, void* stream);
MLA_API mla_status mla_set_stage_events(void* const* events, int32_t n);
MLA_API int64_t mla_kernel_launches(void);

/*
 * mla_decode_absorbed_noalloc -- mla_decode_absorbed for callers that cannot
 * allocate device memory when they decode.  There is no counterpart in the
 * pages; it exists for integration.  Typical callers: a host framework whose
 * own pool owns every device allocation, a plugin that is only handed input
 * and output tensors, a serving loop that forbids allocation on its latency
 * path.  Instead of a caller workspace it uses one array of
 * MLA_DECODE_NOALLOC_SCRATCH_BYTES that the library declares in device memory
 * (every GPU that loads the library holds it until the process exits).
 *
 *   Arguments, layouts and results are those of mla_decode_absorbed without
 *   the workspace pair.
 *   The array holds the partial slots of fewer SM pairs than a full
 *   workspace, so the decode may run on fewer SMs.  Returns MLA_ERR_WORKSPACE
 *   (with mla_last_error_detail naming both sizes) when not even one pair's
 *   layout fits.  On tensor cores the scratch does not depend on max_ctx:
 *   about 304 KiB per sequence of 128 heads plus 0.5 MiB per SM pair, so up
 *   to B = 52 sequences of 128 heads fit (on one pair); B = 64 do not.
 *   The first call on each device looks up that device's copy of the array
 *   (cudaGetSymbolAddress) and caches it; make that first call before any
 *   stream capture.  The call allocates nothing: no cudaMalloc, cudaFree or
 *   allocating library routine.
 *   All calls on a device share the one array and leave the last call's
 *   intermediates in it: calls whose work overlaps on the GPU (different
 *   streams, or host threads racing) corrupt each other -- serialise them.
 *   Device-side status (bounded-wait timeouts, out-of-range cu_ctx) is
 *   recorded in the array but not reported; use mla_decode_absorbed with
 *   mla_check_device_status where that report is needed.
 */
#define MLA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)
MLA_API mla_status mla_decode_absorbed_noalloc(const mla_config* cfg, const void* q_nope,
                                               const void* q_pe, const void* w_kv_b,
                                               const void* latent_cache, const int32_t* cu_ctx,
                                               int32_t B, int32_t max_ctx, const void* w_o,
                                               void* out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
