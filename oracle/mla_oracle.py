"""Plain fp64 NumPy oracle for the MLA forward (prefill and absorbed decode).

Test infrastructure: see the package docstring for who may import this.

Sources (page titles and sections of the reference pages):

* [DSV3] CSDN walkthrough of HF ``DeepseekV3Attention`` (section "代码+流程图"):
  ``__init__`` (projection shapes, the YaRN softmax scale, "eq. 21/22 of the
  YaRN paper") and ``forward`` (q path, kv_a split, kv_b split, RoPE on the
  rot parts, k_rot broadcast, concatenation, FA2 V pad/trim, o_proj).
* [VERL] verl docs, "kimi_vl.py — KimiVL (DeepSeek-V3 架构) 注意力适配":
  "Q 投影和 KV 压缩" (both Q paths) and "V 的 padding 处理".
* [MEGATRON] "Megatron-LM 多潜在注意力MLA实战指南": sections 源码架构 (layer
  table, softmax scale mscale*mscale/sqrt(q_head_dim)), MLA 专属参数详解 (YaRN
  parameters and defaults) and 推理优化 (latent cache, absorption).
* [MINIMIND] MiniMind "Attention 前向传播" blog: section 2 (nn.Linear is
  [out, in], forward x W^T), section 3 (RMSNorm in fp32, rotate_half RoPE),
  section 5 (scaled dot product, triu(1) causal mask, fp32 softmax).
* [KIMI] Kimi-K3 atlas page "Gated MLA › Key and value heads": mla-init,
  mla-forward (no rotary), rmsnorm (eps 1e-6, fp32).

Everything is float64.  Inputs may be torch tensors or numpy arrays of any
float dtype; they are converted with ``np.asarray(..., float64)``.
"""
import math
from typing import Optional, Sequence

import numpy as np


def _f64(t):
    if t is None:
        return None
    try:                                   # torch tensor (bf16 included)
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to(torch.float64).cpu().numpy()
    except ImportError:                    # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def _cfg_get(cfg, name):
    return getattr(cfg, name)


# ---------------------------------------------------------------------------
# Softmax scale (S6)
# ---------------------------------------------------------------------------
def yarn_get_mscale(scale: float, mscale: float) -> float:
    """YaRN attention magnitude factor m(s, a).

    [DSV3] ``__init__`` calls ``yarn_get_mscale(factor, mscale_all_dim)`` and
    squares it into the softmax scale, citing YaRN eqs. 21/22, without showing
    its body.  The closed form used is m = 1 for s <= 1, else
    0.1 * a * ln(s) + 1 (the expression the workload statement gives).
    """
    if scale <= 1.0:
        return 1.0
    return 0.1 * mscale * math.log(scale) + 1.0


def softmax_scale(cfg) -> float:
    """Softmax scale: q_head_dim^-0.5, times mscale^2 under YaRN.

    [DSV3] ``__init__``: ``scaling = qk_head_dim ** -0.5`` and, when
    rope_scaling is set and mscale_all_dim is non-zero,
    ``scaling *= mscale * mscale`` with mscale = m(factor, mscale_all_dim).
    [MEGATRON] 源码架构 states the same: mscale*mscale/sqrt(q_head_dim).
    [KIMI] mla-init: scaling = q_head_dim ** -0.5 (no rotary, no YaRN).
    An explicit ``cfg.softmax_scale`` overrides.
    """
    if cfg.softmax_scale:
        return float(cfg.softmax_scale)
    dq = cfg.qk_nope_head_dim + cfg.qk_rope_head_dim
    s = dq ** -0.5
    if cfg.rope_type == "yarn" and cfg.rope_mscale_all_dim:
        m = yarn_get_mscale(cfg.rope_factor, cfg.rope_mscale_all_dim)
        s = s * m * m
    return s


# ---------------------------------------------------------------------------
# Rotary tables (S9)
# ---------------------------------------------------------------------------
def rope_frequencies(cfg):
    """Per-pair rotation frequencies theta'_i (i < rope/2) and the cos/sin
    magnitude factor.

    Plain RoPE: theta_i = base^(-2i/d) with d = qk_rope_head_dim.
    YaRN ("NTK-by-parts", the reading adopted for pages that list only the
    parameters rotary_base, rotary_scaling_factor,
    original_max_position_embeddings, beta_fast, beta_slow, mscale,
    mscale_all_dim -- [MEGATRON] MLA 专属参数详解):

      corr(b)  = d * ln(L / (2*pi*b)) / (2 * ln base)
      lo = max(floor(corr(beta_fast)), 0), hi = min(ceil(corr(beta_slow)), d-1)
      (hi += 0.001 when lo == hi)
      ramp_i   = clamp((i - lo) / (hi - lo), 0, 1)
      theta'_i = (1 - ramp_i) * theta_i + ramp_i * theta_i / s

    and cos/sin are multiplied by m(s, mscale) / m(s, mscale_all_dim).
    """
    d = cfg.qk_rope_head_dim
    half = d // 2
    base = float(cfg.rope_theta)
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    if cfg.rope_type != "yarn":
        return theta, 1.0
    s = float(cfg.rope_factor)
    L = float(cfg.original_max_position_embeddings)

    def corr(n_rot):
        return d * math.log(L / (n_rot * 2.0 * math.pi)) / (2.0 * math.log(base))

    lo = max(math.floor(corr(cfg.beta_fast)), 0)
    hi = min(math.ceil(corr(cfg.beta_slow)), d - 1)
    lo, hi = float(lo), float(hi)
    if lo == hi:
        hi += 0.001
    ramp = np.clip((i - lo) / (hi - lo), 0.0, 1.0)
    theta_p = (1.0 - ramp) * theta + ramp * (theta / s)
    mag = yarn_get_mscale(s, cfg.rope_mscale) / yarn_get_mscale(
        s, cfg.rope_mscale_all_dim)
    return theta_p, mag


def rope_tables(cfg, max_pos: int):
    """cos/sin tables [max_pos, d] in the rotate_half layout.

    [MINIMIND] section 3: cos and sin have shape [T, d_h] and multiply the
    whole head vector; rotate_half pairs element i with i + d/2, so both
    halves of a row carry the same angle t * theta'_i.  Angles in fp64.
    """
    theta, mag = rope_frequencies(cfg)
    t = np.arange(max_pos, dtype=np.float64)[:, None]
    ang = t * theta[None, :]
    ang = np.concatenate([ang, ang], axis=1)
    return mag * np.cos(ang), mag * np.sin(ang)


def rotate_half(x):
    """[MINIMIND] section 3: cat(-x[..., d/2:], x[..., :d/2])."""
    half = x.shape[-1] // 2
    return np.concatenate([-x[..., half:], x[..., :half]], axis=-1)


def apply_rope(x, cos, sin):
    """[MINIMIND] section 3: x * cos + rotate_half(x) * sin."""
    return x * cos + rotate_half(x) * sin


def _rope_columns(cfg, x):
    """[DSV3] forward: with ``rope_interleave`` the projections emit the rope
    columns as adjacent pairs (2i, 2i+1), and apply_rotary_pos_emb_interleave
    first brings them to rotate_half order [x0, x2, .., x(d-2), x1, x3, ..]
    (pair i becomes columns (i, i + d/2)) and then rotates as usual."""
    if not getattr(cfg, "rope_interleave", False):
        return x
    return np.concatenate([x[..., 0::2], x[..., 1::2]], axis=-1)


# ---------------------------------------------------------------------------
# RMSNorm (S2)
# ---------------------------------------------------------------------------
def rms_norm(x, gamma, eps):
    """gamma * x / sqrt(mean(x^2) + eps) over the last axis.

    [KIMI] rmsnorm and [MINIMIND] section 3 (computed in fp32 there; fp64
    here).  The two pages differ in where the cast back happens; the oracle
    does not round, so the order does not arise.
    """
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    return y if gamma is None else y * gamma


# ---------------------------------------------------------------------------
# Prefill (S1 .. S8)
# ---------------------------------------------------------------------------
def _softmax_rows(s):
    """[MINIMIND] section 5: softmax along the key axis (fp32 there, fp64 here)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def prefill(cfg, inp, rows: Optional[Sequence[int]] = None,
            return_parts: bool = False, return_probs: bool = False):
    """MLA prefill forward, causal, positions 0..T-1 in every batch row.

    Steps, in the order of [DSV3] ``forward`` (same flow in [VERL] and
    [KIMI] mla-forward):

    1. q = q_b_proj(q_a_layernorm(q_a_proj(x))), or q = q_proj(x) when
       q_lora_rank is None; view as [.., heads, q_head_dim]; split nope | rope.
    2. [c | k_pe] = kv_a_proj_with_mqa(x), split [kv_lora_rank, rope].
    3. kv = kv_b_proj(kv_a_layernorm(c)) viewed [.., heads, nope + v],
       split into k_nope and V.
    4. RoPE on q_pe and on the single shared k_pe head (skipped for
       rope_type "none", the Kimi no-rotary variant).
    5. Q_h = [q_nope_h | q_pe_h], K_h = [k_nope_h | k_pe] (k_pe broadcast).
    6. softmax(scale * Q_h K_h^T + causal mask) V_h, V of width v_head_dim
       (zero-padding V to q_head_dim and trimming afterwards, as the FA2
       path does, gives the same numbers).
    7. o_proj over the heads-concatenated output.

    ``rows``: optional list of query positions (within each batch row) whose
    outputs are computed; keys/values are always built for every position.
    Returns out [B, T or len(rows), hidden] and, on request, a dict of parts.
    """
    B, T = inp.B, inp.T
    H, h = cfg.hidden_size, cfg.num_heads
    dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
    dq = dn + dr
    r_kv = cfg.kv_lora_rank
    eps = cfg.rms_eps
    scale = softmax_scale(cfg)

    x = _f64(inp.x).reshape(B, T, H)
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    R = len(rows)

    # Step 2-3: keys and values for every position.
    kva = x @ _f64(inp.w_kv_a).T                       # [B, T, r_kv + dr]
    c, kpe = kva[..., :r_kv], kva[..., r_kv:]
    c_hat = rms_norm(c, _f64(inp.g_kv_a), eps)
    kv = (c_hat @ _f64(inp.w_kv_b).T).reshape(B, T, h, dn + dv)
    k_nope, v = kv[..., :dn], kv[..., dn:]

    # Step 1: queries for the requested rows only.
    xr = x[:, rows, :]
    if cfg.q_lora_rank > 0:
        qa = xr @ _f64(inp.w_q_a).T
        q = rms_norm(qa, _f64(inp.g_q_a), eps) @ _f64(inp.w_q_b).T
    else:
        q = xr @ _f64(inp.w_q).T
    q = q.reshape(B, R, h, dq)
    q_nope, q_pe = q[..., :dn], q[..., dn:]

    # Step 4: RoPE at position t (0-based within the batch row).
    if cfg.rope_type != "none":
        q_pe, kpe = _rope_columns(cfg, q_pe), _rope_columns(cfg, kpe)
        cos, sin = rope_tables(cfg, T)
        kpe = apply_rope(kpe, cos[None, :, :], sin[None, :, :])
        q_pe = apply_rope(q_pe, cos[rows][None, :, None, :],
                          sin[rows][None, :, None, :])

    # Steps 5-6 per batch row and head.
    o = np.empty((B, R, h, dv))
    probs = np.empty((B, h, R, T)) if return_probs else None
    key_pos = np.arange(T)
    mask = key_pos[None, :] > rows[:, None]             # j > i is masked
    for b in range(B):
        for hh in range(h):
            Qh = np.concatenate([q_nope[b, :, hh, :], q_pe[b, :, hh, :]], -1)
            Kh = np.concatenate([k_nope[b, :, hh, :], kpe[b]], -1)
            s = scale * (Qh @ Kh.T)                      # [R, T]
            s = np.where(mask, -np.inf, s)
            p = _softmax_rows(s)
            if return_probs:
                probs[b, hh] = p
            o[b, :, hh, :] = p @ v[b, :, hh, :]

    out = o.reshape(B, R, h * dv) @ _f64(inp.w_o).T
    if not (return_parts or return_probs):
        return out
    parts = dict(q_nope=q_nope, q_pe=q_pe, k_nope=k_nope, k_pe=kpe, v=v,
                 c_hat=c_hat, attn=o, latent_cache=np.concatenate(
                     [c_hat, kpe], -1), scale=scale)
    if return_probs:
        parts["probs"] = probs
    return out, parts


# ---------------------------------------------------------------------------
# Chunked prefill against a cached latent
# ---------------------------------------------------------------------------
def _chunk_positions(T_past, T_new):
    """Positions of the new tokens: they follow the T_past cached ones."""
    return T_past + np.arange(T_new)


def _chunk_latent(past, new_rows):
    """Latent rows of every key position: the cached rows as they are (already
    normalised and roped), then the new tokens' rows."""
    return np.concatenate([past, new_rows], axis=1)


def prefill_chunked(cfg, inp, past_cache, T_past: int,
                    return_parts: bool = False):
    """T_new new tokens per sequence after T_past cached ones.

    [MEGATRON] 推理优化: with cache_mla_latents the cache holds, per token,
    [kv_compressed | k_pos_emb]; prefill against it uncompresses the cached
    latents with the kv up-projection (uncompress_kv_from_cache).  [MINIMIND]
    section 5: with a cache, every history key is visible and the causal mask
    covers only the new T_q x T_q block.  So, for new token i at position
    T_past + i:

    1. q and [c | k_pe] of the new tokens as in ``prefill`` (RoPE at
       positions T_past + i).
    2. Keys/values of all T_past + T_new positions from the latent rows
       [past_cache | RMSNorm(c_new) | roped k_pe_new] uncompressed by kv_b.
    3. softmax over keys 0 .. T_past + i, then o_proj.

    ``past_cache``: [B, T_past, kv_lora_rank + rope] (already normalised and
    roped).  ``inp``: PrefillInputs of the new tokens (inp.T = T_new).
    """
    B, Tn = inp.B, inp.T
    H, h = cfg.hidden_size, cfg.num_heads
    dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
    dq = dn + dr
    r_kv = cfg.kv_lora_rank
    eps = cfg.rms_eps
    scale = softmax_scale(cfg)
    Ta = T_past + Tn
    x = _f64(inp.x).reshape(B, Tn, H)
    past = _f64(past_cache).reshape(B, T_past, r_kv + dr)

    kva = x @ _f64(inp.w_kv_a).T
    c, kpe = kva[..., :r_kv], kva[..., r_kv:]
    c_hat = rms_norm(c, _f64(inp.g_kv_a), eps)
    if cfg.q_lora_rank > 0:
        q = rms_norm(x @ _f64(inp.w_q_a).T, _f64(inp.g_q_a), eps) @ _f64(inp.w_q_b).T
    else:
        q = x @ _f64(inp.w_q).T
    q = q.reshape(B, Tn, h, dq)
    q_nope, q_pe = q[..., :dn], q[..., dn:]
    qpos = _chunk_positions(T_past, Tn)
    if cfg.rope_type != "none":
        q_pe, kpe = _rope_columns(cfg, q_pe), _rope_columns(cfg, kpe)
        cos, sin = rope_tables(cfg, Ta)
        cn, sn = cos[qpos], sin[qpos]
        kpe = apply_rope(kpe, cn[None], sn[None])
        q_pe = apply_rope(q_pe, cn[None, :, None, :], sn[None, :, None, :])
    latent = _chunk_latent(past, np.concatenate([c_hat, kpe], -1))
    kv = (latent[..., :r_kv] @ _f64(inp.w_kv_b).T).reshape(B, Ta, h, dn + dv)
    k_nope, v = kv[..., :dn], kv[..., dn:]
    k_pe = latent[..., r_kv:]
    o = np.empty((B, Tn, h, dv))
    mask = np.arange(Ta)[None, :] > qpos[:, None]
    for b in range(B):
        for hh in range(h):
            Qh = np.concatenate([q_nope[b, :, hh, :], q_pe[b, :, hh, :]], -1)
            Kh = np.concatenate([k_nope[b, :, hh, :], k_pe[b]], -1)
            s = np.where(mask, -np.inf, scale * (Qh @ Kh.T))
            o[b, :, hh, :] = _softmax_rows(s) @ v[b, :, hh, :]
    out = o.reshape(B, Tn, h * dv) @ _f64(inp.w_o).T
    if not return_parts:
        return out
    return out, dict(attn=o, latent=latent, new_cache=latent[:, T_past:])


def _packed_rows(cu_seqlens, N):
    """Sequence index b(m) and in-sequence position of every packed row."""
    cu = np.asarray(_f64(cu_seqlens), dtype=np.int64)
    assert cu[0] == 0 and cu[-1] == N and np.all(np.diff(cu) >= 0)
    seq = np.searchsorted(cu, np.arange(N), side="right") - 1
    return seq, np.arange(N) - cu[seq]


def prefill_varlen(cfg, inp, cu_seqlens, return_parts: bool = False):
    """Packed (THD) prefill: ``inp.x`` holds N tokens of several sequences back
    to back, sequence b owning rows cu_seqlens[b] .. cu_seqlens[b+1]-1.

    [MEGATRON] 训练支持与并行策略 packs variable-length sequences in the THD
    layout described by cumulative sequence lengths.  Every step of
    ``prefill`` is per token except RoPE and attention, so in packed form:
    the position of row m is m - cu_seqlens[b(m)] (positions restart at 0 in
    every sequence), and query m attends to key k only when both rows belong
    to the same sequence and pos(k) <= pos(m) (a block-diagonal causal mask
    over the packed rows).

    ``inp``: PrefillInputs with B = 1, T = N.  Returns out [N, hidden] and, on
    request, the parts (attention output, latent cache rows).
    """
    N = inp.T
    H, h = cfg.hidden_size, cfg.num_heads
    dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
    dq = dn + dr
    r_kv = cfg.kv_lora_rank
    eps = cfg.rms_eps
    scale = softmax_scale(cfg)
    seq, pos = _packed_rows(cu_seqlens, N)

    x = _f64(inp.x).reshape(N, H)
    kva = x @ _f64(inp.w_kv_a).T
    c, kpe = kva[:, :r_kv], kva[:, r_kv:]
    c_hat = rms_norm(c, _f64(inp.g_kv_a), eps)
    kv = (c_hat @ _f64(inp.w_kv_b).T).reshape(N, h, dn + dv)
    k_nope, v = kv[..., :dn], kv[..., dn:]
    if cfg.q_lora_rank > 0:
        q = rms_norm(x @ _f64(inp.w_q_a).T, _f64(inp.g_q_a), eps) @ _f64(inp.w_q_b).T
    else:
        q = x @ _f64(inp.w_q).T
    q = q.reshape(N, h, dq)
    q_nope, q_pe = q[..., :dn], q[..., dn:]
    if cfg.rope_type != "none":
        q_pe, kpe = _rope_columns(cfg, q_pe), _rope_columns(cfg, kpe)
        cos, sin = rope_tables(cfg, int(pos.max()) + 1 if N else 1)
        kpe = apply_rope(kpe, cos[pos], sin[pos])
        q_pe = apply_rope(q_pe, cos[pos][:, None, :], sin[pos][:, None, :])
    visible = (seq[None, :] == seq[:, None]) & (pos[None, :] <= pos[:, None])
    o = np.empty((N, h, dv))
    for hh in range(h):
        Qh = np.concatenate([q_nope[:, hh, :], q_pe[:, hh, :]], -1)
        Kh = np.concatenate([k_nope[:, hh, :], kpe], -1)
        s = np.where(visible, scale * (Qh @ Kh.T), -np.inf)
        o[:, hh, :] = _softmax_rows(s) @ v[:, hh, :]
    out = o.reshape(N, h * dv) @ _f64(inp.w_o).T
    if not return_parts:
        return out
    return out, dict(attn=o, latent_cache=np.concatenate([c_hat, kpe], -1), pos=pos, seq=seq)


# ---------------------------------------------------------------------------
# Decode over the latent cache (D1 .. D4)
# ---------------------------------------------------------------------------
def _split_kv_b(cfg, w_kv_b):
    """[MEGATRON] 推理优化: the kv up-projection splits into up_k (first
    qk_nope rows of each head block) and up_v (last v_head_dim rows)."""
    h, dn, dv = cfg.num_heads, cfg.qk_nope_head_dim, cfg.v_head_dim
    W = _f64(w_kv_b).reshape(h, dn + dv, cfg.kv_lora_rank)
    return W[:, :dn, :], W[:, dn:, :]


def _seq_ids(cu_ctx, batches):
    cu = np.asarray(_f64(cu_ctx), dtype=np.int64)
    B = len(cu) - 1
    return cu, (range(B) if batches is None else list(batches))


def decode_unabsorbed(cfg, q_nope, q_pe, w_kv_b, cache, cu_ctx, w_o=None,
                      batches=None):
    """One decode query per sequence against its cached latents, explicit form.

    The cache row of token j holds [c_hat_j | k_pe_j] (RMS-normalised latent
    and roped shared key part; [MEGATRON] 推理优化, cache_mla_latents).  Per
    head, K_nope = c_hat W_UK^T and V = c_hat W_UV^T are rebuilt (the
    "uncompress" form), then s_j = scale (q_nope.k_nope_j + q_pe.k_pe_j) over
    every cached token j (a single query sees the whole cache: [MINIMIND]
    section 5, the causal block of a one-token query is empty), softmax, and
    o = sum_j p_j V_j.  Returns [nb, heads*v] or, with w_o, [nb, hidden].
    """
    h, dv, r = cfg.num_heads, cfg.v_head_dim, cfg.kv_lora_rank
    scale = softmax_scale(cfg)
    W_UK, W_UV = _split_kv_b(cfg, w_kv_b)
    qn, qp, C = _f64(q_nope), _f64(q_pe), _f64(cache)
    cu, bs = _seq_ids(cu_ctx, batches)
    out = []
    for b in bs:
        Cb = C[cu[b]:cu[b + 1]]
        c, kpe = Cb[:, :r], Cb[:, r:]
        o = np.empty((h, dv))
        for hh in range(h):
            k_nope = c @ W_UK[hh].T                       # [ctx, dn]
            vv = c @ W_UV[hh].T                           # [ctx, dv]
            s = scale * (k_nope @ qn[b, hh] + kpe @ qp[b, hh])
            p = _softmax_rows(s[None, :])[0]
            o[hh] = p @ vv
        out.append(o.reshape(h * dv))
    out = np.stack(out)
    if w_o is not None:
        out = out @ _f64(w_o).T
    return out


def decode_absorbed(cfg, q_nope, q_pe, w_kv_b, cache, cu_ctx, w_o=None,
                    batches=None, return_parts=False):
    """Weight-absorbed decode ([MEGATRON] 推理优化: up_k folded into the
    query, up_v applied after attention).

    D1  q_lat[h] = W_UK[h]^T q_nope[h]                     (kv_lora_rank)
    D2  s_j = scale (q_lat[h].c_j + q_pe[h].k_pe_j),  p = softmax(s),
        o_lat[h] = sum_j p_j c_j
    D4  o[h] = W_UV[h] o_lat[h];  optional o_proj.
    Mathematically identical to ``decode_unabsorbed`` (associativity).
    """
    h, dv, r = cfg.num_heads, cfg.v_head_dim, cfg.kv_lora_rank
    scale = softmax_scale(cfg)
    W_UK, W_UV = _split_kv_b(cfg, w_kv_b)
    qn, qp, C = _f64(q_nope), _f64(q_pe), _f64(cache)
    cu, bs = _seq_ids(cu_ctx, batches)
    out, lat, lses = [], [], []
    for b in bs:
        Cb = C[cu[b]:cu[b + 1]]
        c, kpe = Cb[:, :r], Cb[:, r:]
        q_lat = np.einsum("hd,hdr->hr", qn[b], W_UK)      # [h, r]
        s = scale * (q_lat @ c.T + qp[b] @ kpe.T)          # [h, ctx]
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        o_lat = (e @ c) / l                                # [h, r]
        o = np.einsum("hr,hdr->hd", o_lat, W_UV)           # [h, dv]
        out.append(o.reshape(h * dv))
        lat.append(o_lat)
        lses.append((m + np.log(l))[:, 0])
    out = np.stack(out)
    if w_o is not None:
        out = out @ _f64(w_o).T
    if return_parts:
        return out, dict(o_lat=np.stack(lat), lse=np.stack(lses))
    return out


def max_rel_err(got, ref) -> float:
    """max|got - ref| / max|ref| over a whole tensor (the tolerance metric)."""
    g, r = _f64(got), _f64(ref)
    den = float(np.max(np.abs(r)))
    return float(np.max(np.abs(g - r))) / (den if den > 0 else 1.0)
