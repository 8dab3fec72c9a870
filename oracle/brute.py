"""Loop-level brute-force MLA prefill for tiny shapes (test infrastructure).

This is the check on the vectorised oracle: pure Python loops over explicit
indices, using only ``math``.  It follows the FlashAttention-2 route of the
CSDN ``DeepseekV3Attention`` walkthrough (section "代码+流程图") and the verl
page "kimi_vl.py" (section "拼接最终的 Q 和 K" and "V 的 padding 处理"):
per head it materialises K_h = [k_nope_h | k_pe] with the single k_pe head
copied into every head, zero-pads V_h to the query head dim, runs plain
scaled-dot-product attention with a causal -inf mask, and trims the output
back to v_head_dim.  Linear layers are written out as
y[n] = sum_k W[n][k] x[k] (nn.Linear keeps [out, in]; MiniMind page,
section 2).  RoPE frequencies are base^(-2i/d) (plain) computed here by
loops; YaRN tables are not rebuilt here -- they are pinned separately.
"""
import math


def _lin(W, x):
    return [sum(W[n][k] * x[k] for k in range(len(x))) for n in range(len(W))]


def _rms(x, g, eps):
    ms = sum(v * v for v in x) / len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [x[i] * r * (1.0 if g is None else g[i]) for i in range(len(x))]


def _rope(vec, t, base, rotate):
    d = len(vec)
    half = d // 2
    if not rotate:
        return list(vec)
    out = [0.0] * d
    for i in range(half):
        ang = t * base ** (-2.0 * i / d)
        c, s = math.cos(ang), math.sin(ang)
        a, b = vec[i], vec[i + half]
        # x*cos + rotate_half(x)*sin with rotate_half = [-x2, x1]
        out[i] = a * c - b * s
        out[i + half] = b * c + a * s
    return out


def _tolist(t):
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to(torch.float64).tolist()
    except ImportError:      # pragma: no cover
        pass
    return [list(map(float, r)) if hasattr(r, "__len__") else float(r) for r in t]


def brute_prefill(cfg, inp, scale):
    """Returns out as nested lists [B][T][hidden].  ``scale`` is passed in so
    that this function does not re-derive the YaRN scale."""
    assert cfg.rope_type in ("none", "plain")
    B, T = inp.B, inp.T
    h = cfg.num_heads
    dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
    dq = dn + dr
    r_kv = cfg.kv_lora_rank
    assert not getattr(cfg, "rope_interleave", False)
    rotate = cfg.rope_type == "plain"
    X = _tolist(inp.x)
    Wkva, Wkvb, Wo = _tolist(inp.w_kv_a), _tolist(inp.w_kv_b), _tolist(inp.w_o)
    gkv = _tolist(inp.g_kv_a)
    lora = cfg.q_lora_rank > 0
    if lora:
        Wqa, Wqb, gq = _tolist(inp.w_q_a), _tolist(inp.w_q_b), _tolist(inp.g_q_a)
    else:
        Wq = _tolist(inp.w_q)
    out = []
    for b in range(B):
        Q, K, V = [], [], []          # [t][head][...]
        for t in range(T):
            x = X[b][t]
            qfull = (_lin(Wqb, _rms(_lin(Wqa, x), gq, cfg.rms_eps)) if lora
                     else _lin(Wq, x))
            kva = _lin(Wkva, x)
            c, kpe = kva[:r_kv], kva[r_kv:]
            kv = _lin(Wkvb, _rms(c, gkv, cfg.rms_eps))
            kpe_r = _rope(kpe, t, cfg.rope_theta, rotate)
            qt, kt, vt = [], [], []
            for hh in range(h):
                qh = qfull[hh * dq:(hh + 1) * dq]
                qh = qh[:dn] + _rope(qh[dn:], t, cfg.rope_theta, rotate)
                kvh = kv[hh * (dn + dv):(hh + 1) * (dn + dv)]
                kt.append(kvh[:dn] + kpe_r)                 # shared k_pe copy
                vt.append(kvh[dn:] + [0.0] * (dq - dv))     # V zero-padded
                qt.append(qh)
            Q.append(qt), K.append(kt), V.append(vt)
        rows = []
        for i in range(T):
            concat = []
            for hh in range(h):
                s = []
                for j in range(T):
                    if j > i:
                        s.append(-math.inf)
                    else:
                        s.append(scale * sum(Q[i][hh][d] * K[j][hh][d]
                                             for d in range(dq)))
                m = max(s)
                e = [math.exp(v - m) if v != -math.inf else 0.0 for v in s]
                z = sum(e)
                o = [sum(e[j] / z * V[j][hh][d] for j in range(T))
                     for d in range(dq)]
                concat.extend(o[:dv])                       # trim the pad
            rows.append(_lin(Wo, concat))
        out.append(rows)
    return out
