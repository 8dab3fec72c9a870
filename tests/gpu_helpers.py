"""Shared pieces of the GPU parity tests: run the C ABI on seeded inputs and
bring results back as float64 numpy arrays."""
import numpy as np
import torch

from latent_attention_b200.layer import MlaPrefill, MlaDecode

# Tolerances on max|gpu - oracle| / max|oracle| per output tensor: 1e-5 for
# the fp32 configuration, 2e-2 for bf16 storage with fp32 accumulation.
TOL = {"f32": 1e-5, "bf16": 2e-2}


def f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def weights_of(inp):
    return {k: getattr(inp, k) for k in
            ("w_q_a", "g_q_a", "w_q_b", "w_q", "w_kv_a", "g_kv_a", "w_kv_b",
             "w_o")}


def run_prefill(cfg, inp, latent=True):
    B, T = inp.B, inp.T
    layer = MlaPrefill(cfg, weights_of(inp), B, T)
    x = inp.x.cuda()
    cache = (torch.empty(B * T, cfg.kv_lora_rank + cfg.qk_rope_head_dim,
                         dtype=layer.dtype, device="cuda") if latent else None)
    out = layer(x, latent_cache_out=cache)
    torch.cuda.synchronize()
    layer.check_status()
    return layer, out, cache


def sample_rows(T, n=64, seed=0):
    g = np.random.default_rng(seed)
    k = min(T, n)
    edge = min(T, k // 4)
    rows = set(range(edge)) | set(range(T - edge, T))
    rest = [r for r in range(T) if r not in rows]
    need = k - len(rows)
    if need > 0 and rest:
        rows |= set(g.choice(rest, size=min(need, len(rest)), replace=False).tolist())
    return np.array(sorted(rows))


def run_decode(cfg, di, max_ctx, with_o=False):
    B = di.q_nope.shape[0]
    dec = MlaDecode(cfg, B, max_ctx)
    H = cfg.hidden_size if with_o else cfg.num_heads * cfg.v_head_dim
    out = torch.empty(B, H, dtype=dec.dtype, device="cuda")
    dec(di.q_nope.cuda(), di.q_pe.cuda(), di.w_kv_b.cuda(), di.cache.cuda(),
        di.cu_ctx.cuda(), out, di.w_o.cuda() if with_o else None)
    torch.cuda.synchronize()
    dec.check_status()
    return dec, out


def run_prefill_chunked(cfg, inp, past, T_past):
    """mla_prefill_chunked on the new tokens of ``inp`` after ``past``
    ([B, T_past, r + rope] on the host, or None)."""
    from latent_attention_b200 import (make_config, mla_build_rope_tables,
                                       mla_prefill_chunked,
                                       mla_prefill_chunked_workspace_size)
    B, T = inp.B, inp.T
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    c = make_config(cfg)
    d = cfg.qk_rope_head_dim
    cos = torch.empty(T_past + T, d, device="cuda")
    sin = torch.empty_like(cos)
    mla_build_rope_tables(c, T_past + T, cos, sin)
    n, lay = mla_prefill_chunked_workspace_size(c, B, T, T_past)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.empty(B, T, cfg.hidden_size, dtype=dt, device="cuda")
    cache = torch.empty(B * T, cfg.kv_lora_rank + d, dtype=dt, device="cuda")
    w = {k: (None if v is None else v.cuda()) for k, v in weights_of(inp).items()}
    mla_prefill_chunked(c, w, inp.x.cuda(), B, T,
                        None if past is None else past.cuda().contiguous(), T_past,
                        cos, sin, out, ws, latent_cache_out=cache)
    torch.cuda.synchronize()
    from latent_attention_b200 import mla_check_device_status
    mla_check_device_status(ws)
    return out, cache, ws, lay


def run_prefill_varlen(cfg, inp, cu, max_len, check=True):
    """mla_prefill_varlen on packed inputs (inp.B == 1, inp.T == total)."""
    from latent_attention_b200 import (make_config, mla_build_rope_tables,
                                       mla_prefill_varlen,
                                       mla_prefill_varlen_workspace_size,
                                       mla_check_device_status)
    total, n_seq = inp.T, len(cu) - 1
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    c = make_config(cfg)
    d = cfg.qk_rope_head_dim
    cos = torch.empty(max_len, d, device="cuda")
    sin = torch.empty_like(cos)
    mla_build_rope_tables(c, max_len, cos, sin)
    n, lay = mla_prefill_varlen_workspace_size(c, n_seq, total, max_len)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.empty(total, cfg.hidden_size, dtype=dt, device="cuda")
    cache = torch.empty(total, cfg.kv_lora_rank + d, dtype=dt, device="cuda")
    w = {k: (None if v is None else v.cuda()) for k, v in weights_of(inp).items()}
    mla_prefill_varlen(c, w, inp.x.reshape(total, -1).cuda(), cu.cuda(), n_seq, total, max_len,
                       cos, sin, out, ws, latent_cache_out=cache)
    torch.cuda.synchronize()
    if check:
        mla_check_device_status(ws)
    return out, cache, ws
