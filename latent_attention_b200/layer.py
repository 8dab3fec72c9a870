"""Convenience holders that keep device buffers for repeated calls.

``MlaPrefill`` and ``MlaDecode`` own the device copies of the weights, the
RoPE tables and the workspace (torch allocations), and call the C ABI.  They
do no arithmetic of their own.
"""
import torch

from . import (make_config, mla_build_rope_tables, mla_prefill_workspace_size,
               mla_prefill_forward, mla_decode_workspace_size,
               mla_decode_absorbed, mla_check_device_status)

_WEIGHT_KEYS = ("w_q_a", "g_q_a", "w_q_b", "w_q", "w_kv_a", "g_kv_a", "w_kv_b",
                "w_o")
_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


class MlaPrefill:
    def __init__(self, cfg, weights, B, T, device="cuda", max_pos=None):
        self.cfg, self.B, self.T = cfg, B, T
        self.c = make_config(cfg)
        self.dtype = _DT[cfg.dtype]
        self.device = torch.device(device)
        self.w = {}
        for k in _WEIGHT_KEYS:
            t = weights.get(k) if isinstance(weights, dict) else getattr(weights, k)
            self.w[k] = None if t is None else t.to(self.device).contiguous()
        d = cfg.qk_rope_head_dim
        mp = max_pos or T
        self.cos = torch.empty(mp, d, dtype=torch.float32, device=self.device)
        self.sin = torch.empty_like(self.cos)
        mla_build_rope_tables(self.c, mp, self.cos, self.sin)
        n, self.layout = mla_prefill_workspace_size(self.c, B, T)
        self.ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        self.out = torch.empty(B, T, cfg.hidden_size, dtype=self.dtype,
                               device=self.device)

    def __call__(self, x, out=None, latent_cache_out=None, stream=None):
        out = self.out if out is None else out
        mla_prefill_forward(self.c, self.w, x, self.B, self.T, self.cos,
                            self.sin, out, self.ws, latent_cache_out, stream)
        return out

    def view(self, name, shape, dtype=None):
        """A tensor view of a workspace intermediate (see mla_prefill_layout)."""
        off = self.layout[name]
        if off < 0:
            return None
        dt = dtype or self.dtype
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dt).element_size()
        return self.ws[off:off + nbytes].view(dt).view(*shape)

    def check_status(self, stream=None):
        mla_check_device_status(self.ws, stream)


class MlaDecode:
    def __init__(self, cfg, B, max_ctx, device="cuda"):
        self.cfg, self.B, self.max_ctx = cfg, B, max_ctx
        self.c = make_config(cfg)
        self.dtype = _DT[cfg.dtype]
        self.device = torch.device(device)
        n, self.layout = mla_decode_workspace_size(self.c, B, max_ctx)
        self.ws = torch.empty(n, dtype=torch.uint8, device=self.device)

    def __call__(self, q_nope, q_pe, w_kv_b, cache, cu_ctx, out, w_o=None,
                 stream=None):
        mla_decode_absorbed(self.c, q_nope, q_pe, w_kv_b, cache, cu_ctx,
                            self.B, self.max_ctx, w_o, out, self.ws, stream)
        return out

    def check_status(self, stream=None):
        mla_check_device_status(self.ws, stream)
