"""Out-of-bounds writes, caught without a sanitizer: every output and the
workspace sit between guard regions filled with a known byte pattern, the
outputs themselves start as NaN, and after each call the guards must hold
their pattern bit for bit while the outputs hold no NaN (the library
overwrites every output element, as ``mla.h`` states).  Shapes have ragged
tails so that partial tiles, clamped boxes and partial heads all run."""
import pytest
import torch

import oracle
from mla_inputs import WORKLOADS as W, MlaConfig, make_decode_inputs, make_prefill_inputs, \
    make_varlen_inputs
import latent_attention_b200 as L

pytestmark = pytest.mark.gpu

GUARD = 4096                      # bytes on each side; keeps 256-byte alignment


class Guarded:
    """A tensor of ``shape`` inside a larger buffer with guard regions."""

    def __init__(self, shape, dtype, device, fill):
        es = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD // es
        self.n = 1
        for s in shape:
            self.n *= s
        self.buf = torch.full((2 * self.g + self.n,), fill, dtype=dtype, device=device)
        self.pattern = self.buf[:self.g].clone()
        self.t = self.buf[self.g:self.g + self.n].view(*shape)

    def guards_intact(self):
        a, b = self.buf[:self.g], self.buf[self.g + self.n:]
        if self.buf.dtype.is_floating_point:
            it = {2: torch.int16, 4: torch.int32}[self.buf.element_size()]
            p = self.pattern.view(it)
            return bool(torch.equal(a.view(it), p) and torch.equal(b.view(it), p))
        return bool(torch.equal(a, self.pattern) and torch.equal(b, self.pattern))


def _dt(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def small_bf16(**kw):
    """DeepSeek-V3 head dims at a small hidden size."""
    base = dict(hidden_size=512, num_heads=4, q_lora_rank=256,
                kv_lora_rank=512, qk_nope_head_dim=128, qk_rope_head_dim=64,
                v_head_dim=128, rope_type="yarn", rope_theta=1e4,
                rope_factor=40.0, rope_mscale=1.0, rope_mscale_all_dim=1.0,
                original_max_position_embeddings=4096, dtype="bf16")
    base.update(kw)
    return MlaConfig(**base)


def _weights(inp, dev):
    return {k: (None if getattr(inp, k) is None else getattr(inp, k).to(dev))
            for k in ("w_q_a", "g_q_a", "w_q_b", "w_q", "w_kv_a", "g_kv_a", "w_kv_b", "w_o")}


def _tables(cfg, rows, dev):
    cos = torch.empty(rows, cfg.qk_rope_head_dim, device=dev)
    sin = torch.empty_like(cos)
    L.mla_build_rope_tables(cfg, rows, cos, sin)
    return cos, sin


PREFILL = [
    ("tiny_f32", W["tiny_f32"].cfg, 2, 37),
    ("bf16_dsv3dims_yarn", small_bf16(), 2, 300),
    ("bf16_directq", small_bf16(q_lora_rank=0, rope_type="plain", num_heads=2), 1, 257),
    ("bf16_kimi_norope", small_bf16(rope_type="none", num_heads=3), 1, 200),
]


@pytest.mark.parametrize("name,cfg,B,T", PREFILL, ids=[p[0] for p in PREFILL])
def test_prefill_writes_stay_inside_their_buffers(cuda, name, cfg, B, T):
    inp = make_prefill_inputs(cfg, B, T, seed=71)
    dt, H = _dt(cfg), cfg.hidden_size
    w = cfg.kv_lora_rank + cfg.qk_rope_head_dim
    cos, sin = _tables(cfg, T, cuda)
    n, _ = L.mla_prefill_workspace_size(cfg, B, T)
    ws = Guarded((n,), torch.uint8, cuda, 0xA5)
    out = Guarded((B, T, H), dt, cuda, float("nan"))
    lat = Guarded((B * T, w), dt, cuda, float("nan"))
    L.mla_prefill_forward(cfg, _weights(inp, cuda), inp.x.to(cuda), B, T, cos, sin, out.t,
                          ws.t, latent_cache_out=lat.t)
    torch.cuda.synchronize()
    L.mla_check_device_status(ws.t)
    assert out.guards_intact() and lat.guards_intact() and ws.guards_intact()
    assert not torch.isnan(out.t).any() and not torch.isnan(lat.t).any()
    tol = 1e-5 if cfg.dtype == "f32" else 2e-2
    assert oracle.max_rel_err(out.t, oracle.prefill(cfg, inp)) <= tol


def test_chunked_and_varlen_writes_stay_inside_their_buffers(cuda):
    cfg = small_bf16()
    dt, H = torch.bfloat16, cfg.hidden_size
    w = cfg.kv_lora_rank + cfg.qk_rope_head_dim
    # chunked: 130 new tokens after 257 cached ones, two sequences
    B, T_new, T_past = 2, 130, 257
    inp = make_prefill_inputs(cfg, B, T_new, seed=72)
    past = torch.randn(B, T_past, w, generator=torch.Generator().manual_seed(73)).to(dt)
    cos, sin = _tables(cfg, T_past + T_new, cuda)
    n, _ = L.mla_prefill_chunked_workspace_size(cfg, B, T_new, T_past)
    ws = Guarded((n,), torch.uint8, cuda, 0xA5)
    out = Guarded((B, T_new, H), dt, cuda, float("nan"))
    lat = Guarded((B * T_new, w), dt, cuda, float("nan"))
    L.mla_prefill_chunked(cfg, _weights(inp, cuda), inp.x.to(cuda), B, T_new, past.to(cuda),
                          T_past, cos, sin, out.t, ws.t, latent_cache_out=lat.t)
    torch.cuda.synchronize()
    L.mla_check_device_status(ws.t)
    assert out.guards_intact() and lat.guards_intact() and ws.guards_intact()
    assert not torch.isnan(out.t).any() and not torch.isnan(lat.t).any()
    assert oracle.max_rel_err(out.t, oracle.prefill_chunked(cfg, inp, past, T_past)) <= 2e-2

    # varlen: packed sequences with ragged lengths
    lens = [1, 130, 300, 257, 64]
    vi, cu = make_varlen_inputs(cfg, lens, seed=74)
    total, max_len = vi.T, max(lens)
    cos, sin = _tables(cfg, max_len, cuda)
    n, _ = L.mla_prefill_varlen_workspace_size(cfg, len(lens), total, max_len)
    ws = Guarded((n,), torch.uint8, cuda, 0xA5)
    out = Guarded((total, H), dt, cuda, float("nan"))
    lat = Guarded((total, w), dt, cuda, float("nan"))
    L.mla_prefill_varlen(cfg, _weights(vi, cuda), vi.x.reshape(total, -1).to(cuda),
                         cu.to(cuda), len(lens), total, max_len, cos, sin, out.t, ws.t,
                         latent_cache_out=lat.t)
    torch.cuda.synchronize()
    L.mla_check_device_status(ws.t)
    assert out.guards_intact() and lat.guards_intact() and ws.guards_intact()
    assert not torch.isnan(out.t).any() and not torch.isnan(lat.t).any()
    assert oracle.max_rel_err(out.t, oracle.prefill_varlen(cfg, vi, cu)) <= 2e-2


@pytest.mark.parametrize("with_o", [False, True])
def test_decode_writes_stay_inside_their_buffers(cuda, with_o):
    cfg = W["dsv3_decode"].cfg
    ctx = [1, 63, 700, 4097, 130]
    B, max_ctx = len(ctx), 4097
    di = make_decode_inputs(cfg, B, ctx, seed=75, with_o_proj=with_o)
    H = cfg.hidden_size if with_o else cfg.num_heads * cfg.v_head_dim
    n, _ = L.mla_decode_workspace_size(cfg, B, max_ctx)
    ws = Guarded((n,), torch.uint8, cuda, 0xA5)
    out = Guarded((B, H), torch.bfloat16, cuda, float("nan"))
    L.mla_decode_absorbed(cfg, di.q_nope.to(cuda), di.q_pe.to(cuda), di.w_kv_b.to(cuda),
                          di.cache.to(cuda), di.cu_ctx.to(cuda), B, max_ctx,
                          di.w_o.to(cuda) if with_o else None, out.t, ws.t)
    torch.cuda.synchronize()
    L.mla_check_device_status(ws.t)
    assert out.guards_intact() and ws.guards_intact()
    assert not torch.isnan(out.t).any()
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx,
                                 w_o=di.w_o if with_o else None)
    assert oracle.max_rel_err(out.t, ref) <= 2e-2
