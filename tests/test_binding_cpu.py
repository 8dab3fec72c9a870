"""The Python binding's marshalling, on the host: every tensor is checked
against the dtype and element count that ``mla.h`` declares for its argument
before its pointer reaches the library.  The device placement check and the
library's compute entry points are replaced by fakes here (no GPU), so these
tests see exactly what the binding would pass to the C ABI."""
import pytest
import torch

import latent_attention_b200 as P
from mla_inputs import WORKLOADS, MlaConfig, make_decode_inputs, make_prefill_inputs, \
    make_varlen_inputs


class FakeLib:
    """Records every call; returns MLA_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(P._lib, "load", lambda: lib)
    # host tensors stand in for device tensors
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    return lib


def small_bf16(**kw):
    base = dict(hidden_size=256, num_heads=2, q_lora_rank=64, kv_lora_rank=128,
                qk_nope_head_dim=32, qk_rope_head_dim=16, v_head_dim=32,
                rope_type="yarn", rope_factor=40.0, rope_mscale=1.0,
                rope_mscale_all_dim=1.0, dtype="bf16")
    base.update(kw)
    return MlaConfig(**base)


def weights(inp):
    return {k: getattr(inp, k) for k in ("w_q_a", "g_q_a", "w_q_b", "w_q", "w_kv_a",
                                         "g_kv_a", "w_kv_b", "w_o")}


def _dt(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def prefill_args(cfg, B=2, T=24):
    inp = make_prefill_inputs(cfg, B, T, seed=3)
    d = cfg.qk_rope_head_dim
    return dict(cfg=cfg, weights=weights(inp), x=inp.x, B=B, T=T,
                rope_cos=torch.zeros(T, d), rope_sin=torch.zeros(T, d),
                out=torch.empty(B, T, cfg.hidden_size, dtype=_dt(cfg)),
                workspace=torch.empty(4096, dtype=torch.uint8),
                latent_cache_out=torch.empty(B * T, cfg.kv_lora_rank + d, dtype=_dt(cfg)),
                stream=0)


def decode_args(cfg, ctx=(5, 9, 1), with_o=False):
    di = make_decode_inputs(cfg, len(ctx), list(ctx), seed=4, with_o_proj=with_o)
    B = len(ctx)
    H = cfg.hidden_size if with_o else cfg.num_heads * cfg.v_head_dim
    return dict(cfg=cfg, q_nope=di.q_nope, q_pe=di.q_pe, w_kv_b=di.w_kv_b,
                latent_cache=di.cache, cu_ctx=di.cu_ctx, B=B, max_ctx=max(ctx),
                w_o=di.w_o if with_o else None, out=torch.empty(B, H, dtype=_dt(cfg)),
                workspace=torch.empty(4096, dtype=torch.uint8), stream=0)


@pytest.mark.parametrize("cfg", [WORKLOADS["tiny_f32"].cfg, small_bf16(),
                                 small_bf16(q_lora_rank=0, rope_type="none")],
                         ids=["tiny_f32", "bf16_lora_yarn", "bf16_directq_norope"])
def test_declared_shapes_pass_through(fake, cfg):
    a = prefill_args(cfg)
    P.mla_prefill_forward(**a)
    name, args = fake.calls[-1]
    assert name == "mla_prefill_forward"
    assert args[2].value == a["x"].data_ptr() and args[3] == 2 and args[4] == 24
    assert args[10].value == 4096                     # workspace bytes
    w = args[1]._obj
    assert (w.w_q is None) == bool(cfg.q_lora_rank) and w.w_o == a["weights"]["w_o"].data_ptr()

    P.mla_build_rope_tables(cfg, 24, a["rope_cos"], a["rope_sin"], stream=0)
    assert fake.calls[-1][0] == "mla_build_rope_tables"

    d = cfg.qk_rope_head_dim
    past = torch.zeros(2, 7, cfg.kv_lora_rank + d, dtype=_dt(cfg))
    cos31 = torch.zeros(31, d)
    P.mla_prefill_chunked(cfg, a["weights"], a["x"], 2, 24, past, 7, cos31, cos31,
                          a["out"], a["workspace"], a["latent_cache_out"], stream=0)
    assert fake.calls[-1][0] == "mla_prefill_chunked"

    vi, cu = make_varlen_inputs(cfg, [10, 1, 13], seed=5)
    P.mla_prefill_varlen(cfg, weights(vi), vi.x.reshape(24, -1), cu, 3, 24, 13,
                         a["rope_cos"], a["rope_sin"], a["out"], a["workspace"],
                         a["latent_cache_out"], stream=0)
    assert fake.calls[-1][0] == "mla_prefill_varlen"


@pytest.mark.parametrize("with_o", [False, True])
def test_decode_shapes_pass_through(fake, with_o):
    cfg = small_bf16()
    a = decode_args(cfg, with_o=with_o)
    P.mla_decode_absorbed(**a)
    name, args = fake.calls[-1]
    assert name == "mla_decode_absorbed" and args[6] == 3 and args[7] == 9
    assert (args[8] is None) != with_o
    a.pop("workspace")
    P.mla_decode_absorbed_noalloc(**a)
    assert fake.calls[-1][0] == "mla_decode_absorbed_noalloc"


def _shrink(t):
    return t.reshape(-1)[:-1]


PREFILL_BAD = [
    ("x", lambda a: a["x"].double(), "x must be torch.bfloat16"),
    ("x", lambda a: _shrink(a["x"]), "x holds"),
    ("out", lambda a: _shrink(a["out"]), "out holds"),
    ("out", lambda a: a["out"].float(), "out must be"),
    ("latent_cache_out", lambda a: _shrink(a["latent_cache_out"]), "latent_cache_out holds"),
    ("rope_cos", lambda a: a["rope_cos"][:-1], "rope_cos holds"),
    ("rope_sin", lambda a: a["rope_sin"].bfloat16(), "rope_sin must be torch.float32"),
]


@pytest.mark.parametrize("arg,bad,msg", PREFILL_BAD, ids=[f"{b[0]}-{i}" for i, b in
                                                          enumerate(PREFILL_BAD)])
def test_prefill_rejects_wrong_tensors(fake, arg, bad, msg):
    a = prefill_args(small_bf16())
    a[arg] = bad(a)
    with pytest.raises(ValueError, match=msg):
        P.mla_prefill_forward(**a)
    assert not fake.calls


@pytest.mark.parametrize("field", ["w_q_a", "g_q_a", "w_q_b", "w_kv_a", "g_kv_a",
                                   "w_kv_b", "w_o"])
def test_prefill_rejects_short_or_mistyped_weights(fake, field):
    a = prefill_args(small_bf16())
    w = dict(a["weights"])
    w[field] = _shrink(w[field])
    with pytest.raises(ValueError, match=f"{field} holds"):
        P.mla_prefill_forward(**{**a, "weights": w})
    w[field] = a["weights"][field].float()
    with pytest.raises(ValueError, match=f"{field} must be torch.bfloat16"):
        P.mla_prefill_forward(**{**a, "weights": w})
    assert not fake.calls


def test_chunked_and_varlen_check_their_own_extents(fake):
    cfg = small_bf16()
    a = prefill_args(cfg)
    d = cfg.qk_rope_head_dim
    past = torch.zeros(2, 7, cfg.kv_lora_rank + d, dtype=torch.bfloat16)
    # RoPE tables must reach position T_past + T_new - 1
    cos = torch.zeros(30, d)
    with pytest.raises(ValueError, match="rope_cos holds"):
        P.mla_prefill_chunked(cfg, a["weights"], a["x"], 2, 24, past, 7, cos, cos,
                              a["out"], a["workspace"])
    cos = torch.zeros(31, d)
    with pytest.raises(ValueError, match="past_cache holds"):
        P.mla_prefill_chunked(cfg, a["weights"], a["x"], 2, 24, past[:, :6], 7, cos, cos,
                              a["out"], a["workspace"])
    vi, cu = make_varlen_inputs(cfg, [10, 1, 13], seed=5)
    args = [cfg, weights(vi), vi.x.reshape(24, -1), cu, 3, 24, 13, a["rope_cos"],
            a["rope_sin"], a["out"], a["workspace"]]
    bad = list(args)
    bad[3] = cu.long()
    with pytest.raises(ValueError, match="cu_seqlens must be torch.int32"):
        P.mla_prefill_varlen(*bad)
    bad = list(args)
    bad[3] = cu[:-1]
    with pytest.raises(ValueError, match="cu_seqlens holds"):
        P.mla_prefill_varlen(*bad)
    bad = list(args)
    bad[7] = a["rope_cos"][:12]                       # max_seqlen 13 rows needed
    with pytest.raises(ValueError, match="rope_cos holds"):
        P.mla_prefill_varlen(*bad)
    assert not fake.calls


DECODE_BAD = [
    ("q_nope", lambda a: _shrink(a["q_nope"]), "q_nope holds"),
    ("q_pe", lambda a: a["q_pe"].float(), "q_pe must be"),
    ("w_kv_b", lambda a: _shrink(a["w_kv_b"]), "w_kv_b holds"),
    ("latent_cache", lambda a: _shrink(a["latent_cache"]), "whole rows"),
    ("cu_ctx", lambda a: a["cu_ctx"][:-1], "cu_ctx holds"),
    ("cu_ctx", lambda a: a["cu_ctx"].long(), "cu_ctx must be torch.int32"),
    ("out", lambda a: _shrink(a["out"]), "out holds"),
]


@pytest.mark.parametrize("arg,bad,msg", DECODE_BAD, ids=[f"{b[0]}-{i}" for i, b in
                                                         enumerate(DECODE_BAD)])
def test_decode_rejects_wrong_tensors(fake, arg, bad, msg):
    a = decode_args(small_bf16())
    a[arg] = bad(a)
    with pytest.raises(ValueError, match=msg):
        P.mla_decode_absorbed(**a)
    a.pop("workspace")
    with pytest.raises(ValueError, match=msg):
        P.mla_decode_absorbed_noalloc(**a)
    assert not fake.calls


def test_decode_output_projection_widens_out(fake):
    """With w_o the output is [B, hidden], without it [B, heads * v]."""
    cfg = small_bf16()
    a = decode_args(cfg, with_o=True)
    a["out"] = torch.empty(3, cfg.num_heads * cfg.v_head_dim, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="out holds"):
        P.mla_decode_absorbed(**a)
    a["w_o"] = _shrink(a["w_o"])
    a["out"] = torch.empty(3, cfg.hidden_size, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="w_o holds"):
        P.mla_decode_absorbed(**a)
    assert not fake.calls


def test_device_placement_is_still_required():
    """Without the fake, a host tensor never reaches the library."""
    a = prefill_args(small_bf16())
    with pytest.raises(ValueError, match="CUDA"):
        P.mla_prefill_forward(**a)
