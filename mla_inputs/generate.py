"""Seeded input generators (CPU, torch.Generator), shared by GPU path and oracle.

Every tensor is drawn in fp32 from one ``torch.Generator`` and then rounded to
the configuration dtype, so that the CUDA path and the oracle (which casts the
same rounded tensors to fp64) see identical values.  Distributions follow the
workload statements: weights N(0, 0.02), activations N(0, 1), RMSNorm gains 1
(or, for extra coverage in tests, U(0.5, 1.5)), decode context lengths uniform
over an inclusive integer range, latent cache N(0, 1).

Weights use the ``nn.Linear`` layout ``[out_features, in_features]`` (the
MiniMind attention page, section 2: the stored weight is [out, in] and the
forward computes x W^T).
"""
from dataclasses import dataclass
from typing import Optional

import torch

from .configs import MlaConfig

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, std, dtype):
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


@dataclass
class PrefillInputs:
    x: torch.Tensor                 # [B, T, hidden]
    w_q_a: Optional[torch.Tensor]   # [q_lora_rank, hidden]           (lora)
    g_q_a: Optional[torch.Tensor]   # [q_lora_rank]                   (lora)
    w_q_b: Optional[torch.Tensor]   # [heads*qk_head_dim, q_lora_rank] (lora)
    w_q: Optional[torch.Tensor]     # [heads*qk_head_dim, hidden]     (direct)
    w_kv_a: torch.Tensor            # [kv_lora_rank+rope, hidden]
    g_kv_a: torch.Tensor            # [kv_lora_rank]
    w_kv_b: torch.Tensor            # [heads*(nope+v), kv_lora_rank]
    w_o: torch.Tensor               # [hidden, heads*v_head_dim]
    B: int
    T: int


def make_prefill_inputs(cfg: MlaConfig, B: int, T: int, seed: int = 0,
                        gamma: str = "ones", w_std: float = 0.02,
                        x_std: float = 1.0) -> PrefillInputs:
    dt = _DT[cfg.dtype]
    g = _gen(seed)
    H, h = cfg.hidden_size, cfg.num_heads
    dq = cfg.qk_nope_head_dim + cfg.qk_rope_head_dim
    x = _randn(g, (B, T, H), x_std, dt)
    if cfg.q_lora_rank > 0:
        w_q_a = _randn(g, (cfg.q_lora_rank, H), w_std, dt)
        w_q_b = _randn(g, (h * dq, cfg.q_lora_rank), w_std, dt)
        w_q = None
    else:
        w_q_a = w_q_b = None
        w_q = _randn(g, (h * dq, H), w_std, dt)
    w_kv_a = _randn(g, (cfg.kv_lora_rank + cfg.qk_rope_head_dim, H), w_std, dt)
    w_kv_b = _randn(g, (h * (cfg.qk_nope_head_dim + cfg.v_head_dim),
                        cfg.kv_lora_rank), w_std, dt)
    w_o = _randn(g, (H, h * cfg.v_head_dim), w_std, dt)

    def gain(n):
        if gamma == "ones":
            return torch.ones(n, dtype=dt)
        if gamma == "random":
            return (0.5 + torch.rand(n, generator=g, dtype=torch.float32)).to(dt)
        raise ValueError(gamma)

    g_q_a = gain(cfg.q_lora_rank) if cfg.q_lora_rank > 0 else None
    g_kv_a = gain(cfg.kv_lora_rank)
    return PrefillInputs(x, w_q_a, g_q_a, w_q_b, w_q, w_kv_a, g_kv_a, w_kv_b,
                         w_o, B, T)


def varlen_seq_lengths(n_seq: int, len_min: int, len_max: int,
                       seed: int = 0) -> torch.Tensor:
    """Lengths of packed prefill sequences, uniform on [len_min, len_max]."""
    g = _gen(seed + 6007)
    return torch.randint(len_min, len_max + 1, (n_seq,), generator=g,
                         dtype=torch.int64).to(torch.int32)


def make_varlen_inputs(cfg: MlaConfig, seq_lengths, seed: int = 0,
                       gamma: str = "ones"):
    """Packed (THD) prefill inputs: the sequences' tokens back to back as one
    PrefillInputs with B = 1, T = sum(lengths), plus int32 cu_seqlens [n+1]."""
    lens = torch.as_tensor(seq_lengths, dtype=torch.int64).reshape(-1)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    inp = make_prefill_inputs(cfg, 1, int(cu[-1]), seed=seed, gamma=gamma)
    return inp, cu.to(torch.int32)


def decode_context_lengths(B: int, ctx_min: int, ctx_max: int,
                           seed: int = 0) -> torch.Tensor:
    """Per-sequence cached context lengths, uniform on [ctx_min, ctx_max]."""
    g = _gen(seed + 7919)
    return torch.randint(ctx_min, ctx_max + 1, (B,), generator=g,
                         dtype=torch.int64).to(torch.int32)


@dataclass
class DecodeInputs:
    q_nope: torch.Tensor        # [B, heads, nope]
    q_pe: torch.Tensor          # [B, heads, rope]  (already rotated)
    w_kv_b: torch.Tensor        # [heads*(nope+v), kv_lora_rank]
    cache: torch.Tensor         # [sum ctx, kv_lora_rank+rope]
    cu_ctx: torch.Tensor        # [B+1] int32 prefix sums of the lengths
    ctx: torch.Tensor           # [B] int32
    w_o: Optional[torch.Tensor] # [hidden, heads*v] or None


def make_decode_inputs(cfg: MlaConfig, B: int, ctx_lengths, seed: int = 0,
                       with_o_proj: bool = False,
                       w_std: float = 0.02) -> DecodeInputs:
    dt = _DT[cfg.dtype]
    ctx = torch.as_tensor(ctx_lengths, dtype=torch.int32).reshape(B)
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(ctx.to(torch.int64), 0)
    total = int(cu[-1])
    g = _gen(seed)
    h = cfg.num_heads
    q_nope = _randn(g, (B, h, cfg.qk_nope_head_dim), 1.0, dt)
    q_pe = _randn(g, (B, h, cfg.qk_rope_head_dim), 1.0, dt)
    w_kv_b = _randn(g, (h * (cfg.qk_nope_head_dim + cfg.v_head_dim),
                        cfg.kv_lora_rank), w_std, dt)
    cache = _randn(g, (total, cfg.kv_lora_rank + cfg.qk_rope_head_dim), 1.0, dt)
    w_o = (_randn(g, (cfg.hidden_size, h * cfg.v_head_dim), w_std, dt)
           if with_o_proj else None)
    return DecodeInputs(q_nope, q_pe, w_kv_b, cache, cu.to(torch.int32), ctx,
                        w_o)
