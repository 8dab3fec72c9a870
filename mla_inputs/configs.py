"""MLA layer configurations and the five named workloads.

Field names follow the HF-style DeepSeek-V3 attention module (CSDN
"DeepseekV3Attention" page, ``__init__``): hidden_size, num_attention_heads,
q_lora_rank, kv_lora_rank, qk_nope_head_dim, qk_rope_head_dim, v_head_dim,
rope_theta and rope_scaling{factor, mscale, mscale_all_dim}; the YaRN fields
beta_fast / beta_slow / original_max_position_embeddings are the Megatron-LM
MLA guide's names (section "MLA 专属参数详解").  Megatron calls the nope width
``qk_head_dim`` and the rope width ``qk_pos_emb_head_dim``; the direct-Q
workload below is stated in those names and is mapped to nope=128, rope=64.
"""
from dataclasses import dataclass, field, replace
from typing import Optional


@dataclass(frozen=True)
class MlaConfig:
    hidden_size: int
    num_heads: int
    q_lora_rank: int            # 0 means "None": a direct q_proj
    kv_lora_rank: int
    qk_nope_head_dim: int
    qk_rope_head_dim: int
    v_head_dim: int
    rope_type: str = "plain"    # "none" | "plain" | "yarn"
    rope_theta: float = 10000.0
    rope_factor: float = 1.0
    rope_mscale: float = 1.0
    rope_mscale_all_dim: float = 0.0
    beta_fast: float = 32.0
    beta_slow: float = 1.0
    original_max_position_embeddings: int = 4096
    rms_eps: float = 1e-6
    softmax_scale: Optional[float] = None   # None: derived from head dim + YaRN
    dtype: str = "bf16"                     # "bf16" | "f32"
    rope_interleave: bool = False           # rope columns as adjacent pairs

    @property
    def qk_head_dim(self) -> int:
        return self.qk_nope_head_dim + self.qk_rope_head_dim

    def with_(self, **kw) -> "MlaConfig":
        return replace(self, **kw)


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: MlaConfig
    kind: str                 # "prefill" | "decode"
    batch: int
    seq_len: int = 0          # prefill tokens per batch row
    ctx_min: int = 0          # decode: cached context length range (inclusive)
    ctx_max: int = 0
    note: str = ""
    extra: dict = field(default_factory=dict)


_DSV3 = dict(hidden_size=7168, num_heads=128, q_lora_rank=1536,
             kv_lora_rank=512, qk_nope_head_dim=128, qk_rope_head_dim=64,
             v_head_dim=128)

WORKLOADS = {
    # Tiny fp32 layer: parity at 1e-5.
    "tiny_f32": Workload(
        "tiny_f32",
        MlaConfig(hidden_size=256, num_heads=4, q_lora_rank=64,
                  kv_lora_rank=32, qk_nope_head_dim=32, qk_rope_head_dim=16,
                  v_head_dim=32, rope_type="plain", rope_theta=1e4,
                  dtype="f32"),
        "prefill", batch=1, seq_len=64),
    # DeepSeek-V3-shaped prefill with YaRN (factor 40, mscale_all_dim 1).
    "dsv3_prefill": Workload(
        "dsv3_prefill",
        MlaConfig(**_DSV3, rope_type="yarn", rope_theta=1e4, rope_factor=40.0,
                  rope_mscale=1.0, rope_mscale_all_dim=1.0, beta_fast=32.0,
                  beta_slow=1.0, original_max_position_embeddings=4096),
        "prefill", batch=1, seq_len=4096),
    # q_lora_rank=None: direct q_proj, plain RoPE.
    "directq_prefill": Workload(
        "directq_prefill",
        MlaConfig(hidden_size=4096, num_heads=32, q_lora_rank=0,
                  kv_lora_rank=512, qk_nope_head_dim=128,
                  qk_rope_head_dim=64, v_head_dim=128, rope_type="plain",
                  rope_theta=1e4),
        "prefill", batch=4, seq_len=8192),
    # Kimi-style: shared 64-dim k_pe left unrotated, scale 1/sqrt(192).
    "kimi_prefill": Workload(
        "kimi_prefill",
        MlaConfig(hidden_size=7168, num_heads=96, q_lora_rank=1536,
                  kv_lora_rank=512, qk_nope_head_dim=128,
                  qk_rope_head_dim=64, v_head_dim=128, rope_type="none"),
        "prefill", batch=1, seq_len=16384),
    # Weight-absorbed decode over the compressed latent cache.  The softmax
    # scale is the DeepSeek-V3 YaRN one (same model dimensions).
    "dsv3_decode": Workload(
        "dsv3_decode",
        MlaConfig(**_DSV3, rope_type="yarn", rope_theta=1e4, rope_factor=40.0,
                  rope_mscale=1.0, rope_mscale_all_dim=1.0,
                  original_max_position_embeddings=4096),
        "decode", batch=64, ctx_min=1024, ctx_max=32768),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]
