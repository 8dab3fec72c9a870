"""The allocation-free decode entry point against the regular one.

mla_decode_absorbed_noalloc serves callers that cannot allocate device memory
when they decode (a framework that owns every allocation, a plugin handed only
inputs and outputs, an allocation-free serving loop): it uses the library's
own static device array instead of a caller workspace.  These checks call it
through the C ABI twice in a row -- the second call reuses the array the first
one left behind -- and compare each result with mla_decode_absorbed on the
same inputs and with the fp64 oracle, at the tolerance of the other bf16
decode tests.  This file is
collected last so that a failure here leaves every other test already run.
"""
import pytest
import torch

from latent_attention_b200 import (MlaError, mla_decode_absorbed,
                                   mla_decode_absorbed_noalloc,
                                   mla_decode_workspace_size)
from latent_attention_b200._lib import DECODE_NOALLOC_SCRATCH_BYTES
from mla_inputs import WORKLOADS, make_decode_inputs
import oracle

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _inputs(cfg, ctx, seed, dev, with_o):
    di = make_decode_inputs(cfg, len(ctx), ctx, seed=seed, with_o_proj=with_o)
    return di, [t.to(dev) for t in (di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                                    di.cu_ctx)], (di.w_o.to(dev) if with_o else None)


@pytest.mark.parametrize("with_o", [False, True])
def test_noalloc_matches_workspace_entry_point(cuda, with_o):
    cfg = WORKLOADS["dsv3_decode"].cfg
    max_ctx = 4096
    cases = [([1, 700, 4096, 65], 11), ([3000, 2, 129, 1024, 64], 12)]
    for ctx, seed in cases:                       # two calls in a row
        B = len(ctx)
        di, args, w_o = _inputs(cfg, ctx, seed, cuda, with_o)
        H = cfg.hidden_size if with_o else cfg.num_heads * cfg.v_head_dim
        # the full layout may exceed the array: the array's call then runs on
        # fewer SM pairs, cut at other token positions, so the two agree to
        # rounding
        n, _ = mla_decode_workspace_size(cfg, B, max_ctx)
        ws = torch.empty(n, dtype=torch.uint8, device=cuda)
        ref = torch.empty(B, H, dtype=torch.bfloat16, device=cuda)
        got = torch.full((B, H), float("nan"), dtype=torch.bfloat16, device=cuda)
        mla_decode_absorbed(cfg, *args, B, max_ctx, w_o, ref, ws)
        mla_decode_absorbed_noalloc(cfg, *args, B, max_ctx, w_o, got)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert oracle.max_rel_err(got, ref) <= TOL
        # and both against the fp64 oracle on the same inputs
        want = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                                      di.cu_ctx, w_o=di.w_o if with_o else None)
        assert oracle.max_rel_err(got, want) <= TOL
        assert oracle.max_rel_err(ref, want) <= TOL


def test_noalloc_rejects_oversized_requests(cuda):
    cfg = WORKLOADS["dsv3_decode"].cfg
    B, max_ctx = 64, 32768                        # needs far more than the array
    n, _ = mla_decode_workspace_size(cfg, B, max_ctx)
    assert n > DECODE_NOALLOC_SCRATCH_BYTES
    h, r, dr = cfg.num_heads, cfg.kv_lora_rank, cfg.qk_rope_head_dim
    dn, dv = cfg.qk_nope_head_dim, cfg.v_head_dim
    bf = dict(dtype=torch.bfloat16, device=cuda)
    with pytest.raises(MlaError, match="MLA_ERR_WORKSPACE.*static array"):
        mla_decode_absorbed_noalloc(
            cfg, torch.empty(B, h, dn, **bf), torch.empty(B, h, dr, **bf),
            torch.empty(h * (dn + dv), r, **bf), torch.empty(1, r + dr, **bf),
            torch.zeros(B + 1, dtype=torch.int32, device=cuda), B, max_ctx, None,
            torch.empty(B, h * dv, **bf))
