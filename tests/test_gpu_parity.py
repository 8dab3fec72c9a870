"""GPU parity: the sm_100a library (through the C ABI) against the fp64 oracle
on the same seeded inputs.  Small cases compare every output element; the
full-size workloads compare sampled rows / sequences that the oracle computes
one by one.  Tolerance: max|gpu - oracle| / max|oracle| <= 1e-5 (fp32) or
2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import oracle
from mla_inputs import (MlaConfig, WORKLOADS, make_prefill_inputs,
                        make_decode_inputs, decode_context_lengths)
from gpu_helpers import TOL, f64, run_prefill, run_decode, sample_rows

pytestmark = pytest.mark.gpu

W = WORKLOADS


def small_bf16(**kw):
    """DeepSeek-V3 head dims at a small hidden size."""
    base = dict(hidden_size=512, num_heads=4, q_lora_rank=256,
                kv_lora_rank=512, qk_nope_head_dim=128, qk_rope_head_dim=64,
                v_head_dim=128, rope_type="yarn", rope_theta=1e4,
                rope_factor=40.0, rope_mscale=1.0, rope_mscale_all_dim=1.0,
                original_max_position_embeddings=4096, dtype="bf16")
    base.update(kw)
    return MlaConfig(**base)


# --------------------------------------------------------------------------
# RoPE tables
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name,max_pos", [("tiny_f32", 64), ("dsv3_prefill", 32768),
                                          ("directq_prefill", 8192),
                                          ("kimi_prefill", 16)])
def test_rope_tables(cuda, name, max_pos):
    from latent_attention_b200 import mla_build_rope_tables
    cfg = W[name].cfg
    d = cfg.qk_rope_head_dim
    cos = torch.empty(max_pos, d, device=cuda)
    sin = torch.empty_like(cos)
    mla_build_rope_tables(cfg, max_pos, cos, sin)
    torch.cuda.synchronize()
    if cfg.rope_type == "none":
        assert torch.all(cos == 1) and torch.all(sin == 0)
        return
    rc, rs = oracle.rope_tables(cfg, max_pos)
    # one fp32 rounding of an fp64 value of magnitude <= 1
    assert np.max(np.abs(f64(cos) - rc)) <= 1.2e-7
    assert np.max(np.abs(f64(sin) - rs)) <= 1.2e-7


# --------------------------------------------------------------------------
# Prefill, every element, small shapes (several tiles + ragged tails)
# --------------------------------------------------------------------------
PREFILL_SMALL = [
    ("tiny_f32", W["tiny_f32"].cfg, 1, 64, "ones"),
    ("tiny_f32_b2_ragged_gamma", W["tiny_f32"].cfg, 2, 37, "random"),
    ("tiny_f32_directq", W["tiny_f32"].cfg.with_(q_lora_rank=0), 1, 50, "ones"),
    ("tiny_f32_norope", W["tiny_f32"].cfg.with_(rope_type="none"), 1, 33, "ones"),
    ("tiny_f32_T1", W["tiny_f32"].cfg, 3, 1, "random"),
    ("bf16_dsv3dims_ragged", small_bf16(), 2, 300, "random"),
    ("bf16_directq", small_bf16(q_lora_rank=0, rope_type="plain", num_heads=2),
     1, 257, "ones"),
    ("bf16_kimi_norope", small_bf16(rope_type="none", num_heads=3), 1, 200, "ones"),
    ("bf16_T1", small_bf16(), 2, 1, "ones"),
    ("bf16_96_heads", small_bf16(num_heads=96, hidden_size=256), 1, 130, "random"),
]


@pytest.mark.parametrize("name,cfg,B,T,gamma", PREFILL_SMALL,
                         ids=[c[0] for c in PREFILL_SMALL])
def test_prefill_small(cuda, name, cfg, B, T, gamma):
    inp = make_prefill_inputs(cfg, B, T, seed=1, gamma=gamma)
    layer, out, cache = run_prefill(cfg, inp)
    ref, P = oracle.prefill(cfg, inp, return_parts=True)
    tol = TOL[cfg.dtype]
    assert oracle.max_rel_err(out, ref) <= tol
    # the latent cache handed to decode: [RMSNorm(c) | roped k_pe]
    assert oracle.max_rel_err(cache.view(B, T, -1), P["latent_cache"]) <= tol
    # intermediates: roped queries and the per-head k_nope | V
    N, h = B * T, cfg.num_heads
    dq = cfg.qk_head_dim
    q = f64(layer.view("q", (B, T, h, dq)))
    assert oracle.max_rel_err(q[..., :cfg.qk_nope_head_dim], P["q_nope"]) <= tol
    assert oracle.max_rel_err(q[..., cfg.qk_nope_head_dim:], P["q_pe"]) <= tol
    kv = f64(layer.view("kv", (B, T, h, cfg.qk_nope_head_dim + cfg.v_head_dim)))
    assert oracle.max_rel_err(kv[..., :cfg.qk_nope_head_dim], P["k_nope"]) <= tol
    assert oracle.max_rel_err(kv[..., cfg.qk_nope_head_dim:], P["v"]) <= tol
    attn = f64(layer.view("attn", (B, T, h, cfg.v_head_dim)))
    assert oracle.max_rel_err(attn, P["attn"]) <= tol


@pytest.mark.parametrize("profile", ["growing", "shrinking", "large"])
def test_prefill_softmax_range_stress(cuda, profile):
    """Inputs whose attention scores grow (or shrink) along the sequence, so
    that the running row maximum keeps increasing and the kernels must rescale
    their partial outputs, plus a case with a large score range."""
    cfg = small_bf16(q_lora_rank=0, rope_type="plain", num_heads=2)
    T = 520
    inp = make_prefill_inputs(cfg, 1, T, seed=5)
    t = torch.arange(T, dtype=torch.float32)
    f = {"growing": 1 + 6 * t / T, "shrinking": 7 - 6 * t / T,
         "large": torch.full((T,), 6.0)}[profile]
    inp.x = (inp.x.float() * f[None, :, None]).to(torch.bfloat16)
    layer, out, cache = run_prefill(cfg, inp)
    ref, P = oracle.prefill(cfg, inp, return_parts=True)
    attn = f64(layer.view("attn", (1, T, cfg.num_heads, cfg.v_head_dim)))
    assert oracle.max_rel_err(attn, P["attn"]) <= TOL["bf16"]
    assert oracle.max_rel_err(out, ref) <= TOL["bf16"]


def test_prefill_is_deterministic_and_overwrites(cuda):
    cfg = small_bf16()
    inp = make_prefill_inputs(cfg, 1, 130, seed=2)
    layer, out1, _ = run_prefill(cfg, inp)
    first = out1.clone()
    out1.fill_(float("nan"))
    layer(inp.x.cuda(), out=out1)
    torch.cuda.synchronize()
    assert torch.equal(first, out1)


# --------------------------------------------------------------------------
# Prefill at the full workload sizes: sampled rows
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["dsv3_prefill", "directq_prefill", "kimi_prefill"])
def test_prefill_full_size_sampled_rows(cuda, name):
    wl = W[name]
    cfg = wl.cfg
    inp = make_prefill_inputs(cfg, wl.batch, wl.seq_len, seed=0)
    layer, out, _ = run_prefill(cfg, inp, latent=False)
    rows = sample_rows(wl.seq_len, 48)
    bsel = [0, wl.batch - 1] if wl.batch > 1 else [0]
    sub = type(inp)(**{**inp.__dict__, "x": inp.x[bsel], "B": len(bsel)})
    ref = oracle.prefill(cfg, sub, rows=rows)
    got = out[bsel][:, torch.as_tensor(rows)]
    assert oracle.max_rel_err(got, ref) <= TOL[cfg.dtype]


@pytest.mark.parametrize("name,T", [("dsv3_prefill", 777), ("dsv3_prefill", 1000),
                                    ("directq_prefill", 1000)])
def test_prefill_ragged_rows_on_cta_pairs(cuda, name, T):
    """Row counts that are not a multiple of the 256-row tiles of the CTA-pair
    projections: at 777 rows the last tile's second CTA holds no row, at 1000
    it holds 104 of its 128."""
    cfg = W[name].cfg
    inp = make_prefill_inputs(cfg, 1, T, seed=4)
    layer, out, _ = run_prefill(cfg, inp, latent=False)
    rows = sorted(set(sample_rows(T, 24)) | {255, 256, 511, 512, 767, 768, 895, 896, T - 1})
    rows = [r for r in rows if r < T]
    ref = oracle.prefill(cfg, inp, rows=rows)
    got = out[:, torch.as_tensor(rows)]
    assert oracle.max_rel_err(got, ref) <= TOL[cfg.dtype]


def test_prefill_o_proj_on_224_column_tiles(cuda):
    """o_proj at 4096 rows and 7000 output columns (K = 8 heads x 128): 256 x
    224 pair tiles fill the last wave better than 256 x 256, so they are
    used; each tile's last 32 columns go out by direct stores, and the last
    tile column holds 56 of its 224."""
    cfg = small_bf16(num_heads=8, hidden_size=7000)
    T = 4096
    inp = make_prefill_inputs(cfg, 1, T, seed=7)
    layer, out, _ = run_prefill(cfg, inp, latent=False)
    rows = sorted(set(sample_rows(T, 16)) | {0, 127, 128, 255, 256, 3839, 3840, T - 1})
    ref = oracle.prefill(cfg, inp, rows=rows)
    got = out[:, torch.as_tensor(rows)]
    assert oracle.max_rel_err(got, ref) <= TOL[cfg.dtype]


def test_prefill_one_head_many_row_tiles(cuda):
    """One head: the kv up-projection (K = 512), the q up-projection (K = 256)
    and o_proj (K = 128) are one 256-column tile wide and 313 row tiles deep,
    so every CTA takes two or three tiles of different rows, and the last
    tile is ragged."""
    cfg = small_bf16(num_heads=1)
    T = 40000
    inp = make_prefill_inputs(cfg, 1, T, seed=6)
    layer, out, _ = run_prefill(cfg, inp, latent=False)
    rows = sorted(set(sample_rows(T, 16)) | {0, 255, 256, 511, 20479, 20480, T - 1})
    ref, P = oracle.prefill(cfg, inp, rows=rows, return_parts=True)
    got = out[:, torch.as_tensor(rows)]
    assert oracle.max_rel_err(got, ref) <= TOL[cfg.dtype]
    # every row of the kv up-projection
    kv = f64(layer.view("kv", (1, T, 1, cfg.qk_nope_head_dim + cfg.v_head_dim)))
    assert oracle.max_rel_err(kv[..., :cfg.qk_nope_head_dim], P["k_nope"]) <= TOL[cfg.dtype]
    assert oracle.max_rel_err(kv[..., cfg.qk_nope_head_dim:], P["v"]) <= TOL[cfg.dtype]


# --------------------------------------------------------------------------
# Absorbed decode
# --------------------------------------------------------------------------
DECODE_SMALL = [
    ("tiny_f32", W["tiny_f32"].cfg, [1, 7, 64, 130], 200),
    ("bf16_dsv3dims", small_bf16(), [1, 5, 300, 2049, 77], 4096),
    ("bf16_dsv3_heads", W["dsv3_decode"].cfg, [1, 1000, 33], 1024),
    # chunk (64-token) edges; sequences longer than a slice
    ("bf16_dsv3_heads_edges", W["dsv3_decode"].cfg, [63, 64, 65, 4096, 4097, 8192], 8192),
    # 96 heads (Kimi-K3 MLA): a partial 128-head tile
    ("bf16_96_heads", W["dsv3_decode"].cfg.with_(num_heads=96), [1, 128, 4100], 8192),
]


@pytest.mark.parametrize("name,cfg,ctx,max_ctx", DECODE_SMALL,
                         ids=[c[0] for c in DECODE_SMALL])
@pytest.mark.parametrize("with_o", [False, True])
def test_decode_small(cuda, name, cfg, ctx, max_ctx, with_o):
    B = len(ctx)
    di = make_decode_inputs(cfg, B, ctx, seed=3, with_o_proj=with_o)
    _, out = run_decode(cfg, di, max_ctx, with_o)
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                                 di.cu_ctx, di.w_o if with_o else None)
    assert oracle.max_rel_err(out, ref) <= TOL[cfg.dtype]


def _decode_units():
    return torch.cuda.get_device_properties(0).multi_processor_count // 2


def test_decode_many_short_sequences(cuda):
    """Each CTA pair's slice of the token stream holds many whole sequences:
    the query is reloaded per sequence and the results are final at once."""
    cfg = W["dsv3_decode"].cfg
    rng = np.random.default_rng(11)
    ctx = [int(v) for v in rng.integers(1, 100, size=300)]
    di = make_decode_inputs(cfg, len(ctx), ctx, seed=5)
    _, out = run_decode(cfg, di, 128)
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)
    assert oracle.max_rel_err(out, ref) <= TOL[cfg.dtype]


def test_decode_thousands_of_tiny_sequences(cuda):
    """Dozens of one-chunk segments per CTA pair: the query reload, the
    segment-end hand-over and the per-segment barrier phases cycle many times
    in one launch."""
    cfg = W["dsv3_decode"].cfg
    rng = np.random.default_rng(12)
    ctx = [int(v) for v in rng.integers(1, 13, size=3000)]
    di = make_decode_inputs(cfg, len(ctx), ctx, seed=9)
    _, out = run_decode(cfg, di, 12)
    picks = sorted(set(range(24)) | set(range(len(ctx) - 24, len(ctx))) |
                   set(int(v) for v in rng.integers(0, len(ctx), size=48)))
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx,
                                 batches=picks)
    assert oracle.max_rel_err(out[picks], ref) <= TOL[cfg.dtype]


def test_decode_one_sequence_over_all_units(cuda):
    """One long sequence crosses every slice: one partial per CTA pair."""
    cfg = W["dsv3_decode"].cfg
    ctx = [64 * _decode_units() * 15 + 37]
    di = make_decode_inputs(cfg, 1, ctx, seed=6)
    _, out = run_decode(cfg, di, ctx[0])
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)
    assert oracle.max_rel_err(out, ref) <= TOL[cfg.dtype]


def test_decode_sequences_on_slice_boundaries(cuda):
    """Sequences around the boundaries of the equal slices (1280 positions
    each here; every sequence is charged 288 positions before its tokens):
    one ending on a boundary, one whose tokens start on a boundary, one whose
    charge straddles a boundary, a one-token one, and one long sequence."""
    cfg = W["dsv3_decode"].cfg
    L, C = 1280, 288
    vend = [L, 3 * L - C, 3 * L + 1, 4 * L - 111, 4 * L + C - 111 + 64]
    ctx, pos = [], 0
    for e in vend:
        ctx.append(e - pos - C)
        pos = e
    ctx.append(L * _decode_units() - pos - C)
    assert min(ctx) >= 1
    di = make_decode_inputs(cfg, len(ctx), ctx, seed=7)
    _, out = run_decode(cfg, di, max(ctx))
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)
    assert oracle.max_rel_err(out, ref) <= TOL[cfg.dtype]


@pytest.mark.parametrize("units", [1, 5])
def test_decode_smaller_workspace_uses_fewer_units(cuda, units):
    """A workspace with the partial slots of only `units` SM pairs runs on that
    many pairs; one byte less than one pair's layout is refused."""
    from latent_attention_b200 import (MlaError, make_config, mla_decode_absorbed,
                                       mla_decode_workspace_size)
    cfg = W["dsv3_decode"].cfg
    ctx = [3000, 17, 5000, 640]
    B, max_ctx = len(ctx), 8192
    di = make_decode_inputs(cfg, B, ctx, seed=8)
    c = make_config(cfg)
    n, lay = mla_decode_workspace_size(c, B, max_ctx)
    slot = lay["part_lse"] - lay["part_o"]            # partial o bytes, all slots
    per_unit = 2 * slot // lay["max_splits"]
    lse_all = lay["o_lat"] - lay["part_lse"]
    # the full layout minus the slots of the pairs that are dropped (each
    # buffer rounded up to 256 bytes, so this is an upper bound)
    drop = lay["max_splits"] // 2 - units
    nbytes = n - drop * per_unit - (drop * lse_all) // (lay["max_splits"] // 2)
    ws = torch.empty(nbytes + 4096, dtype=torch.uint8, device=cuda)
    args = [t.cuda() for t in (di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)]
    out = torch.empty(B, cfg.num_heads * cfg.v_head_dim, dtype=torch.bfloat16, device=cuda)
    mla_decode_absorbed(c, *args, B, max_ctx, None, out, ws)
    torch.cuda.synchronize()
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)
    assert oracle.max_rel_err(out, ref) <= TOL[cfg.dtype]
    if units == 1:
        tiny = torch.empty(lay["part_o"] + 256, dtype=torch.uint8, device=cuda)
        with pytest.raises(MlaError, match="MLA_ERR_WORKSPACE"):
            mla_decode_absorbed(c, *args, B, max_ctx, None, out, tiny)


def test_decode_full_size_all_sequences(cuda):
    """The timed decode batch itself (the context lengths of bench.py's rank 0,
    the same slice cut), every one of its 64 sequences element by element."""
    wl = W["dsv3_decode"]
    cfg = wl.cfg
    ctx = decode_context_lengths(wl.batch, wl.ctx_min, wl.ctx_max, seed=0)
    di = make_decode_inputs(cfg, wl.batch, ctx, seed=1)
    _, out = run_decode(cfg, di, wl.ctx_max)
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                                 di.cu_ctx)
    got = out.cpu()
    for b in range(wl.batch):
        assert oracle.max_rel_err(got[b], ref[b]) <= TOL[cfg.dtype], b
    assert oracle.max_rel_err(got, ref) <= TOL[cfg.dtype]


def test_decode_bad_context_is_flagged(cuda):
    from latent_attention_b200 import MlaError
    cfg = small_bf16()
    di = make_decode_inputs(cfg, 2, [5, 9], seed=4)
    from latent_attention_b200.layer import MlaDecode
    dec = MlaDecode(cfg, 2, 8)               # max_ctx 8 < 9
    out = torch.empty(2, cfg.num_heads * cfg.v_head_dim, dtype=torch.bfloat16,
                      device=cuda)
    dec(di.q_nope.cuda(), di.q_pe.cuda(), di.w_kv_b.cuda(), di.cache.cuda(),
        di.cu_ctx.cuda(), out)
    with pytest.raises(MlaError, match="MLA_ERR_SHAPE"):
        dec.check_status()
    dec.check_status()                       # the word was cleared


def test_decode_empty_sequence_is_flagged_and_zeroed(cuda):
    """A sequence with no cached token has nothing to attend to: its output
    row is zero, the status word reports it, and the sequences around it (each
    inside one slice here) are unaffected."""
    from latent_attention_b200 import MlaError
    from latent_attention_b200.layer import MlaDecode
    cfg = W["dsv3_decode"].cfg
    di = make_decode_inputs(cfg, 3, [5, 0, 9], seed=10)
    dec = MlaDecode(cfg, 3, 16)
    out = torch.full((3, cfg.num_heads * cfg.v_head_dim), float("nan"), dtype=torch.bfloat16,
                     device=cuda)
    dec(di.q_nope.cuda(), di.q_pe.cuda(), di.w_kv_b.cuda(), di.cache.cuda(),
        di.cu_ctx.cuda(), out)
    torch.cuda.synchronize()
    with pytest.raises(MlaError, match="MLA_ERR_SHAPE"):
        dec.check_status()
    assert torch.all(out[1] == 0)
    ref = oracle.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx,
                                 batches=[0, 2])
    assert oracle.max_rel_err(out[[0, 2]], ref) <= TOL[cfg.dtype]


def test_bounded_wait_times_out_and_reports(cuda):
    """A device wait that nothing satisfies gives up after its bound, sets the
    status word, and leaves the context usable (failure detection without a
    GPU fault)."""
    import time
    from latent_attention_b200 import MlaError, mla_check_device_status, _lib
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda)
    lib = _lib.load()
    t0 = time.time()
    assert lib.mla_selftest_wait_timeout(ws.data_ptr(), None) == 0
    with pytest.raises(MlaError, match="MLA_ERR_DEVICE_TIMEOUT"):
        mla_check_device_status(ws, torch.cuda.default_stream())
    assert 1.0 < time.time() - t0 < 30.0
    mla_check_device_status(ws, torch.cuda.default_stream())     # cleared
    x = torch.ones(4, device=cuda)                               # context still fine
    assert float((x + 1).sum()) == 8.0


# --------------------------------------------------------------------------
# Chunked prefill against a cached latent
# --------------------------------------------------------------------------
CHUNKED = [
    ("tiny_f32", W["tiny_f32"].cfg, 2, 40, 25),
    ("tiny_f32_nopast", W["tiny_f32"].cfg, 1, 30, 0),
    ("bf16_dsv3dims", small_bf16(), 2, 130, 257),
    ("bf16_one_token", small_bf16(), 3, 1, 300),
    ("bf16_kimi_norope", small_bf16(rope_type="none", num_heads=3), 1, 200, 64),
    ("bf16_directq", small_bf16(q_lora_rank=0, rope_type="plain", num_heads=2),
     2, 64, 129),
]


@pytest.mark.parametrize("name,cfg,B,T_new,T_past", CHUNKED,
                         ids=[c[0] for c in CHUNKED])
def test_prefill_chunked_small(cuda, name, cfg, B, T_new, T_past):
    from gpu_helpers import run_prefill_chunked
    inp = make_prefill_inputs(cfg, B, T_new, seed=21, gamma="random")
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(22)
    past = (torch.randn(B, T_past, cfg.kv_lora_rank + cfg.qk_rope_head_dim,
                        generator=g).to(dt) if T_past else None)
    out, cache, _, _ = run_prefill_chunked(cfg, inp, past, T_past)
    ref, P = oracle.prefill_chunked(
        cfg, inp, past if past is not None else
        torch.zeros(B, 0, cfg.kv_lora_rank + cfg.qk_rope_head_dim), T_past,
        return_parts=True)
    tol = TOL[cfg.dtype]
    assert oracle.max_rel_err(out, ref) <= tol
    assert oracle.max_rel_err(cache.view(B, T_new, -1), P["new_cache"]) <= tol


def test_prefill_chunked_composes_with_prefill(cuda):
    """prefill of the first T_past tokens (its latent cache output) followed by
    a chunked prefill of the rest matches one prefill over all tokens."""
    from gpu_helpers import run_prefill_chunked
    cfg = small_bf16()
    B, T_past, T_new = 2, 200, 120
    full = make_prefill_inputs(cfg, B, T_past + T_new, seed=23)
    first = type(full)(**{**full.__dict__, "x": full.x[:, :T_past], "T": T_past})
    rest = type(full)(**{**full.__dict__, "x": full.x[:, T_past:], "T": T_new})
    _, _, cache = run_prefill(cfg, first)
    out_c, _, _, _ = run_prefill_chunked(cfg, rest, cache.view(B, T_past, -1).cpu(),
                                         T_past)
    _, out_f, _ = run_prefill(cfg, full, latent=False)
    assert oracle.max_rel_err(out_c, out_f[:, T_past:]) <= TOL["bf16"]


def test_prefill_chunked_dsv3_heads(cuda):
    from gpu_helpers import run_prefill_chunked
    cfg = W["dsv3_prefill"].cfg
    B, T_new, T_past = 1, 256, 1024
    inp = make_prefill_inputs(cfg, B, T_new, seed=24)
    g = torch.Generator().manual_seed(25)
    past = torch.randn(B, T_past, cfg.kv_lora_rank + cfg.qk_rope_head_dim,
                       generator=g).to(torch.bfloat16)
    out, _, _, _ = run_prefill_chunked(cfg, inp, past, T_past)
    ref = oracle.prefill_chunked(cfg, inp, past, T_past)
    assert oracle.max_rel_err(out, ref) <= TOL["bf16"]


# --------------------------------------------------------------------------
# Packed (THD) varlen prefill
# --------------------------------------------------------------------------
VARLEN = [
    ("tiny_f32", W["tiny_f32"].cfg, [3, 1, 40, 7]),
    ("tiny_f32_directq_norope", W["tiny_f32"].cfg.with_(q_lora_rank=0, rope_type="none"),
     [17, 2, 33]),
    ("bf16_dsv3dims", small_bf16(), [1, 130, 300, 257, 64]),
    ("bf16_kimi_norope", small_bf16(rope_type="none", num_heads=3), [200, 1, 129]),
    ("bf16_directq", small_bf16(q_lora_rank=0, rope_type="plain", num_heads=2), [256, 255, 3]),
]


@pytest.mark.parametrize("name,cfg,lens", VARLEN, ids=[v[0] for v in VARLEN])
def test_prefill_varlen_small(cuda, name, cfg, lens):
    from gpu_helpers import run_prefill_varlen
    from mla_inputs import make_varlen_inputs
    inp, cu = make_varlen_inputs(cfg, lens, seed=41, gamma="random")
    out, cache, _ = run_prefill_varlen(cfg, inp, cu, max(lens))
    ref, P = oracle.prefill_varlen(cfg, inp, cu, return_parts=True)
    tol = TOL[cfg.dtype]
    assert oracle.max_rel_err(out, ref) <= tol
    assert oracle.max_rel_err(cache, P["latent_cache"]) <= tol


def test_prefill_varlen_matches_separate_prefills(cuda):
    """Each packed sequence gives what a prefill of that sequence alone gives."""
    from gpu_helpers import run_prefill_varlen
    from mla_inputs import make_varlen_inputs
    cfg = small_bf16()
    lens = [300, 1, 129, 512]
    inp, cu = make_varlen_inputs(cfg, lens, seed=42)
    out, _, _ = run_prefill_varlen(cfg, inp, cu, max(lens))
    for b, n in enumerate(lens):
        lo, hi = int(cu[b]), int(cu[b + 1])
        one = type(inp)(**{**inp.__dict__, "x": inp.x[:, lo:hi], "T": n})
        _, o1, _ = run_prefill(cfg, one, latent=False)
        assert oracle.max_rel_err(out[lo:hi], o1[0]) <= 1e-3


def test_prefill_varlen_dsv3_heads_sampled(cuda):
    from gpu_helpers import run_prefill_varlen
    from mla_inputs import make_varlen_inputs, varlen_seq_lengths
    cfg = W["dsv3_prefill"].cfg
    lens = varlen_seq_lengths(6, 1, 700, seed=3).tolist()
    inp, cu = make_varlen_inputs(cfg, lens, seed=43)
    out, _, _ = run_prefill_varlen(cfg, inp, cu, max(lens))
    ref = oracle.prefill_varlen(cfg, inp, cu)
    assert oracle.max_rel_err(out, ref) <= TOL["bf16"]


def test_prefill_varlen_bad_cu_seqlens_is_flagged(cuda):
    """A malformed cu_seqlens (decreasing, too long) is reported through the
    status word; every access stays inside the packed rows."""
    from latent_attention_b200 import MlaError, mla_check_device_status
    from gpu_helpers import run_prefill_varlen
    from mla_inputs import make_varlen_inputs
    cfg = small_bf16()
    inp, _ = make_varlen_inputs(cfg, [50, 50], seed=44)
    bad = torch.tensor([0, 60, 20, 100], dtype=torch.int32)
    _, _, ws = run_prefill_varlen(cfg, inp, bad, 60, check=False)
    with pytest.raises(MlaError, match="SHAPE"):
        mla_check_device_status(ws)
    mla_check_device_status(ws)          # cleared; the context is still usable


# --------------------------------------------------------------------------
# rope_interleave weights
# --------------------------------------------------------------------------
INTERLEAVE = [
    ("tiny_f32", W["tiny_f32"].cfg.with_(rope_interleave=True), 2, 37),
    ("bf16_dsv3dims_yarn", small_bf16(rope_interleave=True), 2, 300),
    ("bf16_directq", small_bf16(q_lora_rank=0, rope_type="plain", num_heads=2,
                                rope_interleave=True), 1, 129),
]


@pytest.mark.parametrize("name,cfg,B,T", INTERLEAVE, ids=[c[0] for c in INTERLEAVE])
def test_prefill_rope_interleave(cuda, name, cfg, B, T):
    inp = make_prefill_inputs(cfg, B, T, seed=52, gamma="random")
    _, out, cache = run_prefill(cfg, inp)
    ref, P = oracle.prefill(cfg, inp, return_parts=True)
    tol = TOL[cfg.dtype]
    assert oracle.max_rel_err(out, ref) <= tol
    assert oracle.max_rel_err(cache.view(B, T, -1), P["latent_cache"]) <= tol


def test_varlen_and_chunked_with_rope_interleave(cuda):
    from gpu_helpers import run_prefill_varlen, run_prefill_chunked
    from mla_inputs import make_varlen_inputs
    cfg = small_bf16(rope_interleave=True)
    inp, cu = make_varlen_inputs(cfg, [70, 1, 200], seed=53)
    out, _, _ = run_prefill_varlen(cfg, inp, cu, 200)
    assert oracle.max_rel_err(out, oracle.prefill_varlen(cfg, inp, cu)) <= TOL["bf16"]
    new = make_prefill_inputs(cfg, 1, 90, seed=54)
    g = torch.Generator().manual_seed(55)
    past = torch.randn(1, 150, cfg.kv_lora_rank + cfg.qk_rope_head_dim,
                       generator=g).to(torch.bfloat16)
    out_c, _, _, _ = run_prefill_chunked(cfg, new, past, 150)
    assert oracle.max_rel_err(out_c, oracle.prefill_chunked(cfg, new, past, 150)) <= TOL["bf16"]


# --------------------------------------------------------------------------
# CUDA-graph capture: the C ABI launches only stream work with parameters
# fixed at the call, so a captured prefill / decode replays bit-identically
# --------------------------------------------------------------------------
def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
        fn()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_prefill_and_decode_replay_from_cuda_graphs(cuda):
    from latent_attention_b200.layer import MlaPrefill, MlaDecode
    from gpu_helpers import weights_of
    cfg = small_bf16()
    inp = make_prefill_inputs(cfg, 2, 300, seed=61)
    layer = MlaPrefill(cfg, weights_of(inp), 2, 300)
    x = inp.x.cuda()
    ref = layer(x).clone()
    out = torch.empty_like(ref)
    g = _capture(lambda: layer(x, out=out))
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    layer.check_status()

    dcfg = W["dsv3_decode"].cfg
    di = make_decode_inputs(dcfg, 4, [1, 700, 4097, 9000], seed=62)
    dec = MlaDecode(dcfg, 4, 9000)
    args = [t.cuda() for t in (di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)]
    dref = torch.empty(4, dcfg.num_heads * dcfg.v_head_dim, dtype=torch.bfloat16, device=cuda)
    dec(*args, dref)
    dout = torch.empty_like(dref)
    gd = _capture(lambda: dec(*args, dout))
    dout.zero_()
    gd.replay()
    torch.cuda.synchronize()
    assert torch.equal(dout, dref)
    dec.check_status()
