"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test names what it pins.  None of them re-derives a value by calling the
same oracle formula twice: values come from the golden closed forms, from
identities of rotations / softmax / RMS normalisation, from library routines
(torch scaled_dot_product_attention in float64) or from the loop-level brute
force in ``oracle.brute``.  The mutation tests at the end plant mistakes in the
oracle (on the CPU) and check that a pin catches each one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as O
from oracle.brute import brute_prefill
from mla_inputs import MlaConfig, WORKLOADS, make_prefill_inputs, \
    make_decode_inputs
from conftest import read_golden

GOLD = read_golden("yarn_closed_forms.txt")


def tiny_cfg(**kw):
    base = dict(hidden_size=16, num_heads=2, q_lora_rank=8, kv_lora_rank=8,
                qk_nope_head_dim=4, qk_rope_head_dim=4, v_head_dim=6,
                rope_type="plain", rope_theta=100.0, dtype="f32")
    base.update(kw)
    return MlaConfig(**base)


# --------------------------------------------------------------------------
# Softmax scale (CSDN DeepseekV3Attention __init__; Megatron 源码架构)
# --------------------------------------------------------------------------
def test_yarn_mscale_closed_form():
    m = O.yarn_get_mscale(40.0, 1.0)
    assert m == pytest.approx(GOLD["mscale_factor40_all_dim1"], rel=1e-15)
    assert m * m == pytest.approx(GOLD["mscale_sq_factor40_all_dim1"], rel=1e-15)
    assert O.yarn_get_mscale(1.0, 1.0) == 1.0        # no scaling: factor 1
    assert O.yarn_get_mscale(0.5, 3.0) == 1.0


def test_softmax_scale_per_workload():
    s2 = O.softmax_scale(WORKLOADS["dsv3_prefill"].cfg)
    assert s2 == pytest.approx(GOLD["softmax_scale_dsv3_yarn"], rel=1e-15)
    s4 = O.softmax_scale(WORKLOADS["kimi_prefill"].cfg)
    assert s4 == pytest.approx(GOLD["softmax_scale_q_head_dim_192"], rel=1e-15)
    s3 = O.softmax_scale(WORKLOADS["directq_prefill"].cfg)
    assert s3 == pytest.approx(GOLD["softmax_scale_q_head_dim_192"], rel=1e-15)
    s1 = O.softmax_scale(WORKLOADS["tiny_f32"].cfg)
    assert s1 == pytest.approx(GOLD["softmax_scale_q_head_dim_48"], rel=1e-15)
    # mscale_all_dim = 0 disables the YaRN factor (the "if mscale_all_dim" branch)
    c = WORKLOADS["dsv3_prefill"].cfg.with_(rope_mscale_all_dim=0.0)
    assert O.softmax_scale(c) == pytest.approx(GOLD["softmax_scale_q_head_dim_192"])
    assert O.softmax_scale(c.with_(softmax_scale=0.25)) == 0.25


# --------------------------------------------------------------------------
# RoPE (MiniMind section 3) and YaRN tables
# --------------------------------------------------------------------------
def test_plain_rope_table_values():
    cfg = tiny_cfg(qk_rope_head_dim=8, rope_theta=10000.0)
    cos, sin = O.rope_tables(cfg, 50)
    t = np.arange(50)
    # pair 0 has theta = base^0 = 1: the angle is the position itself
    np.testing.assert_allclose(cos[:, 0], np.cos(t), rtol=0, atol=1e-15)
    np.testing.assert_allclose(sin[:, 0], np.sin(t), rtol=0, atol=1e-15)
    # pair 3 (last) has theta = 10000^(-6/8) = 1e-3
    np.testing.assert_allclose(cos[:, 3], np.cos(t * 1e-3), atol=1e-15)
    # rotate_half layout: halves carry the same angle
    np.testing.assert_array_equal(cos[:, :4], cos[:, 4:])
    np.testing.assert_array_equal(sin[:, :4], sin[:, 4:])
    assert np.all(cos[0] == 1.0) and np.all(sin[0] == 0.0)
    np.testing.assert_allclose(cos ** 2 + sin ** 2, 1.0, atol=1e-15)


def test_rotate_half_squared_is_minus_identity():
    x = np.random.default_rng(0).standard_normal((5, 16))
    np.testing.assert_array_equal(O.rotate_half(O.rotate_half(x)), -x)
    # and it is a rotation by +90 degrees inside each (i, i+d/2) plane
    y = O.rotate_half(x)
    np.testing.assert_array_equal(y[:, :8], -x[:, 8:])
    np.testing.assert_array_equal(y[:, 8:], x[:, :8])


def test_rope_preserves_norm_and_is_relative():
    cfg = tiny_cfg(qk_rope_head_dim=16, rope_theta=10000.0)
    cos, sin = O.rope_tables(cfg, 300)
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    for t in (0, 7, 299):
        np.testing.assert_allclose(
            np.linalg.norm(O.apply_rope(q, cos[t], sin[t])), np.linalg.norm(q),
            rtol=1e-14)

    def dot(t, u):
        return O.apply_rope(q, cos[t], sin[t]) @ O.apply_rope(k, cos[u], sin[u])
    # <R_t q, R_u k> depends only on t - u
    for (t, u, t2, u2) in [(10, 3, 107, 100), (5, 5, 250, 250), (0, 9, 40, 49)]:
        assert dot(t, u) == pytest.approx(dot(t2, u2), rel=1e-12, abs=1e-12)
    # and R_0 is the identity
    np.testing.assert_array_equal(O.apply_rope(q, cos[0], sin[0]), q)


def test_yarn_factor_one_equals_plain():
    y = WORKLOADS["dsv3_prefill"].cfg.with_(rope_factor=1.0)
    p = y.with_(rope_type="plain")
    cy, sy = O.rope_tables(y, 2000)
    cp, sp = O.rope_tables(p, 2000)
    # (1 - r) theta + r theta / 1 equals theta up to one rounding
    np.testing.assert_allclose(cy, cp, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sy, sp, rtol=0, atol=1e-12)


def test_yarn_ramp_end_points():
    cfg = WORKLOADS["dsv3_prefill"].cfg
    plain = cfg.with_(rope_type="plain")
    th_y, mag = O.rope_frequencies(cfg)
    th_p, mag_p = O.rope_frequencies(plain)
    lo, hi = int(GOLD["yarn_lo_dsv3"]), int(GOLD["yarn_hi_dsv3"])
    assert math.floor(GOLD["corr_dim_beta32"]) == lo
    assert math.ceil(GOLD["corr_dim_beta1"]) == hi
    # dims at or below lo keep the original frequency, dims at or above hi are
    # interpolated by the factor s = 40, and the ramp is linear in between
    np.testing.assert_array_equal(th_y[:lo + 1], th_p[:lo + 1])
    np.testing.assert_allclose(th_y[hi:], th_p[hi:] / 40.0, rtol=1e-15)
    i = 16
    ramp = (i - lo) / (hi - lo)
    assert th_y[i] == pytest.approx(th_p[i] * (1 - ramp + ramp / 40.0), rel=1e-14)
    assert np.all(np.diff(th_y) < 0)
    # mscale == mscale_all_dim -> cos/sin magnitude 1
    assert mag == 1.0 and mag_p == 1.0
    # a magnitude other than 1 is the ratio of the two mscales
    c2 = cfg.with_(rope_mscale=1.0, rope_mscale_all_dim=0.0)
    assert O.rope_frequencies(c2)[1] == pytest.approx(
        GOLD["mscale_factor40_all_dim1"], rel=1e-15)


# --------------------------------------------------------------------------
# RMSNorm (Kimi rmsnorm, MiniMind section 3)
# --------------------------------------------------------------------------
def test_rms_norm_identities():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 33)) * 3.0
    y = O.rms_norm(x, None, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, -1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.rms_norm(5.0 * x, None, 0.0), y, rtol=1e-14)
    g = rng.uniform(0.5, 1.5, 33)
    np.testing.assert_allclose(O.rms_norm(x, g, 0.0), y * g, rtol=1e-14)
    # eps keeps the zero vector finite
    assert np.all(O.rms_norm(np.zeros((1, 4)), None, 1e-6) == 0.0)
    # library routine
    t = torch.from_numpy(x)
    ref = torch.nn.functional.rms_norm(t, (33,), torch.from_numpy(g), eps=1e-6)
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), ref.numpy(), rtol=1e-13)


# --------------------------------------------------------------------------
# Whole forward against the loop-level brute force (FA2 pad/trim route)
# --------------------------------------------------------------------------
BRUTE_CASES = [
    ("lora_plain", tiny_cfg(), 1, 5, "ones"),
    ("lora_plain_gamma_b2", tiny_cfg(), 2, 4, "random"),
    ("direct_q", tiny_cfg(q_lora_rank=0), 1, 5, "ones"),
    ("no_rotary", tiny_cfg(rope_type="none"), 2, 3, "random"),
    ("v_eq_dq", tiny_cfg(v_head_dim=8), 1, 4, "ones"),
]


@pytest.mark.parametrize("name,cfg,B,T,gamma", BRUTE_CASES,
                         ids=[c[0] for c in BRUTE_CASES])
def test_prefill_matches_brute_force(name, cfg, B, T, gamma):
    inp = make_prefill_inputs(cfg, B, T, seed=3, gamma=gamma, w_std=0.3)
    got = O.prefill(cfg, inp)
    ref = np.array(brute_prefill(cfg, inp, O.softmax_scale(cfg)))
    assert got.shape == ref.shape
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_attention_core_matches_library_sdpa():
    cfg = tiny_cfg(num_heads=3, qk_nope_head_dim=8, qk_rope_head_dim=8,
                   v_head_dim=4)
    inp = make_prefill_inputs(cfg, 2, 9, seed=4, w_std=0.4)
    _, P = O.prefill(cfg, inp, return_parts=True)
    q = torch.from_numpy(np.concatenate([P["q_nope"], P["q_pe"]], -1))
    kpe = np.broadcast_to(P["k_pe"][:, :, None, :], P["k_nope"].shape[:3] + (8,))
    k = torch.from_numpy(np.concatenate([P["k_nope"], kpe], -1))
    v = torch.from_numpy(np.ascontiguousarray(P["v"]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
        is_causal=True, scale=P["scale"]).transpose(1, 2)
    np.testing.assert_allclose(P["attn"], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_softmax_rows_sum_to_one_and_are_causal():
    cfg = tiny_cfg()
    inp = make_prefill_inputs(cfg, 2, 6, seed=5, w_std=0.5)
    _, P = O.prefill(cfg, inp, return_probs=True)
    p = P["probs"]
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.triu(np.ones((6, 6)), 1)[None, None] * p == 0)


def test_causality_perturbation():
    cfg = tiny_cfg()
    inp = make_prefill_inputs(cfg, 1, 8, seed=6, w_std=0.4)
    base = O.prefill(cfg, inp)
    j = 5
    x2 = inp.x.clone()
    x2[0, j] += 1.0
    inp2 = type(inp)(**{**inp.__dict__, "x": x2})
    pert = O.prefill(cfg, inp2)
    np.testing.assert_array_equal(base[0, :j], pert[0, :j])   # exactly
    assert np.max(np.abs(base[0, j:] - pert[0, j:])) > 1e-6


def test_single_token_returns_its_value():
    cfg = tiny_cfg()
    inp = make_prefill_inputs(cfg, 3, 1, seed=7, w_std=0.4)
    _, P = O.prefill(cfg, inp, return_parts=True)
    np.testing.assert_allclose(P["attn"][:, 0], P["v"][:, 0], rtol=1e-14)


def test_zero_query_gives_prefix_mean_of_values():
    cfg = tiny_cfg()
    inp = make_prefill_inputs(cfg, 1, 7, seed=8, w_std=0.4)
    inp.w_q_b.zero_()                         # q = 0 -> all scores equal
    _, P = O.prefill(cfg, inp, return_parts=True)
    v = P["v"][0]
    means = np.cumsum(v, axis=0) / np.arange(1, 8)[:, None, None]
    np.testing.assert_allclose(P["attn"][0], means, rtol=1e-13, atol=1e-14)


def test_row_subset_matches_full():
    cfg = tiny_cfg()
    inp = make_prefill_inputs(cfg, 2, 9, seed=9, w_std=0.4)
    full = O.prefill(cfg, inp)
    rows = [0, 4, 8]
    np.testing.assert_allclose(O.prefill(cfg, inp, rows=rows), full[:, rows],
                               rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# Decode (Megatron 推理优化): absorbed == explicit == last prefill row
# --------------------------------------------------------------------------
def test_decode_absorbed_equals_unabsorbed():
    cfg = tiny_cfg(num_heads=3, kv_lora_rank=12, qk_rope_head_dim=4)
    di = make_decode_inputs(cfg, 4, [1, 5, 9, 2], seed=10, with_o_proj=True,
                            w_std=0.3)
    for w_o in (None, di.w_o):
        a = O.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                              di.cu_ctx, w_o)
        u = O.decode_unabsorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                                di.cu_ctx, w_o)
        np.testing.assert_allclose(a, u, rtol=1e-10, atol=1e-12)


def test_decode_single_token_context_returns_value():
    cfg = tiny_cfg(num_heads=2, kv_lora_rank=8)
    di = make_decode_inputs(cfg, 2, [1, 1], seed=11, w_std=0.3)
    got = O.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                            di.cu_ctx)
    W = di.w_kv_b.double().numpy().reshape(2, 10, 8)
    C = di.cache.double().numpy()
    for b in range(2):
        for h in range(2):
            v = W[h, 4:, :] @ C[b, :8]
            np.testing.assert_allclose(got[b, h * 6:(h + 1) * 6], v, rtol=1e-13)


@pytest.mark.parametrize("rope", ["plain", "none"])
def test_decode_matches_last_prefill_row(rope):
    cfg = tiny_cfg(rope_type=rope, num_heads=3)
    T = 7
    inp = make_prefill_inputs(cfg, 1, T, seed=12, w_std=0.4)
    out, P = O.prefill(cfg, inp, return_parts=True)
    cache = P["latent_cache"][0]                          # [T, r_kv + dr]
    cu = torch.tensor([0, T], dtype=torch.int32)
    q_nope = P["q_nope"][0, -1][None]                     # [1, h, dn]
    q_pe = P["q_pe"][0, -1][None]                         # roped
    o = O.decode_absorbed(cfg, q_nope, q_pe, inp.w_kv_b, cache, cu)
    np.testing.assert_allclose(o[0], P["attn"][0, -1].reshape(-1), rtol=1e-11)
    o2 = O.decode_unabsorbed(cfg, q_nope, q_pe, inp.w_kv_b, cache, cu,
                             w_o=inp.w_o)
    np.testing.assert_allclose(o2[0], out[0, -1], rtol=1e-11, atol=1e-13)


def test_decode_library_sdpa():
    cfg = tiny_cfg(num_heads=2, kv_lora_rank=8)
    di = make_decode_inputs(cfg, 3, [3, 6, 4], seed=13, w_std=0.3)
    got = O.decode_unabsorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache,
                              di.cu_ctx)
    W = di.w_kv_b.double().reshape(2, 10, 8)
    C = di.cache.double()
    cu = di.cu_ctx.tolist()
    for b in range(3):
        c, kpe = C[cu[b]:cu[b + 1], :8], C[cu[b]:cu[b + 1], 8:]
        for h in range(2):
            k = torch.cat([c @ W[h, :4].T, kpe], -1)[None, None]
            v = (c @ W[h, 4:].T)[None, None]
            q = torch.cat([di.q_nope[b, h].double(), di.q_pe[b, h].double()])
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[None, None, None], k, v, scale=O.softmax_scale(cfg))
            np.testing.assert_allclose(got[b, h * 6:(h + 1) * 6],
                                       ref.reshape(-1).numpy(), rtol=1e-12)


# --------------------------------------------------------------------------
# Planted mistakes: each must make some pin above fail.
# --------------------------------------------------------------------------
def _brute_gap(cfg, B=1, T=4):
    inp = make_prefill_inputs(cfg, B, T, seed=14, gamma="random", w_std=0.3)
    got = O.prefill(cfg, inp)
    ref = np.array(brute_prefill(cfg, inp, O.softmax_scale(cfg)))
    return float(np.max(np.abs(got - ref)))


MUTANTS = {
    "rotate_half_sign": ("rotate_half",
                         lambda x: np.concatenate([x[..., x.shape[-1] // 2:],
                                                   -x[..., :x.shape[-1] // 2]], -1)),
    "rms_missing_mean": ("rms_norm",
                         lambda x, g, eps: x / np.sqrt(np.sum(x * x, -1,
                                                              keepdims=True) + eps) * g),
    "rope_not_applied": ("apply_rope", lambda x, c, s: x),
    "softmax_no_shift_wrong_axis": ("_softmax_rows",
                                    lambda s: np.nan_to_num(np.exp(s)) /
                                    np.sum(np.nan_to_num(np.exp(s)), 0, keepdims=True)),
}


@pytest.mark.parametrize("mut", sorted(MUTANTS))
def test_planted_mistake_is_caught(monkeypatch, mut):
    assert _brute_gap(tiny_cfg()) < 1e-10
    attr, fn = MUTANTS[mut]
    monkeypatch.setattr(O, attr, fn)
    assert _brute_gap(tiny_cfg()) > 1e-6


def test_planted_scale_mistake_is_caught(monkeypatch):
    # a wrong YaRN scale (mscale not squared) breaks the golden closed form
    monkeypatch.setattr(O, "yarn_get_mscale",
                        lambda s, a: math.sqrt(0.1 * a * math.log(s) + 1)
                        if s > 1 else 1.0)
    s2 = O.softmax_scale(WORKLOADS["dsv3_prefill"].cfg)
    assert abs(s2 - GOLD["softmax_scale_dsv3_yarn"]) > 1e-3


def test_planted_absorption_mistake_is_caught(monkeypatch):
    # using the V rows of kv_b as W_UK (wrong split) breaks absorbed == explicit
    cfg = tiny_cfg(num_heads=2, kv_lora_rank=8, v_head_dim=4)
    di = make_decode_inputs(cfg, 2, [3, 4], seed=15, w_std=0.3)
    orig = O._split_kv_b
    monkeypatch.setattr(O, "_split_kv_b",
                        lambda c, w: (orig(c, w)[1], orig(c, w)[1]))
    a = O.decode_absorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)
    monkeypatch.setattr(O, "_split_kv_b", orig)
    u = O.decode_unabsorbed(cfg, di.q_nope, di.q_pe, di.w_kv_b, di.cache, di.cu_ctx)
    assert np.max(np.abs(a - u)) > 1e-6


# --------------------------------------------------------------------------
# Chunked prefill against a cached latent (Megatron 推理优化 uncompress;
# MiniMind section 5: history keys fully visible, new block causal)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("rope", ["plain", "none"])
@pytest.mark.parametrize("T_past,T_new", [(0, 5), (3, 4), (6, 1)])
def test_chunked_prefill_equals_full_prefill_rows(rope, T_past, T_new):
    cfg = tiny_cfg(rope_type=rope)
    full = make_prefill_inputs(cfg, 2, T_past + T_new, seed=16, gamma="random",
                               w_std=0.4)
    out_full, P = O.prefill(cfg, full, return_parts=True)
    past = P["latent_cache"][:, :T_past]
    new = type(full)(**{**full.__dict__, "x": full.x[:, T_past:], "T": T_new})
    out, Q = O.prefill_chunked(cfg, new, past, T_past, return_parts=True)
    np.testing.assert_allclose(out, out_full[:, T_past:], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(Q["new_cache"], P["latent_cache"][:, T_past:],
                               rtol=1e-12, atol=1e-14)


def test_chunked_prefill_sees_all_history():
    # with zero queries every visible key has equal weight: the output of
    # new token i is the mean of V over positions 0 .. T_past + i
    cfg = tiny_cfg(q_lora_rank=0)
    T_past, T_new = 4, 3
    full = make_prefill_inputs(cfg, 1, T_past + T_new, seed=17, w_std=0.4)
    full.w_q.zero_()
    _, P = O.prefill(cfg, full, return_parts=True)
    new = type(full)(**{**full.__dict__, "x": full.x[:, T_past:], "T": T_new})
    _, Q = O.prefill_chunked(cfg, new, P["latent_cache"][:, :T_past], T_past,
                             return_parts=True)
    v = P["v"][0]
    for i in range(T_new):
        np.testing.assert_allclose(Q["attn"][0, i], v[:T_past + i + 1].mean(0),
                                   rtol=1e-12, atol=1e-14)


CHUNK_MISTAKES = {
    # new tokens placed at positions 0.. instead of after the history (their
    # RoPE angles and their causal mask both shift)
    "positions_not_offset": ("_chunk_positions", lambda T_past, T_new: np.arange(T_new)),
    # the history's latent rows lost
    "history_zeroed": ("_chunk_latent",
                       lambda past, new: np.concatenate([np.zeros_like(past), new], 1)),
    # the cached latents (kv_lora_rank 8 in tiny_cfg) normalised a second
    # time: they are stored normalised, with the gain applied
    "history_normalised_again": ("_chunk_latent", lambda past, new: np.concatenate(
        [np.concatenate([O.rms_norm(past[..., :8], np.ones(8), 1e-6), past[..., 8:]], -1),
         new], 1)),
}


@pytest.mark.parametrize("mistake", sorted(CHUNK_MISTAKES))
def test_planted_chunked_mistake_is_caught(monkeypatch, mistake):
    attr, fn = CHUNK_MISTAKES[mistake]
    monkeypatch.setattr(O, attr, fn)
    with pytest.raises(AssertionError):
        test_chunked_prefill_equals_full_prefill_rows("plain", 3, 4)


# --------------------------------------------------------------------------
# Packed (THD) prefill (Megatron 训练支持与并行策略: cu_seqlens packing)
# --------------------------------------------------------------------------
def _sequence_inputs(inp, lo, hi):
    """PrefillInputs of packed rows lo..hi-1 as one B=1 sequence."""
    return type(inp)(**{**inp.__dict__, "x": inp.x[:, lo:hi], "T": hi - lo})


@pytest.mark.parametrize("rope,q_lora", [("plain", 8), ("none", 0)])
def test_varlen_prefill_equals_brute_force_per_sequence(rope, q_lora):
    # packed with a block-diagonal causal mask vs the loop-level brute force
    # run on every sequence separately (positions restart at 0)
    from mla_inputs import make_varlen_inputs
    cfg = tiny_cfg(rope_type=rope, q_lora_rank=q_lora)
    lens = [3, 1, 6, 2]
    inp, cu = make_varlen_inputs(cfg, lens, seed=31, gamma="random")
    out, P = O.prefill_varlen(cfg, inp, cu, return_parts=True)
    scale = O.softmax_scale(cfg)
    r = cfg.kv_lora_rank
    kva = inp.x[0].double().numpy() @ inp.w_kv_a.double().numpy().T
    for b in range(len(lens)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        ref = np.asarray(brute_prefill(cfg, _sequence_inputs(inp, lo, hi), scale))[0]
        np.testing.assert_allclose(out[lo:hi], ref, rtol=1e-10, atol=1e-12)
        # the first token of every sequence sits at position 0: its cached
        # k_pe is unrotated (R_0 = I)
        np.testing.assert_allclose(P["latent_cache"][lo, r:], kva[lo, r:],
                                   rtol=1e-12, atol=1e-14)


def test_varlen_prefill_single_sequence_is_prefill_and_one_token_is_v():
    from mla_inputs import make_varlen_inputs
    cfg = tiny_cfg()
    inp, cu = make_varlen_inputs(cfg, [7], seed=32)
    np.testing.assert_allclose(O.prefill_varlen(cfg, inp, cu), O.prefill(cfg, inp)[0],
                               rtol=1e-12, atol=1e-14)
    # a one-token sequence attends only to itself: its attention output is its
    # own V = RMSNorm(c) W_UV, per head
    inp, cu = make_varlen_inputs(cfg, [4, 1, 3], seed=33)
    _, P = O.prefill_varlen(cfg, inp, cu, return_parts=True)
    m = int(cu[1])
    h, dn, dv, r = cfg.num_heads, cfg.qk_nope_head_dim, cfg.v_head_dim, cfg.kv_lora_rank
    wkvb = inp.w_kv_b.double().numpy().reshape(h, dn + dv, r)
    c_hat = P["latent_cache"][m, :r]
    for hh in range(h):
        np.testing.assert_allclose(P["attn"][m, hh], wkvb[hh, dn:] @ c_hat,
                                   rtol=1e-12, atol=1e-14)
    assert P["pos"].tolist() == [0, 1, 2, 3, 0, 0, 1, 2]


@pytest.mark.parametrize("mistake", ["no_boundaries", "positions_not_restarted"])
def test_planted_varlen_mistake_is_caught(monkeypatch, mistake):
    orig = O._packed_rows

    def wrong(cu, N):
        seq, pos = orig(cu, N)
        if mistake == "no_boundaries":
            return np.zeros_like(seq), pos
        return seq, np.arange(N)
    monkeypatch.setattr(O, "_packed_rows", wrong)
    with pytest.raises(AssertionError):
        test_varlen_prefill_equals_brute_force_per_sequence("plain", 8)


# --------------------------------------------------------------------------
# rope_interleave (CSDN DeepseekV3Attention forward: "interleaved weights")
# --------------------------------------------------------------------------
def _deinterleave_weights(cfg, inp):
    """The same layer with standard weights: the rope output rows of the q and
    kv_a projections permuted from pair order (2i, 2i+1) to rotate_half order."""
    dr, dn, r = cfg.qk_rope_head_dim, cfg.qk_nope_head_dim, cfg.kv_lora_rank
    perm = list(range(0, dr, 2)) + list(range(1, dr, 2))
    dq = dn + dr
    q_rows = [hh * dq + (i if i < dn else dn + perm[i - dn])
              for hh in range(cfg.num_heads) for i in range(dq)]
    kv_rows = list(range(r)) + [r + p for p in perm]
    kw = dict(w_kv_a=inp.w_kv_a[kv_rows])
    if cfg.q_lora_rank > 0:
        kw["w_q_b"] = inp.w_q_b[q_rows]
    else:
        kw["w_q"] = inp.w_q[q_rows]
    return type(inp)(**{**inp.__dict__, **kw})


@pytest.mark.parametrize("q_lora", [8, 0])
def test_rope_interleave_equals_permuted_weights(q_lora):
    # brute force with the permuted (standard) weights vs the oracle with the
    # interleaved flag on the original weights: outputs and cached k_pe agree
    cfg_i = tiny_cfg(q_lora_rank=q_lora, rope_interleave=True)
    cfg_p = cfg_i.with_(rope_interleave=False)
    inp = make_prefill_inputs(cfg_i, 2, 5, seed=51, gamma="random", w_std=0.4)
    out_i, P = O.prefill(cfg_i, inp, return_parts=True)
    perm_inp = _deinterleave_weights(cfg_i, inp)
    ref = np.asarray(brute_prefill(cfg_p, perm_inp, O.softmax_scale(cfg_p)))
    np.testing.assert_allclose(out_i, ref, rtol=1e-10, atol=1e-12)
    _, Pp = O.prefill(cfg_p, perm_inp, return_parts=True)
    np.testing.assert_allclose(P["latent_cache"], Pp["latent_cache"], rtol=1e-12, atol=1e-14)


def test_planted_interleave_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(O, "_rope_columns", lambda cfg, x: x)
    with pytest.raises(AssertionError):
        test_rope_interleave_equals_permuted_weights(8)
