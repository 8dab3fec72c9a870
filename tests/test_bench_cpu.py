"""bench.py's work accounting, on the host: the algorithmic FLOP and byte
counts behind ``value`` and ``roofline``, checked against counts written out
independently for the DeepSeek-V3 workloads."""
import bench
from mla_inputs import WORKLOADS


def test_prefill_flops_of_the_dsv3_workload():
    # 2N[H r_q + r_q h 192 + H (r_kv + 64) + r_kv h 256 + h 128 H] + B h 320 T (T + 1)
    cfg = WORKLOADS["dsv3_prefill"].cfg
    N, H, h, T = 4096, 7168, 128, 4096
    f = bench.prefill_stage_flops(cfg, 1, T)
    assert f["s1_down_proj"] == 2 * N * H * (1536 + 512 + 64)
    assert f["s3_q_proj"] == 2 * N * 1536 * h * 192
    assert f["s4_kv_up_proj"] == 2 * N * 512 * h * 256
    assert f["s7_attention"] == h * 320 * T * (T + 1)
    assert f["s8_o_proj"] == 2 * N * h * 128 * H
    assert abs(sum(f.values()) - 2.220e12) < 0.001e12


def test_prefill_flops_direct_q():
    cfg = WORKLOADS["directq_prefill"].cfg
    f = bench.prefill_stage_flops(cfg, 4, 8192)
    assert f["s1_down_proj"] == 2 * 4 * 8192 * 4096 * (512 + 64)
    assert f["s3_q_proj"] == 2 * 4 * 8192 * 4096 * 32 * 192
    assert abs(sum(f.values()) - 5.927e12) < 0.001e12


def test_decode_bytes_and_executed_tensor_work():
    cfg = WORKLOADS["dsv3_decode"].cfg
    ctx = 1067537
    w = bench.decode_work(cfg, ctx, 64)
    assert w["cache_bytes"] == ctx * 576 * 2
    # whole decode call: cache, W_kv_b, q_nope | q_pe in, o out
    assert w["bytes"] == ctx * 1152 + 128 * 256 * 512 * 2 + 64 * 128 * (192 + 128) * 2
    # the latent attention kernel alone: cache, q_lat | q_pe in, o_lat out
    # (no W_kv_b: the q-absorb and V-up GEMMs read it)
    assert bench.d2_own_bytes(cfg, ctx, 64) == (ctx * 1152 + 64 * 128 * 576 * 2
                                                + 64 * 128 * 512 * 2)
    v = bench.d2_tensor_view(cfg, ctx, 0.5, 1000.0)
    copies = bench.D2_SCORE_COPIES
    assert copies in (1, 2)
    assert v["flop_executed"] == ctx * 128 * (copies * 2 * 576 + 2 * 512)
    assert v["flop_algorithmic"] == ctx * 128 * 2176
    assert abs(v["achieved"] - v["flop_executed"] / 0.5e-3 / 1e12) < 1e-9
    assert abs(v["frac"] - v["achieved"] / 1000.0) < 1e-12


def test_rooflines_use_the_burst_tensor_peak_and_the_hbm_copy_rate():
    peaks = {"bf16": 1658.8, "bf16_sustained": 1397.3, "hbm": 6550.1}
    r = bench.roof_tensor(2.0e12, 2.0, peaks)          # 1000 TFLOP/s
    assert r["bound"] == "tensor" and r["peak"] == 1658.8
    assert abs(r["frac"] - 1000.0 / 1658.8) < 1e-12
    assert abs(r["frac_sustained"] - 1000.0 / 1397.3) < 1e-12
    h = bench.roof_hbm(3.0e9, 1.0, peaks)              # 3000 GB/s
    assert h["bound"] == "hbm" and h["peak"] == 6550.1
    assert abs(h["frac"] - 3000.0 / 6550.1) < 1e-12
    assert abs(h["frac_of_8tbs"] - 3000.0 / 8000.0) < 1e-12


def test_other_prefill_workloads_are_timed_beside_the_headline():
    assert set(bench.PREFILL_OTHERS) == {"dsv3_prefill", "directq_prefill",
                                         "kimi_prefill"}
    for n in bench.PREFILL_OTHERS:
        assert WORKLOADS[n].kind == "prefill"


def test_reference_arm_and_cpu_baseline_time_the_same_oracle_sample():
    rows = bench.oracle_rows(4096)
    assert rows[:3] == [0, 16, 32] and rows[-1] == 4095 and len(rows) == 257
    assert bench.oracle_rows(64) == [0, 16, 32, 48, 63]
    assert bench.oracle_rows(17) == [0, 16]
