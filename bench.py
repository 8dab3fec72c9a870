#!/usr/bin/env python
"""Benchmark of the MLA hot path on B200: one step = one DeepSeek-V3-shaped
prefill forward (B=1, T=4096, hidden 7168, 128 heads, YaRN) followed by one
weight-absorbed decode step (B=64, context lengths uniform in [1024, 32768]).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  ``value`` is the prefill throughput in
TFLOP/s (algorithmic FLOPs of the forward, causal attention counted for
j <= i only) over all ranks; decode latent-cache GB/s and prefill tokens/s are
reported beside it.  Multi-GPU runs are independent replicas (weak scaling,
no collective on the data path); the timing is the max over ranks.
"""
import argparse
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "dsv3_prefill"
DECODE = "dsv3_decode"
PREFILL_OTHERS = ["dsv3_prefill", "directq_prefill", "kimi_prefill"]
HBM_NOMINAL_GBS = 8000.0          # the ~8 TB/s datasheet HBM3e figure
L2_FLUSH_BYTES = 256 << 20
STAGES_P = ["s1_down_proj", "s3_q_proj", "s4_kv_up_proj", "s7_attention",
            "s8_o_proj"]
STAGES_D = ["d1_q_absorb", "d2_latent_attention", "d3_combine", "d4_v_up",
            "o_proj"]


# ---------------------------------------------------------------------------
# Algorithmic work
# ---------------------------------------------------------------------------
def prefill_stage_flops(cfg, B, T):
    N = B * T
    H, h = cfg.hidden_size, cfg.num_heads
    dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
    dq, rq, rkv = dn + dr, cfg.q_lora_rank, cfg.kv_lora_rank
    down = 2 * N * H * ((rq if rq else 0) + rkv + dr)
    q = 2 * N * (rq * h * dq if rq else H * h * dq)
    kv = 2 * N * rkv * h * (dn + dv)
    attn = B * h * (dq + dv) * T * (T + 1)          # 2 FLOP x causal pairs
    o = 2 * N * h * dv * H
    return {"s1_down_proj": down, "s3_q_proj": q, "s4_kv_up_proj": kv,
            "s7_attention": attn, "s8_o_proj": o}


def decode_work(cfg, ctx_total, B):
    h, r, dr, dn, dv = (cfg.num_heads, cfg.kv_lora_rank, cfg.qk_rope_head_dim,
                        cfg.qk_nope_head_dim, cfg.v_head_dim)
    cache_bytes = ctx_total * (r + dr) * 2
    wkvb = h * (dn + dv) * r * 2
    qio = B * h * (dn + dr) * 2 + B * h * dv * 2
    flops = ctx_total * h * 2 * ((r + dr) + r) + 2 * B * h * r * (dn + dv)
    return {"cache_bytes": cache_bytes, "bytes": cache_bytes + wkvb + qio,
            "flops": flops}


# Score copies the latent attention kernel computes per token and head: each
# CTA of an SM pair computes the partial scores over its own half of the
# r + rope dims and the pair adds the two, so the scores are computed once.
D2_SCORE_COPIES = 1


def d2_own_bytes(cfg, ctx_total, B):
    """Algorithmic DRAM bytes of the latent attention kernel alone: the cache
    rows it streams, the absorbed query it reads (q_lat and q_pe) and the
    latent output it writes.  Partial results of sequences cut between SM
    pairs are the schedule's overhead and are not counted; the kv
    up-projection weights belong to the q-absorb and V-up GEMMs."""
    h, r, dr = cfg.num_heads, cfg.kv_lora_rank, cfg.qk_rope_head_dim
    return ctx_total * (r + dr) * 2 + B * h * (r + dr) * 2 + B * h * r * 2


def d2_tensor_view(cfg, ctx_total, ms, peak_tflops):
    """The latent attention kernel's tensor work as executed: D2_SCORE_COPIES
    x 2 (r + rope) score FLOP plus 2 r FLOP of P.C per token and head (the
    algorithmic count has one copy of the scores)."""
    h, r, dr = cfg.num_heads, cfg.kv_lora_rank, cfg.qk_rope_head_dim
    algo = ctx_total * h * (2 * (r + dr) + 2 * r)
    executed = ctx_total * h * (D2_SCORE_COPIES * 2 * (r + dr) + 2 * r)
    a = executed / (ms * 1e-3) / 1e12
    return {"flop_executed": executed, "flop_algorithmic": algo, "achieved": a,
            "peak": peak_tflops, "unit": "TFLOP/s", "frac": a / peak_tflops}


def roof_tensor(flops, ms, peaks, traffic=None):
    """A tensor-core kernel against the measured burst bf16 peak: the timed
    region lasts tens of milliseconds at the maximum SM clock, not the
    seconds under the power cap that the sustained figure describes (kept
    beside it as frac_sustained)."""
    a = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": a, "peak": peaks["bf16"],
            "unit": "TFLOP/s", "frac": a / peaks["bf16"],
            "peak_sustained": peaks["bf16_sustained"],
            "frac_sustained": a / peaks["bf16_sustained"], "traffic": traffic}


def roof_hbm(nbytes, ms, peaks, traffic=None):
    """A bandwidth-bound kernel against the measured HBM copy rate (and the
    ~8 TB/s datasheet figure)."""
    a = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": a, "peak": peaks["hbm"], "unit": "GB/s",
            "frac": a / peaks["hbm"], "frac_of_8tbs": a / HBM_NOMINAL_GBS,
            "bytes": nbytes, "traffic": traffic}


def time_prefill_workload(wl, seed, K, Wm, flush, dev, world, set_events, tensor_roof,
                          gpu):
    """Time K prefill forwards of one more workload (after Wm warm-up ones),
    the L2 flushed before each, with the library's stage events; returns its
    throughput, stage times, the rooflines of its attention and dominant
    kernels and the clocks sampled while it ran.  Timing is the max over
    ranks."""
    import torch
    from mla_inputs import make_prefill_inputs
    from latent_attention_b200.layer import MlaPrefill
    cfg, B, T = wl.cfg, wl.batch, wl.seq_len
    inp = make_prefill_inputs(cfg, B, T, seed=seed)
    weights = {k: getattr(inp, k) for k in ("w_q_a", "g_q_a", "w_q_b", "w_q",
                                              "w_kv_a", "g_kv_a", "w_kv_b", "w_o")}
    pre = MlaPrefill(cfg, weights, B, T, device=dev)
    x = inp.x.to(dev)
    out = torch.empty(B, T, cfg.hidden_size, dtype=torch.bfloat16, device=dev)
    del inp, weights
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev = [[mk() for _ in range(6)] for _ in range(K)]
    for group in ev:
        for e in group:
            e.record()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu)
    clocks.start()
    t_begin = None
    for i in range(Wm + K):
        flush.zero_()
        if i == Wm:
            if world > 1:
                import torch.distributed as dist
                dist.barrier()
            torch.cuda.synchronize()
            t_begin = time.time()
        set_events(ev[i - Wm] if i >= Wm else None)
        pre(x, out=out)
        set_events(None)
    torch.cuda.synchronize()
    clocks.mark(t_begin, time.time())
    clk = clocks.stop()
    pre.check_status()
    ms = sum(e[0].elapsed_time(e[5]) for e in ev)
    st = {n: sum(e[k].elapsed_time(e[k + 1]) for e in ev) / K
          for k, n in enumerate(STAGES_P)}
    ms = max_over_ranks([ms], world, dev)[0]
    fl = prefill_stage_flops(cfg, B, T)
    dominant = max(STAGES_P, key=lambda n: st[n])
    res = {"B": B, "T": T, "hidden": cfg.hidden_size, "heads": cfg.num_heads,
           "q_lora_rank": cfg.q_lora_rank, "rope": cfg.rope_type,
           "ms": ms / K, "tflops": world * K * sum(fl.values()) / (ms * 1e-3) / 1e12,
           "tokens_per_s": world * K * B * T / (ms * 1e-3),
           "stage_ms": {k: round(v, 4) for k, v in st.items()},
           "attention_roofline": tensor_roof(fl["s7_attention"], st["s7_attention"], None),
           "roofline": dict(tensor_roof(fl[dominant], st[dominant], None), kernel=dominant),
           "clocks": clk}
    res["frac_of_peak"] = res["tflops"] / res["attention_roofline"]["peak"]
    del pre, x, out
    torch.cuda.empty_cache()
    return res


def source_hash():
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "latent_attention_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0,
            "source": "fallback"}


def load_traffic():
    """ncu DRAM bytes per launch, valid only for the sources they were taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    d = json.load(open(p))
    if d.get("source_hash") != source_hash():
        return {}
    return d.get("per_launch_bytes", {})


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 20 ms with timestamps.
    Started before the warm-up and running by the time the timed region
    begins; only samples inside the timed window are summarised (the nearest
    ones, flagged, when the window is shorter than the sampling period)."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0:   # sampler live
                time.sleep(0.01)
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t_begin, t_end):
        self.window = (t_begin, t_end)

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t_read, l in self.lines:
            q = [x.strip() for x in l.split(",")]
            if len(q) < 9:
                continue
            try:
                rows.append((t_read, float(q[1]), float(q[2]), q[5:9]))
            except ValueError:
                continue
        inside = rows
        in_window = None
        if self.window and rows:
            lo, hi = self.window
            inside = [r for r in rows if lo <= r[0] <= hi + 0.025]
            in_window = bool(inside)
            if not inside:                 # window shorter than the period
                inside = sorted(rows, key=lambda r: min(abs(r[0] - lo), abs(r[0] - hi)))[:2]
        reasons = set()
        for r in inside:
            for n, v in zip(self.NAMES, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median([r[1] for r in inside]) if inside else None,
                "sm_max_mhz": inside[-1][2] if inside else None,
                "reasons": sorted(reasons), "samples": len(inside),
                "in_timed_window": in_window}


def gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return local_rank


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_prefill_sample(cfg, inp, rows):
    """Time the fp64 oracle on keys/values for all T positions plus the query
    path, attention and o_proj for ``rows``; returns (seconds, FLOPs done)."""
    import oracle
    import numpy as np
    t0 = time.perf_counter()
    oracle.prefill(cfg, inp, rows=rows)
    dt = time.perf_counter() - t0
    B, T = inp.B, inp.T
    R = len(rows)
    f = prefill_stage_flops(cfg, B, T)
    N = B * T
    H, h = cfg.hidden_size, cfg.num_heads
    dq, dv = cfg.qk_head_dim, cfg.v_head_dim
    done = (2 * N * H * (cfg.kv_lora_rank + cfg.qk_rope_head_dim) +
            f["s4_kv_up_proj"] +
            (f["s1_down_proj"] - 2 * N * H * (cfg.kv_lora_rank + cfg.qk_rope_head_dim)) * R / T +
            f["s3_q_proj"] * R / T +
            B * h * (dq + dv) * 2 * float(np.sum(np.asarray(rows) + 1)) +
            f["s8_o_proj"] * R / T)
    return dt, done


def oracle_rows(T):
    """The stratified query rows the oracle runs on (every 16th and the
    last): keys and values are projected for all T positions, the query
    path, attention and o_proj for these rows.  The reference arm times one
    such sample per step; cpu_baseline repeats it for about ten seconds."""
    return list(range(0, T, 16)) + ([T - 1] if (T - 1) % 16 else [])


def rank_seeds(rank):
    """Seeds of one rank's own synthetic inputs: every replica draws
    different data of the same shapes."""
    return {"prefill": 1000 * rank, "ctx": rank, "decode": 1000 * rank + 1}


def max_over_ranks(values, world, device):
    """Per-rank timings -> their maximum over all ranks (every rank gets it).
    The same collective runs on every rank, in the same order."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def cpu_threads():
    try:
        import torch
        return torch.get_num_threads()
    except Exception:
        return os.cpu_count()


def run_reference(args, rank):
    if rank != 0:
        return 0
    from mla_inputs import WORKLOADS, make_prefill_inputs
    wl = WORKLOADS[PREFILL]
    inp = make_prefill_inputs(wl.cfg, wl.batch, wl.seq_len, seed=0)
    # every 16th query row and the last: the key/value projections for all
    # positions plus a stratified sixteenth of the per-row work, a few seconds
    # per step (the same sample as cpu_baseline)
    rows = oracle_rows(wl.seq_len)
    secs, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        dt, fl = oracle_prefill_sample(wl.cfg, inp, rows)
        if i >= args.warmup:
            secs.append(dt)
            flops = fl
    tot = sum(secs)
    v = flops * len(secs) / tot / 1e12
    sample = (f"fp64 NumPy oracle, {wl.name}: keys/values for all {wl.seq_len} "
              f"positions + query/attention/o_proj for {len(rows)} rows (every 16th "
              f"and the last), each step")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_block(wl, None),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


METRIC = "MLA prefill TFLOP/s + tokens/s; absorbed-decode latent-cache HBM GB/s"


def config_block(wl, dwl):
    c = wl.cfg
    d = {"workload": f"{wl.name} (B={wl.batch}, T={wl.seq_len}) + "
                     f"{DECODE} (B=64, ctx U[1024,32768])",
         "prefill": {"B": wl.batch, "T": wl.seq_len, "hidden": c.hidden_size,
                     "heads": c.num_heads, "q_lora_rank": c.q_lora_rank,
                     "kv_lora_rank": c.kv_lora_rank, "qk_nope": c.qk_nope_head_dim,
                     "qk_rope": c.qk_rope_head_dim, "v_head": c.v_head_dim,
                     "rope": f"{c.rope_type} factor {c.rope_factor}"},
         "l2": "flushed between steps (256 MiB write)",
         "parallelism": "independent replicas, one per GPU"}
    if dwl is not None:
        d["decode"] = dwl
    return d


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", default=PREFILL,
                    choices=["dsv3_prefill", "directq_prefill", "kimi_prefill"],
                    help="prefill workload of the step (default: the headline one)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist
    import ctypes as C
    from datetime import timedelta
    from mla_inputs import (WORKLOADS, make_prefill_inputs, make_decode_inputs,
                            decode_context_lengths)
    import latent_attention_b200 as L
    from latent_attention_b200 import _lib
    from latent_attention_b200.layer import MlaPrefill, MlaDecode

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    lib = _lib.load()

    wl, wd = WORKLOADS[args.prefill], WORKLOADS[DECODE]
    cfg, cfgd = wl.cfg, wd.cfg
    B, T = wl.batch, wl.seq_len
    seeds = rank_seeds(rank)
    inp = make_prefill_inputs(cfg, B, T, seed=seeds["prefill"])
    weights = {k: getattr(inp, k) for k in ("w_q_a", "g_q_a", "w_q_b", "w_q",
                                              "w_kv_a", "g_kv_a", "w_kv_b", "w_o")}
    pre = MlaPrefill(cfg, weights, B, T, device=dev)
    x = inp.x.to(dev)
    out = torch.empty(B, T, cfg.hidden_size, dtype=torch.bfloat16, device=dev)

    ctx = decode_context_lengths(wd.batch, wd.ctx_min, wd.ctx_max, seed=seeds["ctx"])
    di = make_decode_inputs(cfgd, wd.batch, ctx, seed=seeds["decode"])
    dec = MlaDecode(cfgd, wd.batch, wd.ctx_max, device=dev)
    qn, qp = di.q_nope.to(dev), di.q_pe.to(dev)
    wkvb, cache, cu = di.w_kv_b.to(dev), di.cache.to(dev), di.cu_ctx.to(dev)
    dout = torch.empty(wd.batch, cfgd.num_heads * cfgd.v_head_dim,
                       dtype=torch.bfloat16, device=dev)
    ctx_total = int(ctx.sum())
    del inp, di
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    K, Wm = args.steps, args.warmup
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev_p = [[mk() for _ in range(6)] for _ in range(K)]
    ev_d = [[mk() for _ in range(6)] for _ in range(K)]
    ev_s = [(mk(), mk()) for _ in range(K)]
    # torch creates the CUDA event lazily at its first record; the library
    # records through the raw handle, so materialise every handle now.
    for group in ev_p + ev_d:
        for e in group:
            e.record()
    torch.cuda.synchronize()

    def set_events(evs):
        if evs is None:
            lib.mla_set_stage_events(None, 0)
            return
        arr = (C.c_void_p * len(evs))(*[e.cuda_event for e in evs])
        lib.mla_set_stage_events(arr, len(evs))

    def step(i):
        timed = i >= Wm
        j = i - Wm
        if timed:
            ev_s[j][0].record()
        set_events(ev_p[j] if timed else None)
        pre(x, out=out)
        set_events(ev_d[j] if timed else None)
        dec(qn, qp, wkvb, cache, cu, dout)
        set_events(None)
        if timed:
            ev_s[j][1].record()

    clocks = ClockSampler(gpu_index(local))
    clocks.start()                       # live before the warm-up ends
    launches0 = 0
    t_begin = None
    for i in range(Wm + K):
        flush.zero_()
        if i == Wm:
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            launches0 = lib.mla_kernel_launches()
            t_begin = time.time()
        step(i)
    torch.cuda.synchronize()
    clocks.mark(t_begin, time.time())
    launches = lib.mla_kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    pre.check_status()
    dec.check_status()

    step_ms = sum(a.elapsed_time(b) for a, b in ev_s)
    pre_ms = sum(e[0].elapsed_time(e[5]) for e in ev_p)
    dec_ms = sum(e[0].elapsed_time(e[5]) for e in ev_d)
    st_p = {n: sum(e[k].elapsed_time(e[k + 1]) for e in ev_p) / K
            for k, n in enumerate(STAGES_P)}
    st_d = {n: sum(e[k].elapsed_time(e[k + 1]) for e in ev_d) / K
            for k, n in enumerate(STAGES_D)}
    step_ms, pre_ms, dec_ms = max_over_ranks([step_ms, pre_ms, dec_ms], world, dev)

    # ---- end to end through the public API with host buffers -------------
    # Every step copies its input from pinned host memory, runs the prefill
    # through mla_prefill_forward and copies its output back.  The copies of
    # one step overlap the compute of its neighbours (double-buffered device
    # input/output, one stream per copy direction and one for compute), as a
    # serving loop would run; the timed region spans the first step's input
    # copy to the last step's output copy.  The serial form (copy, compute,
    # copy, one step at a time) is reported beside it.
    x_h = torch.empty_like(x, device="cpu").pin_memory()
    x_h.copy_(x.cpu())
    out_h = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(2)]
    x_d = [x, torch.empty_like(x)]
    out_d = [out, torch.empty_like(out)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_cmp = [mk() for _ in range(Wm + K)]
    ev_out = [mk() for _ in range(Wm + K)]

    def pipelined(first, n, t0=None, t1=None):
        for i in range(first, first + n):
            bsel = i % 2
            with torch.cuda.stream(s_in):
                if i - 2 >= first:                  # x_d[bsel] read by step i-2
                    s_in.wait_event(ev_cmp[i - 2])
                if t0 is not None and i == first:
                    t0.record(s_in)
                x_d[bsel].copy_(x_h, non_blocking=True)
            s_cmp.wait_stream(s_in)
            if i - 2 >= first:                      # out_d[bsel] read by step i-2
                s_cmp.wait_event(ev_out[i - 2])
            pre(x_d[bsel], out=out_d[bsel], stream=s_cmp)
            ev_cmp[i].record(s_cmp)
            s_out.wait_event(ev_cmp[i])
            with torch.cuda.stream(s_out):
                out_h[bsel].copy_(out_d[bsel], non_blocking=True)
            ev_out[i].record(s_out)
        if t1 is not None:
            t1.record(s_out)

    torch.cuda.synchronize()
    pipelined(0, Wm)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_t0, e2e_t1 = mk(), mk()
    pipelined(Wm, K, e2e_t0, e2e_t1)
    torch.cuda.synchronize()
    e2e_ms = e2e_t0.elapsed_time(e2e_t1)
    # serial form: one step at a time on the default stream
    ser_ev = [(mk(), mk()) for _ in range(K)]
    for i in range(Wm + K):
        if i >= Wm:
            ser_ev[i - Wm][0].record()
        x.copy_(x_h, non_blocking=True)
        pre(x, out=out)
        out_h[0].copy_(out, non_blocking=True)
        if i >= Wm:
            ser_ev[i - Wm][1].record()
    torch.cuda.synchronize()
    ser_ms = sum(a.elapsed_time(b) for a, b in ser_ev)
    e2e_ms, ser_ms = max_over_ranks([e2e_ms, ser_ms], world, dev)

    fl = prefill_stage_flops(cfg, B, T)
    pflops = sum(fl.values())
    dw = decode_work(cfgd, ctx_total, wd.batch)
    peaks = load_peaks()
    traffic = load_traffic()
    value = world * K * pflops / (pre_ms * 1e-3) / 1e12

    def tensor_roof(flops, ms, stage):
        return roof_tensor(flops, ms, peaks, traffic.get(stage))

    def hbm_roof(nbytes, ms, stage):
        return roof_hbm(nbytes, ms, peaks, traffic.get(stage))

    stages = {n: tensor_roof(fl[n], st_p[n], n) for n in STAGES_P}
    d2_ms = st_d["d2_latent_attention"]
    stages["d2_latent_attention"] = hbm_roof(d2_own_bytes(cfgd, ctx_total, wd.batch),
                                             d2_ms, "d2_latent_attention")
    stages["d2_latent_attention"]["tensor_executed"] = d2_tensor_view(
        cfgd, ctx_total, d2_ms, peaks["bf16"])
    decode_roofline = dict(hbm_roof(dw["bytes"], dec_ms / K, "decode"),
                           what="whole decode call (D1-D4): cache, W_kv_b, q_nope, "
                                "q_pe and the output, over the call's event time")
    dominant = max(STAGES_P, key=lambda n: st_p[n])
    roofline = dict(stages[dominant], kernel=dominant,
                    peak_source=f"{peaks['source']} (bf16 burst / HBM copy)")

    # the other prefill workloads, each timed on its own after the step
    extra = {}
    for name in PREFILL_OTHERS:
        if name == args.prefill:
            continue
        extra[name] = time_prefill_workload(WORKLOADS[name], seeds["prefill"], K, Wm,
                                            flush, dev, world, set_events,
                                            tensor_roof, gpu_index(local))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from mla_inputs import make_prefill_inputs as mpi
        # the reference arm's sample of the step's prefill, repeated for
        # about ten seconds of fp64 work
        inp_c = mpi(cfg, B, T, seed=0)
        rows = oracle_rows(T)
        dt, done, reps = 0.0, 0.0, 0
        while reps == 0 or dt < 10.0:
            d1, f1 = oracle_prefill_sample(cfg, inp_c, rows)
            dt, done, reps = dt + d1, done + f1, reps + 1
        cpu = {"value": done / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
               "kind": "oracle",
               "sample": f"fp64 NumPy oracle, {wl.name} (B={B}, T={T}): keys/values for "
                         f"all {T} positions + query/attention/o_proj for {len(rows)} rows "
                         f"(every 16th and the last), {reps} times; "
                         f"{done / 1e9:.0f} GFLOP in {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": K, "warmup": Wm, "ms_per_step": step_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded; random-init weights of "
                                     "the DeepSeek-V3 MLA layer shapes)",
            "config": config_block(wl, {"B": wd.batch, "ctx_total": ctx_total,
                                        "ctx_range": [wd.ctx_min, wd.ctx_max]}),
            "prefill_ms": pre_ms / K,
            "prefill_tokens_per_s": world * K * B * T / (pre_ms * 1e-3),
            "decode_ms": dec_ms / K,
            "decode_latent_cache_gb_per_s": world * K * dw["cache_bytes"] / (dec_ms * 1e-3) / 1e9,
            "decode_tflops": world * K * dw["flops"] / (dec_ms * 1e-3) / 1e12,
            "stage_ms": {**{k: round(v, 4) for k, v in st_p.items()},
                         **{k: round(v, 4) for k, v in st_d.items()}},
            "roofline": roofline,
            "roofline_stages": stages,
            "decode_roofline": decode_roofline,
            "prefill_configs": extra,
            "clocks": clk,
            "gpu_launches": launches,
            "e2e": {"value": world * K * pflops / (e2e_ms * 1e-3) / 1e12,
                    "unit": "TFLOP/s", "h2d_bytes_per_step": x.numel() * 2,
                    "d2h_bytes_per_step": out.numel() * 2,
                    "serial_value": world * K * pflops / (ser_ms * 1e-3) / 1e12,
                    "what": "prefill through mla_prefill_forward; every step copies its "
                            "input from pinned host memory and its output back, the "
                            "copies overlapping neighbouring steps' compute (double "
                            "buffers, separate copy/compute streams; no L2 flush: weights and "
                            "activations of a step, ~1 GB, exceed L2); serial_value: "
                            "copy, compute, copy one step at a time"},
            "source_hash": source_hash(),
        }
        if cpu:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
