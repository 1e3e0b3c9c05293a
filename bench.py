"""Benchmark of the DSpark draft round on B200s: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dspark|reference] [--workload NAME]

A step is one serving round of the single-request bf16 workload (4 layers,
hidden 3840, 16 x 256 heads, 2 kv heads, vocab 262144, gamma 16, A = 1, a
4096-row context from position 0): the caller crops the cache to 4080 rows
and appends the round's 16 accepted rows at positions 4080..4095
(dspark_append_context_kv: the context K/V projection with its fused
norm/RoPE epilogue), then drafts the next block (dspark_draft_rows: backbone,
KV-injection attention, lm-head with softcap, Markov walk, confidence). Every
row of the hot path runs once per step. The full 4096-row context projection
is timed separately and reported in ``config``.

With N > 1 (launched by torch.distributed.run, one rank per GPU) each rank
serves its own request (rows are independent; there is no collective on the
data path) and ``value`` is the sum over ranks: weak scaling. ``--impl
reference`` times the fp64 CPU oracle on the same round on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("draft tokens/sec (A·γ per round) and µs/round on 1 B200; HBM GB/s, tensor-pipe %")
APPEND_ROWS = 16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--workload", default="single_bf16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, choices=[None, "attention"],
                    help="time one seam alone instead of the round (prints a case line, not the bench line)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def workload_config(wl):
    m = wl.model
    return {"workload": f"{wl.name}: {m.num_hidden_layers} layers, hidden {m.hidden_size}, "
                        f"{m.num_attention_heads}x{m.global_head_dim} heads, {m.num_global_key_value_heads} kv heads, "
                        f"vocab {m.vocab_size}, markov rank {m.markov_rank}, gamma {m.block_size}, A={wl.rows}, "
                        f"Lctx={wl.ctx_len}, softcap {m.final_logit_softcapping}",
            "A": wl.rows, "gamma": m.block_size, "ctx_len": wl.ctx_len, "append_rows_per_step": APPEND_ROWS}


# ----------------------------------------------------------------------------- the oracle (CPU) leg

def oracle_round_seconds(wl, rounds: int = 1):
    """Times the fp64 oracle on `rounds` rounds of the step (append + draft), as it stands."""
    import numpy as np
    from oracle import dspark as O
    from synthetic import make_round_inputs, make_weights
    m = wl.model
    cpu = make_weights(m, wl.seed)
    inp = make_round_inputs(wl)
    W = O.OracleWeights(cpu, m)
    L0 = wl.ctx_len - APPEND_ROWS
    kv = O.project_context_kv(W, inp["hidden"][:, :L0], [0], lengths=[L0])
    times = []
    for _ in range(rounds):
        t = time.perf_counter()
        new = O.project_context_kv(W, inp["hidden"][:, L0:wl.ctx_len], [L0], lengths=[APPEND_ROWS])
        kvr = [[(O.store_rounded(np.concatenate([a[0], b[0]]), m.dtype),
                 O.store_rounded(np.concatenate([a[1], b[1]]), m.dtype)) for a, b in zip(kv[0], new[0])]]
        O.draft_rows(W, kvr, inp["anchors"].tolist(), inp["block_pos"].tolist())
        times.append(time.perf_counter() - t)
    return times


def host_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        n = 1
    return max(n, 1), len(os.sched_getaffinity(0))


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    tok = wl.rows * wl.model.block_size
    # a bounded sample: one fp64 round takes seconds, so at most 8 timed rounds after
    # at most 1 warm-up round keep the whole run within a few minutes
    warm, steps = min(args.warmup, 1), max(1, min(args.steps, 8))
    times = oracle_round_seconds(wl, rounds=warm + steps)[warm:]
    sec = sum(times) / len(times)
    threads, cores = host_threads()
    value = tok / sec
    sample = (f"{len(times)} timed rounds (after {warm} warm-up) of the step: append {APPEND_ROWS} context rows + "
              f"one gamma={wl.model.block_size} draft round, A={wl.rows}, fp64 NumPy oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": len(times), "warmup": warm, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample,
                         "host_cpus": cores},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------- the GPU leg

class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.gpu = gpu_index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def traffic_for(kernel: str):
    """DRAM bytes per launch from the committed ncu summary of `kernel`, if its source is unchanged since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh).get(kernel)
    if not d:
        return None
    h = hashlib.sha256()
    for src in d["sources"]:
        with open(os.path.join(ROOT, src), "rb") as fh:
            h.update(fh.read())
    return d["dram_bytes_per_launch"] if h.hexdigest() == d["sources_sha256"] else None


def run_dspark(args, wl):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    import block_draft_model_dspark_b200 as dsp
    from block_draft_model_dspark_b200 import build as libbuild
    from synthetic import make_round_inputs, make_weights
    libbuild.build()
    m = wl.model
    dev = torch.device("cuda", local)
    cpu = make_weights(m, wl.seed)
    gpu_w = {k: v.to(dev) for k, v in cpu.items()}
    del cpu
    model = dsp.DsparkModel(m, gpu_w)
    inp = make_round_inputs(wl)
    A, G, L, H = wl.rows, m.block_size, wl.ctx_len, m.hidden_size
    L0 = L - APPEND_ROWS
    hidden = inp["hidden"].to(dev)
    pos0 = inp["pos0"].to(dev)
    anchors = inp["anchors"].to(dev)
    block_pos = inp["block_pos"].to(dev)
    stream = torch.cuda.current_stream()

    cache = dsp.KvCache(model, A, L)
    # the full context projection, timed on its own
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(3):
        if i == 2:
            ev0.record()
        model.dspark_project_context_kv(hidden, cache.k, cache.v, pos0=pos0)
        if i == 2:
            ev1.record()
    torch.cuda.synchronize()
    project_full_ms = ev0.elapsed_time(ev1)

    new_rows = hidden[:, L0:L].contiguous()
    tokens = torch.empty(A, G, dtype=torch.int32, device=dev)
    lengths = torch.empty(A, dtype=torch.int32, device=dev)
    conf = torch.empty(A, G, dtype=torch.float32, device=dev)
    crop_host = torch.full((A,), L0, dtype=torch.int32).pin_memory()
    n_new = [APPEND_ROWS] * A
    aws = model.workspace(model.project_workspace_bytes(A * APPEND_ROWS))
    dws = model.workspace(model.draft_workspace_bytes(A, L))

    def step(rows=new_rows, anc=anchors, bpos=block_pos):
        cache.len.copy_(crop_host, non_blocking=True)           # the caller's crop: keep rows [0, L0)
        for b in range(A):
            cache.len_host[b] = L0
        model.dspark_append_context_kv(cache, rows, n_new, pos0, ws=aws)
        model.dspark_draft_rows(cache, anc, bpos, L, tokens, lengths, conf, None, ws=dws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        step()
    barrier()
    # headline: no per-kernel events (they would serialise the kernel chain)
    launches0 = dsp.dspark_kernel_launches()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        barrier()
    launches = dsp.dspark_kernel_launches() - launches0
    ms_total = t0.elapsed_time(t1)
    clocks = clk.summary()

    # per-kernel-class breakdown: the same steps again with an event pair
    # around every launch (on the launching stream)
    dsp.dspark_timer_enable(True)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for _ in range(args.steps):
        step()
    b1.record(stream)
    barrier()
    dsp.dspark_timer_enable(False)
    ms_breakdown = b0.elapsed_time(b1)
    kinds = {}
    for k in dsp.DSPARK_TIMER_KINDS:
        tms, n, by, fl = dsp.dspark_timer_read(k)
        kinds[k] = {"ms": tms, "launches": n, "bytes": by, "flops": fl}

    # separate per-call breakdown (untimed by the headline): draft alone, append alone
    def time_calls(fn, reps=10):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    round_ms = time_calls(lambda: model.dspark_draft_rows(cache, anchors, block_pos, L, tokens, lengths, conf, None,
                                                          ws=dws))

    # e2e: host buffers, copies inside the timed region, result read back every step
    h_rows = new_rows.cpu().pin_memory()
    h_anc = inp["anchors"].pin_memory()
    h_bpos = inp["block_pos"].pin_memory()
    h_tok = torch.empty(A, G, dtype=torch.int32).pin_memory()
    h_len = torch.empty(A, dtype=torch.int32).pin_memory()
    h_conf = torch.empty(A, G, dtype=torch.float32).pin_memory()
    d_rows, d_anc, d_bpos = torch.empty_like(new_rows), torch.empty_like(anchors), torch.empty_like(block_pos)

    def e2e_step():
        d_rows.copy_(h_rows, non_blocking=True)
        d_anc.copy_(h_anc, non_blocking=True)
        d_bpos.copy_(h_bpos, non_blocking=True)
        step(d_rows, d_anc, d_bpos)
        h_tok.copy_(tokens, non_blocking=True)
        h_len.copy_(lengths, non_blocking=True)
        h_conf.copy_(conf, non_blocking=True)
        stream.synchronize()

    for _ in range(3):
        e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    h2d = h_rows.numel() * h_rows.element_size() + h_anc.numel() * 4 + h_bpos.numel() * 4 + crop_host.numel() * 4
    d2h = h_tok.numel() * 4 + h_len.numel() * 4 + h_conf.numel() * 4

    # the job's time is its slowest rank's
    from block_draft_model_dspark_b200.sharding import max_over_ranks
    ms_total = max_over_ranks(ms_total)
    e2e_ms = max_over_ranks(e2e_ms)

    if rank == 0:
        tok_per_step = A * G * world
        ms_per_step = ms_total / args.steps
        value = tok_per_step / (ms_per_step / 1e3)
        hbm, tf_burst, tf_sust, peak_kind = measured_peaks()
        # the dominant kernel (one kernel shape per timer class) by device time
        dom = max(kinds, key=lambda k: kinds[k]["ms"])
        dk = kinds[dom]
        per_launch_ms = dk["ms"] / max(dk["launches"], 1)
        gbs = dk["bytes"] / (dk["ms"] / 1e3) / 1e9 if dk["ms"] > 0 else 0.0
        tfl = dk["flops"] / (dk["ms"] / 1e3) / 1e12 if dk["ms"] > 0 else 0.0
        intensity = dk["flops"] / max(dk["bytes"], 1.0)
        tensor_bound = intensity > (tf_sust * 1e12) / (hbm * 1e9)
        if tensor_bound:
            roof = {"bound": "tensor", "achieved": tfl, "peak": tf_sust, "unit": "TFLOP/s", "frac": tfl / tf_sust}
        else:
            roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}
        roof.update({"kernel": dom, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback", "traffic": traffic_for(dom),
                     "algorithmic_bytes_per_launch": dk["bytes"] / max(dk["launches"], 1),
                     "avg_launch_us": per_launch_ms * 1e3})
        kern = {k: {"ms_per_step": v["ms"] / args.steps, "share": v["ms"] / ms_breakdown if ms_breakdown else 0.0,
                    "launches_per_step": v["launches"] / args.steps,
                    "GB_per_s": v["bytes"] / (v["ms"] / 1e3) / 1e9 if v["ms"] > 0 else None,
                    "TFLOP_per_s": v["flops"] / (v["ms"] / 1e3) / 1e12 if v["ms"] > 0 else None}
                for k, v in kinds.items()}
        cfg = workload_config(wl)
        cfg.update({"parallelism": f"dp{world} (one request per GPU, no collective)",
                    "l2": "inputs larger than L2: 3.7 GB of weights streamed per step",
                    "round_us": round_ms * 1e3, "project_full_context_us": project_full_ms * 1e3,
                    "us_per_step_with_kernel_events": ms_breakdown / args.steps * 1e3,
                    "us_per_step": ms_per_step * 1e3})
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, random-init)",
                "config": cfg, "roofline": roof,
                "e2e": {"value": tok_per_step / (e2e_ms / args.steps / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": launches, "clocks": clocks, "kernels": kern}
        if world == 1 and not args.no_cpu_baseline:
            times = oracle_round_seconds(wl, rounds=1)
            threads, cores = host_threads()
            line["cpu_baseline"] = {"value": A * G / times[0], "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                    "sample": f"1 round of the step (append {APPEND_ROWS} rows + draft), fp64 NumPy "
                                              f"oracle, {times[0]:.2f} s", "host_cpus": cores}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_attention_case(args, wl):
    """The KV-injection attention seam alone (dspark_attend) at a workload's
    attention shape and context lengths: one layer's cache, random bf16 K/V.
    Prints one JSON line with the achieved K/V bandwidth (not the bench line)."""
    import torch
    import block_draft_model_dspark_b200 as dsp
    from block_draft_model_dspark_b200 import build as libbuild
    from synthetic import make_weights, round_meta
    libbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    m0 = wl.model
    # only the attention dimensions matter to the seam: a 1-layer model with small other sizes
    m = m0.replace(num_hidden_layers=1, hidden_size=256, intermediate_size=256, vocab_size=1024, mask_token_id=1023,
                   markov_rank=8, quant_bits=0)
    model = dsp.DsparkModel(m, {k: v.to(dev) for k, v in make_weights(m, wl.seed).items()})
    lens = [int(x) for x in round_meta(wl)[0].tolist()]
    A, G, nH, nKv, hd = wl.rows, m.block_size, m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    L = max(lens)
    cache = dsp.KvCache(model, A, L)
    g = torch.Generator(device=dev).manual_seed(wl.seed)
    cache.k.copy_(torch.randn(cache.k.shape, generator=g, device=dev, dtype=torch.float32).to(cache.k.dtype))
    cache.v.copy_(torch.randn(cache.v.shape, generator=g, device=dev, dtype=torch.float32).to(cache.v.dtype))
    cache.set_lengths(lens)
    q = torch.randn(A, G, nH, hd, generator=g, device=dev).to(torch.bfloat16)
    kb = torch.randn(A, G, nKv, hd, generator=g, device=dev).to(torch.bfloat16)
    vb = torch.randn(A, G, nKv, hd, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(A, G, nH, hd, device=dev, dtype=torch.bfloat16)
    ws = model.workspace(model.draft_workspace_bytes(A, L))
    for _ in range(max(args.warmup, 3)):
        model.dspark_attend(0, cache, q, kb, vb, out, L, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        model.dspark_attend(0, cache, q, kb, vb, out, L, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / args.steps * 1e3
    kv_bytes = sum(lens[b] + G for b in range(A)) * nKv * hd * 2 * 2 + 2 * A * G * nH * hd * 2
    hbm = measured_peaks()[0]
    gbs = kv_bytes / (us * 1e-6) / 1e9
    print(json.dumps({"case": "attention", "workload": wl.name, "A": A, "ctx_lens": lens, "heads": [nH, nKv, hd],
                      "us_per_call": us, "algorithmic_bytes": kv_bytes, "GB_per_s": gbs, "hbm_peak_GB_per_s": hbm,
                      "frac": gbs / hbm, "calls": args.steps, "note": "attention partials + merge kernel; "
                      "cache larger than L2 when its bytes exceed 126 MB"}), flush=True)


def main():
    args = parse()
    from synthetic import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.case == "attention":
        run_attention_case(args, wl)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_dspark(args, wl)


if __name__ == "__main__":
    main()
