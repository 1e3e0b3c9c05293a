"""Benchmark of the DSpark draft round on B200s: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dspark|reference] [--workload NAME]

A step is one serving round of a workload over all its request rows: the
caller crops every row's cache back to where the previous round's accepted
rows begin and appends them (dspark_append_context_kv: the context K/V
projection with its fused norm/RoPE epilogue), then drafts the next block
(dspark_draft_rows: backbone, KV-injection attention, lm-head with softcap,
Markov walk, confidence). Every row of the hot path runs once per round.

Workloads (``--workload``, default ``ragged_bf16``, the largest that the
metric is quoted on at one GPU: A = 32 rows x gamma 16 = 512 drafted tokens
per round):
  * ``single_bf16``: A = 1, a 4096-row context; gamma = 16 rows appended.
  * ``ragged_bf16``: A = 32, per-row context 512..4096 rows at per-row start
    positions (dynamic RoPE); gamma = 16 rows appended per row.
  * ``quant4_bf16``: A = 64, 8192-row contexts, 4-bit weights, gamma = 8.
  * ``long_incremental_bf16``: A = 4, 32768-row contexts; a step is the
    workload's 8 rounds of append(n ~ U[1, 16] per row) + draft.
The full initial context projection is timed separately and reported in
``config``. With N > 1 (torch.distributed.run, one rank per GPU) every rank
serves the whole workload's rows on its own GPU (rows are independent; there
is no collective on the data path) and ``value`` is the sum over ranks: weak
scaling. ``--impl reference`` times the fp64 CPU oracle on the same rounds.
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
DEFAULT_WORKLOAD = "ragged_bf16"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, choices=[None, "attention", "round"],
                    help="attention: time the seam alone; round: run the workload's rounds (for profiling small "
                         "cases with --layers / --vocab); both print a case line, not the bench line")
    ap.add_argument("--layers", type=int, default=0, help="--case round: layers of the model (0: the workload's)")
    ap.add_argument("--vocab", type=int, default=0, help="--case round: vocabulary of the model (0: the workload's)")
    ap.add_argument("--kv-cache", default="kv", choices=["kv", "v_only"],
                    help="context cache layout: kv stores k and v (the default: the faster round); v_only stores v "
                         "alone (half the cache; the attention rebuilds k = rope(v * k_norm))")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


# ----------------------------------------------------------------------------- the step's schedule

class StepPlan:
    """What one step does for a workload: the crop, then its rounds (append + draft).

    All tensors are CPU tensors; ``crop[b]`` is row b's cache length at the
    start of a step, each round is a dict with ``n_new`` [A] int32, ``hidden``
    [A, Lnew_max, H] (rows past n_new are padding), ``anchors`` [A] int32,
    ``block_pos`` [A] int32 and ``max_len`` (the longest row after the append).
    ``init_hidden`` / ``init_len`` hold the initial context (projected once).
    """

    def __init__(self, wl):
        import torch
        from synthetic import make_append_schedule, make_round_inputs
        m = wl.model
        G = m.block_size
        inp = make_round_inputs(wl)
        self.A = wl.rows
        self.pos0 = inp["pos0"]
        lens = inp["ctx_len"].tolist()
        self.init_hidden = inp["hidden"]
        self.init_len = lens
        self.rounds = []
        if wl.append_rounds > 0:
            # the incremental workload: 8 rounds of accepted rows on top of the initial context
            self.crop = list(lens)
            self.capacity = wl.capacity
            cur = list(lens)
            for r in make_append_schedule(wl):
                n = r["n_new"].tolist()
                cur = [c + k for c, k in zip(cur, n)]
                self.rounds.append({"n_new": r["n_new"], "hidden": r["hidden"], "anchors": r["anchors"],
                                    "block_pos": (self.pos0 + torch.tensor(cur, dtype=torch.int32)).to(torch.int32),
                                    "max_len": max(cur)})
            self.append_desc = f"{wl.append_rounds} rounds of append(n ~ U[1, {wl.append_max}] per row) + draft"
        else:
            # one round: the last gamma context rows of every row are its previous round's accepted rows
            self.crop = [L - G for L in lens]
            self.capacity = int(inp["hidden"].shape[1])
            hid = torch.stack([inp["hidden"][b, lens[b] - G:lens[b]] for b in range(self.A)]).contiguous()
            self.rounds.append({"n_new": torch.full((self.A,), G, dtype=torch.int32), "hidden": hid,
                                "anchors": inp["anchors"], "block_pos": inp["block_pos"], "max_len": max(lens)})
            self.append_desc = f"append {G} accepted rows per row + draft"
        self.tokens_per_step = len(self.rounds) * self.A * G


def use_v_only(args, m) -> bool:
    """--kv-cache v_only: needs a bf16 model on the tensor-core attention (head_dim % 64 == 0, <= 256)."""
    ok = m.dtype == "bf16" and m.global_head_dim % 64 == 0 and m.global_head_dim <= 256
    if args.kv_cache == "v_only" and not ok:
        raise SystemExit(f"--kv-cache v_only: unsupported for {m}")
    return args.kv_cache == "v_only"


def workload_config(wl, plan=None):
    m = wl.model
    lens = f"Lctx=U[{wl.ragged_min},{wl.ctx_len}]" if wl.ragged_min else f"Lctx={wl.ctx_len}"
    quant = ", 4-bit affine weights (g64)" if m.quant_bits else ""
    out = {"workload": f"{wl.name}: {m.num_hidden_layers} layers, hidden {m.hidden_size}, "
                       f"{m.num_attention_heads}x{m.global_head_dim} heads, {m.num_global_key_value_heads} kv heads, "
                       f"intermediate {m.intermediate_size}, vocab {m.vocab_size}, markov rank {m.markov_rank}, "
                       f"gamma {m.block_size}, A={wl.rows}, {lens}{quant}, softcap {m.final_logit_softcapping}",
           "A": wl.rows, "gamma": m.block_size, "ctx_len": wl.ctx_len,
           "weights": "synthetic N(0,0.02) matmul/embedding/Markov/confidence weights; RMSNorm gains 1+N(0,0.02) with "
                      "q_norm/k_norm further scaled by head_dim^-1/4 (unit-variance attention logits); layer_scalar 1"}
    if plan is not None:
        out["step"] = plan.append_desc
        out["rounds_per_step"] = len(plan.rounds)
        out["tokens_per_step"] = plan.tokens_per_step
    return out


# ----------------------------------------------------------------------------- the oracle (CPU) leg

def oracle_sample_rows(wl, plan, budget_bytes=4.5e9):
    """Rows of the workload the CPU oracle drafts: all of them when their fp64 cache fits the budget."""
    m = wl.model
    per_row = [(c + sum(int(r["n_new"][b]) for r in plan.rounds)) * m.num_hidden_layers * 2 *
               m.num_global_key_value_heads * m.global_head_dim * 8 for b, c in enumerate(plan.crop)]
    rows, total = [], 0.0
    for b in range(plan.A):
        if rows and total + per_row[b] > budget_bytes:
            break
        rows.append(b)
        total += per_row[b]
    return rows


def oracle_steps(wl, plan, rows, steps, time_budget_s):
    """Times the fp64 oracle on `steps` steps over the sampled `rows`, as it stands.

    The cached context rows are random fp64 values of the workload's lengths
    (the round's cost does not depend on them); each step appends and drafts
    exactly as the GPU step does. Returns the per-step seconds."""
    import numpy as np
    from oracle import dspark as O
    from synthetic import make_weights
    m = wl.model
    W = O.OracleWeights(make_weights(m, wl.seed), m)
    rng = np.random.default_rng(wl.seed)
    nKv, hd = m.num_global_key_value_heads, m.global_head_dim
    base = [[(rng.standard_normal((plan.crop[b], nKv, hd)), rng.standard_normal((plan.crop[b], nKv, hd)))
             for _ in range(m.num_hidden_layers)] for b in rows]
    pos0 = plan.pos0.tolist()
    times = []
    t_start = time.perf_counter()
    for _ in range(steps):
        t = time.perf_counter()
        kv = [list(r) for r in base]
        cur = [plan.crop[b] for b in rows]
        for rnd in plan.rounds:
            n = [int(rnd["n_new"][b]) for b in rows]
            new = O.project_context_kv(W, rnd["hidden"][rows], [pos0[b] + c for b, c in zip(rows, cur)], lengths=n)
            kv = [[(np.concatenate([kv[i][l][0], new[i][l][0]]), np.concatenate([kv[i][l][1], new[i][l][1]]))
                   for l in range(m.num_hidden_layers)] for i in range(len(rows))]
            cur = [c + k for c, k in zip(cur, n)]
            O.draft_rows(W, kv, [int(rnd["anchors"][b]) for b in rows], [int(rnd["block_pos"][b]) for b in rows])
        times.append(time.perf_counter() - t)
        if time.perf_counter() - t_start > time_budget_s:
            break
    return times


def host_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        n = 1
    return max(n, 1), len(os.sched_getaffinity(0))


def cpu_sample_desc(wl, plan, rows, n_steps, warm):
    return (f"{n_steps} timed step(s) (after {warm} warm-up) over {len(rows)} of the {plan.A} request rows: "
            f"{plan.append_desc}, gamma={wl.model.block_size}; fp64 NumPy oracle, random cached context of the "
            f"workload's lengths")


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    plan = StepPlan(wl)
    rows = oracle_sample_rows(wl, plan)
    # a bounded sample: at most 1 warm-up and 4 timed steps, and no more than ~2 minutes of timed steps
    warm, steps = min(args.warmup, 1), max(1, min(args.steps, 4))
    times = oracle_steps(wl, plan, rows, warm + steps, time_budget_s=150.0)
    times = times[warm:] or times
    sec = sum(times) / len(times)
    tok = len(plan.rounds) * len(rows) * wl.model.block_size
    threads, cores = host_threads()
    value = tok / sec
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": len(times), "warmup": warm, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, plan),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": cpu_sample_desc(wl, plan, rows, len(times), warm), "host_cpus": cores},
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


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` at `workload` from the committed ncu summary, if its source is unchanged since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh).get(f"{kernel}@{workload}")
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
    from synthetic import make_weights
    libbuild.build()
    m = wl.model
    dev = torch.device("cuda", local)
    cpu = make_weights(m, wl.seed)
    gpu_w = {k: v.to(dev) for k, v in cpu.items()}
    del cpu
    model = dsp.DsparkModel(m, gpu_w)
    plan = StepPlan(wl)
    A, G = plan.A, m.block_size
    stream = torch.cuda.current_stream()
    pos0 = plan.pos0.to(dev)

    # the initial context, projected once into the cache (timed on its own)
    v_only = use_v_only(args, m)
    cache = dsp.KvCache(model, A, plan.capacity, v_only=v_only, pos0=pos0 if v_only else None)
    init_hidden = plan.init_hidden.to(dev)
    init_n = torch.tensor(plan.init_len, dtype=torch.int32, device=dev)
    pws = model.workspace(model.project_workspace_bytes(A * int(init_hidden.shape[1])))
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(2):
        cache.set_lengths([0] * A)
        if i == 1:
            ev0.record(stream)
        model.dspark_append_context_kv(cache, init_hidden, init_n, pos0, ws=pws)
        if i == 1:
            ev1.record(stream)
    torch.cuda.synchronize()
    project_full_ms = ev0.elapsed_time(ev1)
    project_rows = sum(plan.init_len)
    del init_hidden, pws
    torch.cuda.empty_cache()

    # the step's inputs, resident in HBM before the timed region
    crop = torch.tensor(plan.crop, dtype=torch.int32, device=dev)
    rounds = [{k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in r.items()} for r in plan.rounds]
    outs = [{"tokens": torch.empty(A, G, dtype=torch.int32, device=dev),
             "lengths": torch.empty(A, dtype=torch.int32, device=dev),
             "conf": torch.empty(A, G, dtype=torch.float32, device=dev)} for _ in rounds]
    lnew = max(int(r["hidden"].shape[1]) for r in rounds)
    aws = model.workspace(model.project_workspace_bytes(A * lnew))
    dws = model.workspace(model.draft_workspace_bytes(A, max(r["max_len"] for r in rounds)))

    n_host = [r["n_new"].tolist() for r in plan.rounds]

    def set_host_len(r):
        # the caller's host copy of len (the timers count the attention's bytes from it)
        for b in range(A):
            cache.len_host[b] = plan.crop[b] + sum(n[b] for n in n_host[:r])

    def step(rs=rounds):
        cache.len.copy_(crop, non_blocking=True)         # the caller's crop: keep rows [0, crop[b])
        for i, (r, o) in enumerate(zip(rs, outs)):
            set_host_len(i + 1)
            model.dspark_append_context_kv(cache, r["hidden"], r["n_new"], pos0, ws=aws)
            model.dspark_draft_rows(cache, r["anchors"], r["block_pos"], r["max_len"], o["tokens"], o["lengths"],
                                    o["conf"], None, ws=dws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    warmup = max(args.warmup, 3)
    for _ in range(warmup):
        step()
    barrier()
    assert model.dspark_read_device_status() == 0, "device status set during warm-up"
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

    # the draft call alone (last round's shapes), untimed by the headline
    def time_calls(fn, reps=10):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    r_last, o_last = rounds[-1], outs[-1]
    round_ms = time_calls(lambda: model.dspark_draft_rows(cache, r_last["anchors"], r_last["block_pos"],
                                                          r_last["max_len"], o_last["tokens"], o_last["lengths"],
                                                          o_last["conf"], None, ws=dws))

    # e2e: host buffers, copies inside the timed region, results read back every round
    h_rounds = [{k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in r.items()} for r in plan.rounds]
    d_rounds = [{k: (torch.empty_like(v) if torch.is_tensor(v) else v) for k, v in r.items()} for r in rounds]
    h_outs = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in o.items()} for o in outs]
    h_crop = torch.tensor(plan.crop, dtype=torch.int32).pin_memory()

    def e2e_step():
        cache.len.copy_(h_crop, non_blocking=True)
        for i, (h, d, o, ho) in enumerate(zip(h_rounds, d_rounds, outs, h_outs)):
            set_host_len(i + 1)
            for k in ("hidden", "n_new", "anchors", "block_pos"):
                d[k].copy_(h[k], non_blocking=True)
            model.dspark_append_context_kv(cache, d["hidden"], d["n_new"], pos0, ws=aws)
            model.dspark_draft_rows(cache, d["anchors"], d["block_pos"], d["max_len"], o["tokens"], o["lengths"],
                                    o["conf"], None, ws=dws)
            for k in ("tokens", "lengths", "conf"):
                ho[k].copy_(o[k], non_blocking=True)
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
    h2d = h_crop.numel() * 4 + sum(h[k].numel() * h[k].element_size() for h in h_rounds
                                   for k in ("hidden", "n_new", "anchors", "block_pos"))
    d2h = sum(v.numel() * v.element_size() for o in h_outs for v in o.values())
    assert model.dspark_read_device_status() == 0, "device status set during the timed steps"

    # the job's time is its slowest rank's
    from block_draft_model_dspark_b200.sharding import max_over_ranks
    ms_total = max_over_ranks(ms_total)
    e2e_ms = max_over_ranks(e2e_ms)

    if rank == 0:
        tok_per_step = plan.tokens_per_step * world
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
                     else "fallback (MEASURED_PEAKS.json absent)", "traffic": traffic_for(dom, wl.name),
                     "algorithmic_bytes_per_launch": dk["bytes"] / max(dk["launches"], 1),
                     "algorithmic_flops_per_launch": dk["flops"] / max(dk["launches"], 1),
                     "avg_launch_us": per_launch_ms * 1e3})
        kern = {k: {"ms_per_step": v["ms"] / args.steps, "share": v["ms"] / ms_breakdown if ms_breakdown else 0.0,
                    "launches_per_step": v["launches"] / args.steps,
                    "GB_per_s": v["bytes"] / (v["ms"] / 1e3) / 1e9 if v["ms"] > 0 else None,
                    "TFLOP_per_s": v["flops"] / (v["ms"] / 1e3) / 1e12 if v["ms"] > 0 else None}
                for k, v in kinds.items()}
        cfg = workload_config(wl, plan)
        cfg.update({"parallelism": f"dp{world} (every GPU serves the workload's rows; no collective)",
                    "kv_cache": "v_only (v alone; the attention rebuilds k = rope(v * k_norm))" if v_only
                    else "k and v",
                    "l2": "inputs larger than L2: 3.7 GB of dense weights (1.04 GB at 4 bits) streamed per round",
                    "round_us": round_ms * 1e3, "project_full_context_us": project_full_ms * 1e3,
                    "project_full_context_rows": project_rows,
                    "us_per_step_with_kernel_events": ms_breakdown / args.steps * 1e3,
                    "us_per_step": ms_per_step * 1e3, "us_per_round": ms_per_step * 1e3 / len(plan.rounds)})
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, random-init)",
                "config": cfg, "roofline": roof,
                "e2e": {"value": tok_per_step / (e2e_ms / args.steps / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": launches, "clocks": clocks, "kernels": kern}
        if world == 1 and not args.no_cpu_baseline:
            rows = oracle_sample_rows(wl, plan)
            times = oracle_steps(wl, plan, rows, 1, time_budget_s=60.0)
            threads, cores = host_threads()
            tok = len(plan.rounds) * len(rows) * G
            line["cpu_baseline"] = {"value": tok / times[0], "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                    "sample": cpu_sample_desc(wl, plan, rows, 1, 0) + f", {times[0]:.2f} s",
                                    "host_cpus": cores}
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
    kvt = model.kv_torch_dtype
    q = torch.randn(A, G, nH, hd, generator=g, device=dev).to(kvt)
    kb = torch.randn(A, G, nKv, hd, generator=g, device=dev).to(kvt)
    vb = torch.randn(A, G, nKv, hd, generator=g, device=dev).to(kvt)
    out = torch.empty(A, G, nH, hd, device=dev, dtype=kvt)
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


def run_round_case(args, wl):
    """The workload's step (append + draft rounds) on a model of the workload's shapes, with
    the layer count and the vocabulary optionally reduced (a case small enough for a full ncu
    capture of one launch): warm-up steps, then `--steps` steps timed together. Prints one JSON
    case line (not the bench line: a reduced model is not the workload)."""
    import dataclasses
    import torch
    import block_draft_model_dspark_b200 as dsp
    from block_draft_model_dspark_b200 import build as libbuild
    from synthetic import make_weights
    libbuild.build()
    m = wl.model
    if args.layers:
        m = m.replace(num_hidden_layers=args.layers)
    if args.vocab:
        m = m.replace(vocab_size=args.vocab, mask_token_id=args.vocab - 1)
    wl = dataclasses.replace(wl, model=m)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    model = dsp.DsparkModel(m, {k: v.to(dev) for k, v in make_weights(m, wl.seed).items()})
    plan = StepPlan(wl)
    A, G = plan.A, m.block_size
    pos0 = plan.pos0.to(dev)
    v_only = use_v_only(args, m)
    cache = dsp.KvCache(model, A, plan.capacity, v_only=v_only, pos0=pos0 if v_only else None)
    init_hidden = plan.init_hidden.to(dev)
    init_n = torch.tensor(plan.init_len, dtype=torch.int32, device=dev)
    cache.set_lengths([0] * A)
    model.dspark_append_context_kv(cache, init_hidden, init_n, pos0,
                                   ws=model.workspace(model.project_workspace_bytes(A * int(init_hidden.shape[1]))))
    del init_hidden
    crop = torch.tensor(plan.crop, dtype=torch.int32, device=dev)
    rounds = [{k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in r.items()} for r in plan.rounds]
    outs = [{"tokens": torch.empty(A, G, dtype=torch.int32, device=dev),
             "lengths": torch.empty(A, dtype=torch.int32, device=dev),
             "conf": torch.empty(A, G, dtype=torch.float32, device=dev)} for _ in rounds]
    aws = model.workspace(model.project_workspace_bytes(A * max(int(r["hidden"].shape[1]) for r in rounds)))
    dws = model.workspace(model.draft_workspace_bytes(A, max(r["max_len"] for r in rounds)))

    def step():
        cache.len.copy_(crop, non_blocking=True)
        for r, o in zip(rounds, outs):
            model.dspark_append_context_kv(cache, r["hidden"], r["n_new"], pos0, ws=aws)
            model.dspark_draft_rows(cache, r["anchors"], r["block_pos"], r["max_len"], o["tokens"], o["lengths"],
                                    o["conf"], None, ws=dws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    assert model.dspark_read_device_status() == 0
    print(json.dumps({"case": "round", "workload": wl.name, "layers": m.num_hidden_layers, "vocab": m.vocab_size,
                      "kv_cache": "v_only" if v_only else "kv",
                      "ms_per_step": e0.elapsed_time(e1) / max(args.steps, 1), "steps": args.steps,
                      "note": "reduced model for profiling; not the bench line"}), flush=True)


def main():
    args = parse()
    from synthetic import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.case == "attention":
        run_attention_case(args, wl)
        return
    if args.case == "round":
        run_round_case(args, wl)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_dspark(args, wl)


if __name__ == "__main__":
    main()
