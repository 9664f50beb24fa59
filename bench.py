"""Benchmark of one HARD-KV Cascade Cache decode step on B200.

A *step* is one pass of the whole hot path (score, Logits Calibration, Top-p
budget, compaction, cascade decode attention) over one batch of the
``bf16_b8_ctx16k`` workload (batch 8, 32/8 heads, head dim 128, context 16384 =
dense 256 + condensed 64 + sparse 16064, p = 0.95, clamp [64, 2048]).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch (weak scaling, no data-path
collective); the device time is the max over ranks. Prints one JSON line on
rank 0. ``--impl reference`` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from head_adaptive_kv_b200.workloads import WORKLOADS, make_inputs, to_host_bits  # noqa: E402

WORKLOAD_ID = 2
NSETS = 3  # distinct decode states rotated so that no step re-reads the previous one from L2
GRAPH_STEPS = 12  # steps per replayed CUDA graph (a multiple of NSETS)
METRIC = "decode steps/sec and KV GB/s at 1 B200 (fraction of 8 TB/s HBM roofline)"
NOMINAL_HBM_GBS = 8000.0  # nominal HBM3e bandwidth of the part (DGX figure)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def csrc_hash() -> str:
    """Hash of the kernel sources with comments and blank space removed, so a
    profile stays attached to its kernels across comment-only edits."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "head_adaptive_kv_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(f.encode() + " ".join(text.split()).encode())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel)
        if e and e.get("csrc_hash") == csrc_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---- distributed plumbing ----------------------------------------------------------


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist

    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_value(units_per_rank: int, units_per_step: int, world: int, seconds_max: float, steps: int):
    """Steps/s of the whole job: units all ranks processed / max-over-ranks time."""
    total_units = units_per_rank * world * steps
    return total_units / units_per_step / seconds_max


# ---- algorithmic bytes --------------------------------------------------------------


def logit_floats(G: int) -> int:
    """Floats of one token's per-head logit record (G logits padded to 16 bytes)."""
    return (G + 3) // 4 * 4


def step_bytes(wl, sparse_len, dense_len, cond_len, sel_len) -> int:
    """Bytes one step must move in this design: every sparse key is read once
    and scored (its max-pooled score and its per-head logits written); dense
    and condensed K and V rows are attended; a selected sparse token's V row
    and logit record are read back (its K row is not read again); plus q, the
    outputs and the compacted rows."""
    e = 2 if wl.dtype == torch.bfloat16 else 4
    D = wl.D
    lb = logit_floats(wl.G) * 4
    n = int(np.sum(sparse_len))
    k = int(np.sum(sel_len))
    scored = n * (D * e + 4 + lb)
    attended = int(np.sum(dense_len) + np.sum(cond_len)) * 2 * D * e + k * (D * e + lb)
    q = wl.B * wl.Hq * D * e
    out = wl.B * wl.Hq * (D + 1) * 4
    idx = wl.units * wl.bmax * 4 + wl.units * 4
    return scored + attended + q + out + idx


def score_bytes_of(wl, sparse_len) -> int:
    """Bytes the scoring kernel must move: every sparse key read once, the
    queries read, one fp32 score written per key."""
    e = 2 if wl.dtype == torch.bfloat16 else 4
    n = int(np.sum(sparse_len))
    return n * wl.D * e + wl.B * wl.Hq * wl.D * e + n * 4


# Sparse-tier room kept free while the append is timed (above the launches
# kernel_ms makes: one, 64 captured, 3 + up to 20 replays of 64).
APPEND_ROOM = 2048


def append_bytes(wl) -> int:
    """Algorithmic bytes of one append that rolls the window: per unit the new
    K and V rows read, the oldest window rows read, written to the sparse tier,
    and the new rows written in their place."""
    return wl.units * 8 * wl.D * (2 if wl.dtype == torch.bfloat16 else 4)


def kernel_ms(launch_round, launches_per_round: int, stream, args) -> float:
    """Average device time of one launch: rounds of launches captured in one
    CUDA graph, replayed between CUDA events on the launching stream."""
    rounds = 64
    launch_round()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(rounds):
            launch_round()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, min(20, args.steps // (rounds * launches_per_round)))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / (reps * rounds * launches_per_round)


# ---- clocks -------------------------------------------------------------------------

SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        try:
            self.index = int(vis.split(",")[local_rank]) if vis else local_rank
        except ValueError:
            self.index = local_rank
        self.proc = None
        self.path = os.path.join("/tmp", f"hkv_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9 or not c[0].isdigit() or int(c[0]) != self.index:
                    continue
                try:
                    sm.append(float(c[1]))
                    smax.append(float(c[2]))
                except ValueError:
                    continue
                for n, v in zip(names, c[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.remove(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---- CPU oracle timing ----------------------------------------------------------------


def host_state(x):
    import oracle

    def tier(t):
        return oracle.Tier(to_host_bits(t.k), to_host_bits(t.v), t.len.cpu().numpy())

    return to_host_bits(x.q), tier(x.dense), tier(x.sparse), tier(x.condensed)


def oracle_units(wl, hs, units: list):
    """Run the oracle step on a subset of units (one sub-problem per sequence)."""
    import oracle

    q, dense, sparse, cond = hs
    by_b = {}
    for u in units:
        by_b.setdefault(u // wl.Hkv, []).append(u % wl.Hkv)
    for b, hs_ in by_b.items():
        h0, h1 = min(hs_), max(hs_) + 1
        G = wl.G

        def sub(t):
            ln = t.len.reshape(wl.B, wl.Hkv)[b, h0:h1].copy()
            return oracle.Tier(t.k[b:b + 1, h0:h1], t.v[b:b + 1, h0:h1], ln)

        oracle.step(q[b:b + 1, h0 * G:h1 * G], sub(dense), sub(sparse), sub(cond), 1 / math.sqrt(wl.D),
                    wl.p, wl.bmin, wl.bmax)


def cpu_baseline(wl, hs, min_seconds=10.0):
    """The oracle as it stands on the host cores: whole steps repeated for at
    least min_seconds (at least one)."""
    import oracle

    units = list(range(wl.units))
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_units(wl, hs, units)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    return {"value": reps / dt, "unit": "steps/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} whole step(s) of {wl.name} ({wl.units} units), {dt:.1f} s"}


def config_of(wl, world: int) -> dict:
    """The workload named in every line (both arms)."""
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "D": wl.D,
            "ctx": wl.w_cap + wl.c_cap + wl.n_cap, "dense": wl.w_cap, "condensed": wl.c_cap,
            "sparse": wl.n_cap, "p": wl.p, "clamp": [wl.bmin, wl.bmax], "layout": "pad_max",
            "l2": f"inputs larger than L2 ({wl.units * wl.n_cap * wl.D * 2 / 1e6:.0f} MB of sparse "
                  f"keys per set), {NSETS} distinct sets rotated",
            "parallelism": f"replicas x{world}",
            "timing": f"CUDA graphs of {GRAPH_STEPS} consecutive steps replayed back to back; CUDA events around the K steps"}


# ---- the other workloads, the timeline and the rows beyond the step -----------------


def capture(fn, stream):
    """One call of fn outside capture (warm-up), then fn captured in a CUDA graph."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def replay_ms(g, stream, min_ms=300.0, warm=3) -> float:
    """Mean device time of one replay of g, timed with CUDA events over enough
    replays to last about min_ms."""
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    one = max(e0.elapsed_time(e1), 1e-3)
    reps = int(max(5, min(20000, min_ms / one)))
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def in_step_spans(hkv, prob, x, tiers, out, ws, stream, reps=20) -> dict:
    """Live in-step times of each kernel of one step: the kernels record their
    earliest start and latest end in the workspace (hkv_set_timeline); medians
    over single-step graph replays, relative to the scorer's start (us)."""
    hkv.set_timeline(True)
    try:
        g = capture(lambda: hkv.step(prob, x.q, *tiers, out, ws), stream)
        hkv.read_timeline(ws)
        rows = []
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize()
            rows.append(hkv.read_timeline(ws))
        del g
    finally:
        hkv.set_timeline(False)
    spans = {}
    for kind in rows[0]:
        rel = [(r[kind][0] - r["score"][0], r[kind][1] - r["score"][0]) for r in rows if kind in r]
        st = statistics.median(a for a, _ in rel) / 1e3
        en = statistics.median(b for _, b in rel) / 1e3
        spans[kind] = {"start_us": round(st, 2), "end_us": round(en, 2), "us": round(en - st, 2)}
    step = statistics.median((max(b for _, b in r.values()) - r["score"][0]) for r in rows) / 1e3
    spans["step_us"] = round(step, 2)
    return spans


def oracle_sample(wl, hs, layers: int, seconds: float = 2.0) -> dict:
    """The oracle on as many units of one layer as fit in about `seconds`,
    scaled to steps/s of the whole workload (all units of all layers)."""
    import oracle

    done, t0 = 0, time.perf_counter()
    while True:
        oracle_units(wl, hs, [done % wl.units])
        done += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or done >= wl.units:
            break
    per_unit = dt / done
    return {"value": round(1.0 / (per_unit * wl.units * layers), 6), "unit": "steps/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done} unit(s) of one layer in {dt:.1f} s, scaled to {wl.units} units x {layers} layer(s)"}


def workload_entry(hkv, wl, device, stream, p=None, with_oracle=True) -> dict:
    """Throughput of one workload: all its layers' steps issued back to back on
    one stream, captured in one CUDA graph and replayed."""
    peak, peak_kind = peaks()
    p = wl.p if p is None else p
    xs = [make_inputs(wl, device, layer) for layer in range(wl.layers)]
    prob = hkv.Problem(wl.B, wl.Hq, wl.Hkv, wl.D, wl.dtype, p, wl.bmin, wl.bmax)
    tiers = [[hkv.Tier(t.k, t.v, t.len) for t in (x.dense, x.sparse, x.condensed)] for x in xs]
    outs = [hkv.StepOutputs.allocate(prob, tiers[0][1], device) for _ in xs]
    ws = hkv.Workspace(prob, *tiers[0])

    def all_layers():
        for x, t, o in zip(xs, tiers, outs):
            hkv.step(prob, x.q, *t, o, ws)

    g = capture(all_layers, stream)
    ms = replay_ms(g, stream)
    assert ws.status() == 0, f"device status word set on {wl.name}"
    nbytes, ks = 0, []
    for x, o in zip(xs, outs):
        k = o.sel_len.cpu().numpy()
        ks.append(k)
        nbytes += step_bytes(wl, x.sparse.len.cpu().numpy(), x.dense.len.cpu().numpy(),
                             x.condensed.len.cpu().numpy(), k)
    ks = np.concatenate(ks)
    gbs = nbytes / (ms / 1e3) / 1e9
    e = {"workload": wl.name, "p": p, "layers": wl.layers, "units_per_layer": wl.units,
         "step_us": round(ms * 1e3, 2), "steps_per_s": round(1e3 / ms, 2),
         "bytes_per_step": int(nbytes), "kv_gbs": round(gbs, 1),
         "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4), "frac_of_peak": round(gbs / peak, 4),
         "peak_kind": peak_kind,
         "budgets": {"min": int(ks.min()), "median": int(np.median(ks)), "max": int(ks.max()),
                     "mean": round(float(ks.mean()), 1)}}
    # live in-step kernel spans of the first layer's step
    e["in_step"] = in_step_spans(hkv, prob, xs[0], tiers[0], outs[0], ws, stream, reps=5)
    if with_oracle:
        e["cpu_baseline"] = oracle_sample(wl.with_(p=p), host_state(xs[0]), wl.layers)
    del g
    return e


def mti_entry(hkv, wl, x, prob, tiers, plain_ms, device, stream, horizon=4) -> dict:
    """Rewrite Cache vs Sparse Loading on one decode state: a fresh step that
    also rewrites every unit's selection, a step that reuses the rewrites, and
    the number of reuse steps that pay for a rewrite."""
    st = hkv.MtiState.allocate(prob, device, 0, 0, horizon * max(wl.bmax, 1))
    out = hkv.StepOutputs.allocate(prob, tiers[1], device)
    ws = hkv.Workspace(prob, *tiers)

    def fresh():
        st.left.zero_()
        st.mode.zero_()
        hkv.step_mti(prob, x.q, *tiers, st, out, ws)

    rw_ms = replay_ms(capture(fresh, stream), stream)
    st.left.fill_(1 << 30)  # every unit keeps reusing the rewrite the last fresh step made
    reuse_ms = replay_ms(capture(lambda: hkv.step_mti(prob, x.q, *tiers, st, out, ws), stream), stream)
    assert ws.status() == 0
    gain = plain_ms - reuse_ms
    return {"workload": wl.name, "policy": f"L_lower 0, L_upper 0 (every unit rewrites), horizon {horizon}",
            "plain_step_us": round(plain_ms * 1e3, 2), "rewrite_step_us": round(rw_ms * 1e3, 2),
            "reuse_step_us": round(reuse_ms * 1e3, 2),
            "rewrite_cost_us": round((rw_ms - plain_ms) * 1e3, 2),
            "steps_to_amortize": round((rw_ms - plain_ms) / gain, 3) if gain > 0 else None,
            "cycle_steps_per_s": round(horizon / (rw_ms + (horizon - 1) * reuse_ms) * 1e3, 1)}


def condense_entry(hkv, wl, x, prob, out, device, stream, block=256) -> dict:
    """One condensation pass with every unit's sparse tier full (MERGE)."""
    sk, sv, cv, ck = (t.clone() for t in (x.sparse.k, x.sparse.v, x.condensed.v, x.condensed.k))
    slen0, clen0 = x.sparse.len.clone(), torch.zeros_like(x.condensed.len)
    slen, clen = slen0.clone(), clen0.clone()
    sp, co = hkv.Tier(sk, sv, slen), hkv.Tier(ck, cv, clen)
    w = torch.zeros(wl.units, wl.c_cap, device=device)
    ws = hkv.Workspace(prob, None, sp, co)
    z = torch.zeros(wl.units, wl.n_cap, device=device)
    m = torch.zeros(wl.units, device=device)
    lz = torch.zeros(wl.units, device=device)

    def once():
        slen.copy_(slen0)
        clen.copy_(clen0)
        hkv.condense(prob, sp, co, w, ws, block, wl.n_cap, hkv.CONDENSE_MERGE, z=z, m=m, logZ=lz)

    ms = replay_ms(capture(once, stream), stream, min_ms=100.0)
    assert ws.status() == 0
    e = 2 if wl.dtype == torch.bfloat16 else 4
    moved = int(slen0.sum().item()) - wl.units * block
    nbytes = moved * 2 * wl.D * e * 2 + wl.units * block * 2 * wl.D * e
    return {"workload": wl.name, "block": block, "policy": "merge", "us": round(ms * 1e3, 2),
            "gbs": round(nbytes / (ms / 1e3) / 1e9, 1), "us_per_step_amortized": round(ms * 1e3 / block, 3)}


# ---- our arm ----------------------------------------------------------------------------


def run_ours(args):
    from head_adaptive_kv_b200 import hkv

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    wl = WORKLOADS[WORKLOAD_ID]

    sets = []
    for s in range(NSETS):
        x = make_inputs(wl, device, layer=100 * rank + s)
        prob = hkv.Problem(wl.B, wl.Hq, wl.Hkv, wl.D, wl.dtype, wl.p, wl.bmin, wl.bmax)
        tiers = [hkv.Tier(t.k, t.v, t.len) for t in (x.dense, x.sparse, x.condensed)]
        out = hkv.StepOutputs.allocate(prob, tiers[1], device)
        sets.append((x, prob, tiers, out))
    ws = hkv.Workspace(sets[0][1], *sets[0][2])
    stream = torch.cuda.current_stream()

    # CUDA graphs of GRAPH_STEPS consecutive steps each (the input sets in
    # rotation, every step one full hkv_step over its own decode state), plus
    # one single-step graph per set for a remainder of steps
    for x, prob, tiers, out in sets:
        hkv.step(prob, x.q, *tiers, out, ws)
    torch.cuda.synchronize()
    captured0 = hkv.launch_count()
    multi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(multi):
        for r in range(GRAPH_STEPS):
            x, prob, tiers, out = sets[r % NSETS]
            hkv.step(prob, x.q, *tiers, out, ws)
    singles = []
    for x, prob, tiers, out in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            hkv.step(prob, x.q, *tiers, out, ws)
        singles.append(g)
    torch.cuda.synchronize()
    launches_per_step = (hkv.launch_count() - captured0) // (GRAPH_STEPS + NSETS)

    def run_steps(k):
        """k steps: whole multi-step graphs, then single-step graphs."""
        for _ in range(k // GRAPH_STEPS):
            multi.replay()
        for i in range(k % GRAPH_STEPS):
            singles[i % NSETS].replay()

    run_steps(args.warmup)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    launches0 = hkv.launch_count()
    barrier(dist, device)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    run_steps(args.steps)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(dist, device)
    clk = clocks.stop()
    region_ms = t_start.elapsed_time(t_end)
    per_launch_ms = region_ms / args.steps
    # launches inside the timed region: the library's own kernels recorded in
    # each replayed graph (counted at capture) plus any launched directly
    gpu_launches = args.steps * launches_per_step + (hkv.launch_count() - launches0)
    assert ws.status() == 0, "device status word set during the benchmark"

    region_ms_max = max_over_ranks(region_ms, dist, device)
    launch_ms_max = max_over_ranks(per_launch_ms, dist, device)
    value = whole_job_value(wl.units, wl.units, world, region_ms_max / 1e3, args.steps)

    # algorithmic bytes of one step, from the measured budgets of each set
    nbytes = []
    for x, prob, tiers, out in sets:
        nbytes.append(step_bytes(wl, x.sparse.len.cpu().numpy(), x.dense.len.cpu().numpy(),
                                 x.condensed.len.cpu().numpy(), out.sel_len.cpu().numpy()))
    bytes_per_step = float(np.mean(nbytes))
    step_gbs = bytes_per_step / (launch_ms_max / 1e3) / 1e9

    # The dominant kernel, the scorer, timed on its own: R rounds of one launch
    # per input set, captured in one graph and replayed on the launching stream.
    zbuf = torch.empty(wl.units, sets[0][2][1].cap, dtype=torch.float32, device=device)
    score_ms = kernel_ms(lambda: [hkv.score(prob, x.q, tiers[1], zbuf, ws) for x, prob, tiers, out in sets],
                         NSETS, stream, args)
    score_ms = max_over_ranks(score_ms, dist, device)
    attn_ms = kernel_ms(lambda: [hkv.cascade_decode(prob, x.q, *tiers[:2], out.idx, out.sel_len, tiers[2],
                                                    out.out, ws, lse=out.lse) for x, prob, tiers, out in sets],
                        NSETS, stream, args)
    attn_ms = max_over_ranks(attn_ms, dist, device)
    # the step with the fitted temperature (beta per unit solved before the
    # selection), same rotation of decode states
    fit_outs = []
    for x, prob, tiers, out in sets:
        fo = hkv.StepOutputs.allocate(prob, tiers[1], device)
        fo.beta_fit = torch.zeros(wl.units, device=device)
        fit_outs.append(fo)
    fitted_ms = kernel_ms(lambda: [hkv.step(prob, x.q, *tiers, fo, ws)
                                   for (x, prob, tiers, out), fo in zip(sets, fit_outs)], NSETS, stream, args)
    fitted_ms = max_over_ranks(fitted_ms, dist, device)
    del fit_outs
    # KV append with the dense-window roll, timed on copies of one decode state
    # whose sparse tiers keep room for every append of the timing (so each
    # launch moves a full window row into the sparse tier)
    x0, prob0 = sets[0][0], sets[0][1]
    room = APPEND_ROOM
    a_dense = hkv.Tier(x0.dense.k.clone(), x0.dense.v.clone(), x0.dense.len.clone())
    a_sparse = hkv.Tier(x0.sparse.k.clone(), x0.sparse.v.clone(),
                        torch.clamp(x0.sparse.len - room, min=0).to(torch.int32))
    a_head = torch.zeros(wl.units, dtype=torch.int32, device=device)
    a_new = torch.randn(2, wl.B, wl.Hkv, wl.D, device=device).to(wl.dtype)
    append_ms = kernel_ms(lambda: hkv.append(prob0, a_new[0], a_new[1], a_dense, a_head, a_sparse, ws), 1,
                          stream, args)
    append_ms = max_over_ranks(append_ms, dist, device)
    grew = int((a_sparse.len - torch.clamp(x0.sparse.len - room, min=0)).min().item())
    assert 0 < grew < room, "append timing ran out of sparse room"
    del a_dense, a_sparse
    assert ws.status() == 0, "device status word set during the kernel timing"
    score_bytes = float(np.mean([score_bytes_of(wl, x.sparse.len.cpu().numpy()) for x, *_ in sets]))
    achieved_gbs = score_bytes / (score_ms / 1e3) / 1e9
    peak, peak_kind = peaks()
    kernel = f"k_score_stream<2,{wl.D},{wl.G}>"
    roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved_gbs / peak, 4), "traffic": traffic_from_profile(kernel),
                "peak_kind": peak_kind, "kernel": kernel, "bytes_per_launch": int(score_bytes),
                "launch_us": round(score_ms * 1e3, 2)}
    # the attention again, through the entry point that allocates nothing
    noalloc_ms = kernel_ms(lambda: [hkv.cascade_decode_noalloc(prob, x.q, *tiers[:2], out.idx, out.sel_len,
                                                               tiers[2], out.out, lse=out.lse)
                                    for x, prob, tiers, out in sets], NSETS, stream, args)
    noalloc_ms = max_over_ranks(noalloc_ms, dist, device)
    kernels = {"step_us": round(launch_ms_max * 1e3, 2), "step_gbs": round(step_gbs, 1),
               "score_us": round(score_ms * 1e3, 2), "attn_us": round(attn_ms * 1e3, 2),
               "attn_noalloc_us": round(noalloc_ms * 1e3, 2),
               "append_us": round(append_ms * 1e3, 2),
               "fitted_step_us": round(fitted_ms * 1e3, 2),
               "append_bytes": int(append_bytes(wl))}
    # live in-step spans of every kernel of the step (device timeline)
    kernels["in_step"] = in_step_spans(hkv, *sets[0][1:2], sets[0][0], sets[0][2], sets[0][3], ws, stream)

    # end to end through the public API: per step, copy the step's query and the
    # per-unit lengths from pinned host memory, run, and read the outputs back
    # into pinned host memory. The host does not wait for a step before issuing
    # the next (it issues a step in about a third of the step's device time),
    # and the copies run on two copy streams into and out of two alternating
    # buffers, so step i + 1's inputs travel in and step i - 1's outputs travel
    # back while step i runs; events order each buffer's reuse. Each direction
    # is one copy per step: the inputs sit in one device buffer and the
    # outputs in another.
    x, prob, tiers, out = sets[0]
    lens = [t.len for t in (x.dense, x.sparse, x.condensed)]
    q_bytes = x.q.numel() * x.q.element_size()
    in_bytes = q_bytes + sum(t.numel() * 4 for t in lens)
    n_out, n_lse = out.out.numel(), out.lse.numel()
    out_bytes = (n_out + n_lse + out.sel_len.numel()) * 4
    bufs = []
    for _ in range(2):
        dev_in = torch.empty(in_bytes, dtype=torch.uint8, device=device)
        q_in = dev_in[:q_bytes].view(x.q.dtype).view(x.q.shape)
        q_in.copy_(x.q)
        lens_in, at = [], q_bytes
        for t in lens:
            lens_in.append(dev_in[at:at + t.numel() * 4].view(torch.int32))
            lens_in[-1].copy_(t)
            at += t.numel() * 4
        dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=device)
        oe = hkv.StepOutputs(sel_len=dev_out[(n_out + n_lse) * 4:].view(torch.int32), idx=out.idx,
                             out=dev_out[:n_out * 4].view(torch.float32).view(out.out.shape),
                             lse=dev_out[n_out * 4:(n_out + n_lse) * 4].view(torch.float32).view(out.lse.shape))
        bufs.append({"in": dev_in, "q": q_in, "tiers": [hkv.Tier(t.k, t.v, ln) for t, ln in zip(tiers, lens_in)],
                     "out": dev_out, "o": oe, "ready": torch.cuda.Event(), "done": torch.cuda.Event(),
                     "read": torch.cuda.Event(), "host_out": torch.empty(out_bytes, dtype=torch.uint8).pin_memory()})
    host_in = bufs[0]["in"].cpu().pin_memory()
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    e2e_steps = min(args.steps, 500)
    barrier(dist, device)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)

    def load(i):  # step i's inputs, once step i - 2 has read the buffer
        bf = bufs[i % 2]
        if i >= 2:
            s_in.wait_event(bf["done"])
        with torch.cuda.stream(s_in):
            bf["in"].copy_(host_in, non_blocking=True)
        bf["ready"].record(s_in)

    load(0)
    for i in range(e2e_steps):
        bf = bufs[i % 2]
        if i + 1 < e2e_steps:
            load(i + 1)
        stream.wait_event(bf["ready"])
        if i >= 2:
            stream.wait_event(bf["read"])  # step i - 2's outputs are back on the host
        hkv.step(prob, bf["q"], *bf["tiers"], bf["o"], ws)
        bf["done"].record(stream)
        s_out.wait_event(bf["done"])
        with torch.cuda.stream(s_out):
            bf["host_out"].copy_(bf["out"], non_blocking=True)
        bf["read"].record(s_out)
    for bf in bufs:
        stream.wait_event(bf["read"])
    e1.record(stream)
    torch.cuda.synchronize()
    for bf in bufs:
        assert torch.equal(bf["host_out"][(n_out + n_lse) * 4:].view(torch.int32), out.sel_len.cpu())
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    h2d, d2h = in_bytes, out_bytes
    e2e = {"value": round(whole_job_value(wl.units, wl.units, world, e2e_ms / 1e3, e2e_steps), 2),
           "unit": "steps/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "steps": e2e_steps}

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(wl, host_state(sets[0][0]), args.cpu_seconds)

    # the other workloads, and the rows beyond the step, on one GPU
    extras = None
    if world == 1 and not args.headline_only:
        x0, prob0, tiers0, out0 = sets[0]
        extras = {"mti": mti_entry(hkv, wl, x0, prob0, tiers0, launch_ms_max, device, stream),
                  "condense": condense_entry(hkv, wl, x0, prob0, out0, device, stream)}
        del multi
        singles.clear()
        sets.clear()
        torch.cuda.empty_cache()
        oracle_on = not args.no_cpu_baseline
        per = [workload_entry(hkv, WORKLOADS[1], device, stream, with_oracle=oracle_on)]
        for wid in (3, 5):
            per.append(workload_entry(hkv, WORKLOADS[wid], device, stream, with_oracle=oracle_on))
            torch.cuda.empty_cache()
        for pp in WORKLOADS[4].p_sweep:
            per.append(workload_entry(hkv, WORKLOADS[4], device, stream, p=pp, with_oracle=oracle_on))
            torch.cuda.empty_cache()
        extras["workloads"] = per

    if extras is None:
        del multi
        singles.clear()
    if rank == 0:
        ms = region_ms_max / args.steps
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian decode states with planted heavy hitters)",
            "config": config_of(wl, world),
            "kv_gbs": round(bytes_per_step * world / (region_ms_max / args.steps / 1e3) / 1e9, 1),
            "frac_of_8tbs": round(bytes_per_step / (ms / 1e3) / 1e9 / NOMINAL_HBM_GBS, 4),
            "roofline": roofline,
            "kernels": kernels,
            "cpu_baseline": base,
            "e2e": e2e,
            "gpu_launches": int(gpu_launches),
            "clocks": clk,
            "impl": "ours",
        }
        if extras is not None:
            line["extras"] = extras
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


# ---- reference arm: the CPU oracle ---------------------------------------------------------


def run_reference(args):
    import oracle

    world, rank, local = dist_env()
    if rank != 0:
        return  # rank 0 alone times the oracle
    wl = WORKLOADS[WORKLOAD_ID]
    x = make_inputs(wl, "cpu", layer=0)
    hs = host_state(x)
    # size each step's sample so that warm-up + timed steps take about two minutes
    t0 = time.perf_counter()
    oracle_units(wl, hs, [0])
    t_unit = max(time.perf_counter() - t0, 1e-4)
    per_step = int(max(1, min(wl.units, 120.0 / max(1, args.steps + args.warmup) / t_unit)))
    units = list(range(per_step))
    for _ in range(args.warmup):
        oracle_units(wl, hs, units)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_units(wl, hs, units)
    dt = time.perf_counter() - t0
    value = args.steps * per_step / wl.units / dt
    sample = f"{per_step} of {wl.units} units of {wl.name} per step"
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 / value, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, world), "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "steps/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline workload (no other workloads, trigger or condensation)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
