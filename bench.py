"""Throughput of attention-saliency KV-cache compaction on B200.

One step = one kvc_compress call over one batch of the workload (default: the Llama-3.1-8B
head layout at 128K context, batch 4): window-softmax scoring, group sums, max-pool,
top-k with sinks and recent window, and the K/V gather.  Inputs are seeded synthetic
tensors resident in HBM before timing starts.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvc|reference] [--workload NAME]

With N > 1 it runs under torchrun, one rank per GPU; every rank compacts its own batch of
independent sequences (weak scaling, no collective on the data path) and the time is the
max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_kv_kvc_b200 import synth  # noqa: E402

METRIC = "KV tokens compressed/sec and achieved HBM GB/s (% of peak) at 128K ctx"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- host logic

def rank_seeds(wl: synth.Workload, rank: int) -> tuple:
    """Seeds of the sequences that rank `rank` compacts: rank 0 uses the workload's own
    seeds, rank r the next B seeds after rank r-1's (independent sequences)."""
    return tuple(int(s) + rank * wl.B for s in wl.seeds)


def algorithmic_bytes(wl: synth.Workload) -> dict:
    """Compulsory HBM bytes of one compaction call, by stage.

    score:  every key row of every layer once, the window queries once, and the fp32 score
            rows written once (B * Hs * N * 4);
    select: the score rows read and pooled rows written/read (kept in L2 in practice but
            counted), the kept index lists written;
    gather: the kept K and V rows read and written (and the TSP hidden rows).
    """
    e = 4 if wl.dtype == "f32" else 2
    L, B, Hq, Hkv, N, D, w = wl.n_layers, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.window
    Hs = Hkv if wl.scope == synth.SCOPE_PER_KV_HEAD else 1
    k_read = L * B * Hkv * N * D * e
    q_read = L * B * Hq * w * D * e
    score_write = B * Hs * N * 4
    score = k_read + q_read + score_write
    kb = wl.kv_budget
    gather = 2 * (2 * B * Hkv * kb * D * e)  # K and V, read + write
    idx = B * Hs * kb * 4
    if wl.tsp_rate > 0:
        n_tsp = tsp_count(wl)
        gather += 2 * B * n_tsp * wl.hidden_dim * e
        idx += B * n_tsp * 4
    return {"score": score, "k_read": k_read, "q_read": q_read, "score_write": score_write,
            "gather": gather, "idx": idx, "total": k_read + q_read + gather + idx}


def tsp_count(wl) -> int:
    if wl.tsp_rate <= 0:
        return 0
    sel = int(np.floor(float(np.float32(wl.tsp_rate)) * wl.N))
    sel = min(sel, wl.N - wl.window - wl.n_sink)
    return sel + wl.n_sink + wl.window if sel >= 1 else 0


L2_BYTES = 126 * 2**20  # B200 L2


def measured_peaks() -> tuple:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "long_context_kv_kvc_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, digest: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        rec = d[kernel][workload]
        return rec["dram_bytes_per_launch"] if rec.get("source_digest") == digest else None
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        return summarize_clocks(rows)


def summarize_clocks(rows) -> dict:
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def num(x):
        try:
            return float(x)
        except ValueError:
            return None

    sm = [num(r[1]) for r in rows if num(r[1]) is not None]
    mx = [num(r[2]) for r in rows if num(r[2]) is not None]
    reasons = set()
    for r in rows:
        for i, n in enumerate(names):
            if r[5 + i].lower().startswith("active"):
                reasons.add(n)
    loaded = [s for s, r in zip(sm, rows) if (num(r[3]) or 0) > 300] or sm
    return {"sm_mhz": statistics.median(loaded) if loaded else None,
            "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU legs

def oracle_units(wl: synth.Workload) -> tuple:
    """The CPU sample: as many (sequence, KV head) units as the host has cores (the oracle
    runs one unit per thread), whole sequences first; returns (sequences, KV heads each)."""
    cores = os.cpu_count() or 1
    if cores >= wl.Hkv:
        return max(1, min(wl.B, cores // wl.Hkv)), wl.Hkv
    return 1, cores


def oracle_sample(wl: synth.Workload, inputs: dict, n_seq: int, heads: int) -> tuple:
    """Runs the fp64 oracle on sequences [0, n_seq), KV heads [0, heads) of each (the
    sample), one thread per unit; returns (seconds, equivalent context tokens)."""
    from oracle import oracle as O
    G = wl.G
    q = inputs["q"][:, :n_seq, :heads * G]
    k = inputs["k"][:, :n_seq, :heads]
    v = inputs["v"][:n_seq, :heads]
    t0 = time.perf_counter()
    O.compress(q, k, v, window=wl.window, n_sink=wl.n_sink, pool_kernel=wl.pool_kernel,
               kv_budget=wl.kv_budget, scope=wl.scope, threads=n_seq * heads)
    dt = time.perf_counter() - t0
    return dt, wl.N * n_seq * heads / wl.Hkv


def run_reference(args, wl, rank, world):
    """The oracle as the reference arm: each step is one bounded sample of the workload."""
    if rank != 0:
        return 0
    inputs = synth.make_inputs(wl, seeds=rank_seeds(wl, 0), with_hidden=False)
    cores = os.cpu_count() or 1
    n_seq, heads = oracle_units(wl)
    for _ in range(max(args.warmup, 0)):
        oracle_sample(wl, inputs, n_seq, heads)
    total_t, total_tok = 0.0, 0.0
    for _ in range(args.steps):
        dt, tok = oracle_sample(wl, inputs, n_seq, heads)
        total_t += dt
        total_tok += tok
    value = total_tok / total_t
    sample = (f"sequences 0-{n_seq - 1} of {wl.B}, KV heads 0-{heads - 1} of {wl.Hkv} ({wl.N} tokens each), "
              f"one oracle thread per (sequence, KV head), per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": n_seq * heads, "kind": "oracle",
                             "sample": sample, "host_cores": cores},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, world) -> dict:
    return {"workload": wl.name, "B_per_gpu": wl.B, "global_batch": wl.B * world, "Hq": wl.Hq,
            "Hkv": wl.Hkv, "N": wl.N, "D": wl.D, "window": wl.window, "n_layers": wl.n_layers,
            "kv_budget": wl.kv_budget, "pool_kernel": wl.pool_kernel, "n_sink": wl.n_sink,
            "tsp_rate": wl.tsp_rate, "parallelism": f"batch-sharded replicas x{world} (no collective)",
            "l2": l2_note(wl)}


def l2_note(wl) -> str:
    k_bytes = wl.n_layers * wl.B * wl.Hkv * wl.N * wl.D * (2 if wl.dtype == "bf16" else 4)
    if k_bytes > L2_BYTES:
        return f"inputs larger than L2 ({k_bytes / 2**30:.2f} GiB of K per GPU), no flush"
    return f"K ({k_bytes / 2**20:.0f} MiB per GPU) fits in L2: timed steps re-read it from L2"


# ----------------------------------------------------------------------------- GPU leg

OTHER_CONFIGS = ("llama8b-32k", "structkv-8layer-32k", "fastkv-tsp20-64k")


def time_sharded_scoring(wl, p, dev, steps: int, stream) -> dict:
    import torch
    from long_context_kv_kvc_b200 import kvc
    q, k = dev["q"][0], dev["k"][0]
    U, nq = wl.B * wl.Hkv, wl.G * wl.window
    cuts = (0, wl.N // 2, wl.N)
    blocks = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        kb = k[:, :, a:b].contiguous()
        ws = torch.empty(kvc.kvc_shard_workspace_size(p, b - a), dtype=torch.uint8, device="cuda")
        ml = torch.empty((U, nq, 2), dtype=torch.float32, device="cuda")
        sc = torch.empty((wl.B, wl.Hkv, b - a), dtype=torch.float32, device="cuda")
        blocks.append((a, kb, ws, ml, sc))
    ml_all = torch.empty((len(blocks), U, nq, 2), dtype=torch.float32, device="cuda")
    whole = torch.empty((wl.B, wl.Hkv, wl.N), dtype=torch.float32, device="cuda")
    ws_whole = torch.empty(kvc.kvc_workspace_size(p), dtype=torch.uint8, device="cuda")

    def run_blocks():
        for i, (a, kb, ws, ml, sc) in enumerate(blocks):
            kvc.kvc_shard_stats(p, q, kb, a, ml_all[i], ws)
        for a, kb, ws, ml, sc in blocks:
            kvc.kvc_shard_scores(p, q, kb, a, ml_all, sc, ws)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    t_blocks = timed(run_blocks)
    t_whole = timed(lambda: kvc.kvc_score(p, q, k, whole, ws_whole))
    return {"blocks": len(blocks), "shard_stats_and_scores_ms": t_blocks, "kvc_score_ms": t_whole,
            "ratio": t_blocks / t_whole, "calls": steps}


def time_config(wl, rank: int, steps: int, peak: float) -> dict:
    """Mean time of one kvc_compress step of workload `wl` over `steps` CUDA-event-timed
    steps (after 3 warm-up steps), with enough rotating input copies that the inputs of a
    step are not in L2 from the step before; GB/s against the algorithmic bytes."""
    import torch
    from long_context_kv_kvc_b200 import kvc
    inputs = synth.make_inputs(wl, seeds=rank_seeds(wl, rank))
    e = 2 if wl.dtype == "bf16" else 4
    in_bytes = (wl.n_layers + 1) * wl.B * wl.Hkv * wl.N * wl.D * e
    copies = max(1, -(-3 * L2_BYTES // in_bytes))
    dev = [{k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}]
    for _ in range(copies - 1):
        dev.append({k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in dev[0].items()})
    comp = kvc.Compressor(kvc.params_for(wl))
    stream = torch.cuda.current_stream()
    for i in range(3):
        d = dev[i % copies]
        comp.run_device(d["q"], d["k"], d["v"], d.get("hidden"))
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        d = dev[i % copies]
        ev[i][0].record(stream)
        comp.run_device(d["q"], d["k"], d["v"], d.get("hidden"))
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    ab = algorithmic_bytes(wl)
    gbs = ab["total"] / (ms * 1e-3) / 1e9
    return {"ms": ms, "tokens_per_s": wl.B * wl.N / (ms * 1e-3), "algorithmic_bytes": ab["total"], "gbs": gbs,
            "frac_of_peak": gbs / peak, "steps": steps,
            "l2": (f"{copies} rotating input copies ({in_bytes / 2**20:.0f} MiB of K and V each)" if copies > 1
                   else f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB of K and V)")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvc", choices=["kvc", "reference"])
    ap.add_argument("--workload", default=synth.LLAMA8B_128K_B4.name, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--pivot-steps", type=int, default=5,
                    help="calls timed for the pivot metrics (entropy pass, row statistics); 0 skips")
    ap.add_argument("--config-steps", type=int, default=20,
                    help="timed steps of each other configuration (32K, StructKV 8 layers, FastKV TSP); 0 skips")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flags", type=int, default=0, help="kvc_params.flags (1 = CUDA-core scoring)")
    ap.add_argument("--no-clocks", action="store_true",
                    help="skip nvidia-smi clock sampling and its 1 s warm loop (for profiler runs)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        return run_reference(args, wl, rank, world)

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from long_context_kv_kvc_b200 import kvc

    inputs = synth.make_inputs(wl, seeds=rank_seeds(wl, rank))
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}
    p = kvc.params_for(wl, flags=args.flags)
    comp = kvc.Compressor(p)
    stream = torch.cuda.current_stream()

    # one set of stage events per timed step (score stage = the dominant kernel)
    n_ev = kvc.KVC_STAGE_COUNT + 1
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for evs in events:
        for e in evs:
            e.record(stream)  # materialise the underlying cudaEvent_t
    handles = [(ctypes.c_void_p * n_ev)(*[e.cuda_event for e in evs]) for evs in events]

    def step(i=None):
        p.stage_events = ctypes.cast(handles[i], ctypes.POINTER(ctypes.c_void_p)) if i is not None else None
        comp.run_device(dev["q"], dev["k"], dev["v"], dev.get("hidden"))

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if kvc.kvc_poll_error() != kvc.KVC_OK:
        raise RuntimeError("device-side error during warm-up")

    sampler = None
    if not args.no_clocks:
        sampler = ClockSampler(local)
        sampler.start()
        # keep the GPU busy ~1 s under the sampler before the timed region
        t_end = time.time() + 1.0
        while time.time() < t_end:
            step()
            torch.cuda.synchronize()

    n_before = kvc.kvc_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = (kvc.kvc_launch_count() - n_before) // 1
    clocks = sampler.stop() if sampler else None
    ms = t0.elapsed_time(t1)
    if kvc.kvc_poll_error() != kvc.KVC_OK:
        raise RuntimeError("device-side error during the timed region")

    stage_ms = [[evs[s].elapsed_time(evs[s + 1]) for s in range(n_ev - 1)] for evs in events]
    score_ms = sum(x[kvc.KVC_STAGE_SCORE] for x in stage_ms) / args.steps
    select_ms = sum(x[kvc.KVC_STAGE_SELECT] for x in stage_ms) / args.steps
    gather_ms = sum(x[kvc.KVC_STAGE_GATHER] for x in stage_ms) / args.steps

    t = torch.tensor([ms], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    ms_step = ms_max / args.steps
    tokens = wl.B * wl.N * world
    value = tokens / (ms_step / 1e3)

    ab = algorithmic_bytes(wl)
    peak, peak_kind = measured_peaks()
    achieved = ab["score"] / (score_ms / 1e3) / 1e9
    tc_path = not (args.flags & 1) and wl.dtype == "bf16"
    digest = source_digest("score_tc.cu", "tc_ptx.cuh") if tc_path else source_digest("score_simt.cu")
    kernel_name = "score_tc" if tc_path else "score_simt"
    traffic = recorded_traffic(kernel_name, wl.name, digest)

    # end to end through the public API: pinned host inputs -> device -> compact cache -> host
    e2e = None
    if args.e2e_steps > 0:
        host = {k: v.pin_memory() for k, v in inputs.items() if isinstance(v, torch.Tensor)}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(v.numel() * v.element_size() for v in comp.out.values())
        comp(host["q"], host["k"], host["v"], host.get("hidden"))  # warm-up
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            comp(host["q"], host["k"], host["v"], host.get("hidden"))
        e1.record(stream)
        torch.cuda.synchronize()
        te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device="cuda")
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": tokens / (float(te.item()) / args.e2e_steps / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # the pivot-detection metrics (StructKV sec. 2): cost of the entropy in the scoring pass
    # and of the per-row kept mass / candidate variance, outside the timed region
    pivot = csm_round = decode_att = None
    if args.pivot_steps > 0:
        Hs = wl.Hkv if wl.scope == kvc.KVC_SCOPE_PER_KV_HEAD else 1
        sc = torch.empty((wl.B, Hs, wl.N), dtype=torch.float32, device="cuda")
        ent = torch.empty((wl.n_layers, wl.B, wl.Hq, wl.window), dtype=torch.float32, device="cuda")
        km = torch.empty((wl.B, Hs), dtype=torch.float32, device="cuda")
        cv = torch.empty((wl.B, Hs), dtype=torch.float32, device="cuda")

        def timed(fn):
            fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.pivot_steps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / args.pivot_steps

        t_plain = timed(lambda: kvc.kvc_score(p, dev["q"], dev["k"], sc, comp.ws))
        t_ent = timed(lambda: kvc.kvc_score_entropy(p, dev["q"], dev["k"], sc, ent, comp.ws))
        t_rs = timed(lambda: kvc.kvc_row_stats(sc, wl.n_sink, wl.window, cv, idx=comp.out["idx_out"], kept_mass=km))
        if kvc.kvc_poll_error() != kvc.KVC_OK:
            raise RuntimeError("device-side error in the pivot-metric calls")
        pivot = {"score_ms": t_plain, "score_with_entropy_ms": t_ent, "row_stats_ms": t_rs,
                 "calls": args.pivot_steps}

        # one CentroidKV Chunked Soft Matching round over the last layer's K and V (r = 0.25,
        # chunks of 64): algorithmic bytes = K read to match + K and V read and the kept rows
        # (K, V, degree, position) written; then one decode step's attention (one query per
        # query head) over the centroids with their log-degrees: K, V and degrees read
        if wl.D == 128:
            kl, vl = dev["k"][-1], dev["v"]
            r, ch = 0.25, 64
            m = kvc.kvc_csm_merges(wl.N, wl.n_sink, wl.window, ch, r)
            csm_out = kvc.kvc_csm(kl, vl, wl.n_sink, wl.window, ch, r)
            t_csm = timed(lambda: kvc.kvc_csm(kl, vl, wl.n_sink, wl.window, ch, r, out=csm_out))
            if kvc.kvc_poll_error() != kvc.KVC_OK:
                raise RuntimeError("device-side error in the clustering round")
            row = wl.D * kl.element_size()
            nbytes = wl.B * wl.Hkv * (3 * wl.N * row + (wl.N - m) * (2 * row + 8))  # + degree, position
            csm_round = {"ratio": r, "chunk": ch, "ms": t_csm, "gbs": nbytes / (t_csm * 1e-3) / 1e9,
                         "algorithmic_bytes": nbytes, "frac_of_peak": nbytes / (t_csm * 1e-3) / 1e9 / peak}
            n_c = wl.N - m
            qd = torch.randn((wl.B, wl.Hq, 1, wl.D), generator=torch.Generator().manual_seed(5)).to(kl.dtype).cuda()
            att = torch.empty((wl.B, wl.Hq, 1, wl.D), dtype=torch.float32, device="cuda")
            att_ws = torch.empty(kvc.kvc_decode_attention_workspace_size(wl.B, wl.Hq, wl.Hkv, 1, n_c),
                                 dtype=torch.uint8, device="cuda")
            t_dec = timed(lambda: kvc.kvc_decode_attention(qd, csm_out["k_out"], csm_out["v_out"],
                                                           deg=csm_out["deg_out"], out=att, ws=att_ws))
            if kvc.kvc_poll_error() != kvc.KVC_OK:
                raise RuntimeError("device-side error in the decode attention")
            dbytes = wl.B * wl.Hkv * n_c * (2 * row + 4) + wl.B * wl.Hq * wl.D * (kl.element_size() + 4)  # + q, out
            decode_att = {"cached_rows": n_c, "query_heads": wl.Hq, "ms": t_dec,
                          "gbs": dbytes / (t_dec * 1e-3) / 1e9, "algorithmic_bytes": dbytes,
                          "frac_of_peak": dbytes / (t_dec * 1e-3) / 1e9 / peak}

    # sequence sharding's scoring, outside the timed region: the workload's keys cut into two
    # blocks, both blocks' kvc_shard_stats and kvc_shard_scores on this GPU one after the
    # other (what two ranks would run, without the exchanges), against kvc_score of the
    # whole; the blocks are copied out of the inputs first
    sharded = None
    if args.pivot_steps > 0 and wl.n_layers == 1 and wl.scope == kvc.KVC_SCOPE_PER_KV_HEAD:
        sharded = time_sharded_scoring(wl, p, dev, args.pivot_steps, stream)
        if kvc.kvc_poll_error() != kvc.KVC_OK:
            raise RuntimeError("device-side error in the sharded scoring")

    # the other configurations at their full sizes (outside the timed region above): the
    # whole compress step, inputs resident in HBM; when a configuration's inputs fit in L2,
    # the steps rotate over enough input copies that every step reads its inputs from HBM
    configs = None
    if args.config_steps > 0:
        configs = {}
        for name in OTHER_CONFIGS:
            wl2 = synth.WORKLOADS[name]
            configs[name] = time_config(wl2, rank, args.config_steps, peak)
        if kvc.kvc_poll_error() != kvc.KVC_OK:
            raise RuntimeError("device-side error in the configuration runs")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_seq, heads = oracle_units(wl)
        dt, tok = oracle_sample(wl, inputs, n_seq, heads)
        cpu = {"value": tok / dt, "unit": "tokens/s", "cores": n_seq * heads, "host_cores": os.cpu_count(),
               "kind": "oracle",
               "sample": f"sequences 0-{n_seq - 1} of {wl.B}, KV heads 0-{heads - 1} of {wl.Hkv} ({wl.N} tokens "
                         f"each), fp64 oracle, one thread per (sequence, KV head)", "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic", "config": config_of(wl, world),
            "hbm_gbs": ab["total"] * world / (ms_step / 1e3) / 1e9,
            "hbm_frac_of_peak": ab["total"] / (ms_step / 1e3) / 1e9 / peak,
            "stages_ms": {"score": score_ms, "select": select_ms, "gather": gather_ms},
            "roofline": {"kernel": kernel_name, "bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "algorithmic_bytes_per_launch": ab["score"]},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
            "configs": configs,
            "sharded_scoring": sharded,
            "pivot_metrics": pivot,
            "csm_round": csm_round,
            "decode_attention": decode_att,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
