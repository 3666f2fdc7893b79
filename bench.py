"""Benchmark of the indexer hot path (score + top-K + finalise) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one indexer_topk call over the whole workload (every query row),
inputs resident in HBM.  Prints one JSON line (rank 0).  Under torchrun each
rank runs its own independent problem of the same shape (weak scaling); the
time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from head_weighted_relu_b200 import workloads as W  # noqa: E402

METRIC = "indexer Gpairs/s (causal q·k pairs scored+top-K'd) & % tensor peak; peak HBM GB"
L2_BYTES = 126 * 2 ** 20


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        # wait (at most 3 s) for the first sample, taken before the timed
        # region and left out of the summary, so that sampling is running
        # when the region starts
        if self.proc is not None:
            import select
            ready, _, _ = select.select([self.proc.stdout], [], [], 3.0)
            if ready:
                self.proc.stdout.readline()
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
                self.lines = [ln for ln in out.splitlines() if ln.strip()]
            except Exception:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def rank_workload(wl, rank):
    """Each rank's independent problem: the workload's shape, its own seed."""
    return wl.scaled(seed=wl.seed + 1000 * rank)


def flops_per_pair(wl):
    return 2.0 * wl.H * wl.D


def cpu_baseline(wl, seconds=15.0, max_rows=None):
    """The oracle as it stands, timed on this host's cores on a bounded sample:
    query rows at the end of the workload's query range (the rows that see the
    most keys), drawn with the workload's shapes and distributions."""
    import oracle
    from head_weighted_relu_b200 import indexer as I
    n = 64
    sub = wl.scaled(S=n, q_pos0=wl.q_pos0 + wl.S - n)
    inp = W.generate(sub, "cpu")
    prob = sub.problem()
    hk = W.to_host_bits(inp["k"])
    ks = W.to_host_bits(inp["k_scale"])
    pc = W.to_host_bits(inp["pool_coef"])
    keys = oracle.decode_keys_for(prob, hk, ks, pc)
    done, pairs, t0 = 0, 0, time.perf_counter()
    for t in range(n - 1, -1, -1):
        qs = None if inp["q_scale"] is None else W.to_host_bits(inp["q_scale"][t:t + 1])
        oracle.topk_rows(prob, W.to_host_bits(inp["q"][t:t + 1]), hk, W.to_host_bits(inp["w"][t:t + 1]),
                         np.array([t]), q_scale_rows=qs, k_scale=ks, pool_coef=pc, keys_f64=keys)
        pairs += I.visible_pairs(1, sub.T, sub.visibility, sub.ratio, sub.q_pos0 + t)
        done += 1
        if time.perf_counter() - t0 > seconds or (max_rows and done >= max_rows):
            break
    dt = time.perf_counter() - t0
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count()
    return dict(value=pairs / dt / 1e9, unit="Gpairs/s", cores=cores, kind="oracle",
                sample=f"the last {done} query rows of {wl.name} ({pairs} pairs, {dt:.1f} s); "
                       "NumPy FP64, full score row + stable sort per row, multithreaded BLAS")


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    base = cpu_baseline(wl, seconds=5.0)
    steps = []
    for _ in range(args.warmup):
        cpu_baseline(wl, seconds=2.0, max_rows=2)
    for _ in range(args.steps):
        steps.append(cpu_baseline(wl, seconds=5.0))
    val = statistics.median(s["value"] for s in steps)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "Gpairs/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "S": wl.S, "T": wl.T, "H": wl.H, "D": wl.D, "K": wl.K},
        "cpu_baseline": dict(base, value=val),
        "e2e": {"value": val, "unit": "Gpairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def planned_splits(wl, sms: int) -> int:
    """Key-range splits the library plans for this shape (the host rule in
    capi.cu): with fewer query blocks than half the SMs, SMs / blocks ranges of
    at least 16 key tiles, at most 512.  A split shape adds the merge launch."""
    qb = min(256 // wl.H, 32)
    nb = -(-wl.S // qb)
    if nb * 2 > sms:
        return 1
    g = wl.q_pos0 + wl.S - 1
    n_keys = wl.T // wl.ratio if wl.visibility == W.POOLED else wl.T
    nvis = min(g + 1 if wl.visibility == W.TOKEN else (g + 1) // wl.ratio, n_keys)
    s = min(sms // nb, (nvis + 127) // 128 // 16, 512)
    return s if s >= 2 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsa_prefill_64k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    wl = W.WORKLOADS[args.workload]
    world, rank, local = dist_init()
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    from head_weighted_relu_b200 import indexer as I
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl_r = rank_workload(wl, rank)
    inp = W.generate(wl_r, dev)
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0)
    bufs = I.allocate(prob, dev)
    stream = torch.cuda.current_stream()

    # the FP8 long-context workload also counts, per non-overlapping adjacent
    # query pair, the KV indices the two rows share (binary search)
    shared = torch.empty((wl.S // 2,), dtype=torch.int32, device=dev) if wl.pair_overlap else None

    def step():
        I.topk(inp["q"], inp["k"], inp["w"], wl.K, visibility=wl.visibility, ratio=wl.ratio,
               q_pos0=wl.q_pos0, q_scale=inp["q_scale"], k_scale=inp["k_scale"],
               pool_coef=inp["pool_coef"], buffers=bufs, stream=stream)
        if shared is not None:
            I.indexer_pair_overlap(bufs[0], bufs[1], wl.S, bufs[0].shape[1], shared, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = I.indexer_read_status(bufs[3])

    # ---- timed region: K steps, events per step on the launching stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    pairs = I.visible_pairs(wl.S, wl.T, wl.visibility, wl.ratio, wl.q_pos0)
    value = pairs * world / (ms_step * 1e-3) / 1e9
    peak_mem = torch.cuda.max_memory_allocated(dev) / 1e9

    # the q-cluster preprocessing of the same pairs (shared / left-only /
    # right-only regions), timed on its own on this step's index rows
    regions = None
    if shared is not None:
        width = bufs[0].shape[1]
        outs = [torch.empty((wl.S // 2, width), dtype=torch.int32, device=dev) for _ in range(3)]
        cnt = torch.empty((wl.S // 2, 3), dtype=torch.int32, device=dev)
        for _ in range(3):
            I.indexer_pair_regions(bufs[0], bufs[1], wl.S, width, *outs, cnt, stream)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(10):
            I.indexer_pair_regions(bufs[0], bufs[1], wl.S, width, *outs, cnt, stream)
        r1.record(stream)
        torch.cuda.synchronize()
        r_ms = r0.elapsed_time(r1) / 10
        r_bytes = (bufs[0].numel() + bufs[1].numel() + 3 * outs[0].numel() + cnt.numel()) * 4
        regions = {"ms_per_call": r_ms, "bytes_per_call": r_bytes, "gb_s": r_bytes / (r_ms * 1e-3) / 1e9}
        del outs, cnt

    # decode-like shapes (few query blocks: split key ranges plus a merge) also
    # time indexer_topk_witness, whose seed threshold shortens the per-range
    # selection and the merge without changing the result.  Two seed sources:
    # the same query rows' selection one decode step earlier (one key fewer;
    # queries that change little between steps) and the row above's selection
    # (on these i.i.d. synthetic queries it shares only chance keys).
    splits = planned_splits(wl, torch.cuda.get_device_properties(dev).multi_processor_count)
    witness = None
    if splits > 1 and wl.visibility == W.TOKEN and wl.q_pos0 >= 1:
        prev = I.make_problem(wl.S, wl.T - 1, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0 - 1)
        pb = I.allocate(prev, dev)
        I.indexer_topk(prev, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                       pb[0], pb[1], None, pb[3], stream)
        seed_sets = {"prev_step": pb[0], "row_above": torch.roll(bufs[0], 1, 0).contiguous()}
        wws = torch.empty(I.indexer_witness_workspace_bytes(prob, bufs[0].shape[1]), dtype=torch.uint8, device=dev)
        w_idx, w_len = torch.empty_like(bufs[0]), torch.empty_like(bufs[1])
        witness = {"api": "indexer_topk_witness", "ms_per_call_unseeded": ms_step, "seeds": {
            "prev_step": "the same query rows' output over T - 1 keys",
            "row_above": "output row t - 1 for query row t"}}
        for name, sd in seed_sets.items():
            def wstep():
                I.indexer_topk_witness(prob, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"],
                                       inp["pool_coef"], sd, w_idx, w_len, None, wws, stream)
            for _ in range(3):
                wstep()
            w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            w0.record(stream)
            for _ in range(10):
                wstep()
            w1.record(stream)
            torch.cuda.synchronize()
            witness["ms_per_call_" + name] = w0.elapsed_time(w1) / 10
            witness["identical_" + name] = bool(torch.equal(w_idx, bufs[0]) and torch.equal(w_len, bufs[1]))
        witness["device_status"] = I.indexer_read_status(wws)
        del pb, wws, w_idx, w_len, seed_sets

    pk = _peaks()
    tensor_peak = pk["bf16"] * (2.0 if wl.dtype == "fp8" else 1.0)
    kern_ms = statistics.mean(per)
    achieved = pairs * flops_per_pair(wl) / (kern_ms * 1e-3) / 1e12

    # ---- end to end through the C ABI with host buffers: indexer_topk_host
    # takes page-locked host inputs and outputs; its own copies (keys once,
    # query rows in chunks) run inside the timed region, overlapped with the
    # indexer by the library
    e2e = None
    if not args.no_e2e:
        host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
        h_idx = torch.empty(bufs[0].shape, dtype=torch.int32).pin_memory()
        h_len = torch.empty(bufs[1].shape, dtype=torch.int32).pin_memory()
        hws = torch.empty(I.indexer_host_workspace_bytes(prob), dtype=torch.uint8, device=dev)
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h = h_idx.numel() * 4 + h_len.numel() * 4

        def e2e_step():
            I.indexer_topk_host(prob, host["q"], host["k"], host["w"], host["q_scale"], host["k_scale"],
                                host["pool_coef"], h_idx, h_len, None, hws, stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        n_e2e = max(1, min(args.steps, 5))
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        e2e = {"value": pairs * world / (e2e_ms * 1e-3) / 1e9, "unit": "Gpairs/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "indexer_topk_host (pinned host buffers, copies overlapped with the indexer)"}
        if shared is not None:
            e2e["excludes"] = "the pair-overlap count (it runs on the device rows of the indexer_topk step)"
        del host, hws

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(wl)

    traffic = None
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            traffic = json.load(f).get(wl.name)
    except Exception:
        traffic = None

    launches_per_step = (1 + (1 if splits > 1 else 0) + (1 if wl.visibility == W.POOLED else 0)
                         + (1 if wl.pair_overlap else 0))
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "Gpairs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8-e4m3 (fp32 accumulate)" if wl.dtype == "fp8" else "bf16 (fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": wl.name, "S": wl.S, "T": wl.T, "H": wl.H, "D": wl.D, "K": wl.K,
                       "visibility": ["token", "compressed", "pooled"][wl.visibility], "ratio": wl.ratio,
                       "q_pos0": wl.q_pos0, "pair_overlap": wl.pair_overlap,
                       "parallelism": f"{world} independent problems (one per GPU)",
                       "l2": "inputs larger than L2 (q alone is "
                             f"{inp['q'].numel() * inp['q'].element_size() / 2**30:.2f} GiB)"},
            "pairs_per_step": pairs, "queries_per_s": wl.S * world / (ms_step * 1e-3),
            "tensor_peak_frac": achieved / tensor_peak,
            "peak_hbm_gb": peak_mem,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                         "frac": achieved / tensor_peak, "traffic": traffic,
                         "peak_source": f"{pk['source']} bf16 burst" + (" x2 for fp8 (nominal ratio)" if wl.dtype == "fp8" else ""),
                         "flops_per_pair": flops_per_pair(wl)},
            "clocks": clk.summary(),
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "pair_regions": regions,
            "witness": witness,
            "device_status": status,
            "cpu_baseline": base,
        }
        print(json.dumps(out))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
