#!/usr/bin/env python
"""Benchmark of the DSA lightning indexer (score + top-k) on B200.

One step = one call of the library's dense indexer top-k over one synthetic
dense prefill sequence (T = L = 32768 causal, H = 64, d = 128, k = 2048):
every query scores its whole causal prefix and keeps its top 2048 keys.
The headline `value` is eligible (query, key) pairs per second, in Gpairs/s,
summed over all ranks (each rank processes its own sequence: weak scaling,
no collective on the data path).  Secondary entries (N = 1 only) time the
other workloads of the same library: batched decode at 32K and 128K
(us/step), PIVOT group-proxy prefill at 128K (Reuse and Refine) and HISA
decode at 256K.

Timing: W warm-up steps, then K steps each bracketed by CUDA events on the
launching stream, a 256 MiB L2 flush between steps (outside the events),
a barrier and a device synchronise on both sides of the timed region, and
the max over ranks.  `--impl reference` times the fp64 CPU oracle instead
(rank 0 only) on a bounded sample of the same workload.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "indexer (score+top-k) Gpairs/s prefill"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SM_COUNT, FP32_LANES_PER_SM = 148, 128


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK, sm_max_mhz=1965.0), "fallback"


# ----------------------------------------------------------------- ranks

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over all ranks (device times: the job takes as long as its slowest rank)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(rank: int, T: int):
    """Rank r's own prefill sequence (weak scaling: independent sequences, no data exchange)."""
    return workloads.dense_prefill(seed=2 + 1000 * rank, T=T)


def job_value(pairs_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job Gpairs/s: every rank's pairs over the slowest rank's step time."""
    return pairs_per_rank * world / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.gpu = None

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu:
            cmd += ["-i", self.gpu]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.count(",") >= 7]
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].strip() == "Active"})
        loaded = [s for s in sm if mx and s >= 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------- timing

class L2Flush:
    """Writes a buffer twice the size of L2 (126 MB), then reads another as large: the write evicts
    the step's inputs, the read then evicts the write's dirty lines, so their write-back to HBM
    happens here, outside the timed region, rather than inside the next step."""

    def __init__(self, device, nbytes=256 << 20):
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.clean = torch.ones(nbytes // 4, dtype=torch.float32, device=device)

    def __call__(self):
        self.buf.fill_(1)
        self.clean.max()


def time_steps(step, n, flush):
    """Device time (ms) of n steps, each between CUDA events on the current stream, L2 flushed before each."""
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in ev:
        flush()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


# ------------------------------------------------------------ workloads

class DenseTopk:
    """Dense indexer top-k of a batch (prefill or decode) through the C ABI."""

    def __init__(self, b, device):
        import sparse_attention_indexer_04_b200 as dsa
        self.dsa, self.b, self.k = dsa, b, int(b.params["k"])
        self.lay = dsa.Layout.from_batch(b, device)
        self.Q, self.K, self.W = b.Q.to(device), b.K.to(device), b.W.to(device)
        self.idx = torch.empty(b.n_q, self.k, dtype=torch.int32, device=device)
        self.ws = torch.empty(dsa.index_topk_workspace(self.lay, self.k), dtype=torch.uint8, device=device)
        self.pairs = b.eligible_pairs()
        self.device = device

    def __call__(self):
        self.dsa.index_topk(self.lay, self.Q, self.K, self.W, self.k, idx=self.idx, ws=self.ws)

    def alg_bytes(self):
        b = self.b
        return b.K.numel() * 2 + b.Q.numel() * 2 + b.W.numel() * 4 + b.n_q * self.k * 4

    def e2e(self, steps, flush):
        """The same step from pinned host buffers through the library's host-memory entry point: every
        step copies Q, K, W and the positions in and the indices out, overlapped chunk by chunk with the
        work (two copy streams)."""
        b, dsa = self.b, self.dsa
        hQ, hK, hW = b.Q.pin_memory(), b.K.pin_memory(), b.W.pin_memory()
        hpos = b.q_pos.to(torch.int32).contiguous().pin_memory()
        hidx = torch.empty(b.n_q, self.k, dtype=torch.int32).pin_memory()
        lay = self.lay
        ws = torch.empty(dsa.index_topk_host_workspace(lay, self.k), dtype=torch.uint8, device=self.device)
        s_in, s_out = torch.cuda.Stream(self.device), torch.cuda.Stream(self.device)

        def step():
            dsa.index_topk_host(lay, hpos, hQ, hK, hW, self.k, hidx, ws, in_stream=s_in, out_stream=s_out)

        for _ in range(2):
            step()
        ms = time_steps(step, steps, flush)
        h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hW, hpos)) + 2 * lay.q_off_host.numel() * 4
        out = hidx.numel() * 4
        del ws
        torch.cuda.empty_cache()
        return sum(ms) / steps, h2d, out


class Pivot:
    def __init__(self, b, device, mode):
        import sparse_attention_indexer_04_b200 as dsa
        self.dsa, self.b, self.mode = dsa, b, mode
        p = b.params
        self.k, self.G, self.C = int(p["k"]), int(p["group"]), int(p["n_cand"])
        self.lay = dsa.Layout.from_batch(b, device)
        self.Q, self.K, self.W = b.Q.to(device), b.K.to(device), b.W.to(device)
        self.idx = torch.empty(b.n_q, self.k, dtype=torch.int32, device=device)
        self.ws = torch.empty(dsa.pivot_group_index_workspace(self.lay, self.k, self.G, self.C, mode),
                              dtype=torch.uint8, device=device)

    def __call__(self):
        self.dsa.pivot_group_index(self.lay, self.Q, self.K, self.W, self.k, self.G, self.C, self.mode,
                                   idx=self.idx, ws=self.ws)


class Hisa:
    def __init__(self, b, device):
        import sparse_attention_indexer_04_b200 as dsa
        self.dsa, self.b = dsa, b
        p = b.params
        self.k, self.B, self.keep = int(p["k"]), int(p["block"]), int(p["keep"])
        self.lay = dsa.Layout.from_batch(b, device)
        self.Q, self.K, self.W = b.Q.to(device), b.K.to(device), b.W.to(device)
        self.pooled = dsa.hisa_pool_keys(self.lay, self.K, self.B)
        self.idx = torch.empty(b.n_q, self.k, dtype=torch.int32, device=device)
        self.ws = torch.empty(dsa.hisa_index_workspace(self.lay, self.k, self.B, self.keep), dtype=torch.uint8,
                              device=device)

    def __call__(self):
        self.dsa.hisa_index(self.lay, self.Q, self.K, self.W, self.pooled, self.k, self.B, self.keep,
                            idx=self.idx, ws=self.ws)


def graph_times(step, steps, flush):
    """The step captured once in a CUDA graph: mean device time (us) of a replay with L2 flushed before
    it, and of back-to-back replays (each launch's host latency hidden, as a serving loop would)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    flushed = time_steps(g.replay, steps, flush)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 4 * steps
    e0.record()
    for _ in range(n):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    out = {"us_per_step_l2_flushed": round(1e3 * sum(flushed) / steps, 2),
           "us_per_step_back_to_back": round(1e3 * e0.elapsed_time(e1) / n, 2)}
    del g
    return out


def secondary(device, flush, steps, only=None, pivot_T=131072):
    out = {}

    def run(name, make, extra, graph=False, post=None):
        if only and only not in name:
            return
        try:
            t0 = time.time()
            step = make()
            for _ in range(3):
                step()
            ms = time_steps(step, steps, flush)
            r = {"us_per_step": round(1e3 * sum(ms) / steps, 2), "steps": steps, "setup_s": round(time.time() - t0, 1)}
            r.update(extra(step, sum(ms) / steps))
            if graph:
                try:
                    r["cuda_graph"] = graph_times(step, steps, flush)
                except Exception as e:  # the eager numbers stand without it
                    r["cuda_graph"] = {"error": f"{type(e).__name__}: {e}"[:200]}
            step.dsa.profile_enable(True)                      # a second, separately timed pass per kernel
            time_steps(step, steps, flush)
            prof = step.dsa.profile_read()
            step.dsa.profile_enable(False)
            r["kernels_us_per_step"] = {k: round(1e3 * v[0] / steps, 2) for k, v in prof.items()}
            r["launches_per_step"] = sum(v[1] for v in prof.values()) / steps
            if post:
                r.update(post(step, r["kernels_us_per_step"]))
            out[name] = r
            del step
            torch.cuda.empty_cache()
        except Exception as e:  # keep the headline line even if a secondary workload fails
            out[name] = {"error": f"{type(e).__name__}: {e}"[:300]}

    hbm = load_peaks()[0]["hbm_gbs"]

    def dec_extra(step, ms):
        gbs = step.alg_bytes() / (ms * 1e-3) / 1e9
        return {"alg_bytes": step.alg_bytes(), "achieved_gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}

    run("dense_decode_B16_L32768_mtp2", lambda: DenseTopk(workloads.dense_decode(seed=1), device), dec_extra,
        graph=True)
    run("dense_decode_B16_L131072_mtp2", lambda: DenseTopk(workloads.dense_decode(seed=1, L=131072), device),
        dec_extra, graph=True)
    peaks = load_peaks()[0]
    if not only or "pivot" in only or "reuse" in only or "refine" in only:
        pv = workloads.pivot_prefill(seed=3, T=pivot_T)
        dense_pairs = pv.eligible_pairs()
        for mode, name in ((0, "reuse"), (1, "refine")):
            run(f"pivot_prefill_T{pivot_T}_G16_C8192_{name}", lambda m=mode: Pivot(pv, device, m),
                lambda step, ms: {"dense_equiv_gpairs_s": round(dense_pairs / (ms * 1e-3) / 1e9, 2)},
                post=lambda step, kus, m=mode: pivot_roofline(step.b, m, kus, peaks))
        del pv
    run("hisa_decode_B4_L262144_keep64", lambda: Hisa(workloads.hisa_decode(seed=4), device),
        lambda step, ms: hisa_bytes(step.b, ms, peaks), graph=True)
    return out


def pivot_pairs(b):
    """(proxy scan pairs, Refine pairs) of a PIVOT batch: the proxy of a group scans its sequence's
    keys up to the group's last position; a query of Refine scores the group's candidates inside its
    own prefix, at most min(C, its eligible keys) (exact to within G - 1 per query)."""
    G, C = int(b.params["group"]), int(b.params["n_cand"])
    qo, ko, pos = b.q_offsets.tolist(), b.k_offsets.tolist(), b.q_pos.tolist()
    scan = refine = 0
    for s in range(b.num_seqs):
        L = ko[s + 1] - ko[s]
        for g0 in range(qo[s], qo[s + 1], G):
            g1 = min(g0 + G, qo[s + 1])
            scan += min(L, max(pos[g0:g1]) + 1)
            refine += sum(min(C, L, p + 1) for p in pos[g0:g1])
    return scan, refine


def pivot_roofline(b, mode, kernels_us, peaks):
    """Tensor-pipe fraction of the PIVOT scoring launches (proxy scan; with Refine, also the gathered
    candidate scoring), from their CUDA-event times: 2 H d flop per (row, key) pair against the
    measured bf16 peak; the proxy top-C selection's bytes (each proxy score read once, C candidates
    written per group) against the measured HBM copy bandwidth."""
    scan, refine = pivot_pairs(b)
    flop_pair = 2 * b.H * b.d
    flops = (scan + (refine if mode == 1 else 0)) * flop_pair
    t = kernels_us.get("score_tc", 0.0) * 1e-6
    out = {"proxy_pairs": scan}
    if mode == 1:
        out["refine_pairs"] = refine
    if t > 0:
        tf = flops / t / 1e12
        out["score_tflops"] = round(tf, 1)
        out["score_frac_tensor"] = round(tf / peaks["bf16_tflops"], 4)
    return out


def hisa_bytes(b, ms, peaks):
    """HBM bytes HISA must move per step: each sequence's pooled block keys (fp32, read once for its
    queries), every query's kept blocks' keys (block 0, the `keep` best middle blocks and its own
    block: at most (keep + 2) * B keys of d bf16), Q, W and the index rows; against the measured HBM
    copy bandwidth (the step is latency-bound at this size)."""
    B, keep, k = int(b.params["block"]), int(b.params["keep"]), int(b.params["k"])
    pooled = sum((L + B - 1) // B for L in b.seq_lens()) * b.d * 4
    kept = 0
    for t in range(b.n_q):
        n = int(b.q_pos[t]) + 1
        kept += min(n, (keep + 2) * B) * b.d * 2
    total = pooled + kept + b.Q.numel() * 2 + b.W.numel() * 4 + b.n_q * k * 4
    gbs = total / (ms * 1e-3) / 1e9
    return {"alg_bytes": total, "achieved_gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}


# ------------------------------------------------------------ baselines

def oracle_sample(b, k, budget_s=15.0, max_rows=64):
    """Oracle dense top-k on a growing stratified row sample until ~budget_s of CPU time."""
    import oracle
    threads = oracle.default_threads()
    n = 4
    while True:
        rows = workloads.stratified_rows(b.n_q, n_sample=n, head=1, tail=1)
        pairs = sum(min(int(b.q_pos[r]) + 1, b.seq_lens()[0]) for r in rows)
        t0 = time.perf_counter()
        oracle.dense(b, rows=rows, k=k, threads=threads)
        dt = time.perf_counter() - t0
        if dt > budget_s / 3 or n >= max_rows:
            return pairs, dt, threads, rows
        n *= 2


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    b = workloads.dense_prefill(seed=2)
    k = int(b.params["k"])
    threads = oracle.default_threads()
    rows = workloads.stratified_rows(b.n_q, n_sample=32, head=1, tail=1)
    pairs = sum(int(b.q_pos[r]) + 1 for r in rows)
    for _ in range(args.warmup):
        oracle.dense(b, rows=rows[:2], k=k, threads=threads)
    t = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.dense(b, rows=rows, k=k, threads=threads)
        t.append(time.perf_counter() - t0)
    sec = sum(t) / len(t)
    value = pairs / sec / 1e9
    sample = f"{len(rows)} stratified query rows of the 32K prefill ({pairs} pairs) per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Gpairs/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "dense_prefill_T32768_H64_d128_k2048", "T": 32768, "L": 32768, "H": 64, "d": 128,
                   "k": 2048, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "Gpairs/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "Gpairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ----------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--secondary-steps", type=int, default=5)
    ap.add_argument("--T", type=int, default=32768, help="prefill length (smaller only for profiling captures)")
    ap.add_argument("--only", default=None,
                    help="profiling: run only the secondary workloads whose name contains this (no headline line)")
    ap.add_argument("--pivot-T", type=int, default=131072, help="PIVOT prefill length (smaller for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
        return
    if args.only:
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        sec = secondary(device, L2Flush(device), args.secondary_steps, args.only, args.pivot_T)
        print(json.dumps({"secondary": sec}))
        return

    world, rank, local = dist_setup()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import sparse_attention_indexer_04_b200 as dsa

    peaks, peaks_src = load_peaks()
    b = rank_workload(rank, args.T)
    step = DenseTopk(b, device)
    flush = L2Flush(device)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region
    barrier(world)
    torch.cuda.synchronize()
    n0 = dsa.launch_count()
    with ClockSampler(device) as clk:
        ms = time_steps(step, args.steps, flush)
    launches = dsa.launch_count() - n0
    barrier(world)
    torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(ms), world)
    ms_per_step = total_ms / args.steps
    value = job_value(step.pairs, world, ms_per_step)

    # ---- per-kernel times over a second pass of the same steps (events on the launching stream)
    dsa.profile_enable(True)
    time_steps(step, args.steps, flush)
    prof = dsa.profile_read()
    dsa.profile_enable(False)
    roof, kernels = roofline_entries(prof, step, b, args.steps, peaks, peaks_src)

    e2e_ms, h2d, d2h = step.e2e(max(2, args.steps // 2), flush)
    e2e = {"value": job_value(step.pairs, world, max_over_ranks(e2e_ms, world)), "unit": "Gpairs/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    sec = {}
    if rank == 0 and world == 1:
        if not args.no_secondary:
            del step
            torch.cuda.empty_cache()
            sec = secondary(device, flush, args.secondary_steps)
        pairs, dt, threads, rows = oracle_sample(b, int(b.params["k"]))
        cpu = {"value": pairs / dt / 1e9, "unit": "Gpairs/s", "cores": threads, "kind": "oracle",
               "sample": f"{len(rows)} stratified query rows of the 32K prefill ({pairs} pairs), {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Gpairs/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"dense_prefill_T{args.T}_H64_d128_k2048", "T": args.T, "L": args.T, "H": 64,
                       "d": 128, "k": 2048, "global_batch": world, "seq_len": args.T,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "flushed between timed steps (256 MiB write, then 256 MiB read)",
                       "pairs_per_step_per_gpu": step_pairs(b)},
            "clocks": clk.summary(), "e2e": e2e, "gpu_launches": launches, "roofline": roof, "kernels": kernels,
            "cpu_baseline": cpu, "secondary": sec, "peaks": peaks_src,
        }
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


def step_pairs(b):
    return b.eligible_pairs()


def measured_traffic(kernel, launches_per_step):
    """DRAM bytes per launch of `kernel` on the 32K prefill from the committed ncu capture, or None when
    the kernel's sources or its launches per step changed since (the capture no longer describes it)."""
    import hashlib
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "dram_traffic_dense_prefill_32k.json")
    try:
        rec = json.load(open(path))["kernels"][kernel]
    except (OSError, KeyError, ValueError):
        return None
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sparse_attention_indexer_04_b200", "csrc")
    m = hashlib.sha256()
    for f in rec["sources"]:
        m.update(open(os.path.join(src, f), "rb").read())
    same = m.hexdigest() == rec["sources_sha256"] and rec.get("launches_per_step") == launches_per_step
    return rec["bytes_per_launch"] if same else None


def roofline_entries(prof, step, b, steps, peaks, peaks_src):
    """Per-kernel roofline from the live per-kernel event times; the dominant (most time) is the headline.

    Algorithmic work per step: score kernels do 2*H*d flop per eligible pair (tensor: bf16 peak; CUDA-core:
    fp32 FMA peak); the top-k select reads one fp32 score per eligible pair and writes k indices per row
    (HBM: copy peak).
    """
    clk_max = peaks.get("sm_max_mhz", 1965.0)
    flops = step.pairs * 2 * b.H * b.d
    sel_bytes = step.pairs * 4 + b.n_q * step.k * 4
    total = sum(v[0] for v in prof.values())
    out = []
    for name, (ms, n) in prof.items():
        t = ms / steps * 1e-3
        e = {"kernel": name, "ms_per_step": round(ms / steps, 4), "launches_per_step": n / steps,
             "share": round(ms / total, 4)}
        if name == "score_tc":
            ach = flops / t / 1e12
            e.update(bound="tensor", unit="TFLOP/s", achieved=round(ach, 2), peak=peaks["bf16_tflops"],
                     peak_basis=f"bf16 dense matmul, {peaks_src}", alg_per_step=flops)
        elif name == "score_simt":
            pk = SM_COUNT * FP32_LANES_PER_SM * 2 * clk_max * 1e6 / 1e12
            ach = flops / t / 1e12
            e.update(bound="alu", unit="TFLOP/s", achieved=round(ach, 2), peak=round(pk, 1),
                     peak_basis=f"fp32 FMA: {SM_COUNT} SMs x {FP32_LANES_PER_SM} lanes x 2 x {clk_max:.0f} MHz",
                     alg_per_step=flops)
        elif name == "select_topk":
            ach = sel_bytes / t / 1e9
            e.update(bound="hbm", unit="GB/s", achieved=round(ach, 1), peak=peaks["hbm_gbs"],
                     peak_basis=f"HBM copy, {peaks_src}", alg_per_step=sel_bytes)
        else:
            out.append(e)
            continue
        e["frac"] = round(e["achieved"] / e["peak"], 4)
        # DRAM bytes per launch (ncu), beside the algorithmic work per launch
        e["traffic"] = measured_traffic(name, n / steps) if b.n_q == 32768 else None
        e["alg_per_launch"] = round(e["alg_per_step"] / max(1.0, n / steps))
        out.append(e)
    out.sort(key=lambda e: -e["ms_per_step"])
    dom = next(e for e in out if "bound" in e)
    return dict(dom), out


if __name__ == "__main__":
    main()
