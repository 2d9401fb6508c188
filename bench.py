"""Benchmark of the lightning-indexer decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl li|reference] [--no-sweep]

One step = one DSA decode indexer pass over B=8 requests with 32768 cached
FP8 keys each (H=64 heads, d=128): query quantisation + score of every cache
position (one fused kernel) followed by the top-2048 select (one kernel).
Inputs are synthetic (seeded, shaped as the pages' decode workload) and the
key caches rotate over enough copies to exceed the 126 MB L2, so every step
reads its keys from HBM.  Under torchrun each rank runs its own batch of
requests (weak scaling, no collective on the data path); the time is the max
over ranks.

Prints ONE JSON line (rank 0).  Besides the decode step it carries the L
sweep (8K-128K) and the causal prefill (T = L = 8192: quantise + score, and
the step with its top-2048) against the FP8 tensor peak measured in the same
run (`--no-sweep`, `--no-prefill` skip them).  `--impl reference` times the
fp64 CPU oracle on the same workload instead (a bounded sample of it).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "indexer µs/decode-step and keys scored/s at 8K–128K; % of HBM / FP8-tensor roofline"
WORKLOAD = "dsa_decode_b8_l32k"
B, L, H, D, KTOP = 8, 32768, 64, 128, 2048
L2_BYTES = 126 * 1024 * 1024
SCORER_KERNEL = "stream_score_kernel"
PREFILL_KERNELS = "quantize_query_kernel + prefill_score_kernel"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def decode_bytes_per_key(d=D):
    # key bytes + per-token scale + one fp32 score written
    return d + 4 + 4


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def traffic_for(kernel: str, units: float):
    """DRAM bytes per launch from the committed ncu summary, scaled to `units`
    keys, or None when that summary was taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(kernel)
        if sources_sha256_16(d["sources"]) != d["sources_sha256_16"]:
            return None
        return d["dram_bytes_per_unit"] * units
    except Exception:
        return None


def sources_sha256_16(paths):
    """Hash of the kernel's source files (repo-relative), to detect stale counters."""
    h = hashlib.sha256()
    for rel in paths:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle
# ---------------------------------------------------------------------------
def run_reference(args, rank):
    if rank != 0:
        return
    import oracle
    from sparse_attention_lightning_score_b200 import synth
    nthreads = oracle.nthreads_default()
    case = synth.dsa_decode(B=B, L=L, k_top=KTOP, seed=1)
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    rows_per_step = 1  # bounded sample: one request of the batch per step
    times = []
    for step in range(args.warmup + args.steps):
        r = step % B
        t0 = time.perf_counter()
        q8r, sqr, _ = oracle.quantize_query(case.q[r:r + 1], case.w[r:r + 1].numpy())
        sc = oracle.index_score(q8r, oracle.E4M3, case.w[r:r + 1], case.k8[r], oracle.E4M3, q_scale=sqr,
                                k_scale=case.ks[r], nthreads=nthreads)
        oracle.topk(sc, KTOP)
        t1 = time.perf_counter()
        if step >= args.warmup:
            times.append(t1 - t0)
    t = sum(times) / len(times)
    keys_s = rows_per_step * L / t
    out = {"impl": "reference", "metric": METRIC, "value": keys_s, "unit": "keys/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3 * B / rows_per_step,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "B": B, "L": L, "H": H, "d": D, "k": KTOP},
           "cpu_baseline": {"value": keys_s, "unit": "keys/s", "cores": nthreads, "kind": "oracle",
                            "sample": f"1 of {B} requests per step (L={L}), quantise+score+top-{KTOP}; "
                                      "ms_per_step extrapolated to the full batch"},
           "e2e": {"value": keys_s, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def cpu_baseline_sample(heads=H):
    import oracle
    from sparse_attention_lightning_score_b200 import synth
    nthreads = oracle.nthreads_default()
    case = synth.dsa_decode(B=2, L=L, H=heads, k_top=KTOP, seed=1)
    t0 = time.perf_counter()
    n = 0
    while True:
        r = n % 2
        q8r, sqr, _ = oracle.quantize_query(case.q[r:r + 1], case.w[r:r + 1].numpy())
        sc = oracle.index_score(q8r, oracle.E4M3, case.w[r:r + 1], case.k8[r], oracle.E4M3, q_scale=sqr,
                                k_scale=case.ks[r], nthreads=nthreads)
        oracle.topk(sc, KTOP)
        n += 1
        if time.perf_counter() - t0 > 10.0 or n >= 4096:
            break
    t = time.perf_counter() - t0
    return {"value": n * L / t, "unit": "keys/s", "cores": nthreads, "kind": "oracle",
            "sample": f"{n} request(s) of L={L} (quantise+score+top-{KTOP}) on the host, {t:.1f} s"}


def oracle_sample(kind, case, budget_s=10.0, heads=H):
    """The oracle as it stands, timed on the host cores on a bounded sample of a workload (the
    cpu_baseline object of that workload's JSON line).  `case` is the workload's own synthetic input
    on the host; the sample is whole requests (or whole causal rows) taken until `budget_s` passes,
    so its unit matches the workload's."""
    import numpy as np
    import torch
    import oracle
    nthreads = oracle.nthreads_default()
    t0 = time.perf_counter()
    n, units = 0, 0

    def over():
        return time.perf_counter() - t0 > budget_s

    if kind == "prefill":
        T = case.q.shape[0]
        Lk = case.k8.shape[0]
        while n == 0 or not over():
            r = T - 1 - (n * 997) % T  # rows of every length, the longest first
            q8, sq, _ = oracle.quantize_query(case.q[r:r + 1], case.w[r:r + 1].numpy())
            sc = oracle.index_score(q8, oracle.E4M3, case.w[r:r + 1], case.k8, oracle.E4M3, q_scale=sq,
                                    k_scale=case.ks, causal=True, causal_offset=r, L=Lk, nthreads=nthreads)
            oracle.topk(sc, KTOP, causal=True, causal_offset=r, max_len=Lk)
            units += min(r + 1, Lk)
            n += 1
        t = time.perf_counter() - t0
        return {"value": units / t, "unit": "keys/s (visible pairs)", "cores": nthreads, "kind": "oracle",
                "sample": f"{n} causal row(s) of T={T} (quantise+score+top-{KTOP}), {units} pairs, {t:.1f} s"}
    if kind in ("latent", "latent_glm5", "latent192"):
        fp8 = kind == "latent192"
        Bc = case.q.shape[1]
        Lk = case.c.shape[1]
        while n == 0 or not over():
            b = n % Bc
            qt = oracle.absorb(case.q[0][b:b + 1], case.w_dec[0])
            if fp8:
                qtb = torch.from_numpy(qt).to(torch.bfloat16)
                q8, sq, _ = oracle.quantize_query(qtb, case.w[0][b:b + 1].numpy())
                sc = oracle.index_score(q8, oracle.E4M3, case.w[0][b:b + 1], case.c8[b], oracle.E4M3, q_scale=sq,
                                        k_scale=case.cs[b], nthreads=nthreads)
            else:
                sc = oracle.latent_score(qt, oracle.F64, case.w[0][b:b + 1], case.c[b], nthreads=nthreads)
            oracle.topk(sc, KTOP)
            units += Lk
            n += 1
        t = time.perf_counter() - t0
        return {"value": units / t, "unit": "keys/s", "cores": nthreads, "kind": "oracle",
                "sample": f"{n} request-layer(s) of L={Lk} (absorb+score+top-{KTOP}), {t:.1f} s"}
    if kind in ("hs_b1", "hs_b16"):
        Bc = case.q.shape[1]
        Lk = case.c.shape[1]
        C = case.n_cand if getattr(case, "n_cand", 0) else 8192
        F = case.q.shape[0] - 1
        while n == 0 or not over():
            b = n % Bc
            qt0 = oracle.absorb(case.q[0][b:b + 1], case.w_dec[0])
            sc = oracle.latent_score(qt0, oracle.F64, case.w[0][b:b + 1], case.c[b], nthreads=nthreads)
            cand, _ = oracle.topk(sc, C)
            qtf = np.stack([oracle.absorb(case.q[f][b:b + 1], case.w_dec[f]) for f in range(1, F + 1)])
            oracle.hs_refine(qtf, oracle.F64, case.w[1:, b:b + 1], case.c[b:b + 1], cand, KTOP, nthreads=nthreads)
            units += Lk
            n += 1
        t = time.perf_counter() - t0
        return {"value": units / t, "unit": "keys/s (anchor scan)", "cores": nthreads, "kind": "oracle",
                "sample": f"{n} request(s) of L={Lk}, C={C}, {F} followers (whole HS step), {t:.1f} s"}
    if kind == "sparse_attention":
        q, kv, sel, scale = case
        Bc = q.shape[0]
        while n == 0 or not over():
            b = n % Bc
            oracle.sparse_attention(q[b:b + 1], kv[b:b + 1], sel[b:b + 1], scale)
            n += 1
        t = time.perf_counter() - t0
        return {"value": t / n * Bc * 1e6, "unit": "µs/call", "cores": 1, "kind": "oracle",
                "sample": f"{n} request(s) of {Bc} ({q.shape[1]} heads, {sel.shape[1]} selections, numpy fp64), "
                          f"{t:.1f} s; value extrapolated to the whole call"}
    raise ValueError(kind)


# ---------------------------------------------------------------------------
# li arm
# ---------------------------------------------------------------------------
def make_sets(dev, Lx, seed, heads=H):
    """Key caches for B requests of length Lx, copied until they exceed 1.5x L2."""
    from sparse_attention_lightning_score_b200 import synth
    case = synth.dsa_decode(B=B, L=Lx, H=heads, k_top=KTOP, seed=seed)
    per_set = B * Lx * (D + 4)
    nsets = max(2, math.ceil(1.5 * L2_BYTES / per_set))
    k8 = case.k8.to(dev)
    ks = case.ks.to(dev)
    sets = [(k8, ks)] + [(k8.clone(), ks.clone()) for _ in range(nsets - 1)]
    return case, sets, nsets * per_set


def capture(fns):
    """One CUDA graph replaying the given launches in order (decode steps run
    under graphs in serving; the graph removes host submission from the timing)."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    return g


class DecodeBench:
    """Decode-step launches over rotating key caches, as graphs.

    A step is li_decode_select: the scorer (which also counts each row's first
    radix digit into a histogram) and the top-k that starts from that
    histogram.  The two kernels are also timed
    alone through the call's two halves: the scorer into a scratch workspace,
    the selection from a saved workspace whose histograms are restored by a
    device copy before each launch (the copy's own time is subtracted)."""

    def __init__(self, dev, Lx, seed, heads=H):
        import torch
        from sparse_attention_lightning_score_b200 import api
        self.api = api
        self.Lx = Lx
        self.heads = heads
        self.case, self.sets, self.set_bytes = make_sets(dev, Lx, seed, heads)
        self.n = len(self.sets)
        self.q, self.w = self.case.q.to(dev), self.case.w.to(dev)
        self.sc = torch.empty((B, Lx), dtype=torch.float32, device=dev)
        self.idx = torch.empty((B, KTOP), dtype=torch.int32, device=dev)
        self.ws = api.li_decode_select_workspace(B, dev, Lx)
        # a second set for the pipelined timing: two independent steps in flight on two streams
        self.sc2 = torch.empty_like(self.sc)
        self.idx2 = torch.empty_like(self.idx)
        self.ws2 = api.li_decode_select_workspace(B, dev, Lx)
        self.ws_scratch = api.li_decode_select_workspace(B, dev, Lx)
        # scores + a workspace the scorer filled, for the selection-only timing
        nh = api.li_decode_select_hist_bytes(B)
        self.sc_t = torch.empty_like(self.sc)
        self.idx_t = torch.empty_like(self.idx)
        self.ws_t = api.li_decode_select_workspace(B, dev, Lx)
        kk, ss = self.sets[0]
        api.li_decode_select_score(self.q, self.w, kk, ss, self.ws_t, scores=self.sc_t)
        self.hist_saved = self.ws_t[:nh].clone()
        self.hist_t = self.ws_t[:nh]

    def score(self, i):
        kk, ss = self.sets[i % self.n]
        self.api.li_decode_select_score(self.q, self.w, kk, ss, self.ws_scratch, scores=self.sc)

    def restore(self):
        self.hist_t.copy_(self.hist_saved)

    def topk(self):
        self.restore()
        self.api.li_decode_select_finish(self.sc_t, KTOP, self.ws_t, heads=self.heads, max_len=self.Lx, idx=self.idx_t)

    def step(self, i):
        kk, ss = self.sets[i % self.n]
        self.api.li_decode_select(self.q, self.w, kk, ss, KTOP, scores=self.sc, workspace=self.ws, idx=self.idx)

    def step_on(self, i, stream):
        """Step i on `stream` with the buffer set of its parity (the pipelined timing)."""
        kk, ss = self.sets[i % self.n]
        sc, ws, idx = (self.sc, self.ws, self.idx) if i % 2 == 0 else (self.sc2, self.ws2, self.idx2)
        self.api.li_decode_select(self.q, self.w, kk, ss, KTOP, scores=sc, workspace=ws, idx=idx, stream=stream)

    def build_graphs(self, warmup):
        import torch
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize()
        self.step_graphs = [capture([lambda i=i: self.step(i)]) for i in range(self.n)]
        # one graph holding a step over every rotating set, back to back (as the
        # indexer's kernels sit inside a model's decode graph)
        self.loop_graph = capture([lambda i=i: self.step(i) for i in range(self.n)])
        reps = max(1, 24 // self.n)
        self.score_graph = capture([lambda i=i: self.score(i) for i in range(self.n * reps)])
        self.score_launches = self.n * reps
        self.topk_graph = capture([self.topk] * 16)
        self.topk_launches = 16
        # the same steps, independent, alternating over two streams: step i's top-k overlaps step
        # i+1's scorer (an even number of steps, so that every set is used in both parities)
        self.pipe_n = 2 * self.n
        self.pipe_streams = [torch.cuda.Stream(device=self.sc.device) for _ in range(2)]
        self.pipe_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.pipe_graph):
            main = torch.cuda.current_stream()
            fork = torch.cuda.Event()
            fork.record(main)
            for st in self.pipe_streams:
                st.wait_event(fork)
            for i in range(self.pipe_n):
                st = self.pipe_streams[i % 2]
                with torch.cuda.stream(st):
                    self.step_on(i, st)
            for st in self.pipe_streams:
                ev = torch.cuda.Event()
                ev.record(st)
                main.wait_event(ev)
        self.restore_graph = capture([self.restore] * 16)
        for g in self.step_graphs:
            g.replay()
        self.loop_graph.replay()
        self.score_graph.replay()
        self.topk_graph.replay()
        self.restore_graph.replay()
        self.pipe_graph.replay()
        torch.cuda.synchronize()

    def time_steps(self, steps):
        """Exactly `steps` decode steps: whole loop graphs (one step per rotating
        set each), then single-step graphs for the remainder."""
        import torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps // self.n):
            self.loop_graph.replay()
        for i in range(steps % self.n):
            self.step_graphs[i].replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def time_pipelined(self, steps):
        """At least `steps` independent steps, two in flight (whole pipelined graphs); time per step."""
        reps = max(1, -(-steps // self.pipe_n))
        return self._time_graph(self.pipe_graph, self.pipe_n, reps)

    def time_steps_single(self, steps):
        """The same steps, one graph launch per step."""
        import torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            self.step_graphs[i % self.n].replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def _time_graph(self, g, n, reps):
        import torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * n)

    def time_kernel(self, which, reps=3):
        if which == "score":
            return self._time_graph(self.score_graph, self.score_launches, reps)
        both = self._time_graph(self.topk_graph, self.topk_launches, reps)
        return both - self._time_graph(self.restore_graph, self.topk_launches, reps)

    def time_direct(self, steps):
        import torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            self.step(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps


def run_li(args, rank, world, local_rank):
    import torch
    from sparse_attention_lightning_score_b200 import api

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    from sparse_attention_lightning_score_b200 import dist as li_dist
    dist = li_dist.init("nccl", device=dev) if world > 1 else None

    bench = DecodeBench(dev, L, seed=1 + rank)
    bench.build_graphs(args.warmup)
    assert api.li_get_last_error() == 0

    clocks = ClockSampler(local_rank)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ms = bench.time_steps(args.steps)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist:
        dist.barrier()
    score_ms = bench.time_kernel("score")
    topk_ms = bench.time_kernel("topk")
    direct_ms = bench.time_direct(args.steps)
    single_ms = bench.time_steps_single(args.steps)
    pipe_dev_ms = bench.time_pipelined(args.steps)
    ms, score_ms, topk_ms, direct_ms, single_ms, pipe_dev_ms = li_dist.max_over_ranks(
        [ms, score_ms, topk_ms, direct_ms, single_ms, pipe_dev_ms], device=dev)
    launches = 2 * args.steps

    # ---- end to end through the public API.  Throughput: K independent steps as one DecodePipeline
    # graph, each step copying its own pinned host query/weights in and its selected positions out,
    # the copies of neighbouring steps overlapping its kernels; the headline e2e keeps the steps'
    # kernels on one stream, as `value` does, and the pipelined figure lets two steps' kernels
    # overlap.  Latency: the same step alone as one graph-captured DecodeIndexer step (copy in ->
    # li_decode_select -> copy out), back to back.
    from sparse_attention_lightning_score_b200.step import DecodeIndexer, DecodePipeline
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e = {}
    for nstreams in (1, 2):
        pipe = DecodePipeline([bench.sets[i % bench.n] for i in range(args.steps)], H, KTOP, streams=nstreams)
        for i in range(args.steps):
            pipe.q_host[i].copy_(bench.case.q)
            pipe.w_host[i].copy_(bench.case.w)
        for _ in range(max(1, args.warmup // 2)):
            pipe.run(sync=False)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a0.record()
        pipe.run(sync=False)
        a1.record()
        torch.cuda.synchronize()
        e2e[nstreams] = a0.elapsed_time(a1) / args.steps
        # the selections that came back to the host match the device-side graph's
        bench.step_graphs[(args.steps - 1) % bench.n].replay()
        torch.cuda.synchronize()
        assert torch.equal(pipe.idx_host[args.steps - 1], bench.idx.cpu())
        h2d, d2h = pipe.h2d_bytes_per_step, pipe.d2h_bytes_per_step
        del pipe
    e2e_ms, pipe_e2e_ms = e2e[1], e2e[2]
    indexers = [DecodeIndexer(kk, ss, H, KTOP) for kk, ss in bench.sets]
    for ix in indexers:
        ix.q_host.copy_(bench.case.q)
        ix.w_host.copy_(bench.case.w)
    for i in range(args.warmup):
        indexers[i % len(indexers)].step(sync=False)
    torch.cuda.synchronize()
    a0.record()
    for i in range(args.steps):
        indexers[i % len(indexers)].step(sync=False)
    a1.record()
    torch.cuda.synchronize()
    lat_ms = a0.elapsed_time(a1) / args.steps
    e2e_ms, pipe_e2e_ms, lat_ms = li_dist.max_over_ranks([e2e_ms, pipe_e2e_ms, lat_ms], device=dev)
    del indexers
    assert api.li_get_last_error() == 0
    # every collective of the run is behind us: the group closes before rank 0's sweep and prefill
    # legs, so the other ranks neither wait on them nor run into the group's timeout
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    sweep = None
    if not args.no_sweep and rank == 0:
        sweep = {}
        hbm, _ = peaks()
        for Lx in (8192, 16384, 32768, 65536, 131072):
            bx = DecodeBench(dev, Lx, seed=11)
            bx.build_graphs(3)
            st_ms = bx.time_steps(max(20, args.steps))
            sc_ms = bx.time_kernel("score")
            tk_ms = bx.time_kernel("topk")
            pp_ms = bx.time_pipelined(max(20, args.steps))
            sweep[str(Lx)] = {"us_per_step": round(st_ms * 1e3, 2), "score_us": round(sc_ms * 1e3, 2),
                              "pipelined_us_per_step": round(pp_ms * 1e3, 2),
                              "topk_us": round(tk_ms * 1e3, 2), "keys_per_s": B * Lx / (st_ms * 1e-3),
                              "score_hbm_frac": round(B * Lx * decode_bytes_per_key() / (sc_ms * 1e-3) / 1e9 / hbm,
                                                      3)}
            del bx
    prefill = None
    if not args.no_prefill and rank == 0:
        fp8 = fp8_peak_tflops()
        px = PrefillBench(dev)
        clocks = ClockSampler(local_rank)
        clocks.start()
        time.sleep(0.3)
        r = px.run(max(10, args.steps // 2), args.warmup)
        pclk = clocks.stop()
        prefill = prefill_record(r, px, pclk, fp8)
        del px
        assert api.li_get_last_error() == 0

    hbm, which = peaks()
    units = B * L
    algo_bytes = units * decode_bytes_per_key() + B * H * D * 2 + B * H * 4
    achieved = algo_bytes / (score_ms * 1e-3) / 1e9
    keys_s = world * B * L / (ms * 1e-3)
    out = {
        "metric": METRIC, "value": keys_s, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "L": L, "H": H, "d": D, "k": KTOP,
                   "l2": f"{bench.n} rotating key-cache copies, {bench.set_bytes / 1e6:.0f} MB > 126 MB L2",
                   "launch": "CUDA graphs of back-to-back steps (li_decode_select: score + top-k per step)",
                   "per_rank": "own batch of B requests"},
        "roofline": {"bound": "hbm", "kernel": SCORER_KERNEL, "achieved": achieved, "peak": hbm,
                     "peak_source": which, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": traffic_for(SCORER_KERNEL, units), "algorithmic_bytes": algo_bytes,
                     "kernel_us": score_ms * 1e3},
        "topk": {"us": topk_ms * 1e3, "rows_per_s": B / (topk_ms * 1e-3), "row_len": L, "k": KTOP},
        "direct_us_per_step": direct_ms * 1e3, "graph_per_step_us": single_ms * 1e3,
        "e2e": {"value": world * B * L / (e2e_ms * 1e-3), "unit": "keys/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "api": "DecodePipeline(streams=1).run: K independent steps in one graph, each H2D q,w -> "
                       "li_decode_select -> D2H indices, neighbouring steps' copies overlapping its kernels, "
                       "the steps' kernels one after another",
                "latency_ms_per_step": lat_ms,
                "latency_api": "DecodeIndexer.step (one step per graph: H2D q,w -> li_decode_select -> D2H indices)"},
        "pipelined": {"us_per_step": pipe_dev_ms * 1e3, "keys_per_s": world * B * L / (pipe_dev_ms * 1e-3),
                      "e2e_us_per_step": pipe_e2e_ms * 1e3, "e2e_keys_per_s": world * B * L / (pipe_e2e_ms * 1e-3),
                      "how": "the same independent steps, two in flight on two streams with their own scores and "
                             "workspaces (step i's top-k overlaps step i+1's scorer); device-only, and end to end "
                             "through DecodePipeline(streams=2) with the same copies as e2e"},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if sweep:
        out["sweep"] = sweep
    if prefill:
        out["prefill"] = prefill
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_sample()
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# other configurations (parity-test workloads; timed on request with --workload)
# ---------------------------------------------------------------------------
_FP8_PEAK = None


def fp8_peak_tflops():
    """Dense FP8 (e4m3) tensor-core rate of this GPU, measured the way the bf16 figures of
    MEASURED_PEAKS.json were: an 8192^3 GEMM (2 * 8192^3 flops) timed with CUDA events, the best
    of 10 launches (burst) and the rate of back-to-back launches over 4 s (sustained).  The GEMM
    is torch._scaled_mm, e4m3 x e4m3 -> bf16 with tensor-wise scales, in both of cuBLAS's
    accumulation modes; the faster one is taken.  Measured once per process.
    Returns (burst TF/s, sustained TF/s, source)."""
    global _FP8_PEAK
    if _FP8_PEAK is not None:
        return _FP8_PEAK
    import torch
    try:
        n = 8192
        g = torch.Generator(device="cuda").manual_seed(0)
        a = torch.randn(n, n, device="cuda", generator=g).to(torch.float8_e4m3fn)
        bt = torch.randn(n, n, device="cuda", generator=g).to(torch.float8_e4m3fn)
        one = torch.ones((), device="cuda")
        flops = 2.0 * n ** 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def mm(fast):
            return torch._scaled_mm(a, bt.t(), one, one, out_dtype=torch.bfloat16, use_fast_accum=fast)

        best, best_mode = 0.0, False
        for fast in (False, True):
            for _ in range(3):
                mm(fast)
            torch.cuda.synchronize()
            for _ in range(10):
                e0.record()
                mm(fast)
                e1.record()
                torch.cuda.synchronize()
                tf = flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
                if tf > best:
                    best, best_mode = tf, fast
        count = 0
        t_end = time.time() + 4.0
        e0.record()
        while time.time() < t_end:
            for _ in range(50):
                mm(best_mode)
            count += 50
            e1.record()
            e1.synchronize()
        e1.record()
        torch.cuda.synchronize()
        sust = count * flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
        del a, bt
        src = ("measured: torch._scaled_mm e4m3 8192^3, best of 10 and 4 s back to back "
               f"({'fast' if best_mode else 'fp32'} accumulation)")
        _FP8_PEAK = (best, sust, src)
    except Exception as exc:  # no FP8 GEMM in this torch build: the nominal 2:1 ratio to measured bf16
        p = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(p):
            d = json.load(open(p))
            _FP8_PEAK = (2.0 * float(d["bf16_tflops"]), 2.0 * float(d["bf16_tflops_sustained"]),
                         f"measured bf16 x 2 (FP8 GEMM unavailable: {type(exc).__name__})")
        else:
            _FP8_PEAK = (2 * 1590.0, 2 * 1400.0, "fallback bf16 x 2")
    return _FP8_PEAK


def prefill_record(r, bx, clk, fp8):
    """The causal prefill's figures against the FP8 tensor peak (algorithmic flops: visible
    (t, s) pairs x 2 * H * d)."""
    burst, sust, src = fp8
    flops = bx.pairs * 2 * H * D
    tf = flops / (r["score"] * 1e-3) / 1e12
    return {"workload": "dsa_prefill_t8k", "T": bx.T, "L": bx.L, "H": H, "d": D, "k": KTOP,
            "score_ms": r["score"], "step_ms": r["step"], "topk_ms": r["topk"],
            "tflops": tf, "frac_of_fp8_burst": tf / burst, "frac_of_fp8_sustained": tf / sust,
            "fp8_peak_tflops": {"burst": burst, "sustained": sust, "source": src},
            "pairs_per_s": bx.pairs / (r["step"] * 1e-3), "kernels": PREFILL_KERNELS, "clocks": clk}


class PrefillBench:
    """Causal prefill: T = L = 8192, quantise + score (s <= t) + top-2048 per row."""

    def __init__(self, dev):
        import torch
        from sparse_attention_lightning_score_b200 import api, synth
        self.api = api
        self.T = self.L = 8192
        case = synth.dsa_prefill(T=self.T, L=self.L)
        self.case = case  # host copy, for the oracle's timed sample
        self.q, self.w = case.q.to(dev), case.w.to(dev)
        self.k8, self.ks = case.k8.to(dev), case.ks.to(dev)
        self.sc = torch.empty((self.T, self.L), dtype=torch.float32, device=dev)
        self.idx = torch.empty((self.T, KTOP), dtype=torch.int32, device=dev)
        from sparse_attention_lightning_score_b200 import _lib
        desc = api.score_desc(self.T, H, D, self.L, causal=True)
        import ctypes
        self.ws = torch.empty(_lib.load().li_index_score_workspace(ctypes.byref(desc)), dtype=torch.uint8, device=dev)
        self.pairs = self.T * (self.T + 1) // 2

    def score(self):
        self.api.li_index_score(self.q, self.w, self.k8, self.ks, causal=True, scores=self.sc, workspace=self.ws)

    def topk(self):
        self.api.li_topk(self.sc, KTOP, causal=True, max_len=self.L, idx=self.idx)

    def run(self, steps, warmup):
        import torch
        for _ in range(warmup):
            self.score()
            self.topk()
        torch.cuda.synchronize()
        gs = capture([self.score, self.topk])
        g_sc = capture([self.score])
        g_tk = capture([self.topk])
        res = {}
        for name, g in (("step", gs), ("score", g_sc), ("topk", g_tk)):
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) / steps
        return res


class LatentBench:
    """LatentIndex G=4 group decode: 4 x (absorb + latent score + top-2048), B=4, L=65536; each
    layer's scan counts its first radix digit for the top-k.  kind "bf16": the d_c = 256 bf16
    latent cache; kind "fp8_192": DeepSeek-V3.2's 64 RoPE + 128 NoPE latent as an e4m3 cache
    with per-row scales.  heads = 32 gives GLM-5's indexer shape on the bf16 cache."""

    def __init__(self, dev, B=4, Lx=65536, kind="bf16", heads=H):
        import torch
        from sparse_attention_lightning_score_b200 import api, synth
        self.api = api
        self.B, self.L, self.kind, self.heads = B, Lx, kind, heads
        if kind == "bf16":
            case = synth.latent_group(B=B, L=Lx, H=heads)
            self.c = [(case.c.to(dev), None)]
            per = case.c.numel() * 2
            self.dc, self.key_bytes = 256, 512
        else:
            case = synth.latent_rope_nope(B=B, L=Lx)
            self.c = [(case.c8.to(dev), case.cs.to(dev))]
            per = case.c8.numel() + case.cs.numel() * 4
            self.dc, self.key_bytes = 192, 196
        while len(self.c) * per < 1.5 * L2_BYTES:
            self.c.append(tuple(t.clone() if t is not None else None for t in self.c[0]))
        self.case = case  # host copy, for the oracle's timed sample
        self.q = [case.q[l].to(dev) for l in range(4)]
        self.wd = [case.w_dec[l].to(dev) for l in range(4)]
        self.hist = api.li_decode_select_workspace(B, dev).view(torch.int32)[:B * 2048]
        self.hist_scratch = api.li_decode_select_workspace(B, dev).view(torch.int32)[:B * 2048]
        self.w = [case.w[l].to(dev) for l in range(4)]
        self.qt = torch.empty((B, heads, self.dc), dtype=torch.bfloat16, device=dev)
        self.sc = torch.empty((B, Lx), dtype=torch.float32, device=dev)
        self.idx = torch.empty((4, B, KTOP), dtype=torch.int32, device=dev)

    def score(self, i, l, hist):
        c, cs = self.c[i % len(self.c)]
        if cs is None:
            self.api.li_latent_score_hist(self.qt, self.w[l], c, hist, scores=self.sc)
        else:
            self.api.li_latent_score_fp8(self.qt, self.w[l], c, cs, hist=hist, scores=self.sc)

    def layer(self, i, l):
        self.api.li_absorb_query(self.q[l], self.wd[l], out=self.qt)
        self.score(i, l, self.hist)
        self.api.li_topk_hist(self.sc, KTOP, self.hist, idx=self.idx[l])

    def run(self, steps, warmup):
        import torch
        for i in range(warmup):
            for l in range(4):
                self.layer(i, l)
        torch.cuda.synchronize()
        graphs = [capture([lambda i=i, l=l: self.layer(i, l) for l in range(4)]) for i in range(len(self.c))]
        # the scan alone (its counts go to a scratch histogram nobody reads)
        g_sc = capture([lambda i=i: self.score(i, 0, self.hist_scratch) for i in range(8)])
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        e1.record()
        torch.cuda.synchronize()
        step = e0.elapsed_time(e1) / steps
        e0.record()
        g_sc.replay()
        e1.record()
        torch.cuda.synchronize()
        return {"step": step, "score": e0.elapsed_time(e1) / 8}


class HsBench:
    """HS decode at L=131072: anchor absorb + scan + top-8192, 3 follower absorbs + refine.

    The anchor's scan counts its first radix digit for the top-8192.  Two layouts of the same
    calls, chosen by batch size:
      - B < 8: all four layers are absorbed in one launch, then the anchor's scan and top-k and the
        followers' refine follow on the same stream, so each kernel starts under a programmatic
        dependency on the previous one (at one request the absorption is latency-bound and its
        four layers cost about what one does);
      - B >= 8: the followers' absorption (one launch, three layers) runs on a second stream while
        the anchor absorbs, scans and selects, and the refine waits for both (the followers'
        absorption would lengthen the anchor's chain by several µs)."""

    def __init__(self, dev, B):
        import torch
        from sparse_attention_lightning_score_b200 import api, synth
        self.api = api
        self.B, self.L, self.C = B, 131072, 8192
        case = synth.latent_hs(B=B, L=self.L)
        self.c = [case.c.to(dev)]
        per = case.c.numel() * 2
        while len(self.c) * per < 1.5 * L2_BYTES:
            self.c.append(self.c[0].clone())
        self.case = case  # host copy, for the oracle's timed sample
        self.q = [case.q[l].to(dev) for l in range(4)]
        self.wd = [case.w_dec[l].to(dev) for l in range(4)]
        self.qf = case.q[1:].contiguous().to(dev)
        self.wdf = case.w_dec[1:].contiguous().to(dev)
        self.hist = api.li_decode_select_workspace(B, dev).view(torch.int32)[:B * 2048]
        self.side = torch.cuda.Stream(device=dev)
        self.w0 = case.w[0].to(dev)
        self.wf = case.w[1:].contiguous().to(dev)
        self.qt0 = torch.empty((B, H, 256), dtype=torch.bfloat16, device=dev)
        self.qtf = torch.empty((3, B, H, 256), dtype=torch.bfloat16, device=dev)
        self.sc = torch.empty((B, self.L), dtype=torch.float32, device=dev)
        self.cand = torch.empty((B, self.C), dtype=torch.int32, device=dev)
        self.out = torch.empty((3, B, KTOP), dtype=torch.int32, device=dev)
        self.ws = api.li_hs_refine_workspace(B, self.C, 3, dev)
        self.one_stream = B < 8
        self.q_all = torch.stack(self.q).contiguous()
        self.wd_all = torch.stack(self.wd).contiguous()
        self.qt_all = torch.empty((4, B, H, 256), dtype=torch.bfloat16, device=dev)

    def step(self, i):
        import torch
        c = self.c[i % len(self.c)]
        if self.one_stream:
            self.api.li_absorb_query_layers(self.q_all, self.wd_all, out=self.qt_all)
            self.api.li_latent_score_hist(self.qt_all[0], self.w0, c, self.hist, scores=self.sc)
            self.api.li_topk_hist(self.sc, self.C, self.hist, idx=self.cand)
            self.api.li_hs_refine(c, self.cand, self.qt_all[1:], self.wf, KTOP, out=self.out, workspace=self.ws)
            return
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self.api.li_absorb_query_layers(self.qf, self.wdf, out=self.qtf)
        self.api.li_absorb_query(self.q[0], self.wd[0], out=self.qt0)
        self.api.li_latent_score_hist(self.qt0, self.w0, c, self.hist, scores=self.sc)
        self.api.li_topk_hist(self.sc, self.C, self.hist, idx=self.cand)
        main.wait_stream(self.side)
        self.api.li_hs_refine(c, self.cand, self.qtf, self.wf, KTOP, out=self.out, workspace=self.ws)

    def run(self, steps, warmup):
        import torch
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize()
        graphs = [capture([lambda i=i: self.step(i)]) for i in range(len(self.c))]
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        e1.record()
        torch.cuda.synchronize()
        return {"step": e0.elapsed_time(e1) / steps}


def run_consumer(dev, args, clocks, want_cpu=False):
    """The consumer alone: li_sparse_attention at the decode shape (B = 8 requests, 128 query heads,
    the indexer's 2048 selections out of L = 32768 cached 576-element rows), rotating through 8
    selection sets so that the gathered rows (8 x 18.9 MB) exceed L2."""
    import numpy as np
    import torch
    from sparse_attention_lightning_score_b200 import api
    Ha, D = 128, 576
    g = torch.Generator(device=dev).manual_seed(1)
    q = torch.randn(B, Ha, D, device=dev, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, L, D, device=dev, generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(1)
    sels = [torch.from_numpy(np.stack([np.sort(rng.choice(L, KTOP, replace=False)) for _ in range(B)])
                             .astype(np.int32)).to(dev) for _ in range(8)]
    out = torch.empty(B, Ha, 512, device=dev)
    ws = api.li_sparse_attention_workspace(B, Ha, KTOP, dev)
    scale = 1.0 / 192 ** 0.5
    for i in range(args.warmup):
        api.li_sparse_attention(q, kv, sels[i % 8], scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    gr = capture([lambda i=i: api.li_sparse_attention(q, kv, sels[i % 8], scale, out=out, workspace=ws)
                  for i in range(16)])
    gr.replay()
    torch.cuda.synchronize()
    reps = max(2, args.steps // 16)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        gr.replay()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    us = e0.elapsed_time(e1) * 1e3 / (16 * reps)
    hbm, which = peaks()
    bf16_peak = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"]) \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 1590.0
    byts = B * KTOP * D * 2 + B * Ha * D * 2 + B * Ha * 512 * 4
    flops = B * Ha * KTOP * (D + 512) * 2
    res = {"metric": "sparse attention over the selection, µs per call", "value": us, "unit": "µs/call",
            "higher_is_better": False, "dtype": "bf16",
            "config": {"workload": "sparse_attention_b8_h128_k2048_l32k", "B": B, "heads": Ha, "k": KTOP, "L": L,
                       "row": "576 bf16 (512 latent + 64 RoPE); value = first 512",
                       "l2": "8 rotating selection sets, 151 MB of gathered rows"},
            "roofline": {"bound": "hbm", "kernel": "sparse_attn_kernel + sparse_attn_merge_kernel",
                         "achieved": byts / us / 1e3, "peak": hbm, "peak_source": which, "unit": "GB/s",
                         "frac": byts / us / 1e3 / hbm, "algorithmic_bytes": byts,
                         "tensor_tflops": flops / us / 1e6, "tensor_frac_of_bf16": flops / us / 1e6 / bf16_peak},
            "gpu_launches": 2 * 16 * reps, "clocks": clk}
    if want_cpu:
        res["cpu_baseline"] = oracle_sample("sparse_attention", (q.cpu(), kv.cpu(), sels[0].cpu().numpy(), scale))
    return res


def run_lshard(dev, args, clocks):
    """L-sharding of one long context (B = 8 requests, L = 131072), emulated on one GPU: the per-rank
    step (li_decode_select with values over the rank's L/P slice) and the merge of the P lists
    (li_merge_shards), for P = 2, 4, 8, beside the unsharded step.  The all-gather between them
    (8 B per listed position, P x B x k of them) is not timed: every call here has one GPU."""
    import torch
    from sparse_attention_lightning_score_b200 import api, synth
    Lt = 131072
    case = synth.dsa_decode(B=B, L=Lt, seed=1)
    q, w = case.q.to(dev), case.w.to(dev)
    k8, ks = case.k8.to(dev), case.ks.to(dev)

    def timed(fns, reps):
        g = capture(fns)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (reps * len(fns))

    reps = max(3, args.steps // 4)
    clocks.start()
    ws = api.li_decode_select_workspace(B, dev, Lt)
    sc = torch.empty((B, Lt), dtype=torch.float32, device=dev)
    idx = torch.empty((B, KTOP), dtype=torch.int32, device=dev)
    vals = torch.empty((B, KTOP), dtype=torch.float32, device=dev)
    full_us = timed([lambda: api.li_decode_select(q, w, k8, ks, KTOP, scores=sc, workspace=ws, with_values=True,
                                                  idx=idx, vals=vals)] * 4, reps)
    res = {}
    for P in (2, 4, 8):
        sl = Lt // P
        # every rank's slice as its own cache; copies until the slices read per replay exceed L2
        nset = max(1, math.ceil(1.5 * L2_BYTES / (B * Lt * (D + 4))))
        slices = [(k8[:, p * sl:(p + 1) * sl].contiguous(), ks[:, p * sl:(p + 1) * sl].contiguous())
                  for _ in range(nset) for p in range(P)]
        scp = torch.empty((B, sl), dtype=torch.float32, device=dev)
        lv = torch.empty((P, B, KTOP), dtype=torch.float32, device=dev)
        li = torch.empty((P, B, KTOP), dtype=torch.int32, device=dev)
        for p in range(P):
            api.li_decode_select(q, w, slices[p][0], slices[p][1], KTOP, scores=scp, workspace=ws, with_values=True,
                                 idx=li[p], vals=lv[p])
        ri = torch.empty((B, KTOP), dtype=torch.int32, device=dev)
        rank_us = timed([lambda s=s: api.li_decode_select(q, w, s[0], s[1], KTOP, scores=scp, workspace=ws,
                                                          idx=ri) for s in slices], reps)
        mws = torch.zeros(api._lib.load().li_merge_shards_workspace(P, B, KTOP), dtype=torch.uint8, device=dev)
        oi = torch.empty((B, KTOP), dtype=torch.int32, device=dev)
        merge_us = timed([lambda: api.li_merge_shards(lv, li, sl, KTOP, out_idx=oi, workspace=mws)] * 8, reps)
        # the merged selection is the unsharded one
        assert torch.equal(oi, idx), P
        res[str(P)] = {"rank_step_us": round(rank_us, 2), "merge_us": round(merge_us, 2),
                       "critical_path_us_without_allgather": round(rank_us + merge_us, 2),
                       "allgather_bytes_per_rank": P * B * KTOP * 8}
    clk = clocks.stop()
    return {"metric": "decode step µs at L = 131072 split along L over P ranks (rank step + merge)",
            "value": full_us, "unit": "µs/step (unsharded)", "higher_is_better": False, "dtype": "e4m3",
            "config": {"workload": "lshard_b8_l128k", "B": B, "L": Lt, "k": KTOP,
                       "ranks": "emulated on one GPU, one after another; the all-gather is not timed"},
            "lshard": res, "gpu_launches": None, "clocks": clk}


def run_table4(dev, args, clocks):
    """An in-house analogue of the LatentIndex paper's Table 4 (decode indexer latency by context length):
    one decode token (B = 1) through one 4-layer group, µs per group, at L = 8K..128K:
      dsa         4 layers x li_decode_select (FP8 keys, 64 heads, d = 128, top-2048);
      indexcache  1 indexer layer of the 4 (the other 3 reuse its selection: no kernel);
      latentindex 4 layers x (absorb + bf16 latent scan over the shared d_c = 256 cache + top-2048);
      hs          all four layers absorbed in one launch, the anchor's scan + top-C (C = min(8192, L)),
                  then the 3 followers' gather-once rescoring and top-2048, on one stream;
      *_fp8       the same two over DeepSeek-V3.2's d_c = 192 e4m3 latent with per-row scales.
    Every layer reads its own cache copies, rotated so that a group's working set exceeds L2."""
    import torch
    from sparse_attention_lightning_score_b200 import api, synth
    rows = []
    clocks.start()
    for Lx in (8192, 16384, 32768, 65536, 131072):
        dcase = synth.dsa_decode(B=1, L=Lx, k_top=KTOP, seed=3)
        per = Lx * (D + 4)
        ncopy = max(4, math.ceil(1.5 * L2_BYTES / per))
        k8 = [dcase.k8.to(dev).clone() for _ in range(ncopy)]
        ks = [dcase.ks.to(dev).clone() for _ in range(ncopy)]
        q = [dcase.q.to(dev)] * 4
        w = [dcase.w.to(dev)] * 4
        ws = [api.li_decode_select_workspace(1, dev, Lx) for _ in range(4)]
        sc = torch.empty((1, Lx), dtype=torch.float32, device=dev)
        idx = torch.empty((4, 1, KTOP), dtype=torch.int32, device=dev)
        C = min(8192, Lx)
        lcase = synth.latent_hs(B=1, L=Lx, n_cand=C, seed=4)
        lper = Lx * 512
        lcopy = max(2, math.ceil(1.5 * L2_BYTES / lper))
        cs = [lcase.c.to(dev).clone() for _ in range(lcopy)]
        ql = [lcase.q[l].to(dev) for l in range(4)]
        wdl = [lcase.w_dec[l].to(dev) for l in range(4)]
        wl = [lcase.w[l].to(dev) for l in range(4)]
        wf = lcase.w[1:].contiguous().to(dev)
        qt = torch.empty((1, H, 256), dtype=torch.bfloat16, device=dev)
        ql_all, wdl_all = torch.stack(ql).contiguous(), torch.stack(wdl).contiguous()
        qt_all = torch.empty((4, 1, H, 256), dtype=torch.bfloat16, device=dev)
        hist = api.li_decode_select_workspace(1, dev).view(torch.int32)[:2048]
        lsc = torch.empty((1, Lx), dtype=torch.float32, device=dev)
        cand = torch.empty((1, C), dtype=torch.int32, device=dev)
        out = torch.empty((3, 1, KTOP), dtype=torch.int32, device=dev)
        hws = api.li_hs_refine_workspace(1, C, 3, dev)
        # the same methods over DeepSeek-V3.2's FP8 latent (d_c = 192 e4m3, one scale per row)
        fcase = synth.latent_rope_nope(B=1, L=Lx, G=4, seed=5)
        fper = Lx * 196
        fcopy = max(2, math.ceil(1.5 * L2_BYTES / fper))
        c8s = [(fcase.c8.to(dev).clone(), fcase.cs.to(dev).clone()) for _ in range(fcopy)]
        q8l = [fcase.q[l].to(dev) for l in range(4)]
        wd8 = [fcase.w_dec[l].to(dev) for l in range(4)]
        w8 = [fcase.w[l].to(dev) for l in range(4)]
        wf8 = fcase.w[1:].contiguous().to(dev)
        qt8 = torch.empty((1, H, 192), dtype=torch.bfloat16, device=dev)
        q8_all, wd8_all = torch.stack(q8l).contiguous(), torch.stack(wd8).contiguous()
        qt8_all = torch.empty((4, 1, H, 192), dtype=torch.bfloat16, device=dev)

        def dsa(i, layers=4):
            for l in range(layers):
                j = (4 * i + l) % ncopy
                api.li_decode_select(q[l], w[l], k8[j], ks[j], KTOP, scores=sc, workspace=ws[l], idx=idx[l])

        def latent(i):
            c = cs[i % lcopy]
            for l in range(4):
                api.li_absorb_query(ql[l], wdl[l], out=qt)
                api.li_latent_score_hist(qt, wl[l], c, hist, scores=lsc)
                api.li_topk_hist(lsc, KTOP, hist, idx=idx[l])

        def hs(i):
            c = cs[i % lcopy]
            api.li_absorb_query_layers(ql_all, wdl_all, out=qt_all)
            api.li_latent_score_hist(qt_all[0], wl[0], c, hist, scores=lsc)
            api.li_topk_hist(lsc, C, hist, idx=cand)
            api.li_hs_refine(c, cand, qt_all[1:], wf, KTOP, out=out, workspace=hws)

        def latent8(i):
            c8, cs8 = c8s[i % fcopy]
            for l in range(4):
                api.li_absorb_query(q8l[l], wd8[l], out=qt8)
                api.li_latent_score_fp8(qt8, w8[l], c8, cs8, hist=hist, scores=lsc)
                api.li_topk_hist(lsc, KTOP, hist, idx=idx[l])

        def hs8(i):
            c8, cs8 = c8s[i % fcopy]
            api.li_absorb_query_layers(q8_all, wd8_all, out=qt8_all)
            api.li_latent_score_fp8(qt8_all[0], w8[0], c8, cs8, hist=hist, scores=lsc)
            api.li_topk_hist(lsc, C, hist, idx=cand)
            api.li_hs_refine_fp8(c8, cs8, cand, qt8_all[1:], wf8, KTOP, out=out, workspace=hws)

        res = {"L": Lx}
        for name, fn in (("dsa", lambda i: dsa(i)), ("indexcache", lambda i: dsa(i, 1)), ("latentindex", latent),
                         ("hs", hs), ("latentindex_fp8", latent8), ("hs_fp8", hs8)):
            for i in range(args.warmup):
                fn(i)
            torch.cuda.synchronize()
            nrep = 8
            g = capture([lambda i=i: fn(i) for i in range(nrep)])
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(2, args.steps // nrep)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            res[name + "_us_per_group"] = round(e0.elapsed_time(e1) * 1e3 / (reps * nrep), 2)
            del g
        res["hs_speedup_over_dsa"] = round(res["dsa_us_per_group"] / res["hs_us_per_group"], 3)
        res["hs_fp8_speedup_over_dsa"] = round(res["dsa_us_per_group"] / res["hs_fp8_us_per_group"], 3)
        res["dsa_ms_per_token_61_layers"] = round(res["dsa_us_per_group"] * 61 / 4 / 1e3, 3)
        res["hs_ms_per_token_61_layers"] = round(res["hs_us_per_group"] * 61 / 4 / 1e3, 3)
        rows.append(res)
        del k8, ks, cs, c8s
        torch.cuda.empty_cache()
    clk = clocks.stop()
    return {"metric": "decode indexer µs per 4-layer group, one token (analogue of LatentIndex Table 4)",
            "value": rows[-1]["hs_speedup_over_dsa"], "unit": "x (HS over DSA at L = 131072)",
            "higher_is_better": True, "dtype": "e4m3 (DSA), bf16 (latent)",
            "config": {"workload": "table4_b1_group4", "B": 1, "G": 4, "k": KTOP, "C": "min(8192, L)",
                       "l2": "per-layer cache copies rotated past 1.5 x L2"},
            "table4": rows, "gpu_launches": None, "clocks": clk}


def run_schedules(dev, args, clocks, n_layers=8):
    """Decode steps over n_layers DSA layers (indexer + sparse attention [+ a dense block]) under the
    IndexCache and Multi-layer Indexer schedules: each plan serial and with its indexers on a side
    stream, as one CUDA graph per step."""
    import torch
    from sparse_attention_lightning_score_b200.schedule import (DecodeLayerStack, StepGraph, indexcache_plan,
                                                                mli_plan, priority_streams)
    stack = DecodeLayerStack(n_layers=n_layers, B=B, L=L, k=KTOP, dense=(7168, 4096), device=dev, seed=1)
    plans = {"dsa": mli_plan(n_layers, lag=0), "mli_lag1": mli_plan(n_layers, lag=1),
             "mli_lag2": mli_plan(n_layers, lag=2), "indexcache_half": indexcache_plan(n_layers, retention=0.5),
             "indexcache_half_mli_lag1": mli_plan(n_layers, lag=1, retention=0.5)}
    main, side = priority_streams()
    reps = max(3, args.steps // 5)

    def time_step(plan, overlap, with_rest):
        step = stack.bind(plan, overlap=overlap, with_rest=with_rest)
        with torch.cuda.stream(main):
            for _ in range(args.warmup):
                step.run(main, side)
        torch.cuda.synchronize()
        g = StepGraph(step, main, side)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for _ in range(reps):
            g.replay()
        e1.record(main)
        torch.cuda.synchronize()
        g.close()
        return e0.elapsed_time(e1) * 1e3 / reps

    clocks.start()
    res = {}
    for with_rest in (False, True):
        key = "with_dense" if with_rest else "indexer_and_attention"
        res[key] = {}
        for name, plan in plans.items():
            res[key][name] = {"serial_us": round(time_step(plan, False, with_rest), 2)}
            if name != "dsa":
                res[key][name]["overlapped_us"] = round(time_step(plan, True, with_rest), 2)
    clk = clocks.stop()
    base = res["indexer_and_attention"]["dsa"]["serial_us"]
    best = min(v.get("overlapped_us", v["serial_us"]) for v in res["indexer_and_attention"].values())
    return {"metric": "decode step µs over the layers (indexer + sparse attention per layer)",
            "value": base, "unit": "µs/step (DSA, serial)", "higher_is_better": False,
            "dtype": "e4m3 indexer, bf16 attention",
            "config": {"workload": f"schedules_{n_layers}layers_b{B}_l32k", "layers": n_layers, "B": B, "L": L,
                       "k": KTOP, "indexer_heads": H, "attention_heads": 128, "kv": "576 bf16 per position",
                       "dense_block": "x[B,7168] @ W[7168,4096] bf16 per layer (cuBLAS), in with_dense only",
                       "launch": "one CUDA graph per step, instantiated with node priorities; main stream at the "
                                 "highest priority, overlapped = indexers on a lowest-priority side stream"},
            "schedules": res, "best_over_dsa": round(base / best, 3), "gpu_launches": None, "clocks": clk}


def run_other(args, rank, world, local_rank):
    import torch
    from sparse_attention_lightning_score_b200 import api
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm, which = peaks()
    clocks = ClockSampler(local_rank)
    if args.workload == "glm5_decode":
        # GLM-5's indexer shape (32 heads, d = 128, FP8 keys) on the decode step of the default workload
        bx = DecodeBench(dev, L, seed=1, heads=32)
        bx.build_graphs(args.warmup)
        clocks.start()
        time.sleep(0.3)
        ms = bx.time_steps(args.steps)
        clk = clocks.stop()
        sc_ms, tk_ms = bx.time_kernel("score"), bx.time_kernel("topk")
        algo = B * L * decode_bytes_per_key() + B * 32 * D * 2 + B * 32 * 4
        out = {"metric": METRIC, "value": B * L / (ms * 1e-3), "unit": "keys/s", "ms_per_step": ms,
               "us_per_step": ms * 1e3, "higher_is_better": True, "dtype": "e4m3",
               "config": {"workload": "glm5_decode_b8_l32k", "B": B, "L": L, "H": 32, "d": D, "k": KTOP,
                          "l2": f"{bx.n} rotating key-cache copies"},
               "roofline": {"bound": "hbm", "kernel": SCORER_KERNEL, "achieved": algo / (sc_ms * 1e-3) / 1e9,
                            "peak": hbm, "peak_source": which, "unit": "GB/s",
                            "frac": algo / (sc_ms * 1e-3) / 1e9 / hbm, "kernel_us": sc_ms * 1e3},
               "topk": {"us": tk_ms * 1e3}, "gpu_launches": 2 * args.steps, "clocks": clk}
    elif args.workload == "mli":
        out = run_schedules(dev, args, clocks)
    elif args.workload == "sparse_attention":
        out = run_consumer(dev, args, clocks, want_cpu=rank == 0 and world == 1 and not args.no_cpu_baseline)
    elif args.workload == "table4":
        out = run_table4(dev, args, clocks)
    elif args.workload == "lshard":
        out = run_lshard(dev, args, clocks)
    elif args.workload == "prefill":
        fp8_burst, fp8_sust, fp8_src = fp8_peak_tflops()
        bx = PrefillBench(dev)
        clocks.start()
        r = bx.run(args.steps, args.warmup)
        clk = clocks.stop()
        flops = bx.pairs * 2 * H * D
        achieved = flops / (r["score"] * 1e-3) / 1e12
        out = {"metric": METRIC, "value": bx.pairs / (r["step"] * 1e-3), "unit": "keys/s (visible pairs)",
               "ms_per_step": r["step"], "higher_is_better": True, "dtype": "e4m3",
               "config": {"workload": "dsa_prefill_t8k", "T": bx.T, "L": bx.L, "H": H, "d": D, "k": KTOP},
               "roofline": {"bound": "tensor", "kernel": PREFILL_KERNELS,
                            "achieved": achieved, "peak": fp8_burst, "peak_source": fp8_src, "unit": "TFLOP/s",
                            "frac": achieved / fp8_burst, "frac_of_sustained": achieved / fp8_sust,
                            "score_ms": r["score"]},
               "topk": {"ms": r["topk"], "rows_per_s": bx.T / (r["topk"] * 1e-3)}, "clocks": clk}
    elif args.workload in ("latent", "latent192", "latent_glm5"):
        bx = LatentBench(dev, kind="fp8_192" if args.workload == "latent192" else "bf16",
                         heads=32 if args.workload == "latent_glm5" else H)
        clocks.start()
        r = bx.run(args.steps, args.warmup)
        clk = clocks.stop()
        per_layer_bytes = bx.B * bx.L * (bx.key_bytes + 4)
        achieved = per_layer_bytes / (r["score"] * 1e-3) / 1e9
        fp8 = bx.kind != "bf16"
        out = {"metric": METRIC, "value": 4 * bx.B * bx.L / (r["step"] * 1e-3), "unit": "keys/s",
               "ms_per_step": r["step"], "us_per_layer": r["step"] * 1e3 / 4, "higher_is_better": True,
               "dtype": "e4m3" if fp8 else "bf16",
               "config": {"workload": ("latent_fp8_dc192_g4_b4_l64k" if fp8 else
                                       "latent_h32_g4_b4_l64k" if bx.heads == 32 else "latent_g4_b4_l64k"),
                          "B": bx.B, "L": bx.L, "H": bx.heads, "G": 4, "d_c": bx.dc, "k": KTOP,
                          "l2": f"{len(bx.c)} rotating cache copies"},
               "roofline": {"bound": "hbm", "kernel": "latent8_score_kernel" if fp8 else "stream_score_kernel<bf16>",
                            "achieved": achieved, "peak": hbm, "peak_source": which, "unit": "GB/s",
                            "frac": achieved / hbm, "kernel_us": r["score"] * 1e3}, "clocks": clk}
    else:
        Bx = 1 if args.workload == "hs_b1" else 16
        bx = HsBench(dev, Bx)
        clocks.start()
        r = bx.run(args.steps, args.warmup)
        clk = clocks.stop()
        algo = bx.B * bx.L * (512 + 8) + bx.B * bx.C * (512 + 4 + 3 * 8)
        out = {"metric": METRIC, "value": bx.B * bx.L / (r["step"] * 1e-3), "unit": "keys/s (anchor scan)",
               "ms_per_step": r["step"], "us_per_step": r["step"] * 1e3, "higher_is_better": True,
               "dtype": "bf16", "config": {"workload": f"latent_hs_b{Bx}_l128k", "B": Bx, "L": bx.L, "C": bx.C,
                                           "followers": 3, "k": KTOP, "l2": f"{len(bx.c)} rotating cache copies"},
               "roofline": {"bound": "hbm", "kernel": "whole HS step", "achieved": algo / (r["step"] * 1e-3) / 1e9,
                            "peak": hbm, "peak_source": which, "unit": "GB/s",
                            "frac": algo / (r["step"] * 1e-3) / 1e9 / hbm}, "clocks": clk}
    assert api.li_get_last_error() == 0
    if rank == 0 and world == 1 and not args.no_cpu_baseline and "cpu_baseline" not in out:
        # the oracle on the host cores, on a bounded sample of the same workload
        if args.workload == "glm5_decode":
            out["cpu_baseline"] = cpu_baseline_sample(heads=32)
        elif args.workload in ("prefill", "latent", "latent192", "latent_glm5", "hs_b1", "hs_b16"):
            out["cpu_baseline"] = oracle_sample(args.workload, bx.case)
    out.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup, "scaling": "weak", "vs_baseline": None,
                "data": "synthetic"})
    if rank == 0:
        print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="li", choices=["li", "reference"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the causal prefill record (and the FP8 peak it is measured against)")
    ap.add_argument("--workload", default="decode", choices=["decode", "glm5_decode", "prefill", "latent", "latent192", "latent_glm5", "hs_b1", "hs_b16", "mli", "lshard",
                             "sparse_attention", "table4"],
                    help="decode (default) is the benchmarked configuration; the others time the other "
                         "configurations of the parity tests")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from sparse_attention_lightning_score_b200.dist import env_rank
    rank, world, local_rank = env_rank()
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.workload == "decode":
        run_li(args, rank, world, local_rank)
    else:
        run_other(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
