#!/usr/bin/env python
"""Throughput of the B200 transformer scorer on a seeded request stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload bert-base-len2-100]

One step = one pass of the whole scoring path over one synthetic request
stream: the DP batch scheduler (rm_schedule) groups the stream's requests
(all queued at t = 0, i.e. saturation) into packed varlen batches of at most
Bmax sequences, and every batch is scored by rm_score (embedding, per layer:
QKV GEMM, attention scores, masked softmax, context, output GEMM, residual +
LayerNorm, FFN GEMMs, residual + LayerNorm, then the scalar head).

`value` is sequences/s with the token ids already resident in HBM; `e2e` is
the same metric through rm_score_host with pinned host buffers, the
host->device copy of each batch's ids and the device->host read of its scores
inside the timed region.  Multi-GPU (torchrun): independent replicas, one
stream per rank, no collective on the data path (weak scaling); the time is
the max over ranks.

`repeats` holds five timed regions of this process; `processes` repeats the
measurement in independent processes (default five in total, one after
another on the same GPU), each reporting its first timed region.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same stream (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "sequences scored/sec at 1 B200 (BERT-base, len 2–100); p50 latency"
UNIT = "sequences/s"
# Cost model of the DP scheduler: T(b, L) = C0 + C1*b*L in units of padded
# tokens; C0 stands for the fixed per-batch cost (launch sequence, weight
# streaming) of about 20k token-steps.
SCHED_C0, SCHED_C1 = 20000, 1
KERNEL_NAMES = ("gemm", "attn_scores", "softmax", "attn_context", "layernorm", "embed", "head",
                "attn_fused")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel (tcgen05 GEMM) from one ncu
# capture; valid only for the code it was taken on (code_sha of gemm_tc.cu).  Mean of the 48 projections of one fused call of eight DP
# batches, T = 27829 (the default step's calls average T = 25457).
GEMM_TRAFFIC = {"src_sha": "3db551ef7a0e0283", "workload": "bert-base-len2-100", "fuse": 8,
                "bytes_per_launch": 131929445}


def code_sha(path):
    """sha256 prefix of a source file's code: line comments and blank lines
    dropped, so that editing a comment does not invalidate counters taken on
    the same kernel."""
    lines = []
    for ln in open(path, encoding="utf-8").read().splitlines():
        code = ln.split("//", 1)[0].strip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def replica_workload(w, rank: int):
    """The workload a replica scores: the same model, its own seeded request stream."""
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def reduce_times(vals, dist, device):
    """Max over ranks of per-rank timings (ms); plain values when single-process."""
    vals = np.asarray(vals, dtype=np.float64)
    if dist is None:
        return vals
    import torch
    t = torch.tensor(vals, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().numpy()


def whole_job_rate(world: int, per_rank_units: int, steps: int, max_ms: float) -> float:
    """Units processed by all ranks per second of the slowest rank."""
    return world * per_rank_units * steps / (max_ms / 1000.0)


def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def metric_for(name):
    """The headline metric names the lengths-2..100 BERT-base stream; the other
    workloads name their own model and lengths in the same form."""
    if name == "bert-base-len2-100":
        return METRIC
    w = synth.WORKLOADS[name]
    model = {"tiny-enc": "tiny encoder", "tinybert-b1": "TinyBERT", "bert-base-len5-500": "BERT-base",
             "gpt-1.3b-rm": "GPT-1.3B-shape reward model"}[name]
    lens = (f"len {w.len_lo}\u2013{w.len_hi}" if not w.fixed_lengths
            else "len " + "/".join(str(x) for x in w.fixed_lengths))
    return f"sequences scored/sec at 1 B200 ({model}, {lens}); p50 latency"


def workload_config(name):
    w = synth.WORKLOADS[name]
    s = w.shape
    return {"workload": name,
            "model": {"tiny-enc": "tiny encoder scorer", "tinybert-b1": "TinyBERT-shape encoder",
                      "bert-base-len2-100": "BERT-base-shape scorer",
                      "bert-base-len5-500": "BERT-base-shape scorer",
                      "gpt-1.3b-rm": "GPT-style 1.3B-shape causal reward model"}[name],
            "layers": s.n_layers, "hidden": s.hidden, "heads": s.n_heads, "ffn": s.ffn,
            "vocab": s.vocab, "weights": "random N(0,0.02), bf16" if s.weight_dtype else "random N(0,0.02), fp32",
            "requests_per_step": w.n_requests if not w.fixed_lengths else len(w.fixed_lengths),
            "lengths": f"uniform {w.len_lo}..{w.len_hi}" if not w.fixed_lengths else list(w.fixed_lengths),
            "max_batch": w.max_batch, "arrivals": "all queued at t=0 (saturation)",
            "scheduler": f"DP, T(b,L) = {SCHED_C0} + {SCHED_C1}*b*L",
            "global_batch": w.max_batch, "seq_len": w.len_hi,
            "l2": "inputs larger than L2: every batch streams all weights (BERT-base bf16 218 MB > 126 MB L2)",
            "parallelism": "replicas"}


def clocks_log(args, name):
    """Where the raw nvidia-smi clock samples go (--clocks-dir), or None."""
    return os.path.join(args.clocks_dir, name) if args.clocks_dir else None


def lanes_note(n):
    return f"{n} stream(s) per GPU, consecutive DP batches dealt round-robin"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_path: str | None):
        self.proc = None
        self.path = out_path
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(gpu_index), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if self.path:
            with open(self.path, "w") as f:
                f.write(out)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except ValueError:
                continue
            for k, nm in enumerate(names):
                if r[5 + k].strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


class OracleTimer:
    """The fp64 CPU oracle on the workload's seeded stream (loaded once)."""

    def __init__(self, name: str):
        from oracle import scorer
        self.scorer = scorer
        w = synth.WORKLOADS[name]
        s = w.shape
        self.m = scorer.unpack_weights(synth.make_weights(s, w.seed), s.arch, s.n_layers, s.hidden,
                                       s.n_heads, s.ffn, s.vocab, s.max_pos, s.weight_dtype, s.gelu,
                                       s.ln_eps)
        self.st = synth.make_stream(w)

    def run(self, budget_s: float, min_requests: int = 4, start: int = 0):
        """Score requests one by one until budget_s has elapsed and at least
        min_requests are done; returns (sequences/s, requests, seconds)."""
        st = self.st
        t0 = time.perf_counter()
        k = 0
        while True:
            i = (start + k) % len(st.lengths)
            self.scorer.score_one(self.m, st.ids[st.starts[i]:st.starts[i] + st.lengths[i]])
            k += 1
            el = time.perf_counter() - t0
            if (el >= budget_s and k >= min_requests) or k >= len(st.lengths):
                break
        return k / el, k, el


def reference_arm_prefix(args):
    """The oracle on the best-of-N workload: each step scores one candidate
    as its own prefix + candidate sequence (a bounded sample)."""
    from oracle import best_of_n as OB
    from oracle import scorer as O
    w = synth.PREFIX_WORKLOADS[args.workload]
    s = w.shape
    ids, prefix_len, n_cand, cand_len = synth.make_prefix_groups(w)
    m = O.unpack_weights(synth.make_weights(s, w.weight_seed), s.arch, s.n_layers, s.hidden,
                         s.n_heads, s.ffn, s.vocab, s.max_pos, s.weight_dtype, s.gelu, s.ln_eps)
    groups = OB.split_groups(ids, prefix_len, n_cand, cand_len)
    seqs = [np.concatenate([p, c]) for p, cs in groups for c in cs]
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        OB.score_candidates(m, seqs[it % len(seqs)], [0], [1], [len(seqs[it % len(seqs)])])
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps / total
    cores = oracle_threads()
    sample = (f"one prefix + candidate sequence per step (candidates 0..{args.steps - 1} after "
              f"{args.warmup} warm-up), fp64 numpy oracle, {total:.1f} s")
    line = {"impl": "reference",
            "metric": "candidate sequences scored/sec at 1 B200 (best-of-8 over shared prefixes, GPT-1.3B shape)",
            "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def reference_arm(args):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    if args.workload in synth.PREFIX_WORKLOADS:
        return reference_arm_prefix(args)
    name = args.workload
    w = synth.WORKLOADS[name]
    per_step = 8 if w.shape.hidden >= 768 else 64
    times, done = [], 0
    timer = OracleTimer(name)
    for it in range(args.warmup + args.steps):
        rate, k, el = timer.run(0.0, min_requests=per_step, start=it * per_step)
        if it >= args.warmup:
            times.append(el)
            done += k
    total = sum(times)
    value = done / total
    cores = oracle_threads()
    sample = (f"{per_step} requests per step from the seeded stream, scored one by one by the "
              f"fp64 numpy oracle")
    line = {"impl": "reference", "metric": metric_for(name), "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(name),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# B200 arm
# ---------------------------------------------------------------------------
def stat_summary(vals):
    """Median and a 95% t-interval of the mean of repeated measurements."""
    v = np.asarray(vals, dtype=np.float64)
    n = len(v)
    mean = float(v.mean())
    # two-sided 97.5% quantiles of Student's t for n - 1 = 1..9 degrees of freedom
    tq = {1: 12.706, 2: 4.303, 3: 3.182, 4: 2.776, 5: 2.571, 6: 2.447, 7: 2.365, 8: 2.306, 9: 2.262}
    half = tq.get(n - 1, 1.96) * float(v.std(ddof=1)) / np.sqrt(n) if n > 1 else 0.0
    return {"n": n, "values": [float(x) for x in v], "median": float(np.median(v)), "mean": mean,
            "ci95": [mean - half, mean + half], "min": float(v.min()), "max": float(v.max())}


class StreamExecutor:
    """Scores a request stream as rm_score calls, one per group of request
    indices (a DP batch, or consecutive DP batches fused), dealt round-robin
    to lanes (handles that share the weights, one stream each).  Every step
    re-runs the DP scheduler on the host (S0) and checks it is unchanged."""

    def __init__(self, torch, lanes, streams, st, groups, schedule):
        self.torch = torch
        self.lanes, self.streams, self.stream = lanes, streams, streams[0]
        self.st, self.groups, self.schedule = st, groups, schedule
        self.nb = len(groups)
        self.n_req = int(sum(len(g) for g in groups))
        order = np.concatenate(groups)
        self.order = order
        packed_ids, _ = synth.pack(st, order)
        self.b_tok = np.zeros(self.nb + 1, dtype=np.int64)
        self.b_seq = np.zeros(self.nb + 1, dtype=np.int64)
        self.b_off = []
        for b, g in enumerate(groups):
            lens = st.lengths[g]
            self.b_off.append(synth.offsets_from_lengths(lens))
            self.b_tok[b + 1] = self.b_tok[b] + int(lens.sum())
            self.b_seq[b + 1] = self.b_seq[b] + len(g)
        self.ids_dev = torch.from_numpy(packed_ids).cuda()
        self.out_dev = torch.zeros(self.n_req, dtype=torch.float32, device="cuda")
        self.ev_batch = [torch.cuda.Event(enable_timing=True) for _ in range(self.nb)]
        self.fork_ev = torch.cuda.Event()
        self.join_ev = [torch.cuda.Event() for _ in streams]

    def fork(self):
        # every lane starts after what stream 0 has enqueued so far
        self.fork_ev.record(self.stream)
        for s2 in self.streams[1:]:
            s2.wait_event(self.fork_ev)

    def join(self):
        for k, s2 in enumerate(self.streams[1:], 1):
            self.join_ev[k].record(s2)
            self.stream.wait_event(self.join_ev[k])

    def step(self, record=False):
        bt = self.lanes[0].schedule(self.st.lengths)                  # S0 on the host
        if self.schedule is not None and record and not np.array_equal(bt, self.schedule):
            raise RuntimeError("schedule changed between steps")
        for b in range(self.nb):
            k = b % len(self.lanes)
            self.lanes[k].score(self.ids_dev[self.b_tok[b]:], self.b_off[b],
                                self.out_dev[self.b_seq[b]:], self.streams[k])
            if record:
                self.ev_batch[b].record(self.streams[k])

    def warm(self, n):
        for _ in range(n):
            self.fork()
            self.step()
            self.join()
        self.torch.cuda.synchronize()

    def timed(self, steps, barrier, record_last=False):
        """CUDA-event milliseconds of `steps` steps on stream 0 (all lanes joined)."""
        torch = self.torch
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        self.fork()
        for k in range(steps):
            self.step(record=record_last and k == steps - 1)
        self.join()
        b.record(self.stream)
        torch.cuda.synchronize()
        barrier()
        return a.elapsed_time(b)

    def latency(self, ms_per_step):
        """p50 / p99 request latency in the last recorded step: every request is
        queued at the step's start and completes with its call; the step's start
        is the last call's completion minus the mean step time."""
        per_batch = np.array([self.ev_batch[0].elapsed_time(e) for e in self.ev_batch])
        first_done = ms_per_step - per_batch[-1]
        lat = np.empty(self.n_req)
        for b in range(self.nb):
            lat[self.b_seq[b]:self.b_seq[b + 1]] = per_batch[b] + first_done
        return float(np.median(lat)), float(np.percentile(lat, 99))

    def cupti_step(self, sc):
        """The same single-stream step without events, its kernels timed by CUPTI."""
        def run():
            for b in range(self.nb):
                sc.score(self.ids_dev[self.b_tok[b]:], self.b_off[b], self.out_dev[self.b_seq[b]:],
                         self.stream)
        try:
            return cupti_kernel_times(self.torch, run)
        except Exception as e:                      # a profiler that cannot start
            return {"error": f"{type(e).__name__}: {e}"}

    def profiled_step(self, sc):
        """One step on a single stream with per-launch CUDA events (after timing)."""
        sc.profile(1)
        for b in range(self.nb):
            sc.score(self.ids_dev[self.b_tok[b]:], self.b_off[b], self.out_dev[self.b_seq[b]:],
                     self.stream)
        self.torch.cuda.synchronize()
        prof = sc.profile_read()
        sc.profile(0)
        return prof


# kernel name fragment -> the library's kernel kind (KERNEL_NAMES)
CUPTI_KINDS = (("gemm_bf16_tc_kernel", "gemm"), ("res_ln_kernel", "layernorm"),
               ("attn_tc_kernel", "attn_fused"), ("attn_tile_kernel", "attn_fused"),
               ("attn_fused", "attn_fused"), ("attn_scores_kernel", "attn_scores"),
               ("attn_context_kernel", "attn_context"), ("softmax", "softmax"),
               ("embed_kernel", "embed"), ("head_kernel", "head"), ("best_of_n_kernel", "head"))


def cupti_kernel_times(torch, run):
    """Each kernel's share of the device timeline of run() (one stream), by
    kind, from CUPTI activity records (torch.profiler): a launch's end minus
    the later of its start and the previous kernel's end.  With programmatic
    dependent launch a kernel starts while its predecessor runs and waits for
    it, so its own start-to-end time would count that wait; its share does
    not, and no event sits between two launches.  None where the profiler has
    no CUDA activity."""
    from torch.autograd import DeviceType
    from torch.profiler import ProfilerActivity, profile
    if ProfilerActivity.CUDA not in torch.profiler.supported_activities():
        return None
    with profile(activities=[ProfilerActivity.CUDA]) as p:
        run()
        torch.cuda.synchronize()
    ks = sorted(((e.time_range.start, e.time_range.end, e.name) for e in p.events()
                 if e.device_type == DeviceType.CUDA), key=lambda k: k[0])
    out = {}
    prev_end = None
    for start, end, name in ks:
        share = end - (start if prev_end is None else max(start, prev_end))
        prev_end = end if prev_end is None else max(prev_end, end)
        kind = next((k for frag, k in CUPTI_KINDS if frag in name), None)
        if kind is None:
            continue
        d = out.setdefault(kind, {"launches": 0, "us": 0.0})
        d["launches"] += 1
        d["us"] += max(0.0, float(share))
    return out


def launches_of(lanes):
    return sum(h.profile_read()["total_launches"] for h in lanes)


def arena_line(sc, note):
    reserved, peak, nbuckets = (int(x) for x in sc.arena_stats())
    return {"reserved_bytes": reserved, "peak_planned_bytes": peak, "buckets": nbuckets, "sized_for": note}


def scorer_cfg(rm, s, w, fuse, max_len):
    return rm.RmConfig.make(arch=s.arch, n_layers=s.n_layers, hidden=s.hidden, n_heads=s.n_heads,
                            ffn=s.ffn, vocab=s.vocab, max_pos=s.max_pos,
                            weight_dtype=s.weight_dtype, gelu=s.gelu, ln_eps=s.ln_eps,
                            max_batch_seqs=fuse * w.max_batch,
                            max_tokens=fuse * w.max_batch * max_len, max_len=max_len,
                            sched_max_batch=w.max_batch, sched_c0=SCHED_C0, sched_c1=SCHED_C1)


def fused_groups(groups, fuse):
    return [np.concatenate(groups[k:k + fuse]) for k in range(0, len(groups), fuse)]


def secondary_workloads(args, torch, rm):
    """The pages' other workloads, each on its own handle, one GPU, timed with
    CUDA events after warm-up (reported beside the headline, not in it)."""
    out = {}
    stream = torch.cuda.Stream()
    # lengths 5..500 (TurboTransformers review, main results: 144 req/s on its hardware)
    name = "bert-base-len5-500"
    w = synth.WORKLOADS[name]
    s = w.shape
    st = synth.make_stream(w)
    max_len = min(s.max_pos, 1024, w.len_hi)
    sc = rm.Scorer(scorer_cfg(rm, s, w, args.fuse, max_len), synth.make_weights(s, w.seed))
    lanes = [sc] + [sc.shared() for _ in range(args.lanes - 1)]
    streams = [stream] + [torch.cuda.Stream() for _ in range(args.lanes - 1)]
    batch = sc.schedule(st.lengths)
    groups = [np.nonzero(batch == b)[0] for b in range(int(batch.max()) + 1)]
    row = {"metric": metric_for(name), "unit": UNIT, "config": workload_config(name)}
    for label, gr in (("value", fused_groups(groups, args.fuse)), ("value_unfused", groups)):
        ex = StreamExecutor(torch, lanes, streams, st, gr, batch)
        ex.warm(2)
        l0 = launches_of(lanes)
        ms = ex.timed(args.extra_steps, lambda: None)
        row[label] = ex.n_req * args.extra_steps / (ms / 1000.0)
        row["ms_per_step" if label == "value" else "ms_per_step_unfused"] = ms / args.extra_steps
        if label == "value":
            row["gpu_launches"] = launches_of(lanes) - l0
        del ex
    row["steps"], row["warmup"] = args.extra_steps, 2
    row["executor"] = {"lanes": len(lanes), "fuse": args.fuse, "unfused": "one DP batch (<= 32) per call"}
    row["arena"] = arena_line(sc, f"{args.fuse} x {w.max_batch} sequences x {max_len} tokens")
    for h in lanes:
        h.close()
    out[name] = row
    torch.cuda.empty_cache()

    # GPT-style 1.3B-shape reward model, batches of 64 sequences of 256..560 tokens
    name = "gpt-1.3b-rm"
    w = synth.WORKLOADS[name]
    s = w.shape
    st = synth.make_stream(w)
    sc = rm.Scorer(scorer_cfg(rm, s, w, 1, w.len_hi), synth.make_weights(s, w.seed))
    ex = StreamExecutor(torch, [sc], [stream], st, [np.arange(w.max_batch)], None)
    ex.warm(2)
    l0 = launches_of([sc])
    ms = ex.timed(args.extra_steps, lambda: None)
    n_launch = launches_of([sc]) - l0
    prof = ex.profiled_step(sc)
    pk, pk_kind = peaks()
    g = prof["gemm"]
    tf = g["flops"] / (g["ms"] * 1e-3) / 1e12 if g["ms"] > 0 else None
    out[name] = {"metric": metric_for(name), "unit": UNIT, "value": w.max_batch * args.extra_steps / (ms / 1000.0),
                 "ms_per_step": ms / args.extra_steps, "steps": args.extra_steps, "warmup": 2,
                 "gpu_launches": n_launch,
                 "config": workload_config(name),
                 "gemm_tflops": tf, "gemm_frac_of_sustained": tf / pk["bf16_tflops_sustained"] if tf else None,
                 "arena": arena_line(sc, f"{w.max_batch} sequences x {w.len_hi} tokens")}
    sc.close()
    del ex
    torch.cuda.empty_cache()

    # TinyBERT shape at batch 1, lengths 64 / 128 / 256 (SambaNova blog, Fig. 3)
    name = "tinybert-b1"
    w = synth.WORKLOADS[name]
    s = w.shape
    Lmax = max(w.fixed_lengths)
    cfg = rm.RmConfig.make(arch=s.arch, n_layers=s.n_layers, hidden=s.hidden, n_heads=s.n_heads,
                           ffn=s.ffn, vocab=s.vocab, max_pos=s.max_pos, weight_dtype=s.weight_dtype,
                           gelu=s.gelu, ln_eps=s.ln_eps, max_batch_seqs=1, max_tokens=Lmax,
                           max_len=Lmax, sched_max_batch=1)
    sc = rm.Scorer(cfg, synth.make_weights(s, w.seed))
    o = torch.zeros(1, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lat = {}
    for L in w.fixed_lengths:
        ids = torch.from_numpy(synth.make_token_ids(L, s.vocab, w.seed + L)).cuda()
        off = np.array([0, L], dtype=np.int32)
        vals = []
        for r in range(20 + args.extra_requests):
            torch.cuda.synchronize()
            a.record(stream)
            sc.score(ids, off, o, stream)
            b.record(stream)
            b.synchronize()
            if r >= 20:
                vals.append(a.elapsed_time(b))
        lat[str(L)] = {"p50_ms": float(np.median(vals)), "p99_ms": float(np.percentile(vals, 99))}
    out[name] = {"metric": "batch-1 p50 latency, TinyBERT shape (4 layers, H 312), eager rm_score from an idle GPU",
                 "unit": "ms", "higher_is_better": False, "requests_per_length": args.extra_requests,
                 "warmup": 20, "latency": lat, "value": lat[str(w.fixed_lengths[1])]["p50_ms"],
                 "value_is": f"p50 at length {w.fixed_lengths[1]}",
                 "arena": arena_line(sc, f"1 sequence x {Lmax} tokens")}
    sc.close()
    return out


def b200_arm(args):
    import torch
    import classifier_scoring_b200 as rm
    from classifier_scoring_b200 import build as rmbuild

    rank, world, local = rank_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the scorer has no CPU path)")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    rmbuild.build()

    def barrier():
        if dist is not None:
            dist.barrier()

    name = args.workload
    w = synth.WORKLOADS[name]
    s = w.shape
    flat = synth.make_weights(s, w.seed)
    st = synth.make_stream(replica_workload(w, rank))            # each replica its own requests
    max_len = min(s.max_pos, 1024, max(w.len_hi, int(st.lengths.max())))

    # fusing more batches than the stream has only enlarges the arena
    n_sched = int(rm.schedule(scorer_cfg(rm, s, w, 1, max_len), st.lengths).max()) + 1
    args.fuse = max(1, min(args.fuse, n_sched))
    sc = rm.Scorer(scorer_cfg(rm, s, w, args.fuse, max_len), flat)
    del flat
    lanes = [sc] + [sc.shared() for _ in range(args.lanes - 1)]
    streams = [torch.cuda.Stream() for _ in range(args.lanes)]
    stream = streams[0]

    # the schedule is deterministic: pack the stream in call order once, on the device
    batch = sc.schedule(st.lengths)
    nb = int(batch.max()) + 1
    dp_groups = [np.nonzero(batch == b)[0] for b in range(nb)]
    n_dp_batches = nb
    if args.batch_index is not None:
        # one call only (small profiling case): this DP batch, or the `fuse`
        # consecutive batches starting with it
        keep = np.concatenate(dp_groups[args.batch_index % nb:args.batch_index % nb + args.fuse])
        st = synth.Stream(lengths=st.lengths[keep], ids=st.ids, starts=st.starts[keep])
        batch = None
        groups = [np.arange(len(keep))]
        n_dp_batches = min(args.fuse, n_dp_batches)
        unfused = None
    else:
        # executor: consecutive DP batches run as one forward pass (packed, so
        # the result of every request is the same; the projections get more rows)
        groups = fused_groups(dp_groups, args.fuse)
        unfused = dp_groups if args.fuse > 1 else None
    ex = StreamExecutor(torch, lanes, streams, st, groups, batch)
    n_req = ex.n_req

    # warm-up (plans every length bucket; the kernels are prebuilt)
    ex.warm(args.warmup)
    ex_u = None
    if unfused is not None:
        ex_u = StreamExecutor(torch, lanes, streams, st, unfused, batch)
        ex_u.warm(max(3, args.warmup // 2))

    for h in lanes:
        # per-launch CUDA events inside the timed regions only on request
        # (--profile-every n > 0, a diagnostic that breaks launch overlap)
        h.profile(args.profile_every)
    launches0 = launches_of(lanes)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    clocks = ClockSampler(gpu_index, clocks_log(args, f"clocks_rank{rank}.csv"))
    time.sleep(0.3)
    wall0 = time.perf_counter()
    elapsed_ms = ex.timed(args.steps, barrier, record_last=True)
    wall = time.perf_counter() - wall0
    launches = launches_of(lanes) - launches0
    # further independent timed regions of the same K steps, for a spread
    rep_ms = [elapsed_ms] + [ex.timed(args.steps, barrier) for _ in range(args.repeats - 1)]
    unf_ms = ex_u.timed(args.steps, barrier) if ex_u is not None else None
    clk = clocks.stop()
    p50, p99 = ex.latency(elapsed_ms / args.steps)
    # kernel table and roofline from one extra single-stream step after timing
    prof = ex.profiled_step(sc)
    # and the same step's kernels timed by CUPTI, without per-launch events
    # (not under another profiler such as ncu)
    cup = ex.cupti_step(sc) if not args.no_cupti else None

    # ---- end to end through rm_score_host (pinned host buffers) ----
    b_tok, b_seq, b_off = ex.b_tok, ex.b_seq, ex.b_off
    ids_pin = torch.empty(int(b_tok[-1]), dtype=torch.int32).pin_memory()
    out_pin = torch.empty(n_req, dtype=torch.float32).pin_memory()
    ids_np = ids_pin.numpy()
    host_ids = st.ids
    # position in the arrival-ordered id array of every packed token (call order)
    gather = np.concatenate([np.arange(st.starts[i], st.starts[i] + st.lengths[i]) for i in ex.order])

    def e2e_step():
        sc.schedule(st.lengths)                               # S0
        np.take(host_ids, gather, out=ids_np)                 # S1: host gather into pinned memory
        for b in range(ex.nb):
            k = b % len(lanes)
            lanes[k].score_host(ids_pin[b_tok[b]:], b_off[b], out_pin[b_seq[b]:], streams[k])

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ew0 = time.perf_counter()
    e0.record(stream)
    ex.fork()
    e_steps = max(1, args.steps)
    for _ in range(e_steps):
        e2e_step()
    ex.join()
    e1.record(stream)
    torch.cuda.synchronize()
    e_wall = time.perf_counter() - ew0
    barrier()
    e_ms = max(e0.elapsed_time(e1), 1000 * e_wall)
    if not np.array_equal(out_pin.numpy(), ex.out_dev.cpu().numpy()):
        raise RuntimeError("rm_score_host and rm_score disagree")
    meta_bytes = sum(4 * (len(o)) * 2 + 8 * len(o) for o in b_off)
    h2d = 4 * int(b_tok[-1]) + meta_bytes
    d2h = 4 * n_req

    # ---- reduce over ranks ----
    vals = reduce_times([elapsed_ms, e_ms] + rep_ms + ([unf_ms] if unf_ms is not None else []),
                        dist, "cuda")
    max_ms, max_e_ms = float(vals[0]), float(vals[1])
    max_rep = [float(x) for x in vals[2:2 + len(rep_ms)]]
    max_unf = float(vals[-1]) if unf_ms is not None else None
    value = whole_job_rate(world, n_req, args.steps, max_ms)
    e2e_value = whole_job_rate(world, n_req, e_steps, max_e_ms)

    pk, pk_kind = peaks()
    g = prof["gemm"]
    gemm_tflops = g["flops"] / (g["ms"] * 1e-3) / 1e12 if g["ms"] > 0 else None
    sha = code_sha(os.path.join(ROOT, "classifier_scoring_b200", "csrc", "gemm_tc.cu"))
    traffic = (GEMM_TRAFFIC["bytes_per_launch"]
               if (GEMM_TRAFFIC["src_sha"] == sha and GEMM_TRAFFIC["workload"] == name
                   and GEMM_TRAFFIC["fuse"] == args.fuse and args.batch_index is None) else None)
    roofline = {"kernel": "gemm_bf16_tc_kernel (QKV, output and FFN projections)",
                "measured_on": "one single-stream step with per-launch CUDA events, after the timed "
                               "regions (which ran without per-launch events)",
                "bound": "tensor", "achieved": gemm_tflops, "peak": pk["bf16_tflops_sustained"],
                "unit": "TFLOP/s",
                "frac": (gemm_tflops / pk["bf16_tflops_sustained"]) if gemm_tflops else None,
                "peak_source": f"bf16_tflops_sustained of {pk_kind} (kernel timed inside a long step)",
                "traffic": traffic,
                "launches_timed": g["launches"], "avg_launch_us": 1000 * g["ms"] / max(1, g["launches"])}

    total_ms = max(1e-9, sum(prof[x]["ms"] for x in KERNEL_NAMES))
    kernels = {}
    for kname in KERNEL_NAMES:
        d = prof[kname]
        if d["launches"] == 0:
            continue
        e = {"launches": d["launches"], "avg_us": 1000 * d["ms"] / d["launches"],
             "share": d["ms"] / total_ms}
        if d["flops"] and kname in ("gemm", "attn_scores", "attn_context", "attn_fused"):
            e["tflops"] = d["flops"] / (d["ms"] * 1e-3) / 1e12
        if d["bytes"]:
            e["gbs"] = d["bytes"] / (d["ms"] * 1e-3) / 1e9
            e["hbm_frac_of_measured"] = e["gbs"] / pk["hbm_gbs"]
        c = (cup or {}).get(kname)
        if isinstance(c, dict) and c["launches"] == d["launches"] and c["us"] > 0:
            # the same launches' shares of the device timeline (CUPTI), no events between them
            cu = {"avg_us": c["us"] / c["launches"]}
            if "tflops" in e:
                cu["tflops"] = d["flops"] / (c["us"] * 1e-6) / 1e12
            if d["bytes"]:
                cu["gbs"] = d["bytes"] / (c["us"] * 1e-6) / 1e9
                cu["hbm_frac_of_measured"] = cu["gbs"] / pk["hbm_gbs"]
            e["cupti"] = cu
        kernels[kname] = e

    rep_vals = [whole_job_rate(world, n_req, args.steps, m) for m in max_rep]
    result = {
        "metric": metric_for(name), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(name), lanes=lanes_note(len(lanes)),
                       **({"fuse": f"{args.fuse} consecutive DP batches per rm_score call"}
                          if args.fuse > 1 else {})),
        "repeats": dict(stat_summary(rep_vals), unit=UNIT,
                        method=f"{len(rep_vals)} timed regions of {args.steps} steps each in this "
                               "process (the first is `value`); 95% t-interval of the mean"),
        "p50_latency_ms": p50, "p99_latency_ms": p99, "batches_per_step": n_dp_batches,
        "calls_per_step": ex.nb,
        "tokens_per_step": int(b_tok[-1]),
        "roofline": roofline,
        "kernels": kernels,
        "kernels_method": "avg_us, gbs, tflops: per-launch CUDA events in one single-stream step after "
                          "the timed regions (an event between two launches ends their programmatic "
                          "overlap, so short kernels read slow); cupti: in a second such step without "
                          "events, each launch's share of the device timeline from CUPTI activity "
                          "records (its end minus the later of its start and the previous kernel's end)"
                          + ("" if not (isinstance(cup, dict) and "error" in cup)
                             else f" (unavailable: {cup['error']})"),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "rm_score_host, pinned host ids/scores"},
        "gpu_launches": int(launches),
        "clocks": clk,
        "wall_s_timed": wall,
        "arena": arena_line(sc, f"{args.fuse} x {w.max_batch} sequences x {max_len} tokens"),
        "context": {"turbotransformers_req_s_len2_100": 402, "hardware": "not named on the page"},
    }
    if max_unf is not None:
        result["value_unfused"] = whole_job_rate(world, n_req, args.steps, max_unf)
        result["unfused"] = {"ms_per_step": max_unf / args.steps, "calls_per_step": len(unfused),
                             "executor": f"one DP batch (<= {w.max_batch} sequences) per rm_score call, "
                                         f"{len(lanes)} lanes"}
    for h in lanes:
        h.close()
    del ex, ex_u
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, k, el = OracleTimer(name).run(args.cpu_budget)
        result["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": oracle_threads(),
                                  "kind": "oracle",
                                  "sample": f"first {k} requests of the seeded stream scored one by "
                                            f"one by the fp64 numpy oracle ({el:.1f} s)"}
    if world == 1 and args.batch_index is None and not args.no_extra and name == "bert-base-len2-100":
        result["other_workloads"] = secondary_workloads(args, torch, rm)
    if world == 1 and args.batch_index is None and args.processes > 1:
        result["processes"] = process_repeats(args, name, value)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def process_repeats(args, name, first):
    """The same measurement repeated in independent processes (fresh CUDA
    context, weights and arena each), run one after another on this GPU once
    this process is idle: the value of each process's first timed region,
    with this process's as the first."""
    vals, errors = [first], []
    cmd = [sys.executable, os.path.abspath(__file__), "--workload", name, "--steps", str(args.steps),
           "--warmup", str(args.warmup), "--fuse", str(args.fuse), "--lanes", str(args.lanes),
           "--repeats", "1", "--processes", "1", "--no-extra", "--no-cpu-baseline", "--no-cupti"]
    for _ in range(args.processes - 1):
        r = subprocess.run(cmd, capture_output=True, text=True)
        try:
            vals.append(float(json.loads(r.stdout.strip().splitlines()[-1])["value"]))
        except (ValueError, IndexError, KeyError):
            errors.append(f"exit {r.returncode}: {r.stderr.strip().splitlines()[-1:] or ''}")
    out = dict(stat_summary(vals), unit=UNIT,
               method=f"{len(vals)} independent processes, each: {args.warmup} warm-up and "
                      f"{args.steps} timed steps, one timed region; 95% t-interval of the mean")
    if errors:
        out["errors"] = errors
    return out


# ---------------------------------------------------------------------------
# the two batch reductions alone, on working sets far larger than L2
# ---------------------------------------------------------------------------
def kernel_bench(args):
    import torch
    import classifier_scoring_b200 as rm
    from classifier_scoring_b200 import build as rmbuild

    rmbuild.build()
    torch.cuda.set_device(0)
    pk, pk_kind = peaks()
    st = torch.cuda.Stream()
    reps = max(3, args.steps)
    only = set(args.only.split(",")) if args.only else set()
    out = {"metric": "HBM GB/s of the softmax and residual+LayerNorm kernels alone",
           "unit": "GB/s", "peak_hbm_gbs": pk["hbm_gbs"], "peak_source": f"hbm_gbs of {pk_kind}",
           "kernels": {}}

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(reps):
            fn()
        b.record(st)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    # softmax over the score blocks of sequences with lengths U[5, 500], 12 heads
    rng = np.random.default_rng(7)
    nh = 12
    for label, lo, hi, causal in (("softmax_len5_500", 5, 500, 0), ("softmax_len256_560_causal", 256, 560, 1),
                                  ("softmax_len2_100", 2, 100, 0)):
        lens = []
        tot = 0
        while tot < 1.0e9:                       # about 2 GB of bf16 scores
            L = int(rng.integers(lo, hi + 1))
            lens.append(L)
            tot += nh * L * ((L + 7) // 8 * 8)
        lens = np.array(lens)
        if only and label not in only and label + "_batchwide" not in only:
            continue                             # the lengths are drawn all the same
        off = synth.offsets_from_lengths(lens)
        rb, so = rm.ops.varlen_meta(off, nh)
        S = torch.randn(int(so[-1]), dtype=torch.bfloat16, device="cuda")
        d_off = torch.from_numpy(off).cuda()
        d_so = torch.from_numpy(so).cuda()
        n, T = len(lens), int(off[-1])
        entries = nh * float(np.sum(lens * (lens + 1) / 2 if causal else lens * lens))
        gb = 4.0 * entries / 1e9
        scratch = torch.empty(rm.ops.softmax_scratch_bytes(n, T, nh), dtype=torch.uint8, device="cuda")
        # by length class (the path rm_score takes; the row-index kernels are
        # inside the timing) and with batch-wide lane groups
        for name, fn in (
                (label, lambda: rm.ops.softmax_classes(S, rm.BF16, d_off, d_so, n, T, nh,
                                                       int(lens.max()), causal, scratch, st)),
                (label + "_batchwide", lambda: rm.ops.softmax(S, rm.BF16, d_off, d_so, n, T, nh,
                                                              int(lens.max()), causal, st))):
            if only and name not in only:
                continue
            ms = timed(fn)
            out["kernels"][name] = {"ms": ms, "algorithmic_GB": gb, "gbs": gb / (ms * 1e-3),
                                    "frac_of_measured": gb / (ms * 1e-3) / pk["hbm_gbs"],
                                    "sequences": n, "heads": nh}
        del scratch
        del S
    for label, H, T, mode in (("res_ln_post_H768", 768, 1 << 20, 0), ("res_ln_pre_H2048", 2048, 1 << 18, 1)):
        if only and label not in only:
            continue
        y = torch.randn(T, H, dtype=torch.bfloat16, device="cuda")
        x = torch.randn(T, H, dtype=torch.bfloat16, device="cuda")
        z = torch.empty_like(x) if mode == 1 else None
        g = torch.ones(H, dtype=torch.float32, device="cuda")
        b = torch.zeros(H, dtype=torch.float32, device="cuda")
        ms = timed(lambda: rm.ops.res_ln(y, x, z, g, b, T, H, 1e-5, rm.BF16, mode, st))
        gb = (6.0 if mode == 0 else 8.0) * H * T / 1e9
        out["kernels"][label] = {"ms": ms, "algorithmic_GB": gb, "gbs": gb / (ms * 1e-3),
                                 "frac_of_measured": gb / (ms * 1e-3) / pk["hbm_gbs"],
                                 "rows": T, "hidden": H}
        del y, x, z
    print(json.dumps(out), flush=True)
    return 0


def prefix_bench(args):
    """Best-of-N over shared prefixes (rm_score_prefix) on the GPT-1.3B shape.
    A step scores every candidate of every group and selects each group's best;
    the same candidates scored as independent concatenations through rm_score
    are timed beside it.  Replicas under torchrun: each rank its own groups."""
    import torch
    import classifier_scoring_b200 as rm
    from classifier_scoring_b200 import build as rmbuild

    rank, world, local = rank_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the scorer has no CPU path)")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    rmbuild.build()
    w = synth.PREFIX_WORKLOADS[args.workload]
    s = w.shape
    ids, prefix_len, n_cand, cand_len = synth.make_prefix_groups(w, 1000 * rank)
    n_c, n_g = int(n_cand.sum()), len(n_cand)
    # the unshared comparison: every prefix + candidate as its own sequence
    cat, lens, pos, k = [], [], 0, 0
    for g in range(n_g):
        pre = ids[pos:pos + prefix_len[g]]
        pos += int(prefix_len[g])
        for _ in range(int(n_cand[g])):
            c = ids[pos:pos + cand_len[k]]
            pos += int(cand_len[k])
            k += 1
            cat.append(np.concatenate([pre, c]))
            lens.append(len(cat[-1]))
    cat_ids = np.concatenate(cat).astype(np.int32)
    cat_off = synth.offsets_from_lengths(np.array(lens))
    max_len = int(max(lens))
    cfg = rm.RmConfig.make(arch=s.arch, n_layers=s.n_layers, hidden=s.hidden, n_heads=s.n_heads,
                           ffn=s.ffn, vocab=s.vocab, max_pos=s.max_pos, weight_dtype=s.weight_dtype,
                           gelu=s.gelu, ln_eps=s.ln_eps, max_batch_seqs=n_g + n_c,
                           max_tokens=int(cat_off[-1]), max_len=max_len,
                           sched_max_batch=n_c, sched_c0=SCHED_C0, sched_c1=SCHED_C1)
    flat = synth.make_weights(s, w.weight_seed)
    sc = rm.Scorer(cfg, flat)
    del flat
    stream = torch.cuda.Stream()
    ids_dev = torch.from_numpy(ids).cuda()
    cat_dev = torch.from_numpy(cat_ids).cuda()
    out = torch.zeros(n_c, device="cuda")
    best = torch.zeros(n_g, dtype=torch.int32, device="cuda")
    lo = torch.zeros(n_g, device="cuda")
    out_cat = torch.zeros(n_c, device="cuda")

    def shared():
        sc.score_prefix(ids_dev, prefix_len, n_cand, cand_len, out, best, lo, stream)

    def unshared():
        sc.score(cat_dev, cat_off, out_cat, stream)

    def timed(fn, steps):
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    for _ in range(args.warmup):
        shared()
        unshared()
    torch.cuda.synchronize()
    # the two paths run different attention kernels (bf16 P rounded against
    # other running maxima), each meant to be within 2e-2 of the fp64 oracle:
    # their difference is reported, and only one beyond twice that is an error
    path_diff = float(np.max(np.abs(out.cpu().numpy() - out_cat.cpu().numpy())))
    if path_diff > 4e-2:
        raise RuntimeError(f"shared-prefix and unshared scores disagree by {path_diff}")
    l0 = sc.profile_read()["total_launches"]
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    clocks = ClockSampler(gpu_index, clocks_log(args, f"clocks_prefix_rank{rank}.csv"))
    time.sleep(0.3)
    ms_shared = timed(shared, args.steps)
    clk = clocks.stop()
    launches = sc.profile_read()["total_launches"] - l0
    ms_unshared = timed(unshared, args.steps)
    # end to end: ids from pinned host memory, scores and choices back to the host
    ids_pin = torch.from_numpy(ids).pin_memory()
    res_pin = torch.empty(n_c + 2 * n_g, dtype=torch.float32).pin_memory()
    best_pin = torch.empty(n_g, dtype=torch.int32).pin_memory()

    def e2e():
        with torch.cuda.stream(stream):
            ids_dev.copy_(ids_pin, non_blocking=True)
            shared()
            res_pin[:n_c].copy_(out, non_blocking=True)
            res_pin[n_c:n_c + n_g].copy_(lo, non_blocking=True)
            best_pin.copy_(best, non_blocking=True)

    ms_e2e = timed(e2e, args.steps)
    # kernel shares and the GEMM roofline from one profiled step
    sc.profile(1)
    shared()
    torch.cuda.synchronize()
    prof = sc.profile_read()
    sc.profile(0)
    vals = reduce_times([ms_shared, ms_unshared, ms_e2e], dist, "cuda")
    value = whole_job_rate(world, n_c, args.steps, float(vals[0]))
    pk, pk_kind = peaks()
    g = prof["gemm"]
    gemm_tflops = g["flops"] / (g["ms"] * 1e-3) / 1e12 if g["ms"] > 0 else None
    total_ms = max(1e-9, sum(prof[x]["ms"] for x in KERNEL_NAMES))
    result = {
        "metric": "candidate sequences scored/sec at 1 B200 (best-of-8 over shared prefixes, GPT-1.3B shape)",
        "value": value, "unit": "sequences/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": float(vals[0]) / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "model": "GPT-style 1.3B-shape causal reward model",
                   "groups": n_g, "candidates_per_group": w.n_cand,
                   "prefix_lengths": f"uniform {w.prefix_lo}..{w.prefix_hi}",
                   "candidate_lengths": f"uniform {w.cand_lo}..{w.cand_hi}",
                   "tokens_shared": int(len(ids)), "tokens_unshared": int(cat_off[-1]),
                   "l2": "inputs larger than L2: every step streams all weights (2.6 GB)",
                   "parallelism": "replicas"},
        "unshared": {"value": whole_job_rate(world, n_c, args.steps, float(vals[1])),
                     "ms_per_step": float(vals[1]) / args.steps,
                     "api": "rm_score on the prefix + candidate concatenations",
                     "max_abs_score_diff_vs_shared": path_diff},
        "roofline": {"kernel": "gemm_bf16_tc_kernel (QKV, output and FFN projections)",
                     "measured_on": "one profiled step after the timed region",
                     "bound": "tensor", "achieved": gemm_tflops, "peak": pk["bf16_tflops_sustained"],
                     "unit": "TFLOP/s",
                     "frac": gemm_tflops / pk["bf16_tflops_sustained"] if gemm_tflops else None,
                     "peak_source": f"bf16_tflops_sustained of {pk_kind}", "traffic": None},
        "kernels": {k: {"launches": prof[k]["launches"], "share": prof[k]["ms"] / total_ms}
                    for k in KERNEL_NAMES if prof[k]["launches"]},
        "e2e": {"value": whole_job_rate(world, n_c, args.steps, float(vals[2])), "unit": "sequences/s",
                "h2d_bytes_per_step": 4 * int(len(ids)) + 4 * (3 * n_g + 2 * n_c + 2),
                "d2h_bytes_per_step": 4 * n_c + 8 * n_g,
                "api": "rm_score_prefix, ids from pinned host memory, scores and best/log-odds back"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import best_of_n as OB
        from oracle import scorer as O
        m = O.unpack_weights(synth.make_weights(s, w.weight_seed), s.arch, s.n_layers, s.hidden,
                             s.n_heads, s.ffn, s.vocab, s.max_pos, s.weight_dtype, s.gelu, s.ln_eps)
        t0 = time.perf_counter()
        OB.score_candidates(m, cat[0], [0], [1], [len(cat[0])])
        el = time.perf_counter() - t0
        result["cpu_baseline"] = {"value": 1.0 / el, "unit": "sequences/s", "cores": oracle_threads(),
                                  "kind": "oracle",
                                  "sample": f"candidate 0 of group 0 ({len(cat[0])} tokens) scored "
                                            f"as its own sequence by the fp64 numpy oracle ({el:.1f} s)"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def serve_bench(args):
    """Open-loop serving of the request stream with Poisson arrivals at
    fractions of the saturation rate: whenever the GPU is idle, the host takes
    every queued request, schedules the queue with the DP (throughput or
    latency objective) and launches its batches through rm_score_host (ids
    from pinned host memory, scores back).  Latency = batch completion (CUDA
    event) - arrival.  One GPU; the saturation rate is measured first with
    every request queued at t = 0."""
    import torch
    import classifier_scoring_b200 as rm
    from classifier_scoring_b200 import build as rmbuild

    rank, world, local = rank_env()
    if world > 1:
        raise SystemExit("--serve runs on one GPU")
    torch.cuda.set_device(local)
    rmbuild.build()
    w = synth.WORKLOADS[args.workload]
    s = w.shape
    st = synth.make_stream(w)
    n = len(st.lengths)
    max_len = min(s.max_pos, 1024, max(w.len_hi, int(st.lengths.max())))
    flat = synth.make_weights(s, w.seed)

    def make_cfg(objective, cap):
        return rm.RmConfig.make(arch=s.arch, n_layers=s.n_layers, hidden=s.hidden, n_heads=s.n_heads,
                                ffn=s.ffn, vocab=s.vocab, max_pos=s.max_pos,
                                weight_dtype=s.weight_dtype, gelu=s.gelu, ln_eps=s.ln_eps,
                                max_batch_seqs=w.max_batch, max_tokens=w.max_batch * max_len,
                                max_len=max_len, sched_max_batch=w.max_batch, sched_c0=SCHED_C0,
                                sched_c1=SCHED_C1, sched_objective=objective, sched_max_cost=cap)
    # schedulers: the handle's own DP with each objective (host-only configs)
    sched_cfgs = {"throughput": make_cfg(rm.SCHED_THROUGHPUT, 0),
                  "latency": make_cfg(rm.SCHED_LATENCY, 0)}
    sc = rm.Scorer(make_cfg(rm.SCHED_THROUGHPUT, 0), flat)
    del flat
    stream = torch.cuda.Stream()
    total_tok = int(st.lengths.astype(np.int64).sum())
    ids_pin = torch.empty(total_tok, dtype=torch.int32).pin_memory()
    out_pin = torch.empty(n, dtype=torch.float32).pin_memory()
    ids_np = ids_pin.numpy()

    def run(arrivals, sched_name, warm=False):
        cfg = sched_cfgs[sched_name]
        ev0 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        nxt, queue, last_ev = 0, [], None
        log = []                                     # (event, request indices)
        windows = 0
        while nxt < n or queue:
            now = time.perf_counter() - t0
            while nxt < n and arrivals[nxt] <= now:
                queue.append(nxt)
                nxt += 1
            idle = last_ev is None or last_ev.query()
            if queue and idle:
                q = np.array(queue, dtype=np.int64)
                queue = []
                windows += 1
                batch = rm.schedule(cfg, st.lengths[q])
                tok, oc = 0, 0
                for b in range(int(batch.max()) + 1):
                    members = q[batch == b]
                    lens = st.lengths[members]
                    off = synth.offsets_from_lengths(lens)
                    k = int(off[-1])
                    np.concatenate([st.ids[st.starts[i]:st.starts[i] + st.lengths[i]] for i in members],
                                   out=ids_np[tok:tok + k])
                    sc.score_host(ids_pin[tok:], off, out_pin[oc:], stream)
                    oc += len(members)
                    ev = torch.cuda.Event(enable_timing=True)
                    ev.record(stream)
                    log.append((ev, members))
                    tok += k
                last_ev = log[-1][0]
            elif not queue and nxt < n and idle:
                time.sleep(max(0.0, min(arrivals[nxt] - now, 2e-4)))
        torch.cuda.synchronize()
        lat = np.empty(n)
        done = np.empty(n)
        for ev, members in log:
            t_done = ev0.elapsed_time(ev) / 1000.0
            done[members] = t_done
            lat[members] = t_done - arrivals[members]
        span = float(done.max() - arrivals.min())
        return {"completed_per_s": n / span, "p50_ms": 1000 * float(np.median(lat)),
                "p99_ms": 1000 * float(np.percentile(lat, 99)), "mean_ms": 1000 * float(lat.mean()),
                "max_ms": 1000 * float(lat.max()), "windows": windows, "batches": len(log)}

    zero = np.zeros(n)
    for _ in range(args.warmup):
        run(zero, "throughput")
    sat = run(zero, "throughput")
    sat_rate = sat["completed_per_s"]
    results = []
    for frac in (0.5, 0.9):
        arrivals = synth.make_arrivals(n, frac * sat_rate, w.seed)
        arrivals -= arrivals[0]
        for name in ("throughput", "latency"):
            r = run(arrivals, name)
            r.update({"rate_frac": frac, "rate_req_s": frac * sat_rate, "objective": name})
            results.append(r)
    head = next(r for r in results if r["rate_frac"] == 0.9 and r["objective"] == "latency")
    line = {"metric": "p99 latency at 0.9x of the saturation rate, Poisson arrivals (BERT-base, len 2-100)",
            "value": head["p99_ms"], "unit": "ms", "n_gpus": 1, "steps": 1, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "requests": n, "arrivals": "Poisson (exponential gaps)",
                       "policy": "when the GPU is idle, schedule every queued request with the DP and "
                                 "launch its batches (rm_score_host, pinned host ids)",
                       "scheduler_cost": f"T(b,L) = {SCHED_C0} + {SCHED_C1}*b*L"},
            "saturation": {"completed_per_s": sat_rate, "p50_ms": sat["p50_ms"], "p99_ms": sat["p99_ms"],
                           "batches": sat["batches"]},
            "serving": results,
            "context": {"turbotransformers_mean_latency_ms_at_402_req_s": 7.49}}
    print(json.dumps(line), flush=True)
    return 0


def ensemble_bench(args):
    """Batch-1 latency of one expert and of a K-expert ensemble with majority
    vote on one GPU (the experts run on their own streams at once), per
    input length, over 1000 requests after 50 warm-up requests.  Each request
    is timed from an idle GPU to its decision (CUDA events, synchronised per
    request), so host launch time counts."""
    import torch
    import classifier_scoring_b200 as rm
    from classifier_scoring_b200 import build as rmbuild
    from classifier_scoring_b200.ensemble import Ensemble

    rank, world, local = rank_env()
    if world > 1:
        raise SystemExit("--ensemble runs on one GPU")
    torch.cuda.set_device(local)
    rmbuild.build()
    w = synth.WORKLOADS[args.workload]
    s = w.shape
    K = args.ensemble
    lengths = list(w.fixed_lengths) or [int(w.len_lo), int(w.len_hi)]
    max_len = max(lengths)
    cfg = rm.RmConfig.make(arch=s.arch, n_layers=s.n_layers, hidden=s.hidden, n_heads=s.n_heads,
                           ffn=s.ffn, vocab=s.vocab, max_pos=s.max_pos, weight_dtype=s.weight_dtype,
                           gelu=s.gelu, ln_eps=s.ln_eps, max_batch_seqs=1, max_tokens=max_len,
                           max_len=max_len, sched_max_batch=1)
    experts = [rm.Scorer(cfg, synth.make_weights(s, w.seed + 1000 * k)) for k in range(K)]
    ens = Ensemble(experts)
    main = torch.cuda.Stream()
    scores = torch.zeros(K, 1, device="cuda")
    dec = torch.zeros(1, dtype=torch.int32, device="cuda")
    n_warm, n_req = 50, 1000
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def lat_of(fn):
        out = np.empty(n_req)
        for r in range(n_warm + n_req):
            torch.cuda.synchronize()
            a.record(main)
            fn()
            b.record(main)
            b.synchronize()
            if r >= n_warm:
                out[r - n_warm] = a.elapsed_time(b)
        return out

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    clocks = ClockSampler(gpu_index, clocks_log(args, "clocks_ensemble.csv"))
    time.sleep(0.3)
    l0 = sum(e.profile_read()["total_launches"] for e in experts)
    rows = []
    for L in lengths:
        ids = torch.from_numpy(synth.make_token_ids(L, s.vocab, w.seed + L)).cuda()
        off = np.array([0, L], dtype=np.int32)
        one = lat_of(lambda: experts[0].score(ids, off, scores[0], main))
        many = lat_of(lambda: ens.score_and_vote(ids, off, scores, dec, stream=main))
        # the same two calls captured once into CUDA graphs (rm_plan: kernels only)
        plans = ens.plan(off)
        plans[0].score(ids, scores[0], main)
        ens.score_and_vote(ids, off, scores, dec, stream=main, plans=plans)
        torch.cuda.synchronize()
        g_one, g_many = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_one, stream=main):
            plans[0].score(ids, scores[0], main)
        with torch.cuda.graph(g_many, stream=main):
            ens.score_and_vote(ids, off, scores, dec, stream=main, plans=plans)
        def replay_on_main(g):
            def fn():
                with torch.cuda.stream(main):       # a graph replays on the current stream
                    g.replay()
            return fn
        one_g = lat_of(replay_on_main(g_one))
        many_g = lat_of(replay_on_main(g_many))
        del g_one, g_many
        for p in plans:
            p.close()
        rows.append({"len": L, "one_expert_p50_ms": float(np.median(one)),
                     "one_expert_p99_ms": float(np.percentile(one, 99)),
                     "ensemble_p50_ms": float(np.median(many)),
                     "ensemble_p99_ms": float(np.percentile(many, 99)),
                     "graph_one_expert_p50_ms": float(np.median(one_g)),
                     "graph_one_expert_p99_ms": float(np.percentile(one_g, 99)),
                     "graph_ensemble_p50_ms": float(np.median(many_g)),
                     "graph_ensemble_p99_ms": float(np.percentile(many_g, 99))})
    clk = clocks.stop()
    launches = sum(e.profile_read()["total_launches"] for e in experts) - l0
    head = rows[len(rows) // 2]
    line = {"metric": f"batch-1 p50 latency of a {K}-expert ensemble with majority vote, one B200, "
                      f"CUDA-graph replay ({s.n_layers}-layer H{s.hidden} encoder, length {head['len']})",
            "value": head["graph_ensemble_p50_ms"], "unit": "ms", "n_gpus": 1, "steps": n_req,
            "warmup": n_warm, "ms_per_step": head["graph_ensemble_p50_ms"], "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "experts": K,
                       "weights": f"expert k: random N(0,0.02), seed {w.seed} + 1000k",
                       "vote": "majority of [score > 0], even split by the summed margins",
                       "timing": "per request from an idle GPU to the decision, CUDA events; "
                                 "eager launches and CUDA-graph replay of the same calls"},
            "latency": rows, "gpu_launches": int(launches), "clocks": clk}
    print(json.dumps(line), flush=True)
    for e in experts:
        e.close()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="bert-base-len2-100",
                    choices=list(synth.WORKLOADS) + list(synth.PREFIX_WORKLOADS))
    ap.add_argument("--profile-every", type=int, default=0,
                    help="diagnostic: CUDA events around the launches of every n-th call inside the "
                         "timed regions (0 = off; the kernel table always comes from a separate step)")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed regions of --steps steps each (median and 95%% interval reported)")
    ap.add_argument("--processes", type=int, default=5,
                    help="also repeat the measurement in this many independent processes in total "
                         "(this one included; 1 = none)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads (lengths 5-500, GPT-1.3B shape, TinyBERT batch 1)")
    ap.add_argument("--extra-steps", type=int, default=3, help="timed steps of each other workload")
    ap.add_argument("--extra-requests", type=int, default=200,
                    help="timed batch-1 requests per length of the TinyBERT workload")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cupti", action="store_true",
                    help="skip the CUPTI-timed step of the kernel table (for runs under ncu)")
    ap.add_argument("--clocks-dir", default=None,
                    help="also write the raw clock samples of the timed region as CSV here")
    ap.add_argument("--only", default="",
                    help="with --kernel-bench: comma-separated entries to run (e.g. softmax_len2_100)")
    ap.add_argument("--kernel-bench", action="store_true",
                    help="time the softmax and residual+LayerNorm kernels alone on GB-scale inputs")
    ap.add_argument("--fuse", type=int, default=8,
                    help="consecutive DP batches scored per rm_score call (executor batch fusion)")
    ap.add_argument("--lanes", type=int, default=2,
                    help="handles sharing the weights, one stream each, batches dealt round-robin")
    ap.add_argument("--ensemble", type=int, default=0,
                    help="batch-1 latency of one expert vs this many experts voting (one GPU)")
    ap.add_argument("--serve", action="store_true",
                    help="open-loop Poisson serving at 0.5x and 0.9x of the saturation rate, "
                         "throughput vs latency DP objective (p50/p99)")
    ap.add_argument("--batch-index", type=int, default=None,
                    help="score only this DP batch of the stream per step (small profiling case)")
    args = ap.parse_args()
    args.repeats = max(1, args.repeats)
    if args.warmup < 3 and args.impl == "b200":
        print("note: at least 3 warm-up steps are required; using 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)
    if args.kernel_bench:
        return kernel_bench(args)
    if args.workload in synth.PREFIX_WORKLOADS:
        return prefix_bench(args)
    if args.serve:
        return serve_bench(args)
    if args.ensemble > 0:
        return ensemble_bench(args)
    return b200_arm(args)


if __name__ == "__main__":
    sys.exit(main())
