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
KERNEL_NAMES = ("gemm", "attn_scores", "softmax", "attn_context", "layernorm", "embed", "head")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel (tcgen05 GEMM) from one ncu
# capture; valid only for the source it was taken on (sha256 prefix of
# gemm_tc.cu).  See profiles/gemm_bf16_tc_bert_base_T3264.txt.
GEMM_TRAFFIC = {"src_sha": None, "bytes_per_launch": None}


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
            self.f = open(out_path, "w") if out_path else subprocess.DEVNULL
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


def time_oracle(name: str, budget_s: float, min_requests: int = 4, start: int = 0):
    """Score requests of the workload's stream with the fp64 oracle, one by one,
    until budget_s has elapsed; returns (sequences/s, requests scored)."""
    from oracle import scorer
    w = synth.WORKLOADS[name]
    s = w.shape
    m = scorer.unpack_weights(synth.make_weights(s, w.seed), s.arch, s.n_layers, s.hidden,
                              s.n_heads, s.ffn, s.vocab, s.max_pos, s.weight_dtype, s.gelu, s.ln_eps)
    st = synth.make_stream(w)
    t0 = time.perf_counter()
    k = 0
    while True:
        i = (start + k) % len(st.lengths)
        scorer.score_one(m, st.ids[st.starts[i]:st.starts[i] + st.lengths[i]])
        k += 1
        el = time.perf_counter() - t0
        if (el >= budget_s and k >= min_requests) or k >= len(st.lengths):
            break
    return k / el, k, el


def reference_arm(args):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    name = args.workload
    w = synth.WORKLOADS[name]
    per_step = 8 if w.shape.hidden >= 768 else 64
    times, done = [], 0
    for it in range(args.warmup + args.steps):
        rate, k, el = time_oracle(name, 0.0, min_requests=per_step, start=it * per_step)
        if it >= args.warmup:
            times.append(el)
            done += k
    total = sum(times)
    value = done / total
    cores = oracle_threads()
    sample = (f"{per_step} requests per step from the seeded stream, scored one by one by the "
              f"fp64 numpy oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
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

    name = args.workload
    w = synth.WORKLOADS[name]
    s = w.shape
    flat = synth.make_weights(s, w.seed)
    wr = dataclasses.replace(w, seed=w.seed + 1000 * rank)       # each replica its own requests
    st = synth.make_stream(wr)
    n_req = len(st.lengths)
    max_len = min(s.max_pos, 1024, max(w.len_hi, int(st.lengths.max())))
    cfg = rm.RmConfig.make(arch=s.arch, n_layers=s.n_layers, hidden=s.hidden, n_heads=s.n_heads,
                           ffn=s.ffn, vocab=s.vocab, max_pos=s.max_pos, weight_dtype=s.weight_dtype,
                           gelu=s.gelu, ln_eps=s.ln_eps, max_batch_seqs=w.max_batch,
                           max_tokens=w.max_batch * max_len, max_len=max_len,
                           sched_max_batch=w.max_batch, sched_c0=SCHED_C0, sched_c1=SCHED_C1)
    sc = rm.Scorer(cfg, flat)
    del flat
    stream = torch.cuda.Stream()

    # the schedule is deterministic: pack the stream in batch order once, on the device
    batch = sc.schedule(st.lengths)
    nb = int(batch.max()) + 1
    groups = [np.nonzero(batch == b)[0] for b in range(nb)]
    order = np.concatenate(groups)
    packed_ids, _ = synth.pack(st, order)
    b_tok = np.zeros(nb + 1, dtype=np.int64)
    b_seq = np.zeros(nb + 1, dtype=np.int64)
    b_off = []
    for b, g in enumerate(groups):
        lens = st.lengths[g]
        b_off.append(synth.offsets_from_lengths(lens))
        b_tok[b + 1] = b_tok[b] + int(lens.sum())
        b_seq[b + 1] = b_seq[b] + len(g)
    ids_dev = torch.from_numpy(packed_ids).cuda()
    out_dev = torch.zeros(n_req, dtype=torch.float32, device="cuda")
    ev_batch = [torch.cuda.Event(enable_timing=True) for _ in range(nb)]

    def step(record=False):
        bt = sc.schedule(st.lengths)                          # S0 on the host
        if record and not np.array_equal(bt, batch):
            raise RuntimeError("schedule changed between steps")
        for b in range(nb):
            sc.score(ids_dev[b_tok[b]:], b_off[b], out_dev[b_seq[b]:], stream)
            if record:
                ev_batch[b].record(stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    # warm-up (plans every length bucket, compiles nothing: the kernels are prebuilt)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    sc.profile(args.profile_every)
    launches0 = sc.profile_read()["total_launches"]
    sc.profile(args.profile_every)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    out_dir = os.path.join(ROOT, "gpurun_out")
    clocks = ClockSampler(gpu_index, os.path.join(out_dir, f"clocks_rank{rank}.csv")
                          if os.path.isdir(out_dir) else None)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    t_start.record(stream)
    for k in range(args.steps):
        step(record=(k == args.steps - 1))
    t_end.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier()
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    prof = sc.profile_read()
    launches = prof["total_launches"] - launches0
    sc.profile(0)
    # latency in the last timed step: every request is queued at the step's start
    # and completes with its batch; the step's start is taken as the last
    # batch's completion minus the mean step time
    per_batch = np.array([ev_batch[0].elapsed_time(e) for e in ev_batch])
    first_done = elapsed_ms / args.steps - per_batch[-1]
    lat = np.empty(n_req)
    for b in range(nb):
        lat[b_seq[b]:b_seq[b + 1]] = per_batch[b] + first_done
    p50 = float(np.median(lat))
    p99 = float(np.percentile(lat, 99))

    # ---- end to end through rm_score_host (pinned host buffers) ----
    ids_pin = torch.empty(int(b_tok[-1]), dtype=torch.int32).pin_memory()
    out_pin = torch.empty(n_req, dtype=torch.float32).pin_memory()
    ids_np = ids_pin.numpy()
    host_ids = st.ids

    def e2e_step():
        bt = sc.schedule(st.lengths)
        pos = 0
        for b in range(nb):                                   # S1: host gather into pinned memory
            g = groups[b]
            for i in g:
                L = int(st.lengths[i])
                ids_np[pos:pos + L] = host_ids[st.starts[i]:st.starts[i] + L]
                pos += L
        del bt
        for b in range(nb):
            sc.score_host(ids_pin[b_tok[b]:], b_off[b], out_pin[b_seq[b]:], stream)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ew0 = time.perf_counter()
    e0.record(stream)
    e_steps = max(1, args.steps)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e_wall = time.perf_counter() - ew0
    barrier()
    e_ms = max(e0.elapsed_time(e1), 1000 * e_wall)
    if not np.array_equal(out_pin.numpy(), out_dev.cpu().numpy()):
        raise RuntimeError("rm_score_host and rm_score disagree")
    meta_bytes = sum(4 * (len(o)) * 2 + 8 * len(o) for o in b_off)
    h2d = 4 * int(b_tok[-1]) + meta_bytes
    d2h = 4 * n_req

    # ---- reduce over ranks ----
    vals = np.array([elapsed_ms, e_ms], dtype=np.float64)
    if dist is not None:
        import torch.distributed as tdist
        t = torch.tensor(vals, device="cuda")
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        vals = t.cpu().numpy()
    max_ms, max_e_ms = float(vals[0]), float(vals[1])
    total_seqs = world * n_req * args.steps
    value = total_seqs / (max_ms / 1000.0)
    e2e_value = world * n_req * e_steps / (max_e_ms / 1000.0)

    pk, pk_kind = peaks()
    g = prof["gemm"]
    gemm_tflops = g["flops"] / (g["ms"] * 1e-3) / 1e12 if g["ms"] > 0 else None
    src = open(os.path.join(ROOT, "classifier_scoring_b200", "csrc", "gemm_tc.cu"), "rb").read()
    sha = hashlib.sha256(src).hexdigest()[:16]
    traffic = GEMM_TRAFFIC["bytes_per_launch"] if GEMM_TRAFFIC["src_sha"] == sha else None
    roofline = {"kernel": "gemm_bf16_tc_kernel (QKV, output and FFN projections)",
                "bound": "tensor", "achieved": gemm_tflops, "peak": pk["bf16_tflops_sustained"],
                "unit": "TFLOP/s",
                "frac": (gemm_tflops / pk["bf16_tflops_sustained"]) if gemm_tflops else None,
                "peak_source": f"bf16_tflops_sustained of {pk_kind} (kernel timed inside a long step)",
                "traffic": traffic,
                "launches_timed": g["launches"], "avg_launch_us": 1000 * g["ms"] / max(1, g["launches"])}
    kernels = {}
    for kname in KERNEL_NAMES:
        d = prof[kname]
        if d["launches"] == 0:
            continue
        e = {"launches_timed": d["launches"], "avg_us": 1000 * d["ms"] / d["launches"],
             "share_of_timed": d["ms"] / max(1e-9, sum(prof[x]["ms"] for x in KERNEL_NAMES))}
        if d["flops"] and kname in ("gemm", "attn_scores", "attn_context"):
            e["tflops"] = d["flops"] / (d["ms"] * 1e-3) / 1e12
        if d["bytes"]:
            e["gbs"] = d["bytes"] / (d["ms"] * 1e-3) / 1e9
            e["hbm_frac_of_measured"] = e["gbs"] / pk["hbm_gbs"]
        kernels[kname] = e

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(name),
        "p50_latency_ms": p50, "p99_latency_ms": p99, "batches_per_step": nb,
        "tokens_per_step": int(b_tok[-1]),
        "roofline": roofline,
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "rm_score_host, pinned host ids/scores"},
        "gpu_launches": int(launches),
        "clocks": clk,
        "wall_s_timed": wall,
        "context": {"turbotransformers_req_s_len2_100": 402, "hardware": "not named on the page"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, k, el = time_oracle(name, args.cpu_budget)
        result["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": oracle_threads(),
                                  "kind": "oracle",
                                  "sample": f"first {k} requests of the seeded stream scored one by "
                                            f"one by the fp64 numpy oracle ({el:.1f} s)"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    sc.close()
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="bert-base-len2-100", choices=list(synth.WORKLOADS))
    ap.add_argument("--profile-every", type=int, default=8,
                    help="time the kernels of every n-th batch with CUDA events (0 = off)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "b200":
        print("note: at least 3 warm-up steps are required; using 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)
    return b200_arm(args)


if __name__ == "__main__":
    sys.exit(main())
