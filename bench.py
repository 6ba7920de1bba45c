"""Benchmark: batched speculative-sampling verification on B200.

Default workload (one step = one sv_verify_chain call): Qwen-vocabulary chain
verification, B=32 requests x k=3 drafts, V=151936, bf16 logits, T=0.7.
Metric: verified rows/s (B*(k+1) target rows per step), with the achieved HBM
bandwidth of the verification kernel against the measured copy bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the float64 CPU oracle, same metric

Under torchrun every rank verifies its own batch (weak scaling, no collective
on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speculative_decoding_verification_94_b200 import inputs  # noqa: E402

METRIC = "verified rows/s"
GRAD_METRIC = "kd-gradient draft rows/s"


def metric_of(kind):
    return GRAD_METRIC if kind == "grad" else METRIC
UNIT = "rows/s"
L2_BYTES = 126 * 1024 * 1024
# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, from one capture of the current build on this workload (keyed by
# workload, B, k), with the profiles/ summary that holds it; absent for a
# workload whose kernel changed since its last capture.
NCU_TRAFFIC: dict = {
    ("qwen_chain_verify", 32, 3): (68115200 + 218112,
                                   "profiles/stream_kernel_qwen_chain_B32_k3.md: stream_kernel, "
                                   "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch "
                                   "at commit d7ff710"),
}
# Kernel names of a call's launches, by the library's launch kinds (stream
# pass, finishing kernel, persistent chain kernel).
FINISH_NAME = {"chain": "chain_sample_finish", "kd": "chain_sample_finish",
               "ragged": "chain_sample_finish", "tree_sample": "tree_sample_kernel",
               "tree": "tree_finish", "grad": "kd_grad_kernel"}


def kernel_names(kind):
    return {"stream": "stream_kernel", "finish": FINISH_NAME.get(kind, "finish"),
            "chain": "chain_kernel"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="qwen_chain",
                    choices=["qwen_chain", "kd", "kd_grad", "tree", "tree_sample", "ragged",
                             "tiny", "sweep", "sched_table"])
    ap.add_argument("--table-out", default=None,
                    help="sched_table: write the measured verify-cost table (JSON) here")
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--sigma", type=float, default=1.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--knob", action="append", default=[], metavar="NAME=VALUE",
                    help="library setting for the run (sv_set_knob), e.g. persistent=1")
    ap.add_argument("--min-warm-s", type=float, default=0.5,
                    help="seconds of load before timing (0 for short profiling runs)")
    return ap.parse_args()


def load_peaks():
    """The measured HBM copy bandwidth (GB/s) when the peaks file is present
    (key "hbm_gbs", else the first numeric entry whose key names HBM), else
    the 6650 GB/s fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        if "hbm_gbs" in p:
            return float(p["hbm_gbs"]), "measured"
        for key, v in p.items():
            if "hbm" in key.lower() and isinstance(v, (int, float)):
                return float(v), "measured"
    except Exception:
        pass
    return 6650.0, "fallback"


def rank_seed(rank: int) -> int:
    """Each replica verifies its own batch (weak scaling)."""
    return 1000 * rank


def reduce_max(values, dist, device):
    """Element-wise maximum over ranks of a list of floats (timing only; no
    data-path collective).  Every rank must call it in the same order."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_value(rows_per_rank: int, world: int, steps: int, ms_total: float) -> float:
    """Whole-job rows/s: the rows every rank verified over the slowest rank's time."""
    return rows_per_rank * world * steps / (ms_total * 1e-3)


def make_workload(a, rank):
    seed = rank_seed(rank)
    if a.workload == "qwen_chain":
        B = a.B or 32
        k = a.k or 3
        x = inputs.qwen_chain(B=B, k=k, sigma_d=1.0, seed=seed)
        return "chain", x, dict(workload="qwen_chain_verify", B=B, k=k, V=x.V, input_dtype="bf16",
                                temperature=0.7, draft_sigma=1.0)
    if a.workload == "sweep":
        B = a.B or 8
        k = a.k or 3
        x = inputs.qwen_chain(B=B, k=k, sigma_d=a.sigma, seed=seed)
        return "chain", x, dict(workload="active_batch_sweep_point", B=B, k=k, V=x.V,
                                input_dtype="bf16", temperature=0.7, draft_sigma=a.sigma)
    if a.workload == "kd":
        B = a.B or 256
        k = a.k or 3
        x = inputs.kd_chain(B=B, k=k, seed=seed)
        return "kd", x, dict(workload="fused_verify_kd", B=B, k=k, V=x.V, input_dtype="bf16",
                             temperature=1.0, K=32, weighting="group_norm", group=16)
    if a.workload == "kd_grad":
        B = a.B or 256
        k = a.k or 3
        x = inputs.kd_chain(B=B, k=k, seed=seed)
        return "grad", x, dict(workload="kd_gradient", B=B, k=k, V=x.V, input_dtype="bf16",
                               temperature=1.0, K=32, weighting="group_norm", group=16,
                               output="fp32 [B, k, V]")
    if a.workload == "tiny":
        x = inputs.tiny_chain(seed=seed)
        return "chain", x, dict(workload="tiny_chain_verify", B=4, k=3, V=1024,
                                input_dtype="f32", temperature=1.0)
    if a.workload == "tree":
        t = inputs.make_tree(B=a.B or 8, seed=seed)
        return "tree", t, dict(workload="greedy_tree_verify", B=t.logits.shape[0],
                               n=t.logits.shape[1], V=t.logits.shape[2], depth=t.max_depth,
                               branching=8, input_dtype="bf16", temperature=0.0)
    if a.workload == "ragged":
        B = a.B or 32
        k = a.k or 3
        x = inputs.qwen_chain(B=B, k=k, sigma_d=1.0, seed=seed)
        x.meta["draft_len"], x.meta["active"] = inputs.ragged_lengths(B, k, seed=seed)
        return "ragged", x, dict(workload="ragged_chain_verify", B=B, k=k, V=x.V,
                                 input_dtype="bf16", temperature=0.7, draft_sigma=1.0,
                                 draft_len="uniform on 0..k", idle_fraction=0.15)
    if a.workload == "tree_sample":
        t = inputs.make_tree_sample(B=a.B or 8, seed=seed)
        B, n, V = t.target.shape
        return "tree_sample", t, dict(workload="sampling_tree_verify", B=B, n=n, V=V,
                                      depth=t.max_depth, branching=8, input_dtype="bf16",
                                      temperature=0.7, draft_sigma=1.0)
    raise ValueError(a.workload)


def needed_bytes(kind, x, accepted_len):
    """Bytes verification must read: for each request, target and draft rows
    0..n (n = accepted drafts; draft rows stop at k-1) and the bonus target
    row when every draft was accepted, plus the small inputs and outputs.
    Rows after the first rejection are not part of the computation."""
    if kind == "tree":
        return rows_and_bytes(kind, x)[1]
    if kind == "tree_sample":
        # the target/draft row pairs of the visited nodes (root .. last accepted)
        B, n, V = x.target.shape
        visits = int(np.sum(np.asarray(accepted_len, np.int64) + 1))
        return (visits * V * (x.target.element_size() + x.draft.element_size()) + B * n * 12 +
                B * 4 + 2 * B * (x.max_depth + 1) * 4)
    if kind == "ragged":
        # per active request: pairs 0..min(n, k_b - 1) and the bonus row k_b
        # when n = k_b; idle requests read nothing
        B, P, V = x.target.shape
        te, de = x.target.element_size(), x.draft.element_size()
        kb = x.meta["draft_len"].numpy().astype(np.int64)
        on = x.meta["active"].numpy() != 0
        n = np.asarray(accepted_len, np.int64)
        pairs = np.where(on, np.minimum(n, kb - 1) + 1, 0)
        bonus = on & (n == kb)
        return (int(np.sum(pairs)) * V * (te + de) + int(np.sum(bonus)) * V * te +
                _ragged_io(x))
    if kind == "grad":
        # the draft rows whose gradient is not zero are read once; every row of
        # the fp32 gradient is written; plus the top-K buffers and small inputs
        B, k, V = x.draft.shape
        n = np.asarray(accepted_len, np.int64)
        return int(np.sum(n) * V * x.draft.element_size() + B * k * V * 4 +
                   B * (k + 1) * 32 * 8 + B * 8)
    B, P, V = x.target.shape
    k = P - 1
    te, de = x.target.element_size(), x.draft.element_size()
    n = np.asarray(accepted_len, np.int64)
    pairs = np.minimum(n, k - 1) + 1
    by = int(np.sum(pairs) * V * (te + de) + np.sum(n == k) * V * te)
    by += B * k * 4 + B * P * 4 + B * 4 + B * P * 4
    if kind == "kd":
        by += int(np.sum(n + 1)) * (32 * 8 + 4) + B * k * 4 + B * 4 * 2 + 4
    return by


def _ragged_io(x):
    B, P = x.target.shape[:2]
    return (B * (P - 1) * 4 + B * P * 4 + 2 * B * 4) + B * 4 + B * P * 4


def rows_and_bytes(kind, x):
    """Verified rows per step and the bytes of reading every logit once + I/O."""
    if kind == "ragged":  # the rows the active requests use
        V = x.target.shape[2]
        te, de = x.target.element_size(), x.draft.element_size()
        kb = x.meta["draft_len"].numpy().astype(np.int64)
        on = x.meta["active"].numpy() != 0
        rows = int(np.sum((kb + 1)[on]))
        return rows, (rows * V * te + int(np.sum(kb[on])) * V * de) + _ragged_io(x)
    if kind == "tree":
        B, n, V = x.logits.shape
        es = x.logits.element_size()
        return B * n, B * n * V * es + B * n * 8 + B * 4 + 2 * B * (x.max_depth + 1) * 4
    if kind == "tree_sample":
        B, n, V = x.target.shape
        return B * n, (B * n * V * (x.target.element_size() + x.draft.element_size()) +
                       B * n * 12 + B * 4 + 2 * B * (x.max_depth + 1) * 4)
    if kind == "grad":  # draft rows per step; every draft row read twice, gradient written
        B, k, V = x.draft.shape
        return B * k, B * k * V * (2 * x.draft.element_size() + 4) + B * (k + 1) * 32 * 8 + B * 8
    B, P, V = x.target.shape
    k = P - 1
    te, de = x.target.element_size(), x.draft.element_size()
    by = B * P * V * te + B * k * V * de + B * k * 4 + B * P * 4 + B * 4 + B * P * 4
    if kind == "kd":
        K = 32
        by += B * P * K * 8 + B * P * 4 + B * k * 4 + B * 4 * 2 + 4
    return B * P, by


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [r for (t, r) in self.rows if t0 - 0.15 <= t <= t1 + 0.15] or [r for _, r in self.rows]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if len(r) > 5 + i and r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def oracle_step_fn(kind, x, threads=0):
    from oracle import oracle as O  # CPU baseline only
    if kind == "tree":
        return lambda: O.tree_greedy(x.logits, x.node_tokens, x.parents, x.max_depth,
                                     threads=threads)
    if kind == "tree_sample":
        return lambda: O.tree_sample(x.target, x.draft, x.node_tokens, x.parents, x.uniforms,
                                     x.temperature, x.max_depth, threads=threads)
    if kind == "ragged":
        return lambda: O.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms,
                                      x.temperature, threads=threads,
                                      draft_len=x.meta["draft_len"], active=x.meta["active"])
    if kind == "kd":
        return lambda: O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward,
                                   x.temperature, 32, mode=O.W_GROUP_NORM, group=16,
                                   threads=threads)
    if kind == "grad":
        ref = O.verify_kd(x.target, x.draft, x.draft_tokens, x.uniforms, x.reward, x.temperature,
                          32, mode=O.W_GROUP_NORM, group=16, threads=threads)
        lp, ix, acc = ref["topk_logp"], ref["topk_idx"], ref["accepted_len"]
        r = x.reward.numpy().astype(np.float64)
        return lambda: O.kd_grad(lp, ix, x.draft, acc, r, x.temperature, mode=O.W_GROUP_NORM,
                                 group=16, threads=threads)
    return lambda: O.verify_chain(x.target, x.draft, x.draft_tokens, x.uniforms, x.temperature,
                                  threads=threads)


def cpu_baseline(kind, x, rows, min_seconds=10.0):
    """The oracle as it stands on this host's cores, on a bounded sample."""
    from oracle import oracle as O
    fn = oracle_step_fn(kind, x)
    fn()  # builds / warms up
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds or n >= 1000:
            break
    cores = O.max_threads()
    out = {"value": rows * n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"{n} full batches of the same workload ({rows} rows each) in {dt:.1f} s"}
    # the same oracle on one thread (run last: it leaves the oracle at one thread)
    fn1 = oracle_step_fn(kind, x, threads=1)
    n1, t1 = 0, time.perf_counter()
    while True:
        fn1()
        n1 += 1
        dt1 = time.perf_counter() - t1
        if dt1 >= min_seconds / 2 or n1 >= 1000:
            break
    out["single_thread"] = {"value": rows * n1 / dt1, "unit": UNIT, "cores": 1,
                            "sample": f"{n1} full batches in {dt1:.1f} s"}
    return out


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    kind, x, cfg = make_workload(a, 0)
    rows, _ = rows_and_bytes(kind, x)
    from oracle import oracle as O
    fn = oracle_step_fn(kind, x)
    for _ in range(a.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        fn()
    dt = time.perf_counter() - t0
    value = rows * a.steps / dt
    line = {"impl": "reference", "metric": metric_of(kind), "value": value, "unit": UNIT,
            "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * dt / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(cfg, parallelism=f"dp{a.gpus}" if a.gpus > 1 else "single"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": O.max_threads(),
                             "kind": "oracle",
                             "sample": f"{a.steps} timed full batches ({rows} rows each)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SCHED_KS = (1, 3, 5, 7)
SCHED_BATCHES = (1, 2, 4, 8, 16, 32)
SCHED_SEEDS = 6


def dominant_kernel(kind, x, algo_bytes, kern):
    """The kernel that moves most of the call's algorithmic bytes, and those
    bytes: the streaming pass of a chain or greedy tree (every logit once;
    the finisher re-reads one row pair per request, the tree walk only
    records), the one kernel of a sampling tree or of a persistent chain call,
    and for the KD gradient the gradient kernel (the draft rows once more and
    the fp32 gradient; the statistics pass before it reads the draft rows)."""
    if "chain_kernel" in kern:
        return "chain_kernel", algo_bytes
    if kind == "tree_sample":
        return "tree_sample_kernel", algo_bytes
    if kind == "grad":
        B, k, V = x.draft.shape
        return "kd_grad_kernel", algo_bytes - B * k * V * x.draft.element_size()
    return "stream_kernel", algo_bytes


def kernel_times(step, steps, dev, kind):
    """Mean device time of each kernel of a call, from the library's kernel
    marks: `steps` calls captured in a CUDA graph with the marks on, replayed
    once, every launch's events read back."""
    from speculative_decoding_verification_94_b200 import sv
    with sv.knobs(kernel_marks=1):  # one marked call outside capture creates the events
        step(0)
    torch.cuda.synchronize(dev)
    sv.sv_kernel_times()  # drop its marks
    g = torch.cuda.CUDAGraph()
    with sv.knobs(kernel_marks=1):
        with torch.cuda.graph(g):
            for i in range(steps):
                step(i)
    g.replay()  # the captured event nodes are recorded at replay
    torch.cuda.synchronize(dev)
    marks = sv.sv_kernel_times()
    del g
    names = kernel_names(kind)
    out = {}
    for tag, us in marks:
        n = names.get(tag, tag)
        out.setdefault(n, []).append(us)
    return {n: {"us_per_launch": float(np.mean(v)), "launches_per_step": len(v) / steps}
            for n, v in out.items()}


def graph_time_us(step, steps, dev):
    """Mean device time of one call: `steps` calls captured in a CUDA graph,
    replayed once untimed and once between CUDA events."""
    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            step(i)
    g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s = torch.cuda.current_stream(dev)
    e0.record(s)
    g.replay()
    e1.record(s)
    torch.cuda.synchronize(dev)
    return 1e3 * e0.elapsed_time(e1) / steps


def run_sched_table(a):
    """The measured verify-cost table of the adaptive scheduler's lookup: the
    device time of one verification call for k in SCHED_KS drafts and for
    plain decoding (one token sampled from the target row: the ragged call
    with every draft count 0), at active batches SCHED_BATCHES, V=151936
    bf16, T=0.7, draft noise sigma (default 1.0).  Throughput of a
    configuration = emitted tokens per second of verification, B * mean
    (accepted + 1) / call time (B / call time for plain decoding), the mean
    taken over SCHED_SEEDS batches of the largest size.  Verify
    kernels only: no model forward is timed."""
    from speculative_decoding_verification_94_b200 import sv
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    sv.lib()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    Bmax = max(SCHED_BATCHES)
    rows, table_us, tokens = [], {}, {}
    for k in (0,) + SCHED_KS:
        x = inputs.qwen_chain(B=Bmax, k=max(k, 1), sigma_d=a.sigma, seed=0)
        # tokens emitted per request: a property of the draft/target pair,
        # not of the batch, so estimated once per configuration over
        # SCHED_SEEDS independent batches of Bmax requests
        emitted_k = 1.0
        if k:
            acc = []
            for seed in range(SCHED_SEEDS):
                y = x if seed == 0 else inputs.qwen_chain(B=Bmax, k=k, sigma_d=a.sigma, seed=seed)
                r = sv.sv_verify_chain(y.target.to(dev), y.draft.to(dev), y.draft_tokens.to(dev),
                                       y.uniforms.to(dev), y.temperature, device_status=status)
                acc.append(r["accepted_len"].cpu().numpy().astype(np.float64))
                del y, r
            emitted_k = float(np.mean(np.concatenate(acc) + 1.0))
        for B in SCHED_BATCHES:
            per = x.target[:B].numel() * 2 + (x.draft[:B].numel() * 2 if k else 0)
            ncopy = max(2, math.ceil(2.2 * L2_BYTES / per))
            sets = [dict(t=x.target[:B].contiguous().to(dev), d=x.draft[:B].contiguous().to(dev),
                         tok=x.draft_tokens[:B].contiguous().to(dev),
                         u=x.uniforms[:B].contiguous().to(dev)) for _ in range(ncopy)]
            zeros = torch.zeros(B, dtype=torch.int32, device=dev)
            out = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty(B, max(k, 1) + 1, dtype=torch.int32, device=dev))

            def step(i, s=None):
                s = s or sets[i % ncopy]
                if k == 0:
                    sv.sv_verify_chain_ragged(s["t"], s["d"], s["tok"], s["u"], x.temperature,
                                              draft_len=zeros, out=out, device_status=status)
                else:
                    sv.sv_verify_chain(s["t"], s["d"], s["tok"], s["u"], x.temperature, out=out,
                                       device_status=status)

            us = graph_time_us(step, a.steps, dev)
            emitted = emitted_k
            table_us[(k, B)] = us
            tokens[(k, B)] = emitted
            rows.append(dict(k=k, B=B, call_us=us, mean_emitted=emitted,
                             tokens_per_s=B * emitted / (us * 1e-6)))
            print(json.dumps(rows[-1]), flush=True)
            del sets
    st = int(status.item())
    assert st & sv.SV_DEV_ERROR_MASK == 0, f"device status {st:#x}"
    cfgs = ["plain"] + [f"k={k}" for k in SCHED_KS]
    thr = [[r["tokens_per_s"] for r in rows if r["k"] == k] for k in (0,) + SCHED_KS]
    table = {"what": "verify-kernel cost table: emitted tokens per second of one verification "
                     "call, per configuration (rows) and active batch (columns)",
             "configs": cfgs, "nonspec": 0, "batches": list(SCHED_BATCHES),
             "throughput_tokens_per_s": thr,
             "call_us": [[table_us[(k, B)] for B in SCHED_BATCHES] for k in (0,) + SCHED_KS],
             "mean_emitted": [[tokens[(k, B)] for B in SCHED_BATCHES] for k in (0,) + SCHED_KS],
             "workload": dict(V=inputs.V_QWEN, input_dtype="bf16", temperature=0.7,
                              draft_sigma=a.sigma, seed=0),
             "command": f"python bench.py --workload sched_table --steps {a.steps} "
                        f"--sigma {a.sigma} --table-out <path>"}
    if a.table_out:
        with open(a.table_out, "w") as f:
            json.dump(table, f, indent=1)
            f.write("\n")
    print(json.dumps({"metric": "verify-cost table", "table": table}), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        return run_reference(a)
    if a.workload == "sched_table":
        return run_sched_table(a)
    from speculative_decoding_verification_94_b200 import sv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    sv.lib()
    assert a.warmup >= 3, "at least 3 warm-up steps"
    knobs = {}
    for kv in a.knob:
        name, value = kv.split("=", 1)
        sv.sv_set_knob(getattr(sv, "SV_KNOB_" + name.upper()), int(value))
        knobs[name] = int(value)

    kind, x, cfg = make_workload(a, rank)
    if knobs:
        cfg = dict(cfg, knobs=knobs)
    rows, algo_bytes = rows_and_bytes(kind, x)
    # input copies rotated so that the set exceeds 2x L2: every step reads HBM
    ncopy = max(2, math.ceil(2.2 * L2_BYTES / algo_bytes))
    stream = torch.cuda.current_stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if kind == "tree":
        sets = [dict(logits=x.logits.to(dev), tok=x.node_tokens.to(dev), par=x.parents.to(dev))
                for _ in range(ncopy)]
        outs = dict(accepted_len=torch.empty(x.logits.shape[0], dtype=torch.int32, device=dev),
                    out_tokens=torch.empty(x.logits.shape[0], x.max_depth + 1,
                                           dtype=torch.int32, device=dev),
                    accepted_nodes=torch.empty(x.logits.shape[0], x.max_depth + 1,
                                               dtype=torch.int32, device=dev))

        def step(i, d=None):
            s = d or sets[i % ncopy]
            sv.sv_verify_tree_greedy(s["logits"], s["tok"], s["par"], x.max_depth, out=outs,
                                     device_status=status)
    elif kind == "tree_sample":
        sets = [dict(t=x.target.to(dev), d=x.draft.to(dev), tok=x.node_tokens.to(dev),
                     par=x.parents.to(dev), u=x.uniforms.to(dev)) for _ in range(ncopy)]
        B = x.target.shape[0]
        outs = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=dev),
                    out_tokens=torch.empty(B, x.max_depth + 1, dtype=torch.int32, device=dev),
                    accepted_nodes=torch.empty(B, x.max_depth + 1, dtype=torch.int32,
                                               device=dev))

        def step(i, d=None):
            s = d or sets[i % ncopy]
            sv.sv_verify_tree_sample(s["t"], s["d"], s["tok"], s["par"], s["u"], x.temperature,
                                     x.max_depth, out=outs, device_status=status)
    elif kind == "ragged":
        sets = [dict(t=x.target.to(dev), d=x.draft.to(dev), tok=x.draft_tokens.to(dev),
                     u=x.uniforms.to(dev), kl=x.meta["draft_len"].to(dev),
                     act=x.meta["active"].to(dev)) for _ in range(ncopy)]
        B, P = x.target.shape[0], x.target.shape[1]
        outs = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=dev),
                    out_tokens=torch.empty(B, P, dtype=torch.int32, device=dev))

        def step(i, d=None):
            s = d or sets[i % ncopy]
            sv.sv_verify_chain_ragged(s["t"], s["d"], s["tok"], s["u"], x.temperature,
                                      draft_len=s["kl"], active=s["act"], out=outs,
                                      device_status=status)
    elif kind == "grad":
        B, k, V = x.draft.shape
        sets = [dict(d=x.draft.to(dev)) for _ in range(ncopy)]
        # the top-K buffers and accepted lengths come from one fused verification
        pre = sv.sv_verify_chain(x.target.to(dev), sets[0]["d"], x.draft_tokens.to(dev),
                                 x.uniforms.to(dev), x.temperature,
                                 kd=dict(K=32, reward=x.reward.to(dev), wmode="group_norm",
                                         group=16))
        gin = dict(lp=pre["topk_logp"], ix=pre["topk_idx"], r=x.reward.to(dev))
        outs = dict(grad=torch.empty(B, k, V, device=dev), accepted_len=pre["accepted_len"])
        torch.cuda.synchronize(dev)

        def step(i, d=None):
            s = d or sets[i % ncopy]
            sv.sv_kd_grad(gin["lp"], gin["ix"], s["d"], outs["accepted_len"], gin["r"],
                          x.temperature, wmode="group_norm", group=16, out=outs["grad"],
                          device_status=status)
    else:
        sets = [dict(t=x.target.to(dev), d=x.draft.to(dev), tok=x.draft_tokens.to(dev),
                     u=x.uniforms.to(dev), r=x.reward.to(dev)) for _ in range(ncopy)]
        kdcfg = None
        if kind == "kd":
            kdcfg = dict(K=32, wmode="group_norm", group=16)
        B, P = x.target.shape[0], x.target.shape[1]
        outs = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=dev),
                    out_tokens=torch.empty(B, P, dtype=torch.int32, device=dev))
        if kdcfg:
            outs.update(topk_logp=torch.empty(B, P, 32, device=dev),
                        topk_idx=torch.empty(B, P, 32, dtype=torch.int32, device=dev),
                        lse=torch.empty(B, P, device=dev), kl=torch.empty(B, P - 1, device=dev),
                        loss=torch.empty(B, device=dev), total=torch.empty(1, device=dev))

        def step(i, d=None):
            s = d or sets[i % ncopy]
            kd = None if kdcfg is None else dict(kdcfg, reward=s["r"])
            sv.sv_verify_chain(s["t"], s["d"], s["tok"], s["u"], x.temperature, kd=kd, out=outs,
                               device_status=status)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    # warm-up: at least W steps and at least ~0.5 s of load before timing
    for i in range(a.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    t_end = time.time() + a.min_warm_s
    i = a.warmup
    while time.time() < t_end:
        for _ in range(50):
            step(i)
            i += 1
        torch.cuda.synchronize(dev)

    # The K timed steps are captured once in a CUDA graph (host launch cost
    # of a Python call exceeds the kernel time) and replayed once untimed,
    # then once inside the timed region.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for s_ in range(a.steps):
            step(s_)
    graph.replay()
    torch.cuda.synchronize(dev)
    gstream = torch.cuda.current_stream(dev)
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    start.record(gstream)
    graph.replay()
    end.record(gstream)
    torch.cuda.synchronize(dev)
    tw1 = time.time()
    barrier()
    ms_total = start.elapsed_time(end)
    ms_launch = ms_total / a.steps  # one verification call (stream + finish kernels) per step
    clk = clocks.stop(tw0, tw1)
    ms_total, ms_launch = reduce_max([ms_total, ms_launch], dist, dev)
    st = int(status.item())
    assert st & sv.SV_DEV_ERROR_MASK == 0, f"device status {st:#x}"

    # Per-kernel device times: the same K calls captured again with the
    # library's kernel marks on (an event recorded before and after every
    # launch, on the launching stream) and replayed once.  The marks put an
    # event between the launches, so the sum can exceed the unmarked call.
    kern = kernel_times(step, min(a.steps, 500), dev, kind)
    dom, dom_bytes = dominant_kernel(kind, x, algo_bytes, kern)
    dom_us = kern[dom]["us_per_launch"]
    (dom_us,) = reduce_max([dom_us], dist, dev)

    peak, peak_kind = load_peaks()
    need_bytes = needed_bytes(kind, x, outs["accepted_len"].cpu().numpy())
    # the dominant kernel's share of the algorithmic bytes over its own time
    achieved = dom_bytes / (dom_us * 1e-6) / 1e9
    call_gbs = algo_bytes / (ms_launch * 1e-3) / 1e9
    value = job_value(rows, world, a.steps, ms_total)

    # end to end through the public call: pinned host inputs -> device, verify,
    # results -> pinned host, all inside the timed region.
    e2e = None
    if not a.no_e2e:
        if kind == "tree":
            host = dict(logits=x.logits.pin_memory(), tok=x.node_tokens.pin_memory(),
                        par=x.parents.pin_memory())
        elif kind == "tree_sample":
            host = dict(t=x.target.pin_memory(), d=x.draft.pin_memory(),
                        tok=x.node_tokens.pin_memory(), par=x.parents.pin_memory(),
                        u=x.uniforms.pin_memory())
        elif kind == "ragged":
            host = dict(t=x.target.pin_memory(), d=x.draft.pin_memory(),
                        tok=x.draft_tokens.pin_memory(), u=x.uniforms.pin_memory(),
                        kl=x.meta["draft_len"].pin_memory(), act=x.meta["active"].pin_memory())
        elif kind == "grad":
            host = dict(d=x.draft.pin_memory())
        else:
            host = dict(t=x.target.pin_memory(), d=x.draft.pin_memory(),
                        tok=x.draft_tokens.pin_memory(), u=x.uniforms.pin_memory(),
                        r=x.reward.pin_memory())
        dsts = sets[0]
        res_h = {k2: torch.empty(v.shape, dtype=v.dtype).pin_memory()
                 for k2, v in outs.items()
                 if k2 in (("grad",) if kind == "grad" else ("accepted_len", "out_tokens", "total"))}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(v.numel() * v.element_size() for v in res_h.values())
        n_e2e = max(3, min(a.steps, 50))

        def e2e_step():
            for k2, v in host.items():
                dsts[k2].copy_(v, non_blocking=True)
            step(0, dsts)
            for k2, v in res_h.items():
                v.copy_(outs[k2], non_blocking=True)

        for _ in range(3):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = e0.elapsed_time(e1)
        (ms_e2e,) = reduce_max([ms_e2e], dist, dev)
        e2e = {"value": job_value(rows, world, n_e2e, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e}

    cpu = None
    if rank == 0 and not a.no_cpu:
        cpu = cpu_baseline(kind, x, rows)

    if rank == 0:
        traffic = NCU_TRAFFIC.get((cfg["workload"], cfg.get("B"), cfg.get("k")))
        line = {"metric": metric_of(kind), "value": value, "unit": UNIT, "n_gpus": world,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_total / a.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic",
                "config": dict(cfg, l2=f"{ncopy} rotating input copies "
                                       f"({ncopy * algo_bytes / 2**20:.0f} MiB > 2x L2)",
                               parallelism=f"dp{world}" if world > 1 else "single"),
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                             "unit": "GB/s", "frac": achieved / peak,
                             "kernel": dom, "kernel_us": dom_us, "kernel_bytes": dom_bytes,
                             "call_achieved": call_gbs, "call_frac": call_gbs / peak,
                             "traffic": traffic[0] if traffic else None,
                             "traffic_from": traffic[1] if traffic else None,
                             "peak_kind": peak_kind,
                             "algorithmic_bytes_per_launch": algo_bytes,
                             "needed_bytes_per_launch": need_bytes,
                             "needed_frac": need_bytes / (ms_launch * 1e-3) / 1e9 / peak,
                             "call_us": ms_launch * 1e3},
                "kernels": kern,
                "hbm_gbs": call_gbs, "pct_of_8tbs": 100 * call_gbs / 8000.0,
                "e2e": e2e,
                "gpu_launches": sum(v["launches_per_step"] for v in kern.values()) * a.steps,
                "clocks": clk,
                "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
