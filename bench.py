#!/usr/bin/env python
"""Benchmark: split-KV varlen GQA decode on B200, achieved HBM GB/s and us/call.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|ragged|continuous|shortq|tiny]

One step = one attention call over one batch of the workload (plan made once,
the call captured once in a CUDA graph and replayed).  Inputs are resident in
HBM.  A call whose inputs exceed the 126 MB L2 is timed back to back over
several copies of its inputs used in turn (together several times L2); a
smaller one is timed alone after an L2 flush.  The continuous-batching
workload walks its 100 length draws: before each replay its cu_seqlens_k is
rewritten in place on the device (inside the timed region), so one graph
serves every step.  Bytes counted per call are the algorithmic ones: K and V
over the actual ragged lengths plus Q and O (lse is reported apart).  With N > 1
(torchrun) every rank runs its own copy of the workload (independent
sequences: weak scaling, no collective on the data path) and the time is the
max over ranks.

The timed pass of K calls is repeated (the same number of passes on every
rank, about a quarter of a second of device time in all) and the median pass
gives the value; the spread of the passes and the SM clock sampled throughout
are reported beside it.  Unless --only is given, a one-GPU run also measures
the method's other workloads (ragged, continuous batching over all 100 length
draws, short query, tiny) in the same process and reports them under
"workloads", each with its CPU baseline.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only), on a bounded sample of the same workload per step.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "achieved HBM GB/s and µs/call, varlen GQA split-KV decode, 1×B200 (% of roofline)"
FLUSH_BYTES = 512 << 20
L2_BYTES = 126 << 20          # B200 L2

DESCRIPTIONS = {
    "long": "low-parallelism long-context decode: B=1, q_len=1, Hq=64, Hkv=8, D=128, kv=32768",
    "ragged": "ragged decode batch: B=64, q_len=1, Hq=32, Hkv=8, D=128, kv~U{0..8192}",
    "continuous": "continuous batching: B=256, q_len=1, Hq=64, Hkv=8, D=128, kv~lognormal(mean 2048, "
                  "sigma 1) in [1,16384], step 0",
    "shortq": "short-query varlen: B=32, q_len~U{1..16}, Hq=32, Hkv=4, D=128, kv~U{q_len..4096}, causal",
    "tiny": "tiny decode: B=2, q_len=1, Hq=4, Hkv=1, D=64, kv={37,100}",
    "prefill": "causal prefill (queries longer than one 128-row tile): B=4, q_len=kv~U{512..2048}, Hq=32, "
               "Hkv=4, D=128",
}


def attention_flops(batch: W.Batch) -> int:
    """4 * D flops per visible (query, key) pair and query head (S = Q K^T and
    P V), with the tail-aligned causal mask."""
    sh = batch.shape
    pairs = 0
    for lq, lk in zip(batch.lens_q.tolist(), batch.lens_k.tolist()):
        # query qi sees min(lk, max(0, lk - lq + qi + 1)) keys
        for qi in range(int(lq)):
            pairs += min(int(lk), max(0, int(lk) - int(lq) + qi + 1))
    return 4 * sh.D * sh.Hq * pairs


def algorithmic_bytes(batch: W.Batch) -> dict:
    sh = batch.shape
    kv = int(batch.lens_k.sum()) * sh.Hkv * sh.D * 2 * 2
    tq = int(batch.lens_q.sum())
    qo = tq * sh.Hq * sh.D * 2 * 2
    return {"kv": kv, "qo": qo, "total": kv + qo, "lse": tq * sh.Hq * 4}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running
    (reads only; changes no setting)."""

    REASONS = {0x2: "applications_clocks", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.reasons = 0
        self.sm_max = None
        self.err = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nvml, self._h = pynvml, h
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that, do not guess
            self._nvml = None
            self.err = f"nvml unavailable: {e}"
        self._t = threading.Thread(target=self._run, daemon=True)

    def _reasons_now(self):
        n = self._nvml
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(n, fn):
                return getattr(n, fn)(self._h)
        return 0

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons_now())
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(self._period)

    def __enter__(self):
        if self._nvml:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nvml:
            self._t.join(timeout=2)

    def summary(self) -> dict:
        d = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
             "sm_max_mhz": self.sm_max, "samples": len(self.samples),
             "reasons": [name for bit, name in self.REASONS.items() if self.reasons & bit],
             "source": "nvml, sampled every 10 ms during the timed region"}
        if self.err:
            d["error"] = self.err
        return d


# ------------------------------------------------------------------ peaks / profiles

def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy burst)"
    except Exception:
        return 6650.0, "fallback 6.65 TB/s (pool measurement)"


def measured_tensor_peak():
    """Dense bf16 tensor peak: the burst figure of a cuBLAS GEMM timed alone."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except Exception:
        return 1590.0, "fallback 1.59 PFLOP/s (pool measurement)"


def strip_c_comments(src: str) -> str:
    """The source with // and /* */ comments removed (string and character
    literals kept as they are), trailing blanks cut and blank lines dropped:
    what the compiler sees, up to layout."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (l.rstrip() for l in "".join(out).split("\n"))
    return "\n".join(l for l in lines if l)


def kernel_source_hash() -> str:
    """Hash of the library's C++/CUDA sources without their comments, so that
    a recorded ncu capture stays attached to the code it measured and a
    comment edit does not detach it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "varlen_gqa_split_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h", ".cpp")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + strip_c_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, when it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None, "no ncu record"
    e = rec.get(workload)
    if not e:
        return None, "no ncu record for this workload"
    if e.get("source_hash") != kernel_source_hash():
        return None, "kernel changed since the ncu capture"
    if e.get("kernel") != kernel:
        return None, "ncu record names another kernel"
    return int(e["dram_bytes_per_launch"]), e.get("note", "")


# ------------------------------------------------------------------ distributed

def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun env).  The ranks run independent
    replicas of the workload; the only collectives are the barrier around the
    timed region and the max of the ranks' times.  backend="gloo" runs the
    same logic on CPU (tests)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
        pg = dist
    return rank, world, local, pg


def max_over_ranks(x: float, pg) -> float:
    if pg is None:
        return x
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ------------------------------------------------------------------ reference arm (oracle)

def run_reference(args, batch: W.Batch) -> dict:
    """The oracle as it stands, timed on the host cores: each step computes a
    random sample of the workload's output rows, sized so that warm-up plus
    timed steps take about VGQA_REF_BUDGET_S seconds (default 120)."""
    import oracle
    sh = batch.shape
    qb, kb, vb = W.bits(batch.q), W.bits(batch.k), W.bits(batch.v)
    lens_q, lens_k = batch.lens_q, batch.lens_k
    rows_all = np.array([(b, qi, h) for b in range(len(lens_q)) for qi in range(int(lens_q[b]))
                         for h in range(sh.Hq)], dtype=np.int64)
    # algorithmic bytes of a row: its share of its sequence's K/V for its KV
    # head (read by G * Lq rows) plus its q and out rows
    row_bytes = np.array([lens_k[b] * sh.D * 4 / (sh.G * max(int(lens_q[b]), 1)) + sh.D * 4
                          for b in rows_all[:, 0]])
    budget_s = float(os.environ.get("VGQA_REF_BUDGET_S", "120"))
    t0 = time.perf_counter()
    oracle.attention_rows(qb, kb, vb, batch.cu_q, batch.cu_k, rows_all[:1], B=sh.B, Hq=sh.Hq,
                          Hkv=sh.Hkv, D=sh.D, causal=sh.causal)
    t_row = max(time.perf_counter() - t0, 1e-5)
    n_steps = args.steps + args.warmup
    per_step = max(1, min(len(rows_all), int(budget_s / n_steps / t_row)))
    rng = np.random.default_rng(0)
    times, nbytes = [], []
    for s in range(n_steps):
        pick = rng.choice(len(rows_all), size=per_step, replace=False)
        t0 = time.perf_counter()
        oracle.attention_rows(qb, kb, vb, batch.cu_q, batch.cu_k, rows_all[pick], B=sh.B, Hq=sh.Hq,
                              Hkv=sh.Hkv, D=sh.D, causal=sh.causal)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            nbytes.append(float(row_bytes[pick].sum()))
    total_t = sum(times)
    value = sum(nbytes) / total_t / 1e9
    sample = (f"{per_step} of {len(rows_all)} output rows (b, qi, h) per step, drawn at random; "
              f"bytes attributed per row (K/V share + q + out)")
    return {
        "metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCRIPTIONS[args.workload], "kind": "fp64 CPU oracle (oracle/oracle.c)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def cpu_baseline(batch: W.Batch, bytes_: dict, budget_s: float = 20.0, threads: int | None = None,
                 seed: int = 1) -> dict:
    """The oracle as it stands on the host cores (all of them, or `threads`),
    on a bounded sample of the same workload, scaled to GB/s of the
    workload's algorithmic bytes."""
    import oracle
    sh = batch.shape
    all_threads = oracle.num_threads()
    if threads:
        oracle.set_num_threads(threads)
    try:
        qb, kb, vb = W.bits(batch.q), W.bits(batch.k), W.bits(batch.v)
        lens_q, lens_k = batch.lens_q, batch.lens_k
        rows_all = np.array([(b, qi, h) for b in range(len(lens_q)) for qi in range(int(lens_q[b]))
                             for h in range(sh.Hq)], dtype=np.int64)
        # work per row ~ its visible keys; sample whole rows until the budget is met
        t0 = time.perf_counter()
        oracle.attention_rows(qb, kb, vb, batch.cu_q, batch.cu_k, rows_all[:8], B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv,
                              D=sh.D, causal=sh.causal)
        t8 = max(time.perf_counter() - t0, 1e-4)
        n = int(min(len(rows_all), max(8, 8 * (budget_s / 3) / t8)))
        rng = np.random.default_rng(seed)
        sel = rows_all if n >= len(rows_all) else rows_all[np.sort(rng.choice(len(rows_all), n, replace=False))]
        ts = []
        for _ in range(3):
            t0 = time.perf_counter()
            oracle.attention_rows(qb, kb, vb, batch.cu_q, batch.cu_k, sel, B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv,
                                  D=sh.D, causal=sh.causal)
            ts.append(time.perf_counter() - t0)
        cores = oracle.num_threads()
    finally:
        if threads:
            oracle.set_num_threads(all_threads)
    t = statistics.median(ts)
    # scale: the sample's share of the workload's (row x key) work
    vis = lambda b: int(lens_k[b])  # noqa: E731  (q_len rows see <= Lk keys; decode sees Lk)
    work_sel = sum(vis(b) for b in sel[:, 0])
    work_all = sum(vis(b) for b in rows_all[:, 0])
    frac = work_sel / max(work_all, 1)
    value = bytes_["total"] * frac / t / 1e9
    return {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(sel)} of {len(rows_all)} output rows ({100 * frac:.1f}% of the row x key work), "
                      f"median of 3, scaled to the whole call"}


def cpu_baseline_steps(name: str, batch: W.Batch, budget_s: float, steps=(0, 49, 99)) -> dict:
    """Continuous batching: the oracle at several length draws of the same
    K/V buffer, each a bounded sample; reports the mean GB/s per step."""
    draws = W.lengths(name, seed=0)
    per = []
    for s in steps:
        lq, lk = draws[s]
        b = W.Batch(batch.shape, batch.q[: int(lq.sum())], batch.k, batch.v, W.cu_from_lengths(lq),
                    W.cu_from_lengths(lk), lq, lk)
        per.append(cpu_baseline(b, algorithmic_bytes(b), budget_s / len(steps), seed=1 + s))
    return {"value": statistics.mean(p["value"] for p in per), "unit": "GB/s", "cores": per[0]["cores"],
            "kind": "oracle", "steps": list(steps), "per_step": [p["value"] for p in per],
            "sample": "length draws " + ", ".join(str(s) for s in steps) + ": " + "; ".join(p["sample"] for p in per)}


# ------------------------------------------------------------------ our arm

def make_inputs(name: str, device):
    """Step 0 of the workload.  For continuous batching the K/V buffers hold
    as many tokens as the largest of its steps, so every step's lengths fit."""
    if name != "continuous":
        return W.workload(name, seed=0, gen_device=device)
    steps = W.lengths(name, seed=0)
    cap = max(int(lk.sum()) for _, lk in steps)
    lq, lk = steps[0]
    return W.make_batch(W.SHAPES[name], lq, lk, seed=0, gen_device=device, kv_capacity=cap)


def step_cu_k(name: str, batch: W.Batch):
    """Per-step cu_seqlens_k (host, [S, B+1] int32) and algorithmic bytes."""
    if name != "continuous":
        return batch.cu_k[None, :], [algorithmic_bytes(batch)["total"]]
    cus, byts = [], []
    for lq, lk in W.lengths(name, seed=0):
        b = W.Batch(batch.shape, None, None, None, batch.cu_q, W.cu_from_lengths(lk, batch.shape.B + 1), lq, lk)
        cus.append(b.cu_k)
        byts.append(algorithmic_bytes(b)["total"])
    return np.stack(cus), byts


def max_over_ranks_vec(xs, pg) -> list:
    """Element-wise max over ranks of a list of floats (one collective)."""
    if pg is None:
        return list(xs)
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor(list(xs), dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


KERNELS = {1: "split_simt_kernel", 2: "split_mma_kernel", 3: "split_tc_kernel"}
MIN_TIMED_S = 0.25          # timed passes repeat until about this much device time
MAX_PASSES = 400


class Workload:
    """One workload on one GPU: inputs resident in HBM, a plan, and CUDA
    graphs of its calls, ready to be timed."""

    def __init__(self, name, args, dev, page_size=0):
        from varlen_gqa_split_b200 import Plan
        self.name, self.dev, self.page_size = name, dev, page_size
        batch = make_inputs(name, dev)
        sh = batch.shape
        self.batch, self.sh = batch, sh
        self.bytes = algorithmic_bytes(batch)
        q, k, v = batch.q, batch.k, batch.v
        self.paged = None
        if page_size:
            # the same keys in a paged cache: shuffled pages of page_size tokens,
            # one block-table row per sequence (only step 0's lengths are placed,
            # so one draw of lengths)
            if name == "continuous":
                raise SystemExit("--page-size: the continuous workload changes its lengths every step")
            self.paged = W.paginate(k, v, batch.cu_k, sh.B, page_size, sh.s_max, seed=0, fill=0.0)
            k, v = self.paged.k_cache, self.paged.v_cache
        self.q, self.k, self.v = q, k, v
        self.cu_q = torch.from_numpy(batch.cu_q).to(dev)
        self.cu_k = torch.from_numpy(batch.cu_k).to(dev)
        self.out = torch.empty_like(q)
        self.lse = torch.empty(q.shape[0], sh.Hq, dtype=torch.float32, device=dev)
        self.plan = Plan(sh.B, sh.s_max, sh.Hq, sh.Hkv, sh.D, sh.max_q, nsplit=args.nsplit, variant=args.variant,
                         stages=args.stages, combine=args.combine, ctas=args.ctas,
                         deterministic=int(args.deterministic))
        self.info = self.plan.info
        self.launches_per_call = 2 if self.info["combine"] == 1 else 1     # split (+ combine kernel)
        self.kernel = KERNELS[self.info["variant"]]
        self.stream = torch.cuda.Stream(dev)
        # A call whose inputs exceed L2 is timed in a pipeline: R copies of the
        # inputs (together several times L2), one per layer of a model, and one
        # CUDA graph holding R calls, one per copy -- the attention calls of a
        # decode step over the layers' own caches.  K calls = K/R replays (plus
        # a shorter graph for a remainder) between one pair of events.  A
        # smaller call is timed alone: L2 flushed before each call, events
        # captured inside the graph around the call.  The isolated per-call
        # latency (flush, then one call) is reported for every workload.
        cu_steps_h, self.step_bytes = step_cu_k(name, batch)
        self.n_var = len(self.step_bytes)
        self.pipelined = min(self.step_bytes) >= L2_BYTES
        n_copies = max(2, min(8, -(-4 * L2_BYTES // min(self.step_bytes)))) if self.pipelined else 1
        self.n_copies = n_copies
        self.copies = [(q, k, v, self.out, self.lse)]
        for _ in range(n_copies - 1):
            self.copies.append((q.clone(), k.clone(), v.clone(), torch.empty_like(self.out),
                                torch.empty_like(self.lse)))
        # one cu_seqlens_k row per copy; with several length draws, the rows of
        # the next n_copies draws are written in place before each replay
        cu_ext = np.concatenate([cu_steps_h, cu_steps_h[:n_copies]]) if self.n_var > 1 else cu_steps_h
        self.cu_steps = torch.from_numpy(cu_ext).to(dev)
        self.cu_rows = self.cu_steps[:1].repeat(n_copies, 1).contiguous()
        self.in0 = torch.cuda.Event(enable_timing=True, external=True)
        self.in1 = torch.cuda.Event(enable_timing=True, external=True)
        # L2 flush by reading a buffer four times the L2: the lines it leaves
        # are clean, so the timed call pays no write-back of the flush itself
        # (a flush by writing left ~126 MB of dirty lines that the next call's
        # reads had to evict to DRAM)
        self.flush = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        self.flush_out = torch.zeros((), dtype=torch.int64, device=dev)
        self.graphs = {}
        with torch.cuda.stream(self.stream):
            self.call(q, k, v, self.cu_q, self.cu_rows[0], self.out, self.lse)
            self.stream.synchronize()
            self.g_iso = self._capture(1, events=True)
            self.g_all = self._capture(n_copies) if self.pipelined else None

    def call(self, qq, kk, vv, cq, ck, oo, ll):
        if self.paged is None:
            return self.plan.run(qq, kk, vv, cq, ck, oo, ll)
        return self.plan.run_paged(qq, kk, vv, self.paged.block_table, cq, ck, oo, ll)

    def _capture(self, n_calls, events=False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream, capture_error_mode="global"):
            if events:
                self.in0.record(self.stream)
            for r in range(n_calls):
                qq, kk, vv, oo, ll = self.copies[r]
                self.call(qq, kk, vv, self.cu_q, self.cu_rows[r], oo, ll)
            if events:
                self.in1.record(self.stream)
        return g

    def rem_graph(self, steps):
        rem = steps % self.n_copies
        if not (self.pipelined and rem):
            return None
        if rem not in self.graphs:
            with torch.cuda.stream(self.stream):
                self.graphs[rem] = self._capture(rem)
        return self.graphs[rem]

    def isolated_step(self):
        torch.amax(self.flush, dim=0, out=self.flush_out)
        self.g_iso.replay()
        self.stream.synchronize()
        return self.in0.elapsed_time(self.in1)

    def set_draws(self, j):
        if self.n_var > 1:
            s0 = (j * self.n_copies) % self.n_var
            self.cu_rows.copy_(self.cu_steps[s0:s0 + self.n_copies], non_blocking=True)

    def timed_pass(self, steps, pg):
        """One timed pass of exactly `steps` calls (barrier + synchronise on
        both sides); returns this rank's milliseconds."""
        g_rem = self.rem_graph(steps)
        o0 = torch.cuda.Event(enable_timing=True)
        o1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            self.stream.synchronize()
            barrier(pg)
            torch.cuda.synchronize(self.dev)
            if self.pipelined:
                o0.record(self.stream)
                for j in range(steps // self.n_copies):
                    self.set_draws(j)
                    self.g_all.replay()
                if g_rem is not None:
                    self.set_draws(steps // self.n_copies)
                    g_rem.replay()
                o1.record(self.stream)
                self.stream.synchronize()
                ms = o0.elapsed_time(o1)
            else:
                ms = sum(self.isolated_step() for _ in range(steps))
            torch.cuda.synchronize(self.dev)
            barrier(pg)
        return ms

    def bytes_of(self, steps):
        if self.pipelined:
            return sum(self.step_bytes[i % self.n_var] for i in range(steps))
        return self.bytes["total"] * steps

    def measure(self, steps, warmup, pg, n_iso=200, min_timed_s=MIN_TIMED_S):
        """Warm-up, isolated calls, then repeated timed passes of `steps` calls
        (the same number of passes on every rank), clocks sampled throughout.
        Returns the per-pass milliseconds (max over ranks), the isolated-call
        milliseconds and the clock summary."""
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                self.isolated_step()
            iso_ms = [self.isolated_step() for _ in range(min(steps, n_iso))]
            if self.pipelined:
                for j in range(warmup):
                    self.set_draws(j)
                    self.g_all.replay()
            self.stream.synchronize()
        first = self.timed_pass(steps, pg)
        n_pass = int(min(MAX_PASSES, max(5, math.ceil(min_timed_s * 1e3 / max(first, 1e-3)))))
        n_pass = int(max_over_ranks(float(n_pass), pg))
        local = []
        with ClockSampler(self.dev.index if self.dev.index is not None else 0) as clocks:
            for _ in range(n_pass):
                local.append(self.timed_pass(steps, pg))
        passes = max_over_ranks_vec(local, pg)
        assert self.plan.check_error() == 0, "device error flag set during the benchmark"
        return passes, iso_ms, clocks.summary()

    def summary(self, steps, passes, iso_ms, clocks, world) -> dict:
        """us per call, GB/s and roofline fraction from the median pass."""
        med = statistics.median(passes)
        q10, q90 = np.percentile(passes, [10, 90])
        timed_bytes = self.bytes_of(steps)
        achieved = timed_bytes / (med * 1e-3) / 1e9
        peak, peak_src = measured_peak()
        traffic_key = self.name + (f"_paged{self.page_size}" if self.paged is not None else "")
        traffic, traffic_note = recorded_traffic(traffic_key, self.kernel)
        us = 1e3 * med / steps
        d = {"us_per_call": us, "value_gbs": achieved * world, "frac": achieved / peak,
             "kernel": self.kernel, "calls_per_pass": steps, "passes": len(passes),
             "us_per_call_p10_p90": [1e3 * q10 / steps, 1e3 * q90 / steps],
             "us_per_call_min_max": [1e3 * min(passes) / steps, 1e3 * max(passes) / steps],
             "bytes_per_call": timed_bytes / steps, "length_draws_cycled": self.n_var,
             "traffic": traffic, "clocks": clocks,
             "isolated_call_us": {"median": 1e3 * statistics.median(iso_ms), "min": 1e3 * min(iso_ms),
                                  "max": 1e3 * max(iso_ms), "calls": len(iso_ms),
                                  "value_gbs": self.bytes["total"] / (statistics.median(iso_ms) * 1e-3) / 1e9,
                                  "how": "L2 flushed by a 512 MB read, then one call; CUDA events inside the "
                                         "captured graph"}}
        if clocks.get("sm_mhz"):
            d["kcycles_per_call"] = us * clocks["sm_mhz"] / 1e3
        if traffic is None:
            d["traffic_note"] = traffic_note
        if self.name == "prefill":
            flops = attention_flops(self.batch)
            tpeak, _ = measured_tensor_peak()
            d["tflops"] = flops / (us * 1e-6) / 1e12
            d["tensor_frac"] = d["tflops"] / tpeak
        return d, achieved, peak, peak_src, traffic, traffic_note

    def close(self):
        self.g_iso = self.g_all = None
        self.graphs.clear()
        self.plan.close()


# the workloads the method's ≥70% target names, and the short-query one it
# also asks to report; measured beside the headline workload in one run
EXTRA_WORKLOADS = ("ragged", "continuous", "shortq", "tiny")


def run_ours(args, rank, world, local, pg) -> dict | None:
    from varlen_gqa_split_b200 import build
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = Workload(args.workload, args, dev, args.page_size)
    sh, info, batch, bytes_ = wl.sh, wl.info, wl.batch, wl.bytes
    passes, iso_ms, clocks = wl.measure(args.steps, args.warmup, pg)
    ws, achieved, peak, peak_src, traffic, traffic_note = wl.summary(args.steps, passes, iso_ms, clocks, world)
    ms_per_step = statistics.median(passes) / args.steps
    value = ws["value_gbs"]
    timed_bytes = wl.bytes_of(args.steps)

    # roofline of the split kernel.  One call is one split-kernel launch,
    # followed on the tensor-core path by the LSE combine kernel, launched as a
    # programmatic dependent (it overlaps the split kernel until its wait and
    # then merges the cut units).  The events bracket the whole call, so the
    # achieved figure charges the combine tail to the split kernel: a lower
    # bound on the split kernel's own rate.  Its share of device time is in the
    # committed ncu launch list.
    roofline = {"bound": "hbm", "kernel": wl.kernel, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": timed_bytes / args.steps,
                "timed": ("one call: split kernel + LSE combine kernel (programmatic dependent launch)"
                          if wl.launches_per_call == 2 else "one call: the split kernel alone")}
    if traffic is None:
        roofline["traffic_note"] = traffic_note
    if args.workload == "prefill":
        # queries of up to 2048 tokens: the contraction, not HBM, bounds it
        flops = attention_flops(batch)
        tpeak, tsrc = measured_tensor_peak()
        tach = flops / (ms_per_step * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": wl.kernel, "achieved": tach, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": tach / tpeak, "traffic": traffic, "peak_source": tsrc,
                    "algorithmic_flops_per_launch": flops, "hbm_gbs": achieved,
                    "timed": roofline["timed"]}

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(wl, args, pg, world)

    # the other workloads of the method, in the same process (one GPU)
    extras = {}
    if not args.only and world == 1 and args.page_size == 0:
        for name in EXTRA_WORKLOADS:
            if name == args.workload:
                continue
            other = Workload(name, args, dev)
            # continuous batching: one pass walks all 100 length draws
            st = other.n_var if other.n_var > 1 else args.steps
            p_, iso_, clk_ = other.measure(st, args.warmup, pg, n_iso=50)
            extras[name], *_ = other.summary(st, p_, iso_, clk_, world)
            extras[name]["workload"] = DESCRIPTIONS[name]
            extras[name]["plan"] = {kk: other.info[kk] for kk in ("variant", "ctas", "stages", "combine")}
            if name == "tiny":
                extras[name]["note"] = "latency-bound (37 KB per call): timed alone after an L2 flush"
            if rank == 0 and not args.no_cpu_baseline:
                if name == "continuous":
                    extras[name]["cpu_baseline"] = cpu_baseline_steps(name, other.batch, 12.0)
                elif name != "tiny":
                    extras[name]["cpu_baseline"] = cpu_baseline(other.batch, other.bytes, 8.0)
            other.close()
            del other
            torch.cuda.empty_cache()

    res = None
    if rank == 0:
        cpu = None
        if not (args.no_cpu_baseline or world > 1):
            cpu = cpu_baseline(batch, bytes_)
            cpu["single_thread"] = cpu_baseline(batch, bytes_, budget_s=8.0, threads=1)
        res = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "us_per_call": 1e3 * ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": DESCRIPTIONS[args.workload], "B": sh.B, "Hq": sh.Hq, "Hkv": sh.Hkv,
                       "D": sh.D, "max_q": sh.max_q, "s_max": sh.s_max,
                       "kv_tokens": int(batch.lens_k.sum()), "q_tokens": int(batch.lens_q.sum()),
                       "kv_layout": ("packed THD" if wl.paged is None else
                                     f"paged: {wl.k.shape[0]} pages of {args.page_size} tokens in shuffled "
                                     f"order, one block-table row per sequence"),
                       "bytes_per_call": timed_bytes / args.steps, "lse_bytes_per_call": bytes_["lse"],
                       "length_draws_cycled": wl.n_var,
                       "l2": (f"inputs larger than L2: {wl.n_copies} copies of the inputs ({wl.n_copies} x "
                              f"{bytes_['total'] / 1e6:.0f} MB) used in turn" if wl.pipelined else
                              "flushed before every timed call (512 MB read, outside the timed events)"),
                       "timing": (f"CUDA events around K attn_run calls, captured {wl.n_copies} per CUDA graph "
                                  f"(one per input copy, like the layers of a decode step) and replayed back "
                                  f"to back" +
                                  ("; before each replay one device-to-device copy writes the next draws' "
                                   "cu_seqlens_k in place (timed)" if wl.n_var > 1 else "") if wl.pipelined else
                                  "CUDA events captured inside the graph around the attn_run call, one replay "
                                  "per step after an L2 flush, summed") +
                                 f"; {len(passes)} timed passes of K = {args.steps} calls, each bracketed by a "
                                 f"barrier and synchronisation, value from the median pass",
                       "parallelism": f"replicas x{world} (independent sequences)",
                       "plan": {kk: info[kk] for kk in ("variant", "nsplit", "chunk", "ctas", "stages", "grid_x",
                                                         "grid_y", "grid_z", "combine", "smem_bytes")}},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": wl.launches_per_call * args.steps,
            "clocks": clocks,
            "passes": {k_: ws[k_] for k_ in ("passes", "us_per_call_p10_p90", "us_per_call_min_max")},
            "isolated_call_us": ws["isolated_call_us"],
        }
        if "kcycles_per_call" in ws:
            res["kcycles_per_call"] = ws["kcycles_per_call"]
        if extras:
            res["workloads"] = extras
    wl.close()
    return res


def measure_e2e(wl: Workload, args, pg, world) -> dict:
    """The same call end to end through the public API: pinned host buffers,
    the host-to-device copies of the step's inputs and the device-to-host
    copies of its outputs inside the timed region."""
    batch, sh, plan, paged = wl.batch, wl.sh, wl.plan, wl.paged
    k, v, q = wl.k, wl.v, wl.q
    n_e2e = max(3, min(args.steps, 20))
    # only the tokens this step's lengths cover cross the bus
    tkv = batch.kv_tokens if paged is None else k.shape[0]
    hq = batch.q.cpu().pin_memory()
    hk = k[:tkv].cpu().pin_memory()
    hv = v[:tkv].cpu().pin_memory()
    hcq = torch.from_numpy(batch.cu_q).pin_memory()
    hck = torch.from_numpy(batch.cu_k).pin_memory()
    ho = torch.empty_like(hq).pin_memory()
    hl = torch.empty(hq.shape[0], sh.Hq, dtype=torch.float32).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if paged is not None:
        # the halves of one buffer stay views of one buffer
        dk, dv = torch.empty_like(k.contiguous()), torch.empty_like(v.contiguous())
        hbt = paged.block_table.cpu().pin_memory()
        dbt = torch.empty_like(paged.block_table)
    dcq, dck = torch.empty_like(wl.cu_q), torch.empty_like(wl.cu_k)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcq, hck))
    if paged is not None:
        h2d += hbt.numel() * hbt.element_size()
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    stream = wl.stream
    with torch.cuda.stream(stream):
        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk[:tkv].copy_(hk, non_blocking=True)
            dv[:tkv].copy_(hv, non_blocking=True)
            dcq.copy_(hcq, non_blocking=True)
            dck.copy_(hck, non_blocking=True)
            if paged is None:
                o, l_ = plan.run(dq, dk, dv, dcq, dck, wl.out, wl.lse)
            else:
                dbt.copy_(hbt, non_blocking=True)
                o, l_ = plan.run_paged(dq, dk, dv, dbt, dcq, dck, wl.out, wl.lse)
            ho.copy_(o, non_blocking=True)
            hl.copy_(l_, non_blocking=True)
        for _ in range(2):
            e2e_step()
        stream.synchronize()
        barrier(pg)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg)
    return {"value": wl.bytes["total"] * n_e2e * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
            "us_per_call": 1e3 * e2e_ms / n_e2e}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(DESCRIPTIONS), default="long")
    ap.add_argument("--nsplit", type=int, default=0)
    ap.add_argument("--variant", type=int, default=0)
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--combine", type=int, default=0)
    ap.add_argument("--ctas", type=int, default=0)
    ap.add_argument("--deterministic", action="store_true",
                    help="static shares, bitwise repeatable (no run-time claims)")
    ap.add_argument("--page-size", type=int, default=0,
                    help="read K/V from a paged cache with pages of this many tokens (0: packed)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true",
                    help="time the selected workload alone (no other workloads in the same run)")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        batch = make_inputs(args.workload, "cpu")
        res = run_reference(args, batch)
        print(json.dumps(res), flush=True)
        return

    rank, world, local, pg = dist_setup(args.gpus)
    try:
        res = run_ours(args, rank, world, local, pg)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
