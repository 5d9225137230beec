#!/usr/bin/env python
"""PQ-HSA decode benchmark: µs per decode step and achieved HBM GB/s on B200.

Workload (default): one Llama-3.1-8B-shaped attention layer at 128K context,
32 query / 8 KV heads, head dim 128, paged bf16 K/V (page 16, shuffled pool),
IVF-PQ index with 1024 clusters and 16 x 8-dim subspaces of 256 codes per KV
head, sink 16 + recent 1024 exact, top-k = 1 % of the indexed tokens.
Synthetic seeded data (see synth/). One JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn µs/step & achieved HBM GB/s (% peak) at 128K ctx, 1% budget"
L2_FLUSH_BYTES = 512 << 20
# Eager per-kernel timing: a device-side spin of this many cycles runs before each eager
# step, so the host has queued the whole step before the GPU reaches it and the stage
# events time kernels, not host launch gaps.
QUEUE_AHEAD_CYCLES = 4_000_000
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def dram_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary, or None."""
    try:
        with open(TRAFFIC_FILE) as f:
            entry = json.load(f).get(f"{kernel} {workload}")
    except (OSError, ValueError):
        return None
    return int(entry["dram_bytes_per_launch"]) if entry else None


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_128k")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="bound on the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", choices=["ctx", "budget", "batch"], default=None,
                    help="extra measurements: context-length crossover, budget / background ablation, "
                         "or the 32-sequence batch at 32K")
    ap.add_argument("--append", action="store_true",
                    help="index-append cost on the Qwen3-30B-A3B-shaped workload (512-token batches)")
    ap.add_argument("--train", action="store_true",
                    help="index build cost: k-means centroids + PQ codebooks from raw keys, then encoding")
    ap.add_argument("--train-iters", type=int, default=8, help="Lloyd iterations of each kind for --train")
    return ap.parse_args(argv)


def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the job's time is its slowest rank's)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def bf16_peak():
    """Dense bf16 tensor TFLOP/s: the measured burst figure (a kernel timed alone), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


# ---------------------------------------------------------------------------
# algorithmic bytes (what one step must move at minimum)
# ---------------------------------------------------------------------------

def step_bytes(w, n_idx: int, k: int):
    """Per-step algorithmic HBM bytes of PQ-HSA, of dense decode and of the scan kernel."""
    G, C, D = w.G, w.C, w.D
    R = w.T - w.n_sink - n_idx
    per_unit = (16 * n_idx                       # PQ codes
                + 4 * C * D                      # centroids (q . centroid)
                + 4 * 16 * 256 * 8               # codebook
                + 4 * G * 16 * 256               # LUT written once
                + 4 * C * D + 4 * C              # cluster mean values + counts
                + 512 * (w.n_sink + R + k)       # exact K+V rows (bf16)
                + 8 * G * D)                     # q in, out
    ids = 2 * n_idx
    dense = 512 * w.T + 8 * G * D
    scan = n_idx * (16 + 2 + 4)                  # codes + cluster id read, selection score written
    U = w.B * w.Hkv
    return U * per_unit, U * ids, U * dense, U * scan


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle sample (reported baseline, never the target)
# ---------------------------------------------------------------------------

def oracle_sample(bt, w, budget, seconds: float):
    """Run the float64 oracle on units of the workload until `seconds` elapse; µs per whole step."""
    from threadpoolctl import threadpool_limits
    import oracle as O
    scale = float(np.float32(1.0 / math.sqrt(w.D)))
    done, t0 = 0, time.perf_counter()
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    with threadpool_limits(limits=1):
        while True:
            u = units[done % len(units)]
            O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, bt.centroids,
                            bt.codebooks, bt.codes_rec, bt.ids_rec, bt.n_indexed, w.n_sink, scale,
                            budget=budget, page_size=w.page_size, units=[u])
            done += 1
            el = time.perf_counter() - t0
            if el >= seconds or done >= 4 * len(units):
                break
    us_per_step = el / done * len(units) * 1e6
    return us_per_step, done, el


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import sparse_long_context_pq_b200 as P
    from synth import make_batch, workload
    from synth.device import index_tensors, kv_tensors

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    w = workload(args.workload)
    budget = w.budget
    bt = make_batch(w)
    kv = P.PagedKV(**kv_tensors(bt, dev))
    ix = P.PQIndex(**index_tensors(bt, dev, n_indexed=np.zeros(w.B, dtype=np.int32)))
    stream = torch.cuda.current_stream()

    # ---- index build after prefill: encode every indexed key on the GPU ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ws_idx = P.workspace(P.hsa_index_workspace_bytes(kv, ix, w.n_indexed), dev)
    e0.record()
    P.hsa_append_encode(kv, ix, w.n_indexed, workspace_buf=ws_idx)
    e1.record()
    torch.cuda.synchronize()
    build_ms = e0.elapsed_time(e1)
    assert P.hsa_read_error(ws_idx) == 0

    scale = float(np.float32(1.0 / math.sqrt(w.D)))
    q = torch.from_numpy(bt.q).to(dev)
    out = torch.empty_like(q)
    out_dense = torch.empty_like(q)
    ws = P.workspace(P.hsa_decode_workspace_bytes(kv, ix), dev)
    ws_dense = P.workspace(P.dense_decode_workspace_bytes(kv), dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(P.NUM_STAGES + 1)]
    for e in stage_ev:
        e.record()
    torch.cuda.synchronize()

    def hsa_step(events=None):
        P.hsa_decode(kv, ix, q, out, scale=scale, budget=budget, workspace_buf=ws, stage_events=events)

    def dense_step():
        P.dense_decode(kv, q, out_dense, scale=scale, workspace_buf=ws_dense)

    # warm once outside capture, then capture each step into a CUDA graph
    hsa_step()
    dense_step()
    torch.cuda.synchronize()
    g_hsa, g_dense = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_hsa):
        hsa_step()
    with torch.cuda.graph(g_dense):
        dense_step()
    torch.cuda.synchronize()

    def timed(graph, steps, e2e=None, staging=False):
        """Whole steps: one graph replay each, L2 flushed before, CUDA events around. With
        e2e = (q_host, q, out, out_host) every step also moves q in from pinned host memory
        and out back to it: by the copy engine, or (staging) by kernels that read and write
        mapped views of the pinned buffers."""
        t = []
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(steps):
            flush.zero_()
            a.record()
            if e2e is not None:
                if staging:
                    torch.mul(e2e[0], 1.0, out=e2e[1])
                else:
                    e2e[1].copy_(e2e[0], non_blocking=True)
            graph.replay()
            if e2e is not None:
                if staging:
                    torch.mul(e2e[2], 1.0, out=e2e[3])
                else:
                    e2e[3].copy_(e2e[2], non_blocking=True)
            b.record()
            torch.cuda.synchronize()
            t.append(a.elapsed_time(b))
        return t

    def mapped_view(t_host):
        """A CUDA tensor over a pinned host buffer (unified addressing): a kernel reading or
        writing it moves the bytes over the host link, with no copy-engine round trip."""
        class _Buf:
            pass
        o = _Buf()
        o.__cuda_array_interface__ = {"shape": tuple(t_host.shape), "typestr": "<f4",
                                      "data": (t_host.data_ptr(), False), "version": 3, "strides": None}
        return torch.as_tensor(o, device=dev)

    def timed_stages(steps):
        """Per-kernel times: eager steps with the library's stage events on the launching stream."""
        st = []
        for _ in range(steps):
            flush.zero_()
            torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
            hsa_step(stage_ev)
            torch.cuda.synchronize()
            st.append([stage_ev[i].elapsed_time(stage_ev[i + 1]) for i in range(P.NUM_STAGES)])
        return st

    for _ in range(args.warmup):
        timed(g_hsa, 1)
        timed(g_dense, 1)
        timed_stages(1)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_hsa = timed(g_hsa, args.steps)
        t_stage = timed_stages(args.steps)
        t_dense = timed(g_dense, args.steps)
        q_h = torch.from_numpy(bt.q).pin_memory()
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        t_e2e_ce = timed(g_hsa, args.steps, e2e=(q_h, q, out, out_h))
        try:
            e2e_views = (mapped_view(q_h), q, out, mapped_view(out_h))
        except (RuntimeError, TypeError, ValueError):
            e2e_views = None
        t_e2e = t_e2e_ce
        if e2e_views is not None:
            timed(g_hsa, 2, e2e=e2e_views, staging=True)
            t_staged = timed(g_hsa, args.steps, e2e=e2e_views, staging=True)
            torch.cuda.synchronize()
            if torch.equal(out_h, out.cpu()):      # the last step's result did reach host memory
                t_e2e = t_staged
            else:
                e2e_views = None
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    err = P.hsa_read_error(ws)
    assert err == 0, f"device error word {err}"

    # ---- index build from raw keys: k-means centroids + PQ codebooks (8 + 8 Lloyd
    # iterations), then encoding every indexed key; on a second index, warm, L2 flushed ----
    from synth import train_init_slots
    ix_t = P.PQIndex(**index_tensors(bt, dev, n_indexed=np.zeros(w.B, dtype=np.int32)))
    init_t = torch.from_numpy(train_init_slots(w, w.n_indexed)).to(dev)
    ws_t = P.workspace(P.hsa_train_workspace_bytes(kv, ix_t, w.n_indexed), dev)
    ws_e = P.workspace(P.hsa_index_workspace_bytes(kv, ix_t, w.n_indexed), dev)

    def build_from_keys():
        P.hsa_train_index(kv, ix_t, w.n_indexed, init_t, workspace_buf=ws_t)
        ix_t.n_indexed.zero_()
        ix_t.n_indexed_host.zero_()
        P.hsa_append_encode(kv, ix_t, w.n_indexed, workspace_buf=ws_e)

    build_from_keys()
    flush.zero_()
    e0.record()
    build_from_keys()
    e1.record()
    torch.cuda.synchronize()
    train_build_ms = e0.elapsed_time(e1)
    assert P.hsa_read_error(ws_t) == 0 and P.hsa_read_error(ws_e) == 0
    del ix_t, ws_t, ws_e

    ms_hsa = sum(t_hsa) / len(t_hsa)
    ms_dense = sum(t_dense) / len(t_dense)
    ms_e2e = sum(t_e2e) / len(t_e2e)
    ms_e2e_ce = sum(t_e2e_ce) / len(t_e2e_ce)
    ms_hsa, ms_dense, ms_e2e, ms_e2e_ce = max_over_ranks([ms_hsa, ms_dense, ms_e2e, ms_e2e_ce],
                                                         dist if world > 1 else None, dev)

    stage_ms = [sum(s[i] for s in t_stage) / len(t_stage) for i in range(P.NUM_STAGES)]
    n_idx = int(w.n_indexed)
    k = P.decode_k(budget, n_idx)
    hsa_b, ids_b, dense_b, scan_b = step_bytes(w, n_idx, k)
    peak, peak_kind = measured_peaks()
    dom = int(np.argmax(stage_ms))
    dom_name = P.STAGE_NAMES[dom]
    U = w.B * w.Hkv
    if dom_name == "scan":
        dom_bytes = scan_b
    elif dom_name == "attend":
        dom_bytes = U * (512 * (w.n_sink + (w.T - w.n_sink - n_idx) + k) + 4 * w.C * w.D)
    else:
        dom_bytes = hsa_b
    dom_gbs = dom_bytes / (stage_ms[dom] * 1e-3) / 1e9
    step_gbs = hsa_b / (ms_hsa * 1e-3) / 1e9
    dense_gbs = dense_b / (ms_dense * 1e-3) / 1e9

    res = {
        "metric": METRIC,
        "value": round(ms_hsa * 1e3, 3),
        "unit": "us/step",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_hsa, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 KV, fp32 math",
        "data": "synthetic (seeded; no dataset or weights)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.D, "ctx": w.T,
                   "clusters": w.C, "pq": "16x8/256", "sink": w.n_sink, "recent": w.n_recent,
                   "budget": budget, "k": k, "page_size": w.page_size,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"flushed ({L2_FLUSH_BYTES >> 20} MB write) before every timed step",
                   "timing": "CUDA events per step around a CUDA-graph replay; per-kernel times from "
                             "eager steps with stage events on the launching stream"},
        "percentiles_us": {f"p{q}": round(float(np.percentile(t_hsa, q)) * 1e3, 3) for q in (10, 50, 90)},
        "hbm_gbs": round(step_gbs, 1),
        "hbm_pct_peak": round(100 * step_gbs / peak, 2),
        "bytes_per_step": hsa_b,
        "ids_bytes_per_step": ids_b,
        "dense": {"us_per_step": round(ms_dense * 1e3, 3), "bytes_per_step": dense_b,
                  "hbm_gbs": round(dense_gbs, 1), "pct_peak": round(100 * dense_gbs / peak, 2),
                  "speedup_of_pqhsa": round(ms_dense / ms_hsa, 3)},
        "stages_us": {n: round(v * 1e3, 3) for n, v in zip(P.STAGE_NAMES, stage_ms)},
        "index_build_ms": round(build_ms, 3),
        "index_train_and_encode_ms": round(train_build_ms, 3),
        "roofline": {"kernel": dom_name, "bound": "hbm", "achieved": round(dom_gbs, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                     "traffic": dram_traffic(dom_name + "_kernel", w.name), "algorithmic_bytes": dom_bytes},
        "e2e": {"value": round(ms_e2e * 1e3, 3), "unit": "us/step", "h2d_bytes_per_step": q.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 4,
                "transfer": ("staging kernels read q from and write out to mapped pinned host memory"
                             if e2e_views is not None else "copy engine (cudaMemcpyAsync) from/to pinned memory"),
                "copy_engine_us": round(ms_e2e_ce * 1e3, 3)},
        # per step: the PQ-HSA graph, the eager stage-timed step, the dense graph (attend +
        # merge), the copy-engine end-to-end step, and (when used) the staged one plus 2 warm-ups
        "gpu_launches": args.steps * (3 * P.NUM_STAGES + 2) + (
            (args.steps + 2) * P.NUM_STAGES if e2e_views is not None else 0),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        us, units, el = oracle_sample(bt, w, budget, args.cpu_seconds)
        res["cpu_baseline"] = {"value": round(us, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
                               "sample": f"{units} (sequence, KV head) units of the same workload, "
                                         f"{el:.1f} s of float64 numpy, scaled to a full step"}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


# ---------------------------------------------------------------------------
# extra measurements (one JSON line each; not the headline line)
# ---------------------------------------------------------------------------

class _Setup:
    """One workload on the GPU with its index encoded on the GPU (the build after prefill)."""

    def __init__(self, w, dev):
        import torch
        import sparse_long_context_pq_b200 as P
        from synth import make_batch
        from synth.device import index_tensors, kv_tensors
        self.P, self.torch, self.w, self.dev = P, torch, w, dev
        self.bt = make_batch(w)
        self.kv = P.PagedKV(**kv_tensors(self.bt, dev))
        self.ix = P.PQIndex(**index_tensors(self.bt, dev, n_indexed=np.zeros(w.B, dtype=np.int32)))
        self.ws_idx = P.workspace(P.hsa_index_workspace_bytes(self.kv, self.ix, w.n_indexed), dev)
        P.hsa_append_encode(self.kv, self.ix, w.n_indexed, workspace_buf=self.ws_idx)
        self.scale = float(np.float32(1.0 / math.sqrt(w.D)))
        self.q = torch.from_numpy(self.bt.q).to(dev)
        self.out = torch.empty_like(self.q)
        self.out_dense = torch.empty_like(self.q)
        self.ws = P.workspace(P.hsa_decode_workspace_bytes(self.kv, self.ix), dev)
        self.ws_dense = P.workspace(P.dense_decode_workspace_bytes(self.kv), dev)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def graph(self, fn):
        fn()
        self.torch.cuda.synchronize()
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g):
            fn()
        self.torch.cuda.synchronize()
        return g

    def time_graph(self, g, steps, warmup):
        torch = self.torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t = []
        for i in range(warmup + steps):
            self.flush.zero_()
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            if i >= warmup:
                t.append(a.elapsed_time(b))
        return sum(t) / len(t) * 1e3   # us

    def hsa(self, budget=0.01, background=True):
        return lambda: self.P.hsa_decode(self.kv, self.ix, self.q, self.out, scale=self.scale, budget=budget,
                                         background=background, workspace_buf=self.ws)

    def dense(self):
        return lambda: self.P.dense_decode(self.kv, self.q, self.out_dense, scale=self.scale,
                                           workspace_buf=self.ws_dense)


def run_sweep_ctx(args):
    import torch
    from synth import workload
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, _ = measured_peaks()
    pts = []
    for name in ("llama8b_8k", "llama8b_32k", "llama8b_sweep_128k", "llama8b_512k"):
        w = workload(name)
        S = _Setup(w, dev)
        k = S.P.decode_k(w.budget, w.n_indexed)
        hsa_b, ids_b, dense_b, _ = step_bytes(w, w.n_indexed, k)
        us_h = S.time_graph(S.graph(S.hsa()), args.steps, args.warmup)
        us_d = S.time_graph(S.graph(S.dense()), args.steps, args.warmup)
        assert S.P.hsa_read_error(S.ws) == 0
        print(json.dumps({"sweep": "ctx", "workload": name, "T": w.T, "hsa_us": round(us_h, 3),
                          "dense_us": round(us_d, 3), "speedup": round(us_d / us_h, 3),
                          "hsa_bytes": hsa_b, "ids_bytes": ids_b, "dense_bytes": dense_b,
                          "hsa_gbs": round(hsa_b / us_h / 1e3, 1), "dense_gbs": round(dense_b / us_d / 1e3, 1),
                          "dense_pct_peak": round(100 * dense_b / us_d / 1e3 / peak, 2)}), flush=True)
        pts.append((w, hsa_b, dense_b, us_h, us_d))
        del S
        torch.cuda.empty_cache()
    # Overhead-aware model (crossover article): t = fixed + bytes / BW per method, fitted by
    # least squares; the predicted crossover is the length where the two lines meet.
    def fit(xs, ys):
        xs, ys = np.asarray(xs, float), np.asarray(ys, float)
        A = np.stack([np.ones_like(xs), xs], axis=1)
        (a, b), *_ = np.linalg.lstsq(A, ys, rcond=None)
        return float(a), float(b)
    fh = fit([p_[1] for p_ in pts], [p_[3] for p_ in pts])
    fd = fit([p_[2] for p_ in pts], [p_[4] for p_ in pts])
    w0 = pts[0][0]
    cross = None
    for T in range(2048, 1 << 21, 256):
        wt = w0.scaled(T=T)
        hb, _, db, _ = step_bytes(wt, wt.n_indexed, int(math.floor(wt.budget * wt.n_indexed)))
        if fh[0] + fh[1] * hb <= fd[0] + fd[1] * db:
            cross = T
            break
    print(json.dumps({"sweep": "ctx-model", "hsa_fixed_us": round(fh[0], 2), "hsa_gbs": round(1e-3 / fh[1], 1),
                      "dense_fixed_us": round(fd[0], 2), "dense_gbs": round(1e-3 / fd[1], 1),
                      "predicted_crossover_T": cross}), flush=True)


def run_sweep_batch(args):
    """32 sequences x 32K context (shuffled pages, per-sequence seeds) at 1 %: PQ-HSA vs dense."""
    import torch
    from synth import workload
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, _ = measured_peaks()
    w = workload("batch32_32k")
    S = _Setup(w, dev)
    k = S.P.decode_k(w.budget, w.n_indexed)
    hsa_b, ids_b, dense_b, _ = step_bytes(w, w.n_indexed, k)
    us_h = S.time_graph(S.graph(S.hsa()), args.steps, args.warmup)
    us_d = S.time_graph(S.graph(S.dense()), args.steps, args.warmup)
    assert S.P.hsa_read_error(S.ws) == 0
    print(json.dumps({"sweep": "batch", "workload": w.name, "B": w.B, "T": w.T, "k": k,
                      "hsa_us": round(us_h, 3), "dense_us": round(us_d, 3), "speedup": round(us_d / us_h, 3),
                      "hsa_bytes": hsa_b, "dense_bytes": dense_b,
                      "hsa_gbs": round(hsa_b / us_h / 1e3, 1), "dense_gbs": round(dense_b / us_d / 1e3, 1),
                      "dense_pct_peak": round(100 * dense_b / us_d / 1e3 / peak, 2)}), flush=True)


def run_sweep_budget(args):
    import torch
    from synth import workload
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload(args.workload)
    S = _Setup(w, dev)
    S.dense()()
    torch.cuda.synchronize()
    ref = S.out_dense.clone()
    vmax = float(S.kv.v_cache.float().abs().max())
    for budget in (0.005, 0.01, 0.02, 0.05):
        for bg in (True, False):
            us = S.time_graph(S.graph(S.hsa(budget, bg)), args.steps, args.warmup)
            S.hsa(budget, bg)()
            torch.cuda.synchronize()
            err = float((S.out - ref).abs().max()) / vmax
            rel = float(((S.out - ref).norm(dim=-1) / ref.norm(dim=-1)).mean())
            print(json.dumps({"sweep": "budget", "workload": w.name, "budget": budget, "background": bg,
                              "hsa_us": round(us, 3), "max_abs_err_vs_dense_over_max_v": round(err, 6),
                              "mean_rel_l2_err_vs_dense": round(rel, 6)}), flush=True)


def run_append(args):
    import torch
    from synth import workload
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload("qwen30b_128k_append")
    S = _Setup(w, dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    T = w.T
    for step in range(w.extra_tokens // w.append_batch):
        us_dec = S.time_graph(S.graph(S.hsa()), args.steps, args.warmup)
        T += w.append_batch                      # 512 generated tokens later, the oldest tail tokens move in
        S.kv.seq_lens.fill_(T)
        S.kv.seq_lens_host.fill_(T)
        S.flush.zero_()
        a.record()
        S.P.hsa_append_encode(S.kv, S.ix, w.append_batch, workspace_buf=S.ws_idx)
        b.record()
        torch.cuda.synchronize()
        assert S.P.hsa_read_error(S.ws_idx) == 0
        print(json.dumps({"append": step, "workload": w.name, "T_before": T - w.append_batch,
                          "decode_us": round(us_dec, 3), "append_512_us": round(a.elapsed_time(b) * 1e3, 3),
                          "n_indexed": int(S.ix.n_indexed_host[0])}), flush=True)


def run_train(args):
    """Index build cost from raw prefill keys: Lloyd k-means centroids and residual PQ codebooks
    (hsa_train_index), then encoding every indexed key (hsa_append_encode)."""
    import torch
    import sparse_long_context_pq_b200 as P
    from synth import make_batch, train_init_slots, workload
    from synth.device import index_tensors, kv_tensors
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    for name in ("llama8b_128k", "qwen30b_128k_append"):
        w = workload(name)
        bt = make_batch(w)
        kv = P.PagedKV(**kv_tensors(bt, dev))
        ix = P.PQIndex(**index_tensors(bt, dev, n_indexed=np.zeros(w.B, dtype=np.int32)))
        n_train = w.n_indexed
        init = torch.from_numpy(train_init_slots(w, n_train)).to(dev)
        ws = P.workspace(P.hsa_train_workspace_bytes(kv, ix, n_train), dev)
        ws_idx = P.workspace(P.hsa_index_workspace_bytes(kv, ix, n_train), dev)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def timed(fn, reps):
            t = []
            for i in range(reps + 1):          # the first call is the warm-up
                flush.zero_()
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                if i:
                    t.append(a.elapsed_time(b))
            return sum(t) / len(t)             # ms

        def train(ci, pi):
            return lambda: P.hsa_train_index(kv, ix, n_train, init, coarse_iters=ci, pq_iters=pi, workspace_buf=ws)

        def encode():
            ix.n_indexed.zero_()
            ix.n_indexed_host.zero_()
            P.hsa_append_encode(kv, ix, n_train, workspace_buf=ws_idx)

        reps = max(1, min(args.steps, 3))
        t0 = timed(train(0, 0), reps)           # seeding + one assignment + codeword seeding
        t1 = timed(train(1, 0), reps)
        tp = timed(train(0, 1), reps)
        tf = timed(train(args.train_iters, args.train_iters), reps)
        te = timed(encode, reps)
        assert P.hsa_read_error(ws) == 0 and P.hsa_read_error(ws_idx) == 0
        U = w.B * w.Hkv
        # nearest-centroid search: k.c for every key and centroid, as three bf16 tensor-core
        # products per centroid (the fp32 centroid split in three terms)
        tensor_flop = 6.0 * U * n_train * w.C * w.D
        peak = bf16_peak()
        achieved = tensor_flop / max(t0, 1e-9) / 1e9        # TFLOP/s; t0 also seeds the centres
        traffic = dram_traffic("assign_mma_kernel", name)
        print(json.dumps({
            "train": name, "units": U, "n_train": n_train, "C": w.C, "M": w.M, "ncode": w.ncode,
            "coarse_iters": args.train_iters, "pq_iters": args.train_iters,
            "train_ms": round(tf, 3), "coarse_iter_ms": round(t1 - t0, 3), "pq_iter_ms": round(tp - t0, 3),
            "fixed_ms": round(t0, 3), "encode_ms": round(te, 3), "build_ms": round(tf + te, 3),
            "roofline": {"kernel": "assign_mma_kernel", "bound": "tensor", "achieved": round(achieved, 1),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 3) if peak else None,
                         "traffic": traffic, "note": "achieved is a lower bound: the timed call (no Lloyd "
                         "iterations) also seeds the centroids and codewords and splits the centroids"},
            "timing": "CUDA events, L2 flushed before every call, mean of %d after one warm-up" % reps,
        }), flush=True)


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from synth import make_batch, workload
    w = workload(args.workload)
    bt = make_batch(w)
    per_step_seconds = max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(bt, w, w.budget, per_step_seconds / 4)
    t = []
    units_total = 0
    for _ in range(args.steps):
        us, units, el = oracle_sample(bt, w, w.budget, per_step_seconds)
        t.append(us)
        units_total += units
    us = sum(t) / len(t)
    res = {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us/step",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "ctx": w.T, "budget": w.budget},
        "cpu_baseline": {"value": round(us, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
                         "sample": f"each step: whole (sequence, KV head) units of the workload for "
                                   f"~{per_step_seconds:.1f} s, scaled to a full step of {w.B * w.Hkv} units "
                                   f"({units_total} units timed over {args.steps} steps)"},
        "e2e": {"value": round(us, 1), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.sweep == "ctx":
        run_sweep_ctx(args)
    elif args.sweep == "budget":
        run_sweep_budget(args)
    elif args.sweep == "batch":
        run_sweep_batch(args)
    elif args.append:
        run_append(args)
    elif args.train:
        run_train(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
