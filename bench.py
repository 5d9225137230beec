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
    ap.add_argument("--master-port", type=int, default=29511, help="rendezvous port when --gpus N spawns replicas")
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_128k")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="bound on the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-train-build", action="store_true", help="skip the index-build-from-keys measurement")
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
    """Per-step algorithmic HBM bytes (what one step must move at least) of PQ-HSA and of dense
    decode, the token-major cluster ids (layout overhead, reported apart), and the per-kernel
    split of the PQ-HSA bytes. Intermediates that stay in L2 (scores, partials, cluster
    weights) are not counted."""
    G, C, D = w.G, w.C, w.D
    R = w.T - w.n_sink - n_idx
    lut = 4 * G * 16 * 256                       # PQ look-up table (written once, read once)
    qc = 4 * G * C                               # q . centroid table (written once, read once)
    per_unit = (16 * n_idx                       # PQ codes
                + 4 * C * D                      # centroids (q . centroid)
                + 4 * 16 * 256 * 8               # codebook
                + lut                            # LUT written once
                + 4 * C * D + 4 * C              # cluster mean values + counts
                + 512 * (w.n_sink + R + k)       # exact K+V rows (bf16)
                + 8 * G * D)                     # q in, out
    ids = 2 * n_idx
    dense = 512 * w.T + 8 * G * D
    U = w.B * w.Hkv
    kernels = {
        "tables": U * (4 * C * D + 4 * 16 * 256 * 8 + 4 * G * D + lut + qc),   # reads + table writes
        "scan_select": U * (16 * n_idx + lut + qc),                             # codes + tables
        "attend": U * (512 * (w.n_sink + R + k) + 4 * C * D + 4 * C + 4 * G * D),
        "merge": U * 4 * G * D,                                                # out
    }
    return U * per_unit, U * ids, U * dense, kernels


def scan_wavefronts(G: int, chunks: int) -> int:
    """Shared-memory wavefronts of the scan's LUT gathers (its on-chip algorithmic work): per
    32-slot chunk 16 subspace look-ups, each a 128-bit load per lane per 4 heads (4 wavefronts
    for the 32 lanes of a warp when conflict-free)."""
    return chunks * 16 * 4 * ((G + 3) // 4)


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
# CPU oracle sample (reported baseline, never the target): a process pool over the
# (sequence, KV head) units, one single-threaded worker per core up to the unit count
# and a host-memory bound; the KV pool is shared with the workers, not copied.
# ---------------------------------------------------------------------------

_ORC = {}


def _orc_init(shm, small, n_sink, scale, budget, page_size):
    """Pool worker start: attach the shared K/V pool, keep the small arrays."""
    from multiprocessing import shared_memory
    views = {}
    handles = []
    for name, (shm_name, shape, dtype) in shm.items():
        h = shared_memory.SharedMemory(name=shm_name)
        handles.append(h)
        views[name] = np.ndarray(shape, dtype=dtype, buffer=h.buf)
    _ORC.update(views)
    _ORC.update(small)
    _ORC.update(handles=handles, n_sink=n_sink, scale=scale, budget=budget, page_size=page_size)


def _orc_unit(u):
    """One (sequence, KV head) unit of the oracle's decode step in this worker."""
    import oracle as O
    O.oracle_decode(_ORC["q"], _ORC["k_cache"], _ORC["v_cache"], _ORC["block_table"], _ORC["seq_lens"],
                    _ORC["centroids"], _ORC["codebooks"], _ORC["codes_rec"], _ORC["ids_rec"], _ORC["n_indexed"],
                    _ORC["n_sink"], _ORC["scale"], budget=_ORC["budget"], page_size=_ORC["page_size"], units=[u])
    return u


class OraclePool:
    """The float64 oracle on the host cores: whole decode steps, units spread over a pool of
    spawn-started single-threaded workers (BLAS limited to one thread each)."""

    def __init__(self, bt, w, budget, workers=None):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        import psutil
        self.units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
        # a worker widens one unit's K and V rows to float64 (plus temporaries)
        per_worker = 4 * 8 * w.T * w.D * 2 + (64 << 20)
        mem_cap = max(1, int(0.5 * psutil.virtual_memory().available // per_worker))
        self.workers = workers or max(1, min(os.cpu_count() or 1, len(self.units), mem_cap))
        self._shm = []
        spec = {}
        for name in ("k_cache", "v_cache"):
            arr = getattr(bt, name)
            h = shared_memory.SharedMemory(create=True, size=max(1, arr.nbytes))
            np.ndarray(arr.shape, dtype=arr.dtype, buffer=h.buf)[...] = arr
            self._shm.append(h)
            spec[name] = (h.name, arr.shape, arr.dtype)
        small = {n: getattr(bt, n) for n in ("q", "block_table", "seq_lens", "centroids", "codebooks", "codes_rec",
                                             "ids_rec", "n_indexed")}
        scale = float(np.float32(1.0 / math.sqrt(w.D)))
        env = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in env:
            os.environ[k] = "1"            # inherited by the spawned workers at start
        try:
            self.pool = mp.get_context("spawn").Pool(
                self.workers, initializer=_orc_init, initargs=(spec, small, w.n_sink, scale, budget, w.page_size))
        finally:
            for k, v in env.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v

    def step(self):
        """Wall seconds of one whole decode step (every unit) on the pool."""
        t0 = time.perf_counter()
        self.pool.map(_orc_unit, self.units, chunksize=1)
        return time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()
        for h in self._shm:
            h.close()
            h.unlink()


def oracle_sample(bt, w, budget, seconds: float, warmup: int = 1, min_steps: int = 1, max_steps: int = 1000):
    """Whole oracle steps on the pool until `seconds` elapse (at least min_steps); returns
    (µs per step, steps timed, worker count, seconds)."""
    pool = OraclePool(bt, w, budget)
    try:
        for _ in range(warmup):
            pool.step()
        t, el = [], 0.0
        while len(t) < max_steps and (len(t) < min_steps or el < seconds):
            t.append(pool.step())
            el += t[-1]
        return sum(t) / len(t) * 1e6, len(t), pool.workers, el
    finally:
        pool.close()


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
    # selected tokens per unit as the library counts them (the byte model's k)
    n_sel = P.selected_counts(kv, ix, q, scale=scale, budget=budget, workspace_buf=ws)
    n_chunks = int(ix.list_meta.view(w.B * w.Hkv, -1)[:, 0].sum())   # 32-slot chunks the scan streams
    k = int(n_sel.max())
    assert int(n_sel.min()) == k, "every unit of the workload selects the same count"

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
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(graph, steps, staged=None):
        """Whole steps: one graph replay each, L2 flushed before, CUDA events around. With
        staged = (q_view, out_view) every step also moves q in from and out back to pinned host
        memory by copy kernels that read and write mapped views of the pinned buffers."""
        t = []
        for _ in range(steps):
            flush.zero_()
            a.record()
            if staged is not None:
                torch.mul(staged[0], 1.0, out=q)
            graph.replay()
            if staged is not None:
                torch.mul(out, 1.0, out=staged[1])
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

    q_h = torch.from_numpy(bt.q).pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    prepared = P.DecodeStep(kv, ix, scale=scale, budget=budget)

    def e2e_steps(steps, use_prepared=True):
        """End to end through the public API, per step, by the host's wall clock, from pinned
        host memory to pinned host memory: the prepared step (hsa_decode_step_run: the library
        validates and plans, then replays the recorded host-buffer step as one graph launch), or,
        for comparison, hsa_decode marshalling every argument anew between torch copies in and
        out; then the wait for the result. L2 is flushed, and the flush finished, before each
        step."""
        t_wall, t_dev = [], []
        for _ in range(steps):
            flush.zero_()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            a.record()
            if use_prepared:
                prepared.host(q_h, out_h)
            else:
                q.copy_(q_h, non_blocking=True)
                P.hsa_decode(kv, ix, q, out, scale=scale, budget=budget, workspace_buf=ws)
                out_h.copy_(out, non_blocking=True)
            b.record()
            b.synchronize()
            t_wall.append((time.perf_counter() - t0) * 1e3)
            t_dev.append(a.elapsed_time(b))
        return t_wall, t_dev

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
        e2e_steps(1)
        e2e_steps(1, use_prepared=False)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_hsa = timed(g_hsa, args.steps)
        t_stage = timed_stages(args.steps)
        t_dense = timed(g_dense, args.steps)
        t_e2e, t_e2e_dev = e2e_steps(args.steps)
        t_e2e_call, _ = e2e_steps(args.steps, use_prepared=False)
        try:
            views = (mapped_view(q_h), mapped_view(out_h))
        except (RuntimeError, TypeError, ValueError):
            views = None
        t_staged = None
        if views is not None:
            timed(g_hsa, 2, staged=views)
            t_staged = timed(g_hsa, args.steps, staged=views)
            torch.cuda.synchronize()
            if not torch.equal(out_h, out.cpu()):      # the last step's result did not reach host memory
                t_staged = None
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    err = P.hsa_read_error(ws) | P.hsa_read_error(prepared.workspace_buf)
    assert err == 0, f"device error word {err}"

    train_build_ms = None
    if not args.no_train_build:
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
        train_build_ms = round(e0.elapsed_time(e1), 3)
        assert P.hsa_read_error(ws_t) == 0 and P.hsa_read_error(ws_e) == 0
        del ix_t, ws_t, ws_e

    mean = lambda t: sum(t) / len(t)
    ms_hsa, ms_dense, ms_e2e, ms_e2e_dev, ms_e2e_call = max_over_ranks(
        [mean(t_hsa), mean(t_dense), mean(t_e2e), mean(t_e2e_dev), mean(t_e2e_call)], dist if world > 1 else None,
        dev)

    stage_ms = [mean([s_[i] for s_ in t_stage]) for i in range(P.NUM_STAGES)]
    n_idx = int(w.n_indexed)
    hsa_b, ids_b, dense_b, kern_b = step_bytes(w, n_idx, k)
    peak, peak_kind = measured_peaks()
    dom = int(np.argmax(stage_ms))
    dom_name = P.STAGE_NAMES[dom]
    dom_bytes = kern_b[dom_name]
    dom_gbs = dom_bytes / (stage_ms[dom] * 1e-3) / 1e9
    step_gbs = hsa_b / (ms_hsa * 1e-3) / 1e9
    dense_gbs = dense_b / (ms_dense * 1e-3) / 1e9
    traffic = dram_traffic(dom_name + "_kernel", w.name)
    U = w.B * w.Hkv
    clk_sum = clk.summary()
    onchip = None
    if dom_name == "scan_select":
        # the same launch against its on-chip ceiling: one shared-memory wavefront per clock per SM
        wav = scan_wavefronts(w.G, n_chunks)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        mhz = clk_sum["sm_mhz"] or clk_sum["sm_max_mhz"] or 1965.0
        ceil_g = sms * mhz * 1e6 / 1e9
        ach_g = wav / (stage_ms[dom] * 1e-3) / 1e9
        onchip = {"bound": "shared-memory wavefronts (LUT gathers)", "algorithmic": wav,
                  "achieved": round(ach_g, 1), "peak": round(ceil_g, 1), "unit": "G wavefronts/s",
                  "frac": round(ach_g / ceil_g, 4), "peak_basis": f"{sms} SMs x 1 wavefront/clock x {mhz:.0f} MHz"}

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
        "percentiles_us": {f"p{q_}": round(float(np.percentile(t_hsa, q_)) * 1e3, 3) for q_ in (10, 50, 90)},
        "hbm_gbs": round(step_gbs, 1),
        "hbm_pct_peak": round(100 * step_gbs / peak, 2),
        "bytes_per_step": hsa_b,
        "ids_bytes_per_step": ids_b,
        "dense": {"us_per_step": round(ms_dense * 1e3, 3), "bytes_per_step": dense_b,
                  "hbm_gbs": round(dense_gbs, 1), "pct_peak": round(100 * dense_gbs / peak, 2),
                  "speedup_of_pqhsa": round(ms_dense / ms_hsa, 3)},
        "stages_us": {n: round(v * 1e3, 3) for n, v in zip(P.STAGE_NAMES, stage_ms)},
        "stage_bytes": kern_b,
        "index_build_ms": round(build_ms, 3),
        "index_train_and_encode_ms": train_build_ms,
        "roofline": {"kernel": dom_name, "bound": "hbm", "achieved": round(dom_gbs, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                     "traffic": traffic, "algorithmic_bytes": dom_bytes,
                     "traffic_over_algorithmic": round(traffic / dom_bytes, 3) if traffic else None,
                     "duration_us": round(stage_ms[dom] * 1e3, 3), "onchip": onchip},
        "e2e": {"value": round(ms_e2e * 1e3, 3), "unit": "us/step", "h2d_bytes_per_step": q.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 4,
                "how": "host wall clock per step, page-locked host q to page-locked host out: one C-ABI "
                       "hsa_decode_step_run call through the prepared DecodeStep (validation and split plan "
                       "every call, then one CUDA-graph launch of the host-buffer step: q staged by a copy "
                       "kernel, the four decode kernels, out written to host memory by the merge), then the "
                       "wait",
                "device_us": round(ms_e2e_dev * 1e3, 3),
                "hsa_decode_call_us": round(ms_e2e_call * 1e3, 3),   # torch copies + per-call marshalling
                "graph_staged_us": round(mean(t_staged) * 1e3, 3) if t_staged else None},
        # our kernels in the timed region: graph steps (4 each), eager stage-timed steps (4),
        # dense graph steps (attend + merge), end-to-end calls of both kinds (4 each), staged
        # graph steps (4, + 2 warm)
        "gpu_launches": args.steps * (4 * P.NUM_STAGES + 2) + (
            (args.steps + 2) * P.NUM_STAGES if t_staged is not None else 0),
        "clocks": clk_sum,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        us, steps, workers, el = oracle_sample(bt, w, budget, args.cpu_seconds)
        res["cpu_baseline"] = {"value": round(us, 1), "unit": "us/step", "cores": workers, "kind": "oracle",
                               "sample": f"{steps} whole decode steps ({U} (sequence, KV head) units each, "
                                         f"spread over {workers} single-threaded float64 numpy worker "
                                         f"processes), {el:.1f} s"}
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

    def k_selected(self, budget=0.01):
        """Selected tokens per unit as the library reports them (every unit alike here)."""
        n = self.P.selected_counts(self.kv, self.ix, self.q, scale=self.scale, budget=budget, workspace_buf=self.ws)
        assert int(n.min()) == int(n.max())
        return int(n.max())

    def hsa(self, budget=0.01, background=True):
        return lambda: self.P.hsa_decode(self.kv, self.ix, self.q, self.out, scale=self.scale, budget=budget,
                                         background=background, workspace_buf=self.ws)

    def dense(self):
        return lambda: self.P.dense_decode(self.kv, self.q, self.out_dense, scale=self.scale,
                                           workspace_buf=self.ws_dense)


# Overhead-aware crossover model (rit.work "activation-kv-cache-sparsity-crossover", section
# "Почему один и тот же способ даёт разное ускорение": a byte count gives the direction,
# and adding each kernel's fixed launch and index cost predicts the measured crossover).

def fit_overhead_model(nbytes, times_us):
    """Least-squares fit of t = t0 + nbytes / bw to measured points; returns (t0 in µs, bw in
    bytes per µs)."""
    x = np.asarray(nbytes, dtype=np.float64)
    y = np.asarray(times_us, dtype=np.float64)
    A = np.stack([np.ones_like(x), x], axis=1)
    (t0, slope), *_ = np.linalg.lstsq(A, y, rcond=None)
    return float(t0), float(1.0 / slope) if slope > 0 else float("inf")


def model_time(fit, nbytes):
    t0, bw = fit
    return t0 + nbytes / bw


def predicted_crossover(fit_sparse, fit_dense, bytes_at, lengths):
    """First length (of the increasing `lengths`) where the fitted sparse time is at most the
    fitted dense time; bytes_at(T) gives (sparse bytes, dense bytes) at length T. None if never."""
    for T in lengths:
        hb, db = bytes_at(T)
        if model_time(fit_sparse, hb) <= model_time(fit_dense, db):
            return T
    return None


def measured_crossover(points):
    """Length where the measured sparse and dense times cross, by linear interpolation of
    (dense - sparse) between the two measured lengths that bracket the sign change;
    points = [(T, sparse_us, dense_us)]. None if sparse never overtakes; the first length
    if it already leads there."""
    pts = sorted(points)
    if pts and pts[0][2] - pts[0][1] >= 0:
        return float(pts[0][0])
    for (t0, h0, d0), (t1, h1, d1) in zip(pts, pts[1:]):
        g0, g1 = d0 - h0, d1 - h1
        if g0 < 0 <= g1:
            return float(t0 + (t1 - t0) * (-g0) / (g1 - g0))
    return None


SWEEP_LENGTHS = (8192, 16384, 32768, 49152, 65536, 98304, 131072, 524288)


def run_sweep_ctx(args):
    import torch
    from synth import workload
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, _ = measured_peaks()
    pts = []
    base = workload("llama8b_8k")
    for T in SWEEP_LENGTHS:
        w = base.scaled(T=T, name=f"llama8b_sweep_{T // 1024}k")
        S = _Setup(w, dev)
        k = S.k_selected()
        hsa_b, ids_b, dense_b, _ = step_bytes(w, w.n_indexed, k)
        us_h = S.time_graph(S.graph(S.hsa()), args.steps, args.warmup)
        us_d = S.time_graph(S.graph(S.dense()), args.steps, args.warmup)
        assert S.P.hsa_read_error(S.ws) == 0
        print(json.dumps({"sweep": "ctx", "workload": w.name, "T": w.T, "k": k, "hsa_us": round(us_h, 3),
                          "dense_us": round(us_d, 3), "speedup": round(us_d / us_h, 3),
                          "hsa_bytes": hsa_b, "ids_bytes": ids_b, "dense_bytes": dense_b,
                          "hsa_gbs": round(hsa_b / us_h / 1e3, 1), "dense_gbs": round(dense_b / us_d / 1e3, 1),
                          "dense_pct_peak": round(100 * dense_b / us_d / 1e3 / peak, 2)}), flush=True)
        pts.append((w, hsa_b, dense_b, us_h, us_d))
        del S
        torch.cuda.empty_cache()
    fh = fit_overhead_model([p_[1] for p_ in pts], [p_[3] for p_ in pts])
    fd = fit_overhead_model([p_[2] for p_ in pts], [p_[4] for p_ in pts])

    def bytes_at(T):
        wt = base.scaled(T=T)
        hb, _, db, _ = step_bytes(wt, wt.n_indexed, int(math.floor(wt.budget * wt.n_indexed)))
        return hb, db

    pred = predicted_crossover(fh, fd, bytes_at, range(2048, 1 << 21, 256))
    meas = measured_crossover([(p_[0].T, p_[3], p_[4]) for p_ in pts])
    print(json.dumps({"sweep": "ctx-model", "hsa_fixed_us": round(fh[0], 2), "hsa_gbs": round(fh[1] / 1e3, 1),
                      "dense_fixed_us": round(fd[0], 2), "dense_gbs": round(fd[1] / 1e3, 1),
                      "predicted_crossover_T": pred,
                      "measured_crossover_T": None if meas is None else round(meas),
                      "lengths": list(SWEEP_LENGTHS)}), flush=True)


def run_sweep_batch(args):
    """32 sequences x 32K context (shuffled pages, per-sequence seeds) at 1 %: PQ-HSA vs dense."""
    import torch
    from synth import workload
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, _ = measured_peaks()
    w = workload("batch32_32k")
    S = _Setup(w, dev)
    k = S.k_selected(w.budget)
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
    pool = OraclePool(bt, w, w.budget)
    try:
        for _ in range(args.warmup):
            pool.step()
        t = [pool.step() for _ in range(args.steps)]
    finally:
        pool.close()
    us = sum(t) / len(t) * 1e6
    U = w.B * w.Hkv
    res = {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us/step",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no dataset or weights)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.D, "ctx": w.T,
                   "clusters": w.C, "pq": "16x8/256", "sink": w.n_sink, "recent": w.n_recent,
                   "budget": w.budget, "k": w.k, "page_size": w.page_size, "parallelism": "host cores",
                   "l2": "n/a (host)", "timing": "host wall clock per whole step"},
        "cpu_baseline": {"value": round(us, 1), "unit": "us/step", "cores": pool.workers, "kind": "oracle",
                         "sample": f"{args.steps} whole decode steps ({U} (sequence, KV head) units each, "
                                   f"spread over {pool.workers} single-threaded float64 numpy worker processes)"},
        "e2e": {"value": round(us, 1), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def spawn_replicas(args, argv):
    """`--gpus N` without a launcher: run N replicas, one process per GPU, under torch's launcher
    (the same command the multi-GPU runs use); returns its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={args.master_port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world and args.impl == "ours" and not (args.sweep or args.append or args.train):
        if "WORLD_SIZE" in os.environ:
            sys.exit(f"--gpus {args.gpus} but the launcher started {world} ranks")
        sys.exit(spawn_replicas(args, argv))
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
