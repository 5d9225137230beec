"""PQ-HSA sparse decode attention for B200 (sm_100a): Python binding of libpqhsa.so.

Every step of the decode path runs in the library's CUDA kernels; this module only
marshals torch tensors (device memory) and the current CUDA stream into the C ABI
declared in include/pqhsa.h. There is no CPU fallback: importing works without a
GPU, but every compute call needs the built library and a CUDA device.

Method: rit.work "pq-hsa-long-context-attention" (PQ-HSA).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from . import build as _build

__all__ = [
    "PagedKV", "PQIndex", "HSAError", "load_library", "hsa_decode", "hsa_decode_host", "dense_decode",
    "hsa_build_from_codes", "hsa_append_encode", "hsa_decode_workspace_bytes", "hsa_decode_host_workspace_bytes",
    "dense_decode_workspace_bytes", "hsa_index_workspace_bytes", "hsa_read_error", "hsa_strerror",
    "selected_counts", "DecodeStep", "HSA_DEVERR_PAGE", "HSA_DEVERR_CLUSTER", "HSA_DEVERR_TIMEOUT",
    "HSA_DEVERR_SELECT",
]

HSA_DEVERR_PAGE, HSA_DEVERR_CLUSTER, HSA_DEVERR_TIMEOUT, HSA_DEVERR_SELECT = 1, 2, 4, 8
M_SUB, DSUB, NCODE, HEAD_DIM = 16, 8, 256, 128


class _KV(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("seq_lens_host", ctypes.c_void_p),
                ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("D", ctypes.c_int32), ("page_size", ctypes.c_int32), ("max_pages", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


class _Index(ctypes.Structure):
    _fields_ = [("centroids", ctypes.c_void_p), ("codebooks", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("ids", ctypes.c_void_p), ("sum_v", ctypes.c_void_p), ("mean_v", ctypes.c_void_p),
                ("count", ctypes.c_void_p), ("n_indexed", ctypes.c_void_p), ("n_indexed_host", ctypes.c_void_p),
                ("list_codes", ctypes.c_void_p), ("list_slot", ctypes.c_void_p),
                ("chunk_cluster", ctypes.c_void_p), ("list_meta", ctypes.c_void_p),
                ("C", ctypes.c_int32), ("M", ctypes.c_int32), ("dsub", ctypes.c_int32),
                ("ncode", ctypes.c_int32), ("cap", ctypes.c_int32), ("n_sink", ctypes.c_int32),
                ("list_slots", ctypes.c_int32)]


def index_list_slots(cap: int, C: int) -> int:
    """List slots per unit the cluster-ordered code lists need: 32 * (ceil(cap / 32) + C)."""
    return 32 * ((cap + 31) // 32 + C)


class _Params(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("budget", ctypes.c_double), ("k_override", ctypes.c_int32),
                ("background", ctypes.c_int32)]


class _Debug(ctypes.Structure):
    _fields_ = [("approx_logits", ctypes.c_void_p), ("selected", ctypes.c_void_p),
                ("n_selected", ctypes.c_void_p), ("stage_events", ctypes.c_void_p)]


NUM_STAGES = 4
STAGE_NAMES = ("tables", "scan_select", "attend", "merge")


EXPORTS = ("hsa_decode", "hsa_decode_host", "hsa_decode_step_create", "hsa_decode_step_run",
           "hsa_decode_step_destroy", "dense_decode", "hsa_build_from_codes", "hsa_append_encode",
           "hsa_index_list_slots", "hsa_decode_workspace_bytes", "hsa_decode_host_workspace_bytes",
           "dense_decode_workspace_bytes", "hsa_index_workspace_bytes",
           "hsa_read_error", "hsa_strerror", "hsa_abi_sizes")

_lib = None


class HSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {hsa_strerror(status)} (status {status})")
        self.status = status


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libpqhsa.so (built in-tree by sparse_long_context_pq_b200.build). Raises if missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or os.environ.get("PQHSA_LIB", _build.LIB_PATH)
    if not os.path.exists(path):
        raise RuntimeError(f"libpqhsa.so not found at {path}; build it with "
                           f"`python -m sparse_long_context_pq_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.hsa_decode.argtypes = [P(_KV), P(_Index), vp, vp, P(_Params), P(_Debug), vp, sz, vp]
    lib.hsa_decode_host.argtypes = [P(_KV), P(_Index), vp, vp, P(_Params), vp, sz, vp]
    lib.hsa_decode_host_workspace_bytes.argtypes = [P(_KV), P(_Index)]
    lib.hsa_decode_step_create.argtypes = [P(_KV), P(_Index), P(_Params), vp, sz, P(vp)]
    lib.hsa_decode_step_run.argtypes = [vp, vp, vp, vp]
    lib.hsa_decode_step_destroy.argtypes = [vp]
    lib.hsa_decode_step_destroy.restype = None
    lib.dense_decode.argtypes = [P(_KV), vp, vp, ctypes.c_float, vp, sz, vp]
    lib.hsa_build_from_codes.argtypes = [P(_KV), P(_Index), vp, sz, vp]
    lib.hsa_append_encode.argtypes = [P(_KV), P(_Index), i32, vp, sz, vp]
    lib.hsa_train_workspace_bytes.argtypes = [P(_KV), P(_Index), i32]
    lib.hsa_train_index.argtypes = [P(_KV), P(_Index), i32, vp, i32, i32, vp, vp, sz, vp]
    lib.hsa_decode_workspace_bytes.argtypes = [P(_KV), P(_Index)]
    lib.dense_decode_workspace_bytes.argtypes = [P(_KV)]
    lib.hsa_index_workspace_bytes.argtypes = [P(_KV), P(_Index), i32]
    lib.hsa_read_error.argtypes = [vp, P(i32), vp]
    lib.hsa_strerror.argtypes = [ctypes.c_int]
    lib.hsa_abi_sizes.argtypes = [P(ctypes.c_int64)] * 4
    for f in ("hsa_decode", "hsa_decode_host", "hsa_decode_step_create", "hsa_decode_step_run", "dense_decode",
              "hsa_build_from_codes", "hsa_append_encode", "hsa_read_error", "hsa_train_index"):
        getattr(lib, f).restype = ctypes.c_int
    for f in ("hsa_decode_workspace_bytes", "hsa_decode_host_workspace_bytes", "dense_decode_workspace_bytes",
              "hsa_index_workspace_bytes", "hsa_train_workspace_bytes"):
        getattr(lib, f).restype = sz
    lib.hsa_strerror.restype = ctypes.c_char_p
    lib.hsa_abi_sizes.restype = None
    sizes = [ctypes.c_int64() for _ in range(4)]
    lib.hsa_abi_sizes(*[ctypes.byref(s) for s in sizes])
    mine = [ctypes.sizeof(t) for t in (_KV, _Index, _Params, _Debug)]
    if [s.value for s in sizes] != mine:
        raise RuntimeError(f"ABI struct size mismatch: library {[s.value for s in sizes]} vs binding {mine}")
    if path == _build.LIB_PATH or "PQHSA_LIB" in os.environ:
        _lib = lib
    return lib


def hsa_strerror(status: int) -> str:
    return load_library().hsa_strerror(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _on_gpu(*ts: Optional[torch.Tensor]) -> None:
    """The library dereferences these on the device: a host tensor here would be a bad address."""
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("expected a CUDA tensor, got one on " + str(t.device))


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, status: int):
    if status != 0:
        raise HSAError(fn, status)


@dataclass
class PagedKV:
    """Paged bf16 KV cache [num_pages][Hkv][page_size][D] plus the block table and lengths."""

    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: torch.Tensor      # int32 [B, max_pages] (device)
    seq_lens: torch.Tensor         # int32 [B] (device)
    seq_lens_host: torch.Tensor    # int32 [B] (cpu)
    Hq: int

    def struct(self) -> _KV:
        P, Hkv, ps, D = self.k_cache.shape
        B, maxp = self.block_table.shape
        assert self.k_cache.dtype == torch.bfloat16 and self.v_cache.dtype == torch.bfloat16
        assert self.block_table.dtype == torch.int32 and self.seq_lens.dtype == torch.int32
        assert self.seq_lens_host.dtype == torch.int32 and self.seq_lens_host.device.type == "cpu"
        assert self.k_cache.is_contiguous() and self.v_cache.is_contiguous() and self.block_table.is_contiguous()
        _on_gpu(self.k_cache, self.v_cache, self.block_table, self.seq_lens)
        return _KV(_ptr(self.k_cache), _ptr(self.v_cache), _ptr(self.block_table), _ptr(self.seq_lens),
                   _ptr(self.seq_lens_host), B, self.Hq, Hkv, D, ps, maxp, P)

    @property
    def B(self) -> int:
        return self.block_table.shape[0]

    @property
    def Hkv(self) -> int:
        return self.k_cache.shape[1]


@dataclass
class PQIndex:
    """Per-(sequence, KV head) IVF-PQ index storage (caller-owned device tensors)."""

    centroids: torch.Tensor        # fp32 [B, Hkv, C, D]
    codebooks: torch.Tensor        # fp32 [B, Hkv, M, 256, 8]
    codes: torch.Tensor            # uint8 [B, Hkv, cap, M]
    ids: torch.Tensor              # int16 storage of u16 cluster ids [B, Hkv, cap]
    sum_v: torch.Tensor            # fp32 [B, Hkv, C, D]
    mean_v: torch.Tensor           # fp32 [B, Hkv, C, D]
    count: torch.Tensor            # int32 [B, Hkv, C]
    n_indexed: torch.Tensor        # int32 [B] (device)
    n_indexed_host: torch.Tensor   # int32 [B] (cpu)
    n_sink: int
    list_codes: Optional[torch.Tensor] = None     # uint8 [B, Hkv, list_slots, M]  (library-maintained)
    list_slot: Optional[torch.Tensor] = None      # int32 [B, Hkv, list_slots]
    chunk_cluster: Optional[torch.Tensor] = None  # int16 storage of u16 [B, Hkv, list_slots / 32]
    list_meta: Optional[torch.Tensor] = None      # int32 [B, Hkv, 2 + 2C]

    def __post_init__(self):
        if self.list_codes is None:
            B, Hkv, cap, _ = self.codes.shape
            C = self.centroids.shape[2]
            ls = index_list_slots(cap, C)
            dev = self.codes.device
            self.list_codes = torch.zeros(B, Hkv, ls, M_SUB, device=dev, dtype=torch.uint8)
            self.list_slot = torch.full((B, Hkv, ls), -1, device=dev, dtype=torch.int32)
            self.chunk_cluster = torch.zeros(B, Hkv, ls // 32, device=dev, dtype=torch.int16)
            self.list_meta = torch.zeros(B, Hkv, 2 + 2 * C, device=dev, dtype=torch.int32)

    @staticmethod
    def allocate(B: int, Hkv: int, C: int, cap: int, n_sink: int, device) -> "PQIndex":
        f = dict(device=device, dtype=torch.float32)
        return PQIndex(
            centroids=torch.zeros(B, Hkv, C, HEAD_DIM, **f),
            codebooks=torch.zeros(B, Hkv, M_SUB, NCODE, DSUB, **f),
            codes=torch.zeros(B, Hkv, cap, M_SUB, device=device, dtype=torch.uint8),
            ids=torch.zeros(B, Hkv, cap, device=device, dtype=torch.int16),
            sum_v=torch.zeros(B, Hkv, C, HEAD_DIM, **f),
            mean_v=torch.zeros(B, Hkv, C, HEAD_DIM, **f),
            count=torch.zeros(B, Hkv, C, device=device, dtype=torch.int32),
            n_indexed=torch.zeros(B, device=device, dtype=torch.int32),
            n_indexed_host=torch.zeros(B, dtype=torch.int32),
            n_sink=n_sink,
        )

    @property
    def C(self) -> int:
        return self.centroids.shape[2]

    @property
    def cap(self) -> int:
        return self.codes.shape[2]

    def struct(self) -> _Index:
        for t in (self.centroids, self.codebooks, self.codes, self.ids, self.sum_v, self.mean_v, self.count,
                  self.list_codes, self.list_slot, self.chunk_cluster, self.list_meta):
            assert t.is_contiguous()
        assert self.n_indexed_host.device.type == "cpu" and self.n_indexed_host.dtype == torch.int32
        _on_gpu(self.centroids, self.codebooks, self.codes, self.ids, self.sum_v, self.mean_v, self.count,
                self.n_indexed, self.list_codes, self.list_slot, self.chunk_cluster, self.list_meta)
        return _Index(_ptr(self.centroids), _ptr(self.codebooks), _ptr(self.codes), _ptr(self.ids),
                      _ptr(self.sum_v), _ptr(self.mean_v), _ptr(self.count), _ptr(self.n_indexed),
                      _ptr(self.n_indexed_host), _ptr(self.list_codes), _ptr(self.list_slot),
                      _ptr(self.chunk_cluster), _ptr(self.list_meta), self.C, M_SUB, DSUB, NCODE, self.cap,
                      self.n_sink, self.list_codes.shape[2])


def hsa_decode_workspace_bytes(kv: PagedKV, index: PQIndex) -> int:
    kvs, ixs = kv.struct(), index.struct()
    n = load_library().hsa_decode_workspace_bytes(ctypes.byref(kvs), ctypes.byref(ixs))
    if n == 0:
        raise HSAError("hsa_decode_workspace_bytes", 1)
    return int(n)


def hsa_decode_host_workspace_bytes(kv: PagedKV, index: PQIndex) -> int:
    kvs, ixs = kv.struct(), index.struct()
    n = load_library().hsa_decode_host_workspace_bytes(ctypes.byref(kvs), ctypes.byref(ixs))
    if n == 0:
        raise HSAError("hsa_decode_host_workspace_bytes", 1)
    return int(n)


def _check_host_io(t: torch.Tensor, shape, name: str) -> None:
    """hsa_decode_host reads and writes these on the host (pinned memory keeps the copies
    asynchronous)."""
    if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected a contiguous fp32 host tensor {list(shape)}")


def dense_decode_workspace_bytes(kv: PagedKV) -> int:
    kvs = kv.struct()
    n = load_library().dense_decode_workspace_bytes(ctypes.byref(kvs))
    if n == 0:
        raise HSAError("dense_decode_workspace_bytes", 1)
    return int(n)


def hsa_index_workspace_bytes(kv: PagedKV, index: PQIndex, n_new: int = 0) -> int:
    """Workspace of hsa_append_encode(kv, index, n_new) (n_new = 0: of hsa_build_from_codes)."""
    kvs, ixs = kv.struct(), index.struct()
    return int(load_library().hsa_index_workspace_bytes(ctypes.byref(kvs), ctypes.byref(ixs), int(n_new)))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed workspace buffer (torch allocations are 256-byte aligned)."""
    return torch.zeros(max(256, (nbytes + 255) // 256 * 256), dtype=torch.uint8, device=device)


def hsa_decode(kv: PagedKV, index: PQIndex, q: torch.Tensor, out: Optional[torch.Tensor] = None, *,
               scale: float, budget: float = 0.01, k_override: int = -1, background: bool = True,
               approx_logits: Optional[torch.Tensor] = None, selected: Optional[torch.Tensor] = None,
               n_selected: Optional[torch.Tensor] = None, workspace_buf: Optional[torch.Tensor] = None,
               stage_events=None, stream=None) -> torch.Tensor:
    """One PQ-HSA decode step (see hsa_decode in include/pqhsa.h). q, out: fp32 [B, Hq, D]."""
    assert q.dtype == torch.float32 and q.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    kvs, ixs = kv.struct(), index.struct()
    lib = load_library()
    if workspace_buf is None:
        workspace_buf = workspace(hsa_decode_workspace_bytes(kv, index), q.device)
    prm = _Params(float(scale), float(budget), int(k_override), 1 if background else 0)
    ev_arr = None
    if stage_events is not None:
        assert len(stage_events) == NUM_STAGES + 1
        ev_arr = (ctypes.c_void_p * (NUM_STAGES + 1))(*[e.cuda_event for e in stage_events])
    _on_gpu(q, out, approx_logits, selected, n_selected, workspace_buf)
    dbg = _Debug(_ptr(approx_logits), _ptr(selected), _ptr(n_selected),
                 ctypes.cast(ev_arr, ctypes.c_void_p) if ev_arr is not None else None)
    st = lib.hsa_decode(ctypes.byref(kvs), ctypes.byref(ixs), q.data_ptr(), out.data_ptr(), ctypes.byref(prm),
                        ctypes.byref(dbg), workspace_buf.data_ptr(), workspace_buf.numel(), _stream(stream))
    _check("hsa_decode", st)
    return out


class DecodeStep:
    """hsa_decode prepared for one cache, index and workspace, for a decode loop: the C-ABI
    views of the cache and the index, the parameters and the workspace are checked and
    marshalled once here, and each call passes only q, out and the stream (the library still
    validates every call, lengths included). The tensors must keep their storage while the
    step is in use; their contents (lengths, appended tokens, lists) may change between calls.
    Calling the step runs it on device q / out: by default as one hsa_decode call, or with
    graph=True as the library's prepared step (hsa_decode_step_run: one CUDA graph launch per
    call while the split plan and the buffers stay the same - worth it when a loop reuses
    the same q and out tensors). .host() runs it on page-locked host q / out: by default as
    the prepared step, or with graph=False as one hsa_decode_host call. The workspace is
    sized for all of them.
    """

    def __init__(self, kv: PagedKV, index: PQIndex, *, scale: float, budget: float = 0.01, k_override: int = -1,
                 background: bool = True, workspace_buf: Optional[torch.Tensor] = None):
        self.kv, self.index = kv, index          # keep the tensors behind the views alive
        self._kvs, self._ixs = kv.struct(), index.struct()
        if workspace_buf is None:
            workspace_buf = workspace(hsa_decode_host_workspace_bytes(kv, index), kv.k_cache.device)
        _on_gpu(workspace_buf)
        self.workspace_buf = workspace_buf
        self._prm = _Params(float(scale), float(budget), int(k_override), 1 if background else 0)
        self._shape = (kv.B, kv.Hq, kv.k_cache.shape[3])
        self._device = kv.k_cache.device
        self._fn = load_library().hsa_decode
        self._fn_host = load_library().hsa_decode_host
        self._kv_ref, self._ix_ref = ctypes.byref(self._kvs), ctypes.byref(self._ixs)
        self._prm_ref = ctypes.byref(self._prm)
        self._ws_ptr, self._ws_len = workspace_buf.data_ptr(), workspace_buf.numel()
        self._lib = load_library()
        self._handle = ctypes.c_void_p(None)
        self._host_ok = None   # (q_host, out_host, their data pointers) last checked

    def _check_io(self, t: torch.Tensor, name: str) -> None:
        if (t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != self._shape
                or t.device != self._device):
            raise ValueError(f"{name}: expected a contiguous fp32 tensor {list(self._shape)} on {self._device}")

    def __call__(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None,
                 graph: bool = False) -> torch.Tensor:
        self._check_io(q, "q")
        if out is None:
            out = torch.empty_like(q)
        else:
            self._check_io(out, "out")
        if graph:
            self._run_step(q, out, stream)
            return out
        st = self._fn(self._kv_ref, self._ix_ref, q.data_ptr(), out.data_ptr(), self._prm_ref, None, self._ws_ptr,
                      self._ws_len, _stream(stream))
        _check("hsa_decode", st)
        return out

    def _run_step(self, q: torch.Tensor, out: torch.Tensor, stream) -> None:
        if not self._handle.value:
            _check("hsa_decode_step_create",
                   self._lib.hsa_decode_step_create(self._kv_ref, self._ix_ref, self._prm_ref, self._ws_ptr,
                                                    self._ws_len, ctypes.byref(self._handle)))
        _check("hsa_decode_step_run",
               self._lib.hsa_decode_step_run(self._handle, q.data_ptr(), out.data_ptr(), _stream(stream)))

    def host(self, q_host: torch.Tensor, out_host: torch.Tensor, stream=None, graph: bool = True) -> torch.Tensor:
        """q in from and out back to host memory, queued on the stream (out_host holds the result
        once the stream has reached it). A decode loop passes the same two buffers every step:
        they are checked once, and again whenever another tensor or storage comes in."""
        ok = self._host_ok
        if (ok is None or ok[0] is not q_host or ok[1] is not out_host or ok[2] != q_host.data_ptr()
                or ok[3] != out_host.data_ptr()):
            _check_host_io(q_host, self._shape, "q_host")
            _check_host_io(out_host, self._shape, "out_host")
            self._host_ok = (q_host, out_host, q_host.data_ptr(), out_host.data_ptr())
        if not graph:
            st = self._fn_host(self._kv_ref, self._ix_ref, q_host.data_ptr(), out_host.data_ptr(), self._prm_ref,
                               self._ws_ptr, self._ws_len, _stream(stream))
            _check("hsa_decode_host", st)
            return out_host
        self._run_step(q_host, out_host, stream)
        return out_host

    def close(self) -> None:
        """Release the library's prepared step (after its queued work has finished)."""
        if getattr(self, "_handle", None) is not None and self._handle.value:
            self._lib.hsa_decode_step_destroy(self._handle)
            self._handle = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def hsa_decode_host(kv: PagedKV, index: PQIndex, q_host: torch.Tensor, out_host: torch.Tensor, *, scale: float,
                    budget: float = 0.01, k_override: int = -1, background: bool = True,
                    workspace_buf: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """hsa_decode with q and out in host memory (see hsa_decode_host in include/pqhsa.h).
    Queued on the stream: out_host holds the result once the stream has reached it."""
    shape = (kv.B, kv.Hq, kv.k_cache.shape[3])
    _check_host_io(q_host, shape, "q_host")
    _check_host_io(out_host, shape, "out_host")
    kvs, ixs = kv.struct(), index.struct()
    if workspace_buf is None:
        workspace_buf = workspace(hsa_decode_host_workspace_bytes(kv, index), kv.k_cache.device)
    _on_gpu(workspace_buf)
    prm = _Params(float(scale), float(budget), int(k_override), 1 if background else 0)
    st = load_library().hsa_decode_host(ctypes.byref(kvs), ctypes.byref(ixs), q_host.data_ptr(), out_host.data_ptr(),
                                        ctypes.byref(prm), workspace_buf.data_ptr(), workspace_buf.numel(),
                                        _stream(stream))
    _check("hsa_decode_host", st)
    return out_host


def selected_counts(kv: PagedKV, index: PQIndex, q: torch.Tensor, *, scale: float, budget: float = 0.01,
                    k_override: int = -1, background: bool = True,
                    workspace_buf: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Selected tokens per (sequence, KV head) as hsa_decode reports them: int32 [B, Hkv] on the
    host, from one decode step with the n_selected debug output (synchronises the stream)."""
    n_sel = torch.full((kv.B, kv.Hkv), -1, dtype=torch.int32, device=q.device)
    hsa_decode(kv, index, q, scale=scale, budget=budget, k_override=k_override, background=background,
               n_selected=n_sel, workspace_buf=workspace_buf)
    return n_sel.cpu()


def dense_decode(kv: PagedKV, q: torch.Tensor, out: Optional[torch.Tensor] = None, *, scale: float,
                 workspace_buf: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense split-K GQA decode over every token (see dense_decode in include/pqhsa.h)."""
    assert q.dtype == torch.float32 and q.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    kvs = kv.struct()
    if workspace_buf is None:
        workspace_buf = workspace(dense_decode_workspace_bytes(kv), q.device)
    _on_gpu(q, out, workspace_buf)
    st = load_library().dense_decode(ctypes.byref(kvs), q.data_ptr(), out.data_ptr(), ctypes.c_float(scale),
                                     workspace_buf.data_ptr(), workspace_buf.numel(), _stream(stream))
    _check("dense_decode", st)
    return out


def hsa_build_from_codes(kv: PagedKV, index: PQIndex, workspace_buf: Optional[torch.Tensor] = None,
                         stream=None) -> None:
    """count / sum_v / mean_v of every cluster from the caller's codes and ids."""
    kvs, ixs = kv.struct(), index.struct()
    if workspace_buf is None:
        workspace_buf = workspace(hsa_index_workspace_bytes(kv, index), index.centroids.device)
    _on_gpu(workspace_buf)
    st = load_library().hsa_build_from_codes(ctypes.byref(kvs), ctypes.byref(ixs), workspace_buf.data_ptr(),
                                             workspace_buf.numel(), _stream(stream))
    _check("hsa_build_from_codes", st)


def hsa_append_encode(kv: PagedKV, index: PQIndex, n_new: int, workspace_buf: Optional[torch.Tensor] = None,
                      stream=None) -> None:
    """Encode the next n_new tokens of every sequence into the index (advances n_indexed)."""
    kvs, ixs = kv.struct(), index.struct()
    if workspace_buf is None:
        workspace_buf = workspace(hsa_index_workspace_bytes(kv, index, n_new), index.centroids.device)
    _on_gpu(workspace_buf)
    st = load_library().hsa_append_encode(ctypes.byref(kvs), ctypes.byref(ixs), int(n_new),
                                          workspace_buf.data_ptr(), workspace_buf.numel(), _stream(stream))
    _check("hsa_append_encode", st)


def hsa_train_workspace_bytes(kv: PagedKV, index: PQIndex, n_train: int) -> int:
    kvs, ixs = kv.struct(), index.struct()
    n = load_library().hsa_train_workspace_bytes(ctypes.byref(kvs), ctypes.byref(ixs), int(n_train))
    if n == 0:
        raise HSAError("hsa_train_workspace_bytes", 1)
    return int(n)


def hsa_train_index(kv: PagedKV, index: PQIndex, n_train: int, init_slots: torch.Tensor, *,
                    coarse_iters: int = 8, pq_iters: int = 8, assign_out: Optional[torch.Tensor] = None,
                    workspace_buf: Optional[torch.Tensor] = None, stream=None) -> None:
    """Train index.centroids / index.codebooks by Lloyd k-means on the keys at positions
    [n_sink, n_sink + n_train) (see hsa_train_index in include/pqhsa.h).
    init_slots: int32 [B, Hkv, C + 16 * 256] training slots seeding the centroids, then the codewords."""
    assert init_slots.dtype == torch.int32 and init_slots.is_contiguous()
    if assign_out is not None:
        assert assign_out.dtype == torch.int32 and assign_out.is_contiguous()
    kvs, ixs = kv.struct(), index.struct()
    if workspace_buf is None:
        workspace_buf = workspace(hsa_train_workspace_bytes(kv, index, n_train), index.centroids.device)
    _on_gpu(init_slots, assign_out, workspace_buf)
    st = load_library().hsa_train_index(ctypes.byref(kvs), ctypes.byref(ixs), int(n_train), init_slots.data_ptr(),
                                        int(coarse_iters), int(pq_iters), _ptr(assign_out),
                                        workspace_buf.data_ptr(), workspace_buf.numel(), _stream(stream))
    _check("hsa_train_index", st)


def hsa_read_error(workspace_buf: torch.Tensor, stream=None) -> int:
    """Read and clear the device error word of a workspace (synchronises the stream)."""
    v = ctypes.c_int32(0)
    _on_gpu(workspace_buf)
    st = load_library().hsa_read_error(workspace_buf.data_ptr(), ctypes.byref(v), _stream(stream))
    _check("hsa_read_error", st)
    return int(v.value)


def dense_decode_static(kv: PagedKV, q: torch.Tensor, out: Optional[torch.Tensor] = None, *, scale: float,
                        stream=None) -> torch.Tensor:
    """dense_decode with the library's static scratch array: no workspace, no allocation in the
    library (see dense_decode_static in include/pqhsa.h for its limit and its sharing rules)."""
    assert q.dtype == torch.float32 and q.is_contiguous()
    if out is None:
        out = torch.empty_like(q)
    lib = load_library()
    fn = lib.dense_decode_static
    fn.argtypes = [ctypes.POINTER(_KV), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    kvs = kv.struct()
    _on_gpu(q, out)
    _check("dense_decode_static", fn(ctypes.byref(kvs), q.data_ptr(), out.data_ptr(), ctypes.c_float(scale),
                                     _stream(stream)))
    return out
