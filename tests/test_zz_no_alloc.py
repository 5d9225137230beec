"""dense_decode_static, the entry point that allocates nothing, against the oracle and dense_decode.

Some callers cannot hand the library a device workspace: a plain host program with no
device allocator, a runtime whose memory pool is fixed before serving, a decode loop
that must not call cudaMalloc. dense_decode_static keeps its split-K scratch in a
static array inside the library. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import sparse_long_context_pq_b200 as P
from synth import make_batch, workload
from synth.device import kv_tensors
from helpers import DENSE_TOL, max_abs_v, scale_for

pytestmark = pytest.mark.gpu

CASES = [
    dict(name="qwen30b_128k_append", B=2, T=8192, extra_tokens=0, append_batch=0),   # 8 units x G=8
    dict(name="tiny_4k"),                                                            # 1 unit x G=4
]


def _entry():
    fn = P.load_library().dense_decode_static
    fn.argtypes = [ctypes.POINTER(P._KV), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _problem(case):
    w = workload(**case)
    bt = make_batch(w)
    dev = torch.device("cuda:0")
    kv = P.PagedKV(**kv_tensors(bt, dev))
    q = torch.from_numpy(bt.q).to(dev)
    return w, bt, kv, q


def _call_static(kv, q, scale):
    out = torch.full_like(q, float("nan"))
    kvs = kv.struct()
    st = _entry()(ctypes.byref(kvs), q.data_ptr(), out.data_ptr(), ctypes.c_float(scale),
                  torch.cuda.current_stream().cuda_stream)
    assert st == 0, P.hsa_strerror(st)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _oracle(w, bt, scale, units=None):
    ref = O.oracle_dense(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, scale, page_size=w.page_size,
                         units=units)
    return ref


def test_static_scratch_matches_oracle_and_dense_decode_across_shapes(cuda_device):
    """Two shapes, each called twice, the larger first: the array keeps the previous call's
    partials at other offsets, and no call may read them. Each output is checked against
    the float64 oracle and against dense_decode (the same kernels with a workspace)."""
    for case in CASES:
        w, bt, kv, q = _problem(case)
        scale = scale_for(w.D)
        ref = _oracle(w, bt, scale)
        ws_out = P.dense_decode(kv, q, scale=scale).cpu().numpy()
        tol = DENSE_TOL * max_abs_v(bt)
        for _ in range(2):
            got = _call_static(kv, q, scale)
            assert np.isfinite(got).all()
            for (b, h), r in ref.items():
                rows = slice(h * w.G, (h + 1) * w.G)
                assert float(np.abs(got[b, rows] - r).max()) <= tol, (case["name"], b, h)
            assert float(np.abs(got - ws_out).max()) <= tol


def test_static_scratch_at_its_largest_shape(cuda_device):
    """B * Hkv * G = 16000 (250 sequences x 8 KV heads x 8 query heads per KV head, 64 tokens):
    one split-K chunk is all the 8 MiB array holds; sampled units against the oracle."""
    case = dict(name="qwen30b_128k_append", B=250, Hq=64, Hkv=8, T=64, C=4, n_recent=16, n_needles=0,
                extra_tokens=0, append_batch=0)
    w, bt, kv, q = _problem(case)
    scale = scale_for(w.D)
    got = _call_static(kv, q, scale)
    units = [(0, 0), (123, 4), (249, 7)]
    ref = _oracle(w, bt, scale, units=units)
    tol = DENSE_TOL * max_abs_v(bt)
    for (b, h), r in ref.items():
        assert float(np.abs(got[b, h * w.G:(h + 1) * w.G] - r).max()) <= tol
    ws_out = P.dense_decode(kv, q, scale=scale).cpu().numpy()
    assert float(np.abs(got - ws_out).max()) <= tol
