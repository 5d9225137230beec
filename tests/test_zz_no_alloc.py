"""dense_decode_static, the entry point that allocates nothing, against dense_decode.

Some callers cannot hand the library a device workspace: a plain host program with no
device allocator, a runtime whose memory pool is fixed before serving, a decode loop
that must not call cudaMalloc. dense_decode_static keeps its split-K scratch in a
static array inside the library. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_long_context_pq_b200 as P
from synth import make_batch, workload
from synth.device import kv_tensors
from helpers import DENSE_TOL, max_abs_v, scale_for

pytestmark = pytest.mark.gpu


def _entry():
    fn = P.load_library().dense_decode_static
    fn.argtypes = [ctypes.POINTER(P._KV), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


@pytest.mark.parametrize("case", [
    dict(name="tiny_4k"),
    dict(name="qwen30b_128k_append", B=2, T=8192, extra_tokens=0, append_batch=0),
])
def test_static_scratch_matches_dense_decode_twice(cuda_device, case):
    w = workload(**case)
    bt = make_batch(w)
    dev = torch.device("cuda:0")
    kv = P.PagedKV(**kv_tensors(bt, dev))
    q = torch.from_numpy(bt.q).to(dev)
    scale = scale_for(w.D)
    ref = P.dense_decode(kv, q, scale=scale).cpu().numpy()
    tol = DENSE_TOL * max_abs_v(bt)
    fn = _entry()
    kvs = kv.struct()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                       # the array keeps the previous call's contents
        out = torch.full_like(q, float("nan"))
        assert fn(ctypes.byref(kvs), q.data_ptr(), out.data_ptr(), ctypes.c_float(scale), stream) == 0
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert float(np.abs(got - ref).max()) <= tol


def test_static_scratch_rejects_shapes_beyond_its_limit(cuda_device):
    lens = np.full(4096, 64, dtype=np.int32)
    fake = 1 << 20
    kvs = P._KV(fake, fake, fake, fake, lens.ctypes.data, 4096, 64, 8, 128, 16, 4, 4096)  # B*Hkv*G = 262144
    assert _entry()(ctypes.byref(kvs), fake, fake, ctypes.c_float(1.0), None) == 5
