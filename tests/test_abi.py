"""The C-ABI library loads, exports every function include/pqhsa.h declares, and rejects bad
arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import sparse_long_context_pq_b200 as P
from sparse_long_context_pq_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pqhsa.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return P.load_library()


@pytest.fixture(scope="module")
def host_only(lib):
    """Tests that pass fake device pointers expect the call to refuse on the host before any
    launch; they run only where no GPU is visible, so a validation regression can never
    launch a kernel on addresses that are not device memory."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-validation test with fake device pointers: CPU-only")
    return lib


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("hsa_build_from_codes", "hsa_append_encode", "hsa_decode", "dense_decode", "hsa_strerror"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_abi_struct_sizes_match_binding(lib):
    sizes = [ctypes.c_int64() for _ in range(4)]
    lib.hsa_abi_sizes(*[ctypes.byref(s) for s in sizes])
    assert [s.value for s in sizes] == [ctypes.sizeof(t) for t in (P._KV, P._Index, P._Params, P._Debug)]


def test_list_capacity(lib):
    lib.hsa_index_list_slots.restype = ctypes.c_int64
    lib.hsa_index_list_slots.argtypes = [ctypes.c_int32, ctypes.c_int32]
    assert lib.hsa_index_list_slots(130032, 1024) == 32 * (4064 + 1024) == P.index_list_slots(130032, 1024)
    assert lib.hsa_index_list_slots(0, 4) == 0


def test_strerror(lib):
    assert P.hsa_strerror(0) == "ok"
    assert P.hsa_strerror(2) == "unsupported shape"


# ---- host-side validation (fake device pointers are never dereferenced on these paths) ----

FAKE = 1 << 20   # 256-byte aligned, never touched


def _kv(B=1, Hq=4, Hkv=1, D=128, page_size=16, max_pages=8, num_pages=8, seq=100, aligned=True):
    lens = np.full(B, seq, dtype=np.int32)
    base = FAKE if aligned else FAKE + 8
    kv = P._KV(base, FAKE, FAKE, FAKE, lens.ctypes.data, B, Hq, Hkv, D, page_size, max_pages, num_pages)
    return kv, lens


def _ix(B=1, C=16, cap=128, n_idx=50, n_sink=4, M=16, dsub=8, list_slots=None, list_slot=FAKE,
        chunk_cluster=FAKE):
    nh = np.full(B, n_idx, dtype=np.int32)
    ls = P.index_list_slots(cap, max(C, 1)) if list_slots is None else list_slots
    ix = P._Index(centroids=FAKE, codebooks=FAKE, codes=FAKE, ids=FAKE, sum_v=FAKE, mean_v=FAKE, count=FAKE,
                  n_indexed=FAKE, n_indexed_host=nh.ctypes.data, list_codes=FAKE, list_slot=list_slot,
                  chunk_cluster=chunk_cluster, list_meta=FAKE, C=C, M=M, dsub=dsub, ncode=256, cap=cap,
                  n_sink=n_sink,
                  list_slots=ls)
    return ix, nh


def _decode(lib, kv, ix, ws_bytes=1 << 30, q=FAKE):
    prm = P._Params(0.088, 0.01, -1, 1)
    return lib.hsa_decode(ctypes.byref(kv), ctypes.byref(ix), q, FAKE, ctypes.byref(prm), None, FAKE, ws_bytes, None)


@pytest.mark.parametrize("mutate,status", [
    (dict(Hq=6, Hkv=4), 1),            # Hq not a multiple of Hkv
    (dict(Hq=12, Hkv=1), 2),           # group of 12 heads unsupported
    (dict(D=64), 2),                   # head dim 64
    (dict(page_size=24), 2),           # page size not a power of two
    (dict(seq=1000), 3),               # longer than the block table
    (dict(aligned=False), 4),          # cache pointer not 256-byte aligned
])
def test_decode_rejects_bad_cache(host_only, mutate, status):
    lib = host_only
    kv, lens = _kv(**mutate)
    ix, nh = _ix()
    assert _decode(lib, kv, ix) == status


@pytest.mark.parametrize("mutate,status", [
    (dict(M=8, dsub=16), 2),
    (dict(C=0), 1),
    (dict(n_idx=200), 3),              # more than cap
    (dict(n_idx=99), 3),               # n_sink + N > T
    (dict(list_slots=32 * 4), 3),      # cluster lists too small
    (dict(C=5000), 2),                 # too many clusters for the list builder
    (dict(list_slot=FAKE + 4), 4),     # list slots are streamed by 16-byte async copies
    (dict(chunk_cluster=FAKE + 2), 4), # cluster ids are fetched as aligned 4-byte words
])
def test_decode_rejects_bad_index(host_only, mutate, status):
    lib = host_only
    kv, lens = _kv()
    ix, nh = _ix(**mutate)
    assert _decode(lib, kv, ix) == status


def test_decode_rejects_small_workspace_and_null_q(host_only):
    lib = host_only
    kv, lens = _kv()
    ix, nh = _ix()
    assert _decode(lib, kv, ix, ws_bytes=16) == 5
    assert _decode(lib, kv, ix, q=None) == 1
    need = lib.hsa_decode_workspace_bytes(ctypes.byref(kv), ctypes.byref(ix))
    assert need > 0 and need % 256 == 0


def test_decode_host_validates_before_queuing(host_only):
    """hsa_decode_host checks everything before its first copy: a bad cache, a null host
    pointer or a workspace without room for q and out is refused (fake device pointers
    are never touched). Its workspace is hsa_decode's plus two 256-byte aligned q/out areas."""
    lib = host_only
    kv, lens = _kv()
    ix, nh = _ix()
    q = np.zeros((1, 4, 128), dtype=np.float32)
    out = np.zeros_like(q)
    prm = P._Params(0.088, 0.01, -1, 1)
    need = lib.hsa_decode_workspace_bytes(ctypes.byref(kv), ctypes.byref(ix))
    need_host = lib.hsa_decode_host_workspace_bytes(ctypes.byref(kv), ctypes.byref(ix))
    assert need_host == need + 2 * 2048   # 1 x 4 x 128 fp32 = 2048 bytes each

    def call(kv_, ix_, qp, op, ws_bytes):
        return lib.hsa_decode_host(ctypes.byref(kv_), ctypes.byref(ix_), qp, op, ctypes.byref(prm), FAKE, ws_bytes,
                                   None)

    assert call(kv, ix, None, out.ctypes.data, need_host) == 1
    assert call(kv, ix, q.ctypes.data, None, need_host) == 1
    assert call(kv, ix, q.ctypes.data, out.ctypes.data, need) == 5      # no room for q and out
    bad_kv, _ = _kv(D=64)
    assert call(bad_kv, ix, q.ctypes.data, out.ctypes.data, need_host) == 2
    bad_ix, _ = _ix(n_idx=200)
    assert call(kv, bad_ix, q.ctypes.data, out.ctypes.data, need_host) == 3


def test_decode_step_validates_without_cuda(host_only):
    """hsa_decode_step_create checks its arguments and makes no CUDA call; every run checks
    the views and the current lengths again before anything is recorded or launched."""
    lib = host_only
    kv, lens = _kv()
    ix, nh = _ix()
    prm = P._Params(0.088, 0.01, -1, 1)
    need_host = lib.hsa_decode_host_workspace_bytes(ctypes.byref(kv), ctypes.byref(ix))
    h = ctypes.c_void_p()
    assert lib.hsa_decode_step_create(ctypes.byref(kv), ctypes.byref(ix), ctypes.byref(prm), FAKE, need_host - 256,
                                      ctypes.byref(h)) == 5 and not h.value
    bad_kv, _ = _kv(D=64)
    assert lib.hsa_decode_step_create(ctypes.byref(bad_kv), ctypes.byref(ix), ctypes.byref(prm), FAKE, need_host,
                                      ctypes.byref(h)) == 2 and not h.value
    assert lib.hsa_decode_step_create(ctypes.byref(kv), ctypes.byref(ix), ctypes.byref(prm), FAKE, need_host,
                                      None) == 1
    assert lib.hsa_decode_step_create(ctypes.byref(kv), ctypes.byref(ix), ctypes.byref(prm), FAKE, need_host,
                                      ctypes.byref(h)) == 0 and h.value
    q = np.zeros((1, 4, 128), dtype=np.float32)
    out = np.zeros_like(q)
    assert lib.hsa_decode_step_run(h, None, out.ctypes.data, None) == 1
    assert lib.hsa_decode_step_run(None, q.ctypes.data, out.ctypes.data, None) == 1
    lens[0] = 1000                    # grown past the block table after the step was made
    assert lib.hsa_decode_step_run(h, q.ctypes.data, out.ctypes.data, None) == 3
    lib.hsa_decode_step_destroy(h)
    lib.hsa_decode_step_destroy(None)


def test_append_checks_capacity(host_only):
    lib = host_only
    kv, lens = _kv(seq=100)
    ix, nh = _ix(n_idx=50, n_sink=4, cap=60)
    big = 1 << 30
    assert lib.hsa_append_encode(ctypes.byref(kv), ctypes.byref(ix), 20, FAKE, big, None) == 3   # cap 60 < 70
    ix2, nh2 = _ix(n_idx=50, n_sink=4, cap=128)
    assert lib.hsa_append_encode(ctypes.byref(kv), ctypes.byref(ix2), 50, FAKE, big, None) == 3  # beyond T
    assert lib.hsa_append_encode(ctypes.byref(kv), ctypes.byref(ix2), -1, FAKE, big, None) == 1
    assert nh2[0] == 50                                                                           # untouched


def test_append_workspace(host_only):
    lib = host_only
    kv, lens = _kv(seq=100)
    ix, nh = _ix(n_idx=40, n_sink=4, cap=128, C=16)
    q = lambda k, i, n: lib.hsa_index_workspace_bytes(ctypes.byref(k), ctypes.byref(i), n)
    assert q(kv, ix, 0) == 256                                  # build from codes: the error word
    need = q(kv, ix, 20)                                        # tensor-core encoding: terms, norms, assignment
    assert need >= 256 + 3 * 256 * 128 * 2 + 256 * 4 + 20 * 4 and need % 256 == 0
    assert lib.hsa_append_encode(ctypes.byref(kv), ctypes.byref(ix), 20, FAKE, need - 256, None) == 5
    kv4, _ = _kv(seq=100, page_size=4, max_pages=32, num_pages=32)
    assert q(kv4, ix, 20) == 256                                # 4-row pages: CUDA-core encoding


def test_dense_rejects_bad_args(host_only):
    lib = host_only
    kv, lens = _kv()
    assert lib.dense_decode(ctypes.byref(kv), FAKE + 4, FAKE, ctypes.c_float(1.0), FAKE, 1 << 30, None) == 4
    assert lib.dense_decode(ctypes.byref(kv), FAKE, FAKE, ctypes.c_float(1.0), FAKE, 8, None) == 5


def _train(lib, kv, ix, n_train=40, coarse=2, pq=2, ws_bytes=1 << 30, init=FAKE, assign_out=None):
    return lib.hsa_train_index(ctypes.byref(kv), ctypes.byref(ix), n_train, init, coarse, pq, assign_out, FAKE,
                               ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(n_train=0), 1),
    (dict(coarse=-1), 1),
    (dict(pq=1001), 1),
    (dict(init=None), 1),
    (dict(n_train=97), 3),             # n_sink 4 + 97 > T = 100
    (dict(init=FAKE + 2), 4),          # init slots are 4-byte words
    (dict(assign_out=FAKE + 2), 4),
    (dict(ws_bytes=64), 5),
])
def test_train_rejects_bad_args(host_only, kw, status):
    lib = host_only
    kv, lens = _kv()
    ix, nh = _ix()
    assert _train(lib, kv, ix, **kw) == status


def test_train_rejects_unsupported_index(host_only):
    lib = host_only
    kv, lens = _kv(seq=2 << 20, max_pages=(2 << 20) // 16, num_pages=(2 << 20) // 16)
    ix, nh = _ix(cap=2 << 20)
    assert _train(lib, kv, ix, n_train=65535 * 32 + 1) == 2   # beyond the longest training set
    ix2, nh2 = _ix(M=8, dsub=16)
    kv2, lens2 = _kv()
    assert _train(lib, kv2, ix2) == 2
    assert lib.hsa_train_workspace_bytes(ctypes.byref(kv2), ctypes.byref(ix), 0) == 0
    assert lib.hsa_train_workspace_bytes(ctypes.byref(kv2), ctypes.byref(ix), 40) % 256 == 0


def test_binding_rejects_host_tensors_for_device_arrays():
    """A host tensor where the library expects device memory is refused before any call."""
    import torch
    B, Hkv, ps, pages = 1, 1, 16, 4
    kv = P.PagedKV(k_cache=torch.zeros(pages, Hkv, ps, 128, dtype=torch.bfloat16),
                   v_cache=torch.zeros(pages, Hkv, ps, 128, dtype=torch.bfloat16),
                   block_table=torch.zeros(B, pages, dtype=torch.int32), seq_lens=torch.zeros(B, dtype=torch.int32),
                   seq_lens_host=torch.zeros(B, dtype=torch.int32), Hq=4)
    with pytest.raises(ValueError):
        kv.struct()
    ix = P.PQIndex.allocate(B, Hkv, 4, 32, 4, "cpu")
    with pytest.raises(ValueError):
        ix.struct()
    with pytest.raises(ValueError):     # the prepared step marshals the same views, once
        P.DecodeStep(kv, ix, scale=0.1)


def test_static_dense_decode_validates_like_dense_decode(host_only):
    """dense_decode_static checks the KV-cache view with the same validation as dense_decode:
    a misaligned block table or length array is refused on the host, before any launch."""
    lib = host_only
    fn = lib.dense_decode_static
    fn.argtypes = [ctypes.POINTER(P._KV), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    lens = np.full(1, 100, dtype=np.int32)
    for bt, sl in ((FAKE + 2, FAKE), (FAKE, FAKE + 2)):
        kv = P._KV(FAKE, FAKE, bt, sl, lens.ctypes.data, 1, 4, 1, 128, 16, 8, 8)
        assert fn(ctypes.byref(kv), FAKE, FAKE, ctypes.c_float(1.0), None) == 4
    kv, _ = _kv(Hq=12, Hkv=1)
    assert fn(ctypes.byref(kv), FAKE, FAKE, ctypes.c_float(1.0), None) == 2
    kv, _ = _kv()
    assert fn(ctypes.byref(kv), FAKE + 4, FAKE, ctypes.c_float(1.0), None) == 4


def test_static_dense_decode_rejects_shapes_beyond_its_array(host_only):
    """The split-K partials of one chunk need B * Hkv * G * 520 bytes plus 768 of alignment
    slack in the 8 MiB array (after a 256-byte header): B * Hkv * G <= 16129 fits, 16130 does
    not. Refused shapes return HSA_ERR_WORKSPACE before any CUDA call (the pointers here are
    never dereferenced: only refused shapes are passed)."""
    lib = host_only
    fn = lib.dense_decode_static
    fn.argtypes = [ctypes.POINTER(P._KV), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    limit = ((8 << 20) - 256 - 768) // 520
    assert limit == 16129
    for B, Hq, Hkv in ((4096, 64, 8), (253, 64, 8), (16130, 1, 1)):
        assert B * Hq >= limit + 1                    # B * Hkv * G = B * Hq
        lens = np.full(B, 64, dtype=np.int32)
        kv = P._KV(FAKE, FAKE, FAKE, FAKE, lens.ctypes.data, B, Hq, Hkv, 128, 16, 4, 4096)
        assert fn(ctypes.byref(kv), FAKE, FAKE, ctypes.c_float(1.0), None) == 5
