"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle on the same seeded inputs.

Gates: approximate logits within 1e-4 of the row's max |logit|; the selected set
identical except near-ties within 1e-5 of the k-th score; the attention output
within 2e-3 * max|V|; cluster counts exact; encoded ids/codes identical except
documented near-ties.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import sparse_long_context_pq_b200 as P
from synth import make_batch, workload
from synth.device import index_tensors, kv_tensors
from helpers import (DENSE_TOL, LOGIT_RTOL, OUT_TOL, assert_sorted_positions, compare_logits, compare_selection,
                     max_abs_v, reference_codes, scale_for)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_4k": dict(name="tiny_4k"),
    "llama8b_16k": dict(name="llama8b_128k", T=16384, n_needles=16),
    "batch_4x4k": dict(name="batch32_32k", B=4, T=4096),
    "qwen_g8_8k": dict(name="qwen30b_128k_append", B=2, T=8192, extra_tokens=0, append_batch=0),
    "ragged_5003": dict(name="tiny_4k", T=5003, n_recent=101, C=32, n_needles=3),
    "mha_g1_4k": dict(name="tiny_4k", Hq=2, Hkv=2),                   # one query head per KV head
    "gqa_g2_4k": dict(name="tiny_4k", Hq=4, Hkv=2),
    "page4_4k": dict(name="tiny_4k", page_size=4),                    # dense path gathers rows
    "page64_3000": dict(name="tiny_4k", T=3000, page_size=64, n_recent=64, C=48),
}


def _setup(case, seq_lens=None, n_indexed=None, n_sink=None):
    w = workload(**case)
    if n_sink is not None:
        w = w.scaled(n_sink=n_sink)
    bt = make_batch(w)
    if seq_lens is not None:
        bt.seq_lens[:] = seq_lens
    if n_indexed is not None:
        bt.n_indexed[:] = n_indexed
    codes, ids = reference_codes(bt)
    dev = torch.device("cuda:0")
    kv = P.PagedKV(**kv_tensors(bt, dev))
    ix = P.PQIndex(**index_tensors(bt, dev, codes, ids))
    return w, bt, codes, ids, kv, ix, dev


def _run_hsa(w, bt, codes, ids, kv, ix, dev, budget=0.01, k_override=-1, background=True):
    scale = scale_for(w.D)
    ws_idx = P.workspace(P.hsa_index_workspace_bytes(kv, ix), dev)
    P.hsa_build_from_codes(kv, ix, workspace_buf=ws_idx)
    q = torch.from_numpy(bt.q).to(dev)
    cap = ix.cap
    approx = torch.full((w.B, w.Hq, cap), float("nan"), device=dev)
    sel = torch.full((w.B, w.Hkv, cap), -1, dtype=torch.int32, device=dev)
    nsel = torch.full((w.B, w.Hkv), -1, dtype=torch.int32, device=dev)
    ws = P.workspace(P.hsa_decode_workspace_bytes(kv, ix), dev)
    out = P.hsa_decode(kv, ix, q, scale=scale, budget=budget, k_override=k_override, background=background,
                       approx_logits=approx, selected=sel, n_selected=nsel, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    assert P.hsa_read_error(ws_idx) == 0
    orc = O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, bt.centroids, bt.codebooks,
                          codes, ids, bt.n_indexed, w.n_sink, scale, budget=budget,
                          k_override=k_override if k_override >= 0 else None, background=background,
                          page_size=w.page_size)
    return (out.cpu().numpy(), approx.cpu().numpy(), sel.cpu().numpy(), nsel.cpu().numpy(), orc,
            ix.mean_v.cpu().numpy(), ix.count.cpu().numpy())


def _check_all(w, bt, res, check_means=True, ids=None):
    out, approx, sel, nsel, orc, mean_v, count = res
    vmax = max_abs_v(bt)
    worst_logit = worst_out = 0.0
    for (b, h), r in orc.items():
        N = int(bt.n_indexed[b])
        G = w.G
        rows = slice(h * G, (h + 1) * G)
        if r["s_hat"].shape[1]:
            worst_logit = max(worst_logit, compare_logits(approx[b, rows, :N], r["s_hat"]))
        k = r["k"]
        assert nsel[b, h] == k
        gsel = sel[b, h, :k]
        assert_sorted_positions(gsel)
        compare_selection(gsel, r, w.n_sink)
        worst_out = max(worst_out, float(np.abs(out[b, rows] - r["out"]).max()))
        if check_means and ids is not None and N > 0:
            V = O.unit_rows(bt.v_cache, bt.block_table[b], h, w.n_sink + np.arange(N), w.page_size)
            cnt, _, mu = O.cluster_means(V, ids[b, h, :N].astype(np.int64), w.C)
            np.testing.assert_array_equal(count[b, h], cnt)
            np.testing.assert_allclose(mean_v[b, h], mu, rtol=0, atol=1e-5)
    assert worst_logit <= LOGIT_RTOL, worst_logit
    assert worst_out <= OUT_TOL * vmax, (worst_out, vmax)
    return worst_logit, worst_out


@pytest.mark.parametrize("name", list(CASES))
def test_hsa_decode_matches_oracle(cuda_device, name):
    w, bt, codes, ids, kv, ix, dev = _setup(CASES[name])
    res = _run_hsa(w, bt, codes, ids, kv, ix, dev)
    _check_all(w, bt, res, ids=ids)


@pytest.mark.parametrize("name", ["tiny_4k", "qwen_g8_8k", "ragged_5003"])
def test_dense_decode_matches_oracle(cuda_device, name):
    w, bt, codes, ids, kv, ix, dev = _setup(CASES[name])
    scale = scale_for(w.D)
    q = torch.from_numpy(bt.q).to(dev)
    ws = P.workspace(P.dense_decode_workspace_bytes(kv), dev)
    out = P.dense_decode(kv, q, scale=scale, workspace_buf=ws).cpu().numpy()
    assert P.hsa_read_error(ws) == 0
    ref = O.oracle_dense(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, scale, page_size=w.page_size)
    vmax = max_abs_v(bt)
    for (b, h), r in ref.items():
        err = float(np.abs(out[b, h * w.G:(h + 1) * w.G] - r).max())
        assert err <= DENSE_TOL * vmax, (b, h, err)


def test_full_budget_equals_dense_on_gpu(cuda_device):
    w, bt, codes, ids, kv, ix, dev = _setup(CASES["tiny_4k"])
    out, approx, sel, nsel, orc, *_ = _run_hsa(w, bt, codes, ids, kv, ix, dev, budget=1.0)
    q = torch.from_numpy(bt.q).to(dev)
    dense = P.dense_decode(kv, q, scale=scale_for(w.D)).cpu().numpy()
    assert nsel[0, 0] == w.n_indexed
    np.testing.assert_allclose(out, dense, rtol=0, atol=DENSE_TOL * max_abs_v(bt))


@pytest.mark.parametrize("budget,k_override,background", [
    (0.0, -1, True),      # k = 0: every indexed token approximate
    (0.05, -1, True),
    (0.01, -1, False),    # plain top-k sparse attention
    (0.01, 1, True),      # single selected token
    (0.5, -1, True),
])
def test_hsa_decode_budgets_and_ablation(cuda_device, budget, k_override, background):
    w, bt, codes, ids, kv, ix, dev = _setup(CASES["ragged_5003"])
    res = _run_hsa(w, bt, codes, ids, kv, ix, dev, budget=budget, k_override=k_override, background=background)
    _check_all(w, bt, res, check_means=False)


def test_ragged_batch_lengths(cuda_device):
    case = dict(name="batch32_32k", B=3, T=3000, C=64)
    T = np.array([3000, 2890, 1963], dtype=np.int32)
    n_idx = np.maximum(T - 16 - 256, 0).astype(np.int32)
    w, bt, codes, ids, kv, ix, dev = _setup(case, seq_lens=T, n_indexed=n_idx)
    res = _run_hsa(w, bt, codes, ids, kv, ix, dev)
    _check_all(w, bt, res, ids=ids)


def test_no_index_and_no_sink(cuda_device):
    # sequence 0: nothing indexed (dense); sequence 1: indexed but no sink and no tail
    case = dict(name="batch32_32k", B=2, T=1500, C=16, n_needles=0)
    w, bt, codes, ids, kv, ix, dev = _setup(case, seq_lens=np.array([1500, 1500]),
                                            n_indexed=np.array([0, 1500]), n_sink=0)
    res = _run_hsa(w, bt, codes, ids, kv, ix, dev, budget=0.02)
    _check_all(w, bt, res, ids=ids)


def test_prepared_step_matches_hsa_decode(cuda_device):
    """DecodeStep (the cache and index views marshalled once) gives hsa_decode's output, on
    device and on host buffers (hsa_decode_host), eagerly and as the graph-replayed prepared
    step, and still does after the lengths change in place behind its views. Two decode calls agree to rounding, not bit for bit: the
    cluster-weight sums are fp32 atomics in arrival order."""
    w, bt, codes, ids, kv, ix, dev = _setup(CASES["qwen_g8_8k"])
    ws_idx = P.workspace(P.hsa_index_workspace_bytes(kv, ix), dev)
    P.hsa_build_from_codes(kv, ix, workspace_buf=ws_idx)
    scale = scale_for(w.D)
    q = torch.from_numpy(bt.q).to(dev)
    step = P.DecodeStep(kv, ix, scale=scale, budget=w.budget)
    for _ in range(2):
        ref = P.hsa_decode(kv, ix, q, scale=scale, budget=w.budget)
        got = step(q)
        out = torch.full_like(q, float("nan"))
        assert step(q, out) is out
        out_g = torch.full_like(q, float("nan"))
        step(q, out_g, graph=True)              # prepared step on device buffers: records, then replays
        step(q, out_g, graph=True)
        torch.cuda.synchronize()
        tol = 1e-6 * float(ref.abs().max()) + 1e-7
        for o in (got, out, out_g):
            assert float((o - ref).abs().max()) <= tol
        # the host-buffer entry: q in from and out back to pinned host memory
        q_h = q.cpu().pin_memory()
        outs = [torch.full(q.shape, float("nan")).pin_memory() for _ in range(4)]
        step.host(q_h, outs[0])                 # prepared step: records its graph
        step.host(q_h, outs[1])                 # replays it
        step.host(q_h, outs[2], graph=False)    # one hsa_decode_host call
        P.hsa_decode_host(kv, ix, q_h, outs[3], scale=scale, budget=w.budget)
        q_pageable = q.cpu()                    # not page-locked: copied by cudaMemcpyAsync
        out_pageable = torch.full(q.shape, float("nan"))
        P.hsa_decode_host(kv, ix, q_pageable, out_pageable, scale=scale, budget=w.budget)
        torch.cuda.synchronize()
        ref_h = ref.cpu()
        for o in outs + [out_pageable]:
            assert float((o - ref_h).abs().max()) <= tol
        with pytest.raises(P.HSAError):         # the graph-replayed step needs page-locked buffers
            step.host(q_pageable, out_pageable)
        # a replay reads the host buffer's current contents
        q2 = (q * 0.5).contiguous()
        ref2 = P.hsa_decode(kv, ix, q2, scale=scale, budget=w.budget)
        q_h.copy_(q2.cpu())
        step.host(q_h, outs[0])
        torch.cuda.synchronize()
        assert float((outs[0] - ref2.cpu()).abs().max()) <= 1e-6 * float(ref2.abs().max()) + 1e-7
        assert P.hsa_read_error(step.workspace_buf) == 0
        kv.seq_lens.sub_(700)                  # a shorter tail (and another split plan), same storage
        kv.seq_lens_host.sub_(700)
    with pytest.raises(ValueError):
        step(q[:, :1].contiguous())
    step.close()
