"""Full-size GPU parity: every workload at its real size, through the same hsa_decode call the
bench times; the float64 oracle recomputes a sample of (sequence, KV head) units in full."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_long_context_pq_b200 as P
from synth import make_batch, workload
from synth.device import index_tensors, kv_tensors
from helpers import (LOGIT_RTOL, OUT_TOL, assert_sorted_positions, compare_logits, compare_selection, max_abs_v,
                     reference_codes, scale_for)

pytestmark = pytest.mark.gpu


def _decode_and_check(w, bt, codes, ids, units, dev):
    kv = P.PagedKV(**kv_tensors(bt, dev))
    ix = P.PQIndex(**index_tensors(bt, dev, codes, ids))
    P.hsa_build_from_codes(kv, ix)
    scale = scale_for(w.D)
    q = torch.from_numpy(bt.q).to(dev)
    approx = torch.zeros(w.B, w.Hq, ix.cap, device=dev)
    sel = torch.zeros(w.B, w.Hkv, ix.cap, dtype=torch.int32, device=dev)
    nsel = torch.zeros(w.B, w.Hkv, dtype=torch.int32, device=dev)
    ws = P.workspace(P.hsa_decode_workspace_bytes(kv, ix), dev)
    out = P.hsa_decode(kv, ix, q, scale=scale, budget=w.budget, approx_logits=approx, selected=sel,
                       n_selected=nsel, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    out, approx, sel, nsel = out.cpu().numpy(), approx.cpu().numpy(), sel.cpu().numpy(), nsel.cpu().numpy()
    orc = O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, bt.centroids, bt.codebooks,
                          codes, ids, bt.n_indexed, w.n_sink, scale, budget=w.budget, page_size=w.page_size,
                          units=units)
    vmax = max_abs_v(bt)
    for (b, h), r in orc.items():
        N = int(bt.n_indexed[b])
        rows = slice(h * w.G, (h + 1) * w.G)
        assert compare_logits(approx[b, rows, :N], r["s_hat"]) <= LOGIT_RTOL
        assert nsel[b, h] == r["k"] == O.decode_k(w.budget, N)
        assert_sorted_positions(sel[b, h, :r["k"]])
        compare_selection(sel[b, h, :r["k"]], r, w.n_sink)
        assert float(np.abs(out[b, rows] - r["out"]).max()) <= OUT_TOL * vmax
    # every unit, sampled or not: a complete, sorted selection of the right size and finite outputs
    assert np.isfinite(out).all()
    for b in range(w.B):
        for h in range(w.Hkv):
            k = O.decode_k(w.budget, int(bt.n_indexed[b]))
            assert nsel[b, h] == k
            s = sel[b, h, :k]
            assert_sorted_positions(s)
            assert s[0] >= w.n_sink and s[-1] < w.n_sink + bt.n_indexed[b]
    return kv, ix


@pytest.mark.parametrize("name,units", [
    ("llama8b_8k", [(0, 0), (0, 7)]),        # context sweep: exact tail (1024 rows) larger than k
    ("llama8b_32k", [(0, 2), (0, 6)]),
    ("llama8b_128k", [(0, 0), (0, 5)]),
    ("llama8b_512k", [(0, 3)]),
    ("batch32_32k", [(0, 0), (13, 7), (31, 2)]),
])
def test_fullsize_decode(cuda_device, name, units):
    w = workload(name)
    bt = make_batch(w)
    codes, ids = reference_codes(bt)
    _decode_and_check(w, bt, codes, ids, units, torch.device("cuda:0"))


def test_fullsize_qwen_append(cuda_device):
    """Qwen3-30B-A3B shape at 128K, batch 4, G=8: decode, then one 512-token append
    (context grown by 512) and decode again; sampled units checked in full."""
    w = workload("qwen30b_128k_append")
    bt = make_batch(w)
    dev = torch.device("cuda:0")
    codes, ids = reference_codes(bt)
    units = [(1, 2)]
    kv, ix = _decode_and_check(w, bt, codes, ids, units, dev)
    # grow every sequence by 512 tokens, encode the oldest 512 tail tokens on the GPU
    T2 = w.T + 512
    kv.seq_lens.fill_(T2)
    kv.seq_lens_host.fill_(T2)
    ws = P.workspace(P.hsa_index_workspace_bytes(kv, ix, 512), dev)
    P.hsa_append_encode(kv, ix, 512, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    N0 = w.n_indexed
    res = O.oracle_append(bt.k_cache, bt.block_table, bt.centroids, bt.codebooks, bt.n_indexed, 512, w.n_sink,
                          page_size=w.page_size)
    gids = ix.ids.cpu().numpy().view(np.uint16)
    gcodes = ix.codes.cpu().numpy()
    excused = 0
    for (b, h), (ii, cc, gaps) in res.items():
        bad = np.nonzero(gids[b, h, N0:N0 + 512].astype(np.int64) != ii)[0]
        for j in bad:
            assert gaps["gap_c"][j] < 1e-5 * max(gaps["best_c"][j], 1.0)
        ok = np.setdiff1d(np.arange(512), bad)
        mism = np.argwhere(gcodes[b, h, N0 + ok].astype(np.int64) != cc[ok])
        for r_, s_ in mism:
            j = ok[r_]
            assert gaps["gap_m"][j, s_] < 1e-5 * max(gaps["best_m"][j, s_], 1.0)
        excused += len(bad) + len(mism)
        codes[b, h, N0:N0 + 512] = cc
        ids[b, h, N0:N0 + 512] = ii
    bt.seq_lens[:] = T2
    bt.n_indexed[:] = N0 + 512
    assert ix.n_indexed_host.tolist() == [N0 + 512] * w.B
    # decode the grown context from the oracle's own encoding on both sides
    _decode_and_check(w, bt, codes, ids, units, dev)
