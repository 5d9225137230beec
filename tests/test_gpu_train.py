"""GPU parity of index training (Lloyd k-means centroids on the keys, per-subspace k-means
codebooks on the residuals) against the oracle, and decode from a GPU-trained index.

One Lloyd step is compared element by element; an assignment may differ only where the
oracle's best and runner-up distances nearly tie, and only the centres such a token touches
may then differ. Several steps are compared through the k-means objective and the share of
agreeing assignments (near-tie flips make later steps drift apart legitimately).
"""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_long_context_pq_b200 as P
from synth import make_batch, train_init_slots, workload
from synth.device import index_tensors, kv_tensors
from helpers import OUT_TOL, compare_logits, compare_selection, max_abs_v, scale_for

pytestmark = pytest.mark.gpu

TIE = 1e-5
CENTRE_TOL = 1e-4


def _ties(X, Cn):
    """Rows whose nearest centre is ambiguous: the oracle's best and runner-up distances lie
    within TIE of each other (relative, floored at 1). Centres equal to the winner bit for bit
    are not rivals: both sides compute the same distance for them and keep the lower index.
    Returns ({row: (winner, runner-up)}, the centres such rows touch)."""
    X64 = X.astype(np.float64)
    C64 = Cn.astype(np.float64)
    inv = np.unique(Cn, axis=0, return_inverse=True)[1].reshape(-1)
    same = inv[:, None] == inv[None, :]
    rows, centres = {}, set()
    for i in range(0, len(X), 256):
        d = ((X64[i:i + 256, None, :] - C64[None]) ** 2).sum(axis=2)
        win = np.argmin(d.astype(np.float32), axis=1)
        rival = np.where(same[win], np.inf, d)
        run = np.argmin(rival, axis=1)
        best = d[np.arange(len(win)), win]
        gap = rival[np.arange(len(win)), run] - best
        for j in np.nonzero(gap < TIE * np.maximum(best, 1.0))[0]:
            rows[i + int(j)] = (int(win[j]), int(run[j]))
            centres.update((int(win[j]), int(run[j])))
    return rows, centres


def _setup(case):
    case = {k: v for k, v in case.items() if k != "n_train"}
    w = workload(**case)
    bt = make_batch(w)
    dev = torch.device("cuda:0")
    kv = P.PagedKV(**kv_tensors(bt, dev))
    ix = P.PQIndex(**index_tensors(bt, dev, n_indexed=np.zeros(w.B, np.int32)))
    return w, bt, dev, kv, ix


def _train(w, dev, kv, ix, n_train, init, coarse, pq):
    ws = P.workspace(P.hsa_train_workspace_bytes(kv, ix, n_train), dev)
    aout = torch.full((w.B, w.Hkv, n_train), -1, dtype=torch.int32, device=dev)
    P.hsa_train_index(kv, ix, n_train, torch.from_numpy(init).to(dev), coarse_iters=coarse, pq_iters=pq,
                      assign_out=aout, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    return ix.centroids.cpu().numpy(), ix.codebooks.cpu().numpy(), aout.cpu().numpy()


def _keys(bt, w, b, h, n_train):
    return O.unit_rows(bt.k_cache, bt.block_table[b], h, w.n_sink + np.arange(n_train), w.page_size).astype(np.float32)


CASES = [dict(name="tiny_4k"), dict(name="qwen30b_128k_append", B=2, T=4096, extra_tokens=0, append_batch=0, C=128),
         dict(name="tiny_4k", n_sink=13, page_size=8, C=300),   # unaligned first key; C not a tile multiple
         dict(name="tiny_4k", page_size=4),                      # CUDA-core assignment
         dict(name="tiny_4k", C=1),                              # one centroid: the mean of all keys
         dict(name="tiny_4k", n_sink=0, n_train=200),            # no sink; a partial, ragged training set
         dict(name="tiny_4k", n_train=1, C=1)]                   # a single training key


@pytest.mark.parametrize("case", CASES + [dict(name="tiny_4k", C=4096)])   # the largest C: 16 centroid tiles
def test_one_coarse_step_matches_oracle(cuda_device, case):
    w, bt, dev, kv, ix = _setup(case)
    n_train = case.get("n_train", w.n_indexed)
    init = train_init_slots(w, n_train)
    cen, books, aout = _train(w, dev, kv, ix, n_train, init, coarse=1, pq=0)
    orc = O.oracle_train(bt.k_cache, bt.block_table, w.n_sink, n_train, init, w.C, 1, 0, page_size=w.page_size)
    checked = 0
    for (b, h), (cen_o, books_o, a_o) in orc.items():
        X = _keys(bt, w, b, h, n_train)
        _, loose = _ties(X, X[init[b, h, :w.C]])                          # their update may differ
        diff = np.abs(cen[b, h] - cen_o).max(axis=1)
        bad = [c for c in np.nonzero(diff > CENTRE_TOL)[0] if c not in loose]
        assert not bad, f"unit {(b, h)}: centroids {bad[:5]} differ by {diff[bad[:5]]}"
        if loose:
            continue                                                      # everything after depends on the tie
        tie_rows, _ = _ties(X, cen_o)
        mism = [j for j in np.nonzero(aout[b, h] != a_o)[0] if j not in tie_rows]
        assert not mism, f"unit {(b, h)}: final assignment differs at {mism[:5]}"
        # pq_iters = 0: codeword m of subspace s is the residual of its seed row
        seeds = init[b, h, w.C:].reshape(w.M, w.ncode)
        ok = ~np.isin(seeds, list(tie_rows))
        err = np.abs(books[b, h] - books_o).max(axis=2)
        assert float(err[ok].max()) <= CENTRE_TOL
        checked += 1
    assert checked >= 1


@pytest.mark.parametrize("case", CASES)
def test_one_codebook_step_matches_oracle(cuda_device, case):
    w, bt, dev, kv, ix = _setup(case)
    n_train = case.get("n_train", w.n_indexed)
    init = train_init_slots(w, n_train, seed=1)
    cen, books, aout = _train(w, dev, kv, ix, n_train, init, coarse=0, pq=1)
    orc = O.oracle_train(bt.k_cache, bt.block_table, w.n_sink, n_train, init, w.C, 0, 1, page_size=w.page_size)
    checked = 0
    for (b, h), (cen_o, books_o, a_o) in orc.items():
        X = _keys(bt, w, b, h, n_train)
        np.testing.assert_array_equal(cen[b, h], cen_o)                   # the seed keys, unchanged
        tie_rows, _ = _ties(X, cen_o)
        mism = [j for j in np.nonzero(aout[b, h] != a_o)[0] if j not in tie_rows]
        assert not mism, f"unit {(b, h)}: assignment differs at {mism[:5]}"
        R = (X.astype(np.float64) - cen_o[a_o].astype(np.float64)).astype(np.float32)
        for s in range(w.M):
            sub = slice(s * w.dsub, (s + 1) * w.dsub)
            Z = R[:, sub]
            seeds = init[b, h, w.C + s * w.ncode:w.C + (s + 1) * w.ncode]
            W0 = Z[seeds]
            _, loose = _ties(Z, W0)
            # a row whose centroid was a near-tie has one of two residuals: the codewords
            # either would join, and any codeword it seeds, may differ
            for j, pair in tie_rows.items():
                loose.update(np.nonzero(seeds == j)[0].tolist())
                for c in pair:
                    z = X[j, sub].astype(np.float64) - cen_o[c, sub].astype(np.float64)
                    loose.add(int(np.argmin(((z[None] - W0.astype(np.float64)) ** 2).sum(1).astype(np.float32))))
            diff = np.abs(books[b, h, s] - books_o[s]).max(axis=1)
            bad = [m for m in np.nonzero(diff > CENTRE_TOL)[0] if m not in loose]
            assert not bad, f"unit {(b, h)} subspace {s}: codewords {bad[:5]} differ by {diff[bad[:5]]}"
        checked += 1
    assert checked >= 1


def test_several_steps_track_the_oracle(cuda_device):
    w, bt, dev, kv, ix = _setup(CASES[0])
    n_train = w.n_indexed
    init = train_init_slots(w, n_train, seed=2)
    cen, books, aout = _train(w, dev, kv, ix, n_train, init, coarse=4, pq=4)
    orc = O.oracle_train(bt.k_cache, bt.block_table, w.n_sink, n_train, init, w.C, 4, 4, page_size=w.page_size)
    for (b, h), (cen_o, books_o, a_o) in orc.items():
        X = _keys(bt, w, b, h, n_train)
        obj_g = O.kmeans_objective(X, cen[b, h], O.lloyd_assign(X, cen[b, h]))
        obj_o = O.kmeans_objective(X, cen_o, a_o)
        assert abs(obj_g - obj_o) <= 1e-3 * obj_o, (obj_g, obj_o)
        assert np.mean(aout[b, h] == a_o) >= 0.99
        seed = X[init[b, h, :w.C]]
        assert obj_g < O.kmeans_objective(X, seed, O.lloyd_assign(X, seed))   # training lowered it


def test_trained_index_encodes_and_decodes(cuda_device):
    """Train on the prefill keys, encode them with the trained index, decode: matches the
    oracle run on the same trained centroids and codebooks with the oracle's own encoding."""
    w, bt, dev, kv, ix = _setup(dict(name="qwen30b_128k_append", B=1, T=4096, extra_tokens=0, append_batch=0,
                                     C=128))
    n_train = w.n_indexed
    init = train_init_slots(w, n_train, seed=3)
    cen, books, _ = _train(w, dev, kv, ix, n_train, init, coarse=4, pq=4)
    ws = P.workspace(P.hsa_index_workspace_bytes(kv, ix, w.n_indexed), dev)
    P.hsa_append_encode(kv, ix, w.n_indexed, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    res = O.oracle_append(bt.k_cache, bt.block_table, cen, books, np.zeros(w.B, int), w.n_indexed, w.n_sink,
                          page_size=w.page_size)
    orc_ids = np.zeros((w.B, w.Hkv, w.index_cap), np.uint16)
    orc_codes = np.zeros((w.B, w.Hkv, w.index_cap, w.M), np.uint8)
    for (b, h), (ii, cc, _) in res.items():
        orc_ids[b, h, :w.n_indexed] = ii
        orc_codes[b, h, :w.n_indexed] = cc
    gids = ix.ids.cpu().numpy().view(np.uint16)
    gcodes = ix.codes.cpu().numpy()
    agree = np.mean(gcodes[:, :, :w.n_indexed] == orc_codes[:, :, :w.n_indexed])
    assert agree >= 0.999, agree
    if not (np.array_equal(gids, orc_ids) and np.array_equal(gcodes, orc_codes)):
        # near-tie encodings differ: decode both sides from the oracle's index
        ix.ids.copy_(torch.from_numpy(orc_ids.view(np.int16)))
        ix.codes.copy_(torch.from_numpy(orc_codes))
        P.hsa_build_from_codes(kv, ix, workspace_buf=ws)
    scale = scale_for(w.D)
    q = torch.from_numpy(bt.q).to(dev)
    approx = torch.zeros(w.B, w.Hq, w.index_cap, device=dev)
    sel = torch.zeros(w.B, w.Hkv, w.index_cap, dtype=torch.int32, device=dev)
    nsel = torch.zeros(w.B, w.Hkv, dtype=torch.int32, device=dev)
    wsd = P.workspace(P.hsa_decode_workspace_bytes(kv, ix), dev)
    out = P.hsa_decode(kv, ix, q, scale=scale, budget=0.01, approx_logits=approx, selected=sel,
                       n_selected=nsel, workspace_buf=wsd).cpu().numpy()
    assert P.hsa_read_error(wsd) == 0
    orc = O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, cen, books, orc_codes,
                          orc_ids, np.full(w.B, w.n_indexed), w.n_sink, scale, budget=0.01, page_size=w.page_size)
    a, s_, ns = approx.cpu().numpy(), sel.cpu().numpy(), nsel.cpu().numpy()
    vmax = max_abs_v(bt)
    for (b, h), r in orc.items():
        rows = slice(h * w.G, (h + 1) * w.G)
        assert compare_logits(a[b, rows, :w.n_indexed], r["s_hat"]) <= 1e-4
        assert ns[b, h] == r["k"]
        compare_selection(s_[b, h, :r["k"]], r, w.n_sink)
        assert float(np.abs(out[b, rows] - r["out"]).max()) <= OUT_TOL * vmax
