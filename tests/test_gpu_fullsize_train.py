"""Full-size GPU checks of the index build from raw keys (Llama-3.1-8B shape at 128K: 8 units
x 130032 keys, C = 1024), in the launch configuration the build bench uses.

The oracle cannot rerun Lloyd iterations over 130K keys x 1024 centroids per unit in seconds,
so these tests check what must hold at any size, on sampled units, in float64:
* one coarse step: every centroid is the mean of the keys its seed key attracts (the
  assignment to the seeds recomputed here in float64);
* the returned assignment is the nearest of the GPU's final centroids (sampled keys);
* one codebook step: every codeword is the mean of the residual sub-vectors its seed
  residual attracts, residuals taken against the GPU's own centroids and assignment;
* encoding all keys: sampled keys' ids and codes equal the oracle encoder's.
Near-ties (best and runner-up within 1e-5 relative) are excused as everywhere else.
"""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_long_context_pq_b200 as P
from synth import make_batch, train_init_slots, workload
from synth.device import index_tensors, kv_tensors

pytestmark = pytest.mark.gpu

TIE = 1e-5
TOL = 1e-4


def _nearest(X, Cn, rows=8192):
    """Nearest centre of every row in float64 (|x|^2 - 2 x.c + |c|^2 by blocks): returns
    (argmin, runner-up, best distance, gap to the runner-up); exact ties go to the lower index."""
    X = X.astype(np.float64)
    # a centre equal bit for bit to a lower-indexed one never wins (both sides compute the
    # same distance for the two and keep the lower index), so it is no rival either
    _, first = np.unique(Cn, axis=0, return_index=True)
    shadow = np.ones(len(Cn), bool)
    shadow[first] = False
    Cn = Cn.astype(np.float64)
    cn = (Cn ** 2).sum(1)
    cn[shadow] = np.inf
    a = np.empty(len(X), np.int64)
    r = np.empty(len(X), np.int64)
    best = np.empty(len(X))
    gap = np.empty(len(X))
    for i in range(0, len(X), rows):
        x = X[i:i + rows]
        d = (x ** 2).sum(1)[:, None] - 2.0 * (x @ np.where(shadow[:, None], 0.0, Cn).T) + cn[None, :]
        two = np.argpartition(d, 1, axis=1)[:, :2]
        dv = np.take_along_axis(d, two, axis=1)
        swap = (dv[:, 1] < dv[:, 0]) | ((dv[:, 1] == dv[:, 0]) & (two[:, 1] < two[:, 0]))
        two[swap] = two[swap][:, ::-1]
        dv[swap] = dv[swap][:, ::-1]
        a[i:i + rows], r[i:i + rows] = two[:, 0], two[:, 1]
        best[i:i + rows] = np.maximum(dv[:, 0], 0.0)
        gap[i:i + rows] = dv[:, 1] - dv[:, 0]
    return a, r, best, gap


def _means_check(X, a, r, best, gap, seeds, got):
    """got[c] must be the mean of the rows nearest to seed c (a centre with no rows keeps its
    seed). A near-tie row (gap < 1e-5 relative) may belong to either of its two nearest
    seeds: a centre touched by such rows passes if the mean over its certain rows plus some
    subset of them matches."""
    C = len(seeds)
    X = X.astype(np.float64)
    tie = gap < TIE * np.maximum(best, 1.0)
    sure = ~tie
    sums = np.zeros((C, X.shape[1]))
    np.add.at(sums, a[sure], X[sure])
    cnt = np.bincount(a[sure], minlength=C).astype(np.float64)
    maybe = {}
    for j in np.nonzero(tie)[0]:
        maybe.setdefault(int(a[j]), []).append(int(j))
        maybe.setdefault(int(r[j]), []).append(int(j))
    got = got.astype(np.float64)
    bad = []
    for c in range(C):
        opts = maybe.get(c, [])[:10]
        ok = False
        for mask in range(1 << len(opts)):
            sel = [opts[i] for i in range(len(opts)) if mask >> i & 1]
            n = cnt[c] + len(sel)
            want = (sums[c] + X[sel].sum(0)) / n if n > 0 else seeds[c].astype(np.float64)
            if np.abs(got[c] - want).max() <= TOL:
                ok = True
                break
        if not ok:
            bad.append(c)
    assert not bad, f"centres {bad[:5]} are not the mean of their rows"
    return int(tie.sum())


def _setup():
    w = workload("llama8b_128k")
    bt = make_batch(w)
    dev = torch.device("cuda:0")
    kv = P.PagedKV(**kv_tensors(bt, dev))
    ix = P.PQIndex(**index_tensors(bt, dev, n_indexed=np.zeros(w.B, np.int32)))
    return w, bt, dev, kv, ix


def _train(w, dev, kv, ix, init, coarse, pq):
    n = w.n_indexed
    ws = P.workspace(P.hsa_train_workspace_bytes(kv, ix, n), dev)
    aout = torch.full((w.B, w.Hkv, n), -1, dtype=torch.int32, device=dev)
    P.hsa_train_index(kv, ix, n, torch.from_numpy(init).to(dev), coarse_iters=coarse, pq_iters=pq,
                      assign_out=aout, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    return ix.centroids.cpu().numpy(), ix.codebooks.cpu().numpy(), aout.cpu().numpy()


def _keys(bt, w, b, h):
    return O.unit_rows(bt.k_cache, bt.block_table[b], h, w.n_sink + np.arange(w.n_indexed), w.page_size)


def test_fullsize_coarse_step(cuda_device):
    w, bt, dev, kv, ix = _setup()
    init = train_init_slots(w, w.n_indexed, seed=11)
    cen, books, aout = _train(w, dev, kv, ix, init, coarse=1, pq=0)
    rng = np.random.default_rng(5)
    for (b, h) in [(0, 0), (0, 6)]:
        u = b * w.Hkv + h
        X = _keys(bt, w, b, h)
        seeds = X[init[b, h, :w.C]]
        _means_check(X, *_nearest(X, seeds), seeds, cen[b, h])
        # the returned assignment: nearest of the GPU's final centroids (sampled keys)
        js = rng.choice(w.n_indexed, 8192, replace=False)
        a1, _, best1, gap1 = _nearest(X[js], cen[b, h])
        ok = (aout[b, h, js] == a1) | (gap1 < TIE * np.maximum(best1, 1.0))
        assert ok.all(), f"unit {u}: assignment differs at {js[~ok][:5]}"
        # pq_iters = 0: codeword m of subspace s is the residual of its seed key
        for s in (0, 7, 15):
            sl = slice(8 * s, 8 * s + 8)
            sd = init[b, h, w.C + s * w.ncode:w.C + (s + 1) * w.ncode]
            want = (X[sd, sl].astype(np.float32) - cen[b, h][aout[b, h, sd], sl]).astype(np.float32)
            np.testing.assert_allclose(books[b, h, s], want, rtol=0, atol=1e-6)


def test_fullsize_codebook_step(cuda_device):
    w, bt, dev, kv, ix = _setup()
    init = train_init_slots(w, w.n_indexed, seed=12)
    cen, books, aout = _train(w, dev, kv, ix, init, coarse=2, pq=1)
    for (b, h) in [(0, 3)]:
        X = _keys(bt, w, b, h)
        a = aout[b, h].astype(np.int64)
        assert a.min() >= 0 and a.max() < w.C
        R = (X.astype(np.float32) - cen[b, h][a]).astype(np.float64)
        for s in range(w.M):
            Z = R[:, 8 * s:8 * s + 8]
            seeds = Z[init[b, h, w.C + s * w.ncode:w.C + (s + 1) * w.ncode]]
            _means_check(Z, *_nearest(Z, seeds), seeds, books[b, h, s])


def test_fullsize_encode_all_keys(cuda_device):
    """The build the decode bench times: every indexed key encoded on the GPU with the
    workload's index; sampled keys of two units against the oracle's encoder."""
    w, bt, dev, kv, ix = _setup()
    ws = P.workspace(P.hsa_index_workspace_bytes(kv, ix, w.n_indexed), dev)
    P.hsa_append_encode(kv, ix, w.n_indexed, workspace_buf=ws)
    torch.cuda.synchronize()
    assert P.hsa_read_error(ws) == 0
    gids = ix.ids.cpu().numpy().view(np.uint16)
    gcodes = ix.codes.cpu().numpy()
    rng = np.random.default_rng(9)
    for (b, h) in [(0, 1), (0, 7)]:
        js = np.sort(rng.choice(w.n_indexed, 2048, replace=False))
        keys = O.unit_rows(bt.k_cache, bt.block_table[b], h, w.n_sink + js, w.page_size)
        ids, codes, gaps = O.encode_keys(keys, bt.centroids[b, h], bt.codebooks[b, h])
        tie_c = gaps["gap_c"] < TIE * np.maximum(gaps["best_c"], 1.0)
        ok_id = (gids[b, h, js].astype(np.int64) == ids) | tie_c
        assert ok_id.all(), f"ids differ at slots {js[~ok_id][:5]}"
        same = gids[b, h, js].astype(np.int64) == ids
        tie_m = gaps["gap_m"] < TIE * np.maximum(gaps["best_m"], 1.0)
        ok_code = (gcodes[b, h, js].astype(np.int64) == codes) | tie_m
        assert ok_code[same].all(), "codes differ beyond near-ties"
