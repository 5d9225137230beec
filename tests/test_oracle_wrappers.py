"""Pins for the oracle's batch wrappers (oracle_decode, oracle_dense, oracle_build_means,
oracle_append, oracle_train) at B = 2 sequences, Hkv = 2 KV heads, G = 2 query heads per
KV head, with different lengths and indexed counts per sequence and a shuffled page pool.

What is pinned is the wrappers' own arithmetic: which query rows belong to unit (b, h), which
block-table row, length, indexed count and per-unit index arrays it reads, and at which
positions new tokens start. Every expected value is built here from per-unit arrays laid out
by hand (no paging, no wrapper), or fixed by construction (keys placed exactly on centroid +
codewords, values constant per cluster), and every unit's data differs from every other
unit's, so routing one unit's inputs to another fails. No GPU needed.
"""
import numpy as np
import pytest

import oracle as O
from synth import f32_to_bf16_bits

B, HKV, G, D, PS = 2, 2, 2, 128, 4
M, DSUB, NCODE = 16, 8, 256


def _grid(rng, shape, lim=8, step=0.125):
    """Values on a 1/8 grid with |x| < 1 (sums of two stay exact in bf16)."""
    return (rng.integers(-lim + 1, lim, size=shape) * step).astype(np.float64)


def _page_pool(per_unit_k, per_unit_v, lens, rng):
    """Scatter per-unit [T_b][D] rows (bf16-exact) into one shuffled pool [pages][Hkv][PS][D].

    Returns (k_cache, v_cache, block_table). Sequence b's logical page i is pool page
    block_table[b, i]; the two sequences' pages are interleaved in the pool."""
    max_pages = -(-max(lens) // PS)
    n_pages = B * max_pages + 3
    perm = rng.permutation(n_pages).astype(np.int32)
    bt = perm[:B * max_pages].reshape(B, max_pages)
    kc = np.zeros((n_pages, HKV, PS, D), np.uint16)
    vc = np.zeros_like(kc)
    for b in range(B):
        for h in range(HKV):
            for t in range(lens[b]):
                kc[bt[b, t // PS], h, t % PS] = f32_to_bf16_bits(per_unit_k[b][h][t].astype(np.float32))
                vc[bt[b, t // PS], h, t % PS] = f32_to_bf16_bits(per_unit_v[b][h][t].astype(np.float32))
    return kc, vc, bt


def _one_unit_pool(K, V):
    """A unit's rows alone in an unshuffled pool of one KV head (identity block table)."""
    T = K.shape[0]
    npg = -(-T // PS)
    kc = np.zeros((npg, 1, PS, D), np.uint16)
    vc = np.zeros_like(kc)
    kb = np.zeros((npg * PS, D), np.uint16)
    vb = np.zeros_like(kb)
    kb[:T] = f32_to_bf16_bits(K.astype(np.float32))
    vb[:T] = f32_to_bf16_bits(V.astype(np.float32))
    kc[:, 0] = kb.reshape(npg, PS, D)
    vc[:, 0] = vb.reshape(npg, PS, D)
    return kc, vc, np.arange(npg, dtype=np.int32)


@pytest.fixture(scope="module")
def batch():
    """Random per-unit keys/values/index, different lengths and indexed counts per sequence."""
    rng = np.random.default_rng(2024)
    lens = [61, 47]
    n_sink = 3
    n_idx = np.array([50, 31], dtype=np.int32)
    C = 5
    K = [[_grid(rng, (lens[b], D)) for h in range(HKV)] for b in range(B)]
    V = [[_grid(rng, (lens[b], D)) + (b * HKV + h) for h in range(HKV)] for b in range(B)]
    kc, vc, bt = _page_pool(K, V, lens, rng)
    q = rng.standard_normal((B, HKV * G, D)) / np.sqrt(D)
    cent = rng.standard_normal((B, HKV, C, D))
    cb = 0.3 * rng.standard_normal((B, HKV, M, NCODE, DSUB))
    cap = 64
    codes = rng.integers(0, NCODE, size=(B, HKV, cap, M)).astype(np.uint8)
    ids = rng.integers(0, C, size=(B, HKV, cap)).astype(np.uint16)
    return dict(lens=lens, n_sink=n_sink, n_idx=n_idx, C=C, K=K, V=V, kc=kc, vc=vc, bt=bt, q=q, cent=cent,
                cb=cb, codes=codes, ids=ids, seq_lens=np.array(lens, dtype=np.int32))


def test_dense_wrapper_routes_every_unit(batch):
    d = batch
    scale = 0.09
    got = O.oracle_dense(d["q"], d["kc"], d["vc"], d["bt"], d["seq_lens"], scale, page_size=PS)
    assert sorted(got) == [(b, h) for b in range(B) for h in range(HKV)]
    for b in range(B):
        for h in range(HKV):
            Kb = O.widen_bf16(f32_to_bf16_bits(d["K"][b][h].astype(np.float32)))
            Vb = O.widen_bf16(f32_to_bf16_bits(d["V"][b][h].astype(np.float32)))
            rows = d["q"][b, h * G:(h + 1) * G]           # query heads of KV head h
            want = O.dense_unit(rows, Kb, Vb, scale)
            np.testing.assert_allclose(got[(b, h)], want, rtol=0, atol=1e-12)
            # the values carry a per-unit offset, so a unit routed elsewhere is off by >= 1
            assert abs(float(got[(b, h)].mean()) - (b * HKV + h)) < 0.5


@pytest.mark.parametrize("budget,background", [(0.1, True), (0.3, False), (1.0, True)])
def test_decode_wrapper_matches_hand_sliced_units(batch, budget, background):
    d = batch
    scale = 0.11
    got = O.oracle_decode(d["q"], d["kc"], d["vc"], d["bt"], d["seq_lens"], d["cent"], d["cb"], d["codes"],
                          d["ids"], d["n_idx"], d["n_sink"], scale, budget=budget, background=background,
                          page_size=PS)
    for b in range(B):
        for h in range(HKV):
            kc1, vc1, bt1 = _one_unit_pool(d["K"][b][h], d["V"][b][h])
            N = int(d["n_idx"][b])
            k = int(np.floor(budget * N))
            want = O.decode_unit(d["q"][b, h * G:(h + 1) * G], kc1, vc1, bt1, 0, d["lens"][b], PS,
                                 d["cent"][b, h], d["cb"][b, h], d["codes"][b, h][:N], d["ids"][b, h][:N], N,
                                 d["n_sink"], scale, k, background)
            r = got[(b, h)]
            assert r["k"] == k
            np.testing.assert_array_equal(r["sel"], want["sel"])
            np.testing.assert_allclose(r["s_hat"], want["s_hat"], rtol=0, atol=1e-12)
            np.testing.assert_allclose(r["out"], want["out"], rtol=0, atol=1e-12)


def test_decode_wrapper_closed_form_equals_dense_per_unit():
    """Keys exactly on centroid + codewords and values constant within each cluster: the
    approximate logits are exact and the background is exact, so every unit's PQ-HSA output
    equals dense attention over its own rows, whatever the budget (see the per-unit closed
    form in the oracle pins); here at B = 2, Hkv = 2, G = 2 with per-unit indexes."""
    rng = np.random.default_rng(7)
    lens = [44, 57]
    n_sink, C = 2, 3
    n_idx = np.array([lens[0] - n_sink - 5, lens[1] - n_sink - 9], dtype=np.int32)
    cap = 60
    cent = np.zeros((B, HKV, C, D))
    cb = np.zeros((B, HKV, M, NCODE, DSUB))
    codes = np.zeros((B, HKV, cap, M), np.uint8)
    ids = np.zeros((B, HKV, cap), np.uint16)
    K = [[None] * HKV for _ in range(B)]
    Vv = [[None] * HKV for _ in range(B)]
    for b in range(B):
        for h in range(HKV):
            T, N = lens[b], int(n_idx[b])
            cent[b, h] = _grid(rng, (C, D), lim=4)
            cb[b, h] = _grid(rng, (M, NCODE, DSUB), lim=4)
            a = rng.integers(0, C, size=N)
            cd = rng.integers(0, NCODE, size=(N, M))
            keys = _grid(rng, (T, D))
            vals = _grid(rng, (T, D))
            cvals = _grid(rng, (C, D)) + 2 * (b * HKV + h)      # per-cluster constant value, per unit
            for j in range(N):
                keys[n_sink + j] = cent[b, h, a[j]] + cb[b, h][np.arange(M), cd[j]].reshape(D)
                vals[n_sink + j] = cvals[a[j]]
            ids[b, h, :N] = a
            codes[b, h, :N] = cd
            K[b][h], Vv[b][h] = keys, vals
    kc, vc, bt = _page_pool(K, Vv, lens, rng)
    q = rng.standard_normal((B, HKV * G, D)) / np.sqrt(D)
    scale = 0.2
    for budget in (0.0, 0.05, 0.5):
        got = O.oracle_decode(q, kc, vc, bt, np.array(lens, np.int32), cent, cb, codes, ids, n_idx, n_sink, scale,
                              budget=budget, page_size=PS)
        for b in range(B):
            for h in range(HKV):
                Kb = O.widen_bf16(f32_to_bf16_bits(K[b][h].astype(np.float32)))
                Vb = O.widen_bf16(f32_to_bf16_bits(Vv[b][h].astype(np.float32)))
                want = O.dense_unit(q[b, h * G:(h + 1) * G], Kb, Vb, scale)
                np.testing.assert_allclose(got[(b, h)]["out"], want, rtol=0, atol=1e-10)


def test_build_means_wrapper_counts_only_the_indexed_range():
    """Values constant per (unit, cluster) on the indexed positions and different on the sink
    and the tail: each unit's means are its own constants and its counts the histogram of its
    own first N ids; a wrong position offset or length pulls in a sink or tail value."""
    rng = np.random.default_rng(11)
    lens = [40, 33]
    n_sink, C = 4, 6
    n_idx = np.array([29, 17], dtype=np.int32)
    cap = 40
    ids = rng.integers(0, C, size=(B, HKV, cap)).astype(np.uint16)
    consts = np.zeros((B, HKV, C, D))
    K = [[None] * HKV for _ in range(B)]
    Vv = [[None] * HKV for _ in range(B)]
    for b in range(B):
        for h in range(HKV):
            consts[b, h] = _grid(rng, (C, D)) + 3 * (b * HKV + h)
            vals = np.full((lens[b], D), -50.0)                     # sink and tail
            for j in range(int(n_idx[b])):
                vals[n_sink + j] = consts[b, h, ids[b, h, j]]
            K[b][h], Vv[b][h] = np.zeros((lens[b], D)), vals
    kc, vc, bt = _page_pool(K, Vv, lens, rng)
    got = O.oracle_build_means(vc, bt, ids, n_idx, n_sink, C, page_size=PS)
    for b in range(B):
        for h in range(HKV):
            cnt, _, mean = got[(b, h)]
            want_cnt = np.bincount(ids[b, h, :n_idx[b]].astype(np.int64), minlength=C)
            np.testing.assert_array_equal(cnt, want_cnt)
            for c in range(C):
                want = consts[b, h, c] if want_cnt[c] else np.zeros(D)
                np.testing.assert_array_equal(mean[c], want)


def test_append_wrapper_encodes_the_positions_after_each_sequences_index():
    """New keys placed exactly on (centroid + codewords) of well separated per-unit centroids:
    the encoding of each unit's n_new tokens after its own n_indexed is known by construction;
    the tokens before and after them are far from every centroid and would change the ids."""
    rng = np.random.default_rng(5)
    lens = [70, 58]
    n_sink, C, n_new = 2, 4, 9
    n_idx = np.array([40, 27], dtype=np.int32)
    cent = np.zeros((B, HKV, C, D))
    cb = np.zeros((B, HKV, M, NCODE, DSUB))
    want_ids = np.zeros((B, HKV, n_new), np.int64)
    want_codes = np.zeros((B, HKV, n_new, M), np.int64)
    K = [[None] * HKV for _ in range(B)]
    for b in range(B):
        for h in range(HKV):
            cent[b, h] = 8.0 * np.eye(C, D) * (1 + b * HKV + h) / 4      # far apart, per unit
            # codewords: distinct one-hot patterns on a 1/8 grid, far apart relative to rounding
            cb[b, h] = 0.0
            for s in range(M):
                for m in range(NCODE):
                    cb[b, h, s, m, m % DSUB] = 0.125 * (1 + m // DSUB)
            keys = np.full((lens[b], D), 30.0)                            # far from everything
            a = rng.integers(0, C, size=n_new)
            cd = rng.integers(0, NCODE, size=(n_new, M))
            for j in range(n_new):
                keys[n_sink + n_idx[b] + j] = cent[b, h, a[j]] + cb[b, h][np.arange(M), cd[j]].reshape(D)
            want_ids[b, h], want_codes[b, h] = a, cd
            K[b][h] = keys
    kc, vc, bt = _page_pool(K, K, lens, rng)
    got = O.oracle_append(kc, bt, cent, cb, n_idx, n_new, n_sink, page_size=PS)
    for b in range(B):
        for h in range(HKV):
            ii, cc, _ = got[(b, h)]
            np.testing.assert_array_equal(ii, want_ids[b, h])
            np.testing.assert_array_equal(cc, want_codes[b, h])


def test_train_wrapper_matches_train_unit_on_hand_sliced_keys():
    """oracle_train per (b, h) equals train_unit on that unit's training keys laid out by hand
    (positions [n_sink, n_sink + n_train) of its own rows), with per-unit seed slots."""
    rng = np.random.default_rng(9)
    lens = [150, 140]
    n_sink, C, n_train = 3, 4, 120
    K = [[_grid(rng, (lens[b], D)) + (b * HKV + h) for h in range(HKV)] for b in range(B)]
    kc, vc, bt = _page_pool(K, K, lens, rng)
    init = np.stack([np.stack([rng.integers(0, n_train, size=C + M * NCODE) for h in range(HKV)])
                     for b in range(B)]).astype(np.int64)
    got = O.oracle_train(kc, bt, n_sink, n_train, init, C, 2, 1, page_size=PS)
    for b in range(B):
        for h in range(HKV):
            keys = O.widen_bf16(f32_to_bf16_bits(K[b][h][n_sink:n_sink + n_train].astype(np.float32)))
            want = O.train_unit(keys.astype(np.float32), init[b, h], C, 2, 1)
            for x, y in zip(got[(b, h)], want):
                np.testing.assert_array_equal(x, y)
            # per-unit offsets: each unit's centroids sit near its own offset
            assert abs(float(got[(b, h)][0].mean()) - (b * HKV + h)) < 0.5
