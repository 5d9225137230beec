"""Pins for the float64 oracle: closed forms, brute force and a hand-derived case.

Each test checks the oracle against something other than its own formulas, so
that a dropped term, a wrong sign or index, or a transposed operand in it fails
at least one of them. No GPU needed.
"""
import itertools
import math

import numpy as np
import pytest

import oracle as O
from synth import f32_to_bf16_bits, workload, make_batch


# ---------------------------------------------------------------------------
# helpers: a small paged problem built from arbitrary float arrays
# ---------------------------------------------------------------------------

def _paged(keys, vals, page_size, rng, Hkv=1):
    """Lay [Hkv][T][D] float arrays (already bf16-exact) into a shuffled paged pool."""
    keys = np.asarray(keys, dtype=np.float32)
    vals = np.asarray(vals, dtype=np.float32)
    if keys.ndim == 2:
        keys, vals = keys[None], vals[None]
    H, T, D = keys.shape
    npg = -(-T // page_size)
    perm = rng.permutation(npg + 3)[:npg].astype(np.int32)        # spare pages stay unused
    kc = np.zeros((npg + 3, H, page_size, D), np.uint16)
    vc = np.zeros_like(kc)
    pad = npg * page_size
    for h in range(H):
        kb = np.zeros((pad, D), np.uint16)
        vb = np.zeros((pad, D), np.uint16)
        kb[:T] = f32_to_bf16_bits(keys[h])
        vb[:T] = f32_to_bf16_bits(vals[h])
        kc[perm, h] = kb.reshape(npg, page_size, D)
        vc[perm, h] = vb.reshape(npg, page_size, D)
    assert np.array_equal(O.widen_bf16(f32_to_bf16_bits(keys)), keys.astype(np.float64)), "keys not bf16-exact"
    return kc, vc, perm


def _grid_values(rng, shape, step=0.125, lim=8):
    """Values on a 1/8 grid with |x| < 1: sums of a few stay exactly representable in bf16."""
    return (rng.integers(-lim + 1, lim, size=shape) * step).astype(np.float64)


# ---------------------------------------------------------------------------
# 1. hand-derived example (scale 1, logits on a ln2 grid so every weight is a power of 2)
# ---------------------------------------------------------------------------

def test_hand_derived_example():
    # D=2, one 2-dim subspace, 2 codewords, 2 clusters; sink = position 0, indexed
    # positions 1..4, tail = position 5. q = (ln 2, 0) so a key with first coord x
    # has weight 2^x.
    #   slot  pos  id code  recon-x  actual-x   v
    #    0     1    0   0      0        0       2
    #    1     2    1   1      2        3      10   <- top-1 by approx score
    #    2     3    1   0      1        1       4
    #    3     4    0   1      1        1       6
    #   sink pos0 x=0 v=1; tail pos5 x=1 v=3; second value coordinate is 1 everywhere.
    # Cluster means over ALL members: mu0 = (2+6)/2 = 4, mu1 = (10+4)/2 = 7.
    # Exact set {0, 2, 5}: weights 1, 8, 2.  Unselected: slot0 (w 1, c0), slot2 (w 2, c1),
    # slot3 (w 2, c0) -> W0 = 3, W1 = 2.
    #   num = 1*1 + 8*10 + 2*3 + 3*4 + 2*7 = 113, den = 1 + 8 + 2 + 3 + 2 = 16.
    # Background off: 87 / 11. Dense: (1*1+1*2+8*10+2*4+2*6+2*3)/16 = 109/16.
    ln2 = math.log(2.0)
    q = np.array([[ln2, 0.0]])
    keys = np.array([[0, 0], [0, 0], [3, 0], [1, 0], [1, 0], [1, 0]], dtype=np.float64)
    vals = np.array([[1, 1], [2, 1], [10, 1], [4, 1], [6, 1], [3, 1]], dtype=np.float64)
    cent = np.array([[0.0, 0.0], [1.0, 0.0]])
    cb = np.array([[[0.0, 0.0], [1.0, 0.0]]])            # [M=1][ncode=2][dsub=2]
    ids = np.array([0, 1, 1, 0])
    codes = np.array([[0], [1], [0], [1]], dtype=np.uint8)
    kc, vc, bt = _paged(keys, vals, 2, np.random.default_rng(0))
    r = O.decode_unit(q, kc, vc, bt, 0, 6, 2, cent, cb, codes, ids, 4, 1, 1.0, k=1)
    assert list(r["sel"]) == [1]
    np.testing.assert_allclose(r["out"][0], [113 / 16, 1.0], rtol=1e-12)
    np.testing.assert_allclose(r["s_hat"][0], [0, 2 * ln2, ln2, ln2], rtol=1e-12, atol=1e-15)
    r0 = O.decode_unit(q, kc, vc, bt, 0, 6, 2, cent, cb, codes, ids, 4, 1, 1.0, k=1, background=False)
    np.testing.assert_allclose(r0["out"][0], [87 / 11, 1.0], rtol=1e-12)
    d = O.dense_unit(q, O.widen_bf16(f32_to_bf16_bits(keys)), vals, 1.0)
    np.testing.assert_allclose(d[0], [109 / 16, 1.0], rtol=1e-12)
    cnt, sm, mu = O.cluster_means(vals[1:5], ids, 2)
    np.testing.assert_array_equal(cnt, [2, 2])
    np.testing.assert_allclose(mu[:, 0], [4.0, 7.0])


# ---------------------------------------------------------------------------
# 2. approximate logits on zero-noise keys equal exact logits
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,dsub,ncode,C", [(16, 8, 256, 64), (4, 4, 8, 3), (2, 3, 5, 7)])
def test_zero_noise_keys_give_exact_logits(M, dsub, ncode, C):
    rng = np.random.default_rng(1)
    D = M * dsub
    G, N = 3, 200
    q = rng.standard_normal((G, D))
    cent = rng.standard_normal((C, D))
    cb = 0.3 * rng.standard_normal((M, ncode, dsub))
    ids = rng.integers(0, C, N)
    codes = rng.integers(0, ncode, (N, M)).astype(np.uint8)
    # reconstruct every key explicitly, then take plain dot products
    keys = np.stack([cent[ids[j]] + np.concatenate([cb[s, codes[j, s]] for s in range(M)]) for j in range(N)])
    scale = 1.0 / math.sqrt(D)
    exact = scale * q @ keys.T
    approx = O.approx_logits(q, cent, cb, codes, ids, scale)
    np.testing.assert_allclose(approx, exact, rtol=0, atol=1e-12)


def test_lut_is_subspace_dot_product():
    rng = np.random.default_rng(2)
    M, ncode, dsub = 4, 6, 3
    q = rng.standard_normal(M * dsub)
    cb = rng.standard_normal((M, ncode, dsub))
    lut = O.pq_lut(q, cb)
    for s in range(M):
        for m in range(ncode):
            assert lut[s, m] == pytest.approx(float(np.dot(q[s * dsub:(s + 1) * dsub], cb[s, m])), abs=1e-13)


# ---------------------------------------------------------------------------
# 3. full budget == dense;  equal values per cluster + zero-noise keys == dense at any budget
# ---------------------------------------------------------------------------

def test_full_budget_equals_dense_on_generated_workload():
    w = workload("tiny_4k", T=600, C=8, n_recent=40, n_needles=4)
    bt = make_batch(w)
    scale = 1.0 / math.sqrt(w.D)
    res = O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, bt.centroids,
                          bt.codebooks, bt.codes_rec, bt.ids_rec, bt.n_indexed, w.n_sink, scale,
                          budget=1.0)
    dense = O.oracle_dense(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, scale)
    for key, r in res.items():
        assert r["k"] == w.n_indexed
        np.testing.assert_allclose(r["out"], dense[key], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("k", [0, 1, 5, 17])
def test_equal_cluster_values_and_exact_keys_equal_dense(k):
    rng = np.random.default_rng(3)
    M, dsub, ncode, C, D = 4, 4, 8, 3, 16
    s0, N, R = 3, 26, 5
    T = s0 + N + R
    cent = _grid_values(rng, (C, D))
    cb = _grid_values(rng, (M, ncode, dsub))
    ids_all = rng.integers(0, C, T)
    codes_all = rng.integers(0, ncode, (T, M))
    keys = np.stack([cent[ids_all[j]] + np.concatenate([cb[s, codes_all[j, s]] for s in range(M)])
                     for j in range(T)])
    mu = _grid_values(rng, (C, D))
    vals = mu[ids_all]                                   # every member of a cluster has the same value
    q = rng.standard_normal((2, D)).astype(np.float32).astype(np.float64)
    kc, vc, bt = _paged(keys, vals, 4, rng)
    scale = 0.25
    r = O.decode_unit(q, kc, vc, bt, 0, T, 4, cent, cb, codes_all[s0:s0 + N].astype(np.uint8),
                      ids_all[s0:s0 + N], N, s0, scale, k=k)
    d = O.dense_unit(q, keys, vals, scale)
    np.testing.assert_allclose(r["out"], d, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# 4. special cases
# ---------------------------------------------------------------------------

def test_single_cluster_no_exact_tokens_gives_cluster_mean():
    rng = np.random.default_rng(4)
    D, N = 8, 30
    keys = _grid_values(rng, (N, D))
    vals = _grid_values(rng, (N, D))
    kc, vc, bt = _paged(keys, vals, 4, rng)
    cent = rng.standard_normal((1, D))
    cb = rng.standard_normal((2, 5, 4))
    codes = rng.integers(0, 5, (N, 2)).astype(np.uint8)
    q = 3.0 * rng.standard_normal((3, D))
    r = O.decode_unit(q, kc, vc, bt, 0, N, 4, cent, cb, codes, np.zeros(N, int), N, 0, 0.7, k=0)
    for g in range(3):
        np.testing.assert_allclose(r["out"][g], vals.mean(axis=0), rtol=1e-12, atol=1e-14)


def test_identical_query_heads_give_identical_outputs():
    w = workload("tiny_4k", T=400, C=8, n_recent=30, n_needles=0)
    bt = make_batch(w)
    bt.q[0, :] = bt.q[0, 0]
    res = O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, bt.centroids,
                          bt.codebooks, bt.codes_rec, bt.ids_rec, bt.n_indexed, w.n_sink, 0.088)
    out = res[(0, 0)]["out"]
    for g in range(1, w.G):
        np.testing.assert_array_equal(out[g], out[0])


def test_no_index_is_dense():
    w = workload("tiny_4k", T=100, C=4, n_recent=84, n_needles=0)   # n_indexed = 0
    bt = make_batch(w)
    assert w.n_indexed == 0
    res = O.oracle_decode(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, bt.centroids,
                          bt.codebooks, bt.codes_rec, bt.ids_rec, bt.n_indexed, w.n_sink, 0.088)
    dense = O.oracle_dense(bt.q, bt.k_cache, bt.v_cache, bt.block_table, bt.seq_lens, 0.088)
    np.testing.assert_allclose(res[(0, 0)]["out"], dense[(0, 0)], rtol=1e-13)


def test_k_is_floor_of_budget_times_indexed_count():
    assert O.decode_k(0.01, 3952) == 39
    assert O.decode_k(0.01, 130032) == 1300
    assert O.decode_k(0.01, 100) == 1
    assert O.decode_k(0.01, 99) == 0
    assert O.decode_k(1.0, 57) == 57
    assert O.decode_k(0.3, 10, k_override=4) == 4
    assert O.decode_k(0.3, 10, k_override=40) == 10


# ---------------------------------------------------------------------------
# 5. brute force on tiny inputs
# ---------------------------------------------------------------------------

def _beats(key, a, b):
    return key[a] > key[b] or (key[a] == key[b] and a < b)


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_subset_enumeration(seed):
    rng = np.random.default_rng(10 + seed)
    n = int(rng.integers(1, 13))
    sigma = rng.integers(-3, 4, n) * 0.25 if seed % 2 else rng.standard_normal(n)   # ties in half the cases
    key = sigma.astype(np.float32)
    for k in range(0, min(3, n) + 1):
        winners = [S for S in itertools.combinations(range(n), k)
                   if all(_beats(key, a, b) for a in S for b in range(n) if b not in S)]
        assert len(winners) == 1
        assert list(O.select_topk(sigma, k)) == list(winners[0])


def test_topk_float32_decision():
    # two scores distinct in float64 but equal in float32: the smaller index wins
    sigma = np.array([0.5, 0.5 + 1e-12, 0.1])
    assert list(O.select_topk(sigma, 1)) == [0]


@pytest.mark.parametrize("seed", range(4))
def test_encode_matches_loops(seed):
    rng = np.random.default_rng(20 + seed)
    C, M, dsub, ncode = 5, 2, 3, 6
    D = M * dsub
    cent = _grid_values(rng, (C, D))
    cb = _grid_values(rng, (M, ncode, dsub))
    keys = list(_grid_values(rng, (12, D)))
    keys.append((cent[1] + cent[3]) / 2)                   # exact centroid tie -> lower id
    keys = np.array(keys)
    ids, codes, _ = O.encode_keys(keys, cent, cb)
    for j, kv in enumerate(keys):
        best, bi = None, -1
        for c in range(C):
            d = sum((float(kv[i]) - float(cent[c, i])) ** 2 for i in range(D))
            if best is None or d < best:
                best, bi = d, c
        assert ids[j] == bi
        r = [float(kv[i]) - float(cent[bi, i]) for i in range(D)]
        for s in range(M):
            best, bm = None, -1
            for m in range(ncode):
                d = sum((r[s * dsub + i] - float(cb[s, m, i])) ** 2 for i in range(dsub))
                if best is None or d < best:
                    best, bm = d, m
            assert codes[j, s] == bm
    assert ids[-1] == 1


def _loop_decode(q, keys, vals, cent, cb, codes, ids, s0, N, T, scale, k):
    """Per-token loop: every weight and every mean written out."""
    G, D = q.shape
    M, ncode, dsub = cb.shape
    C = cent.shape[0]
    shat = [[scale * (sum(q[g, d] * cent[ids[j], d] for d in range(D)) +
                      sum(sum(q[g, s * dsub + d] * cb[s, codes[j, s], d] for d in range(dsub)) for s in range(M)))
             for j in range(N)] for g in range(G)]
    sig = [max(shat[g][j] for g in range(G)) for j in range(N)]
    order = sorted(range(N), key=lambda j: (-float(np.float32(sig[j])), j))
    sel = set(order[:k])
    mu = []
    for c in range(C):
        mem = [j for j in range(N) if ids[j] == c]
        mu.append([sum(vals[s0 + j, d] for j in mem) / len(mem) if mem else 0.0 for d in range(D)])
    out = np.zeros((G, D))
    for g in range(G):
        terms = []                                   # (logit, value vector)
        for t in range(T):
            if s0 <= t < s0 + N:
                j = t - s0
                if j in sel:
                    terms.append((scale * sum(q[g, d] * keys[t, d] for d in range(D)), vals[t]))
                else:
                    terms.append((shat[g][j], mu[ids[j]]))
            else:
                terms.append((scale * sum(q[g, d] * keys[t, d] for d in range(D)), vals[t]))
        m = max(l for l, _ in terms)
        den = sum(math.exp(l - m) for l, _ in terms)
        for d in range(D):
            out[g, d] = sum(math.exp(l - m) * v[d] for l, v in terms) / den
    return out, sorted(sel)


@pytest.mark.parametrize("seed,k", [(0, 0), (1, 2), (2, 3), (3, 7)])
def test_decode_matches_per_token_loop(seed, k):
    rng = np.random.default_rng(30 + seed)
    M, dsub, ncode, C = 2, 3, 4, 3
    D = M * dsub
    s0, N, R = 2, 16, 6
    T = s0 + N + R
    keys = _grid_values(rng, (T, D))
    vals = _grid_values(rng, (T, D))
    cent = rng.standard_normal((C, D))
    cb = rng.standard_normal((M, ncode, dsub))
    ids = rng.integers(0, C, N)
    codes = rng.integers(0, ncode, (N, M)).astype(np.uint8)
    q = rng.standard_normal((2, D))
    kc, vc, bt = _paged(keys, vals, 4, rng)
    r = O.decode_unit(q, kc, vc, bt, 0, T, 4, cent, cb, codes, ids, N, s0, 0.6, k=k)
    ref, sel = _loop_decode(q, keys, vals, cent, cb, codes, ids, s0, N, T, 0.6, k)
    assert list(r["sel"]) == sel
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-12)


def test_cluster_means_by_loop():
    rng = np.random.default_rng(40)
    V = rng.standard_normal((50, 4))
    ids = rng.integers(0, 6, 50)
    ids[ids == 5] = 4                                    # cluster 5 empty
    cnt, sm, mu = O.cluster_means(V, ids, 6)
    for c in range(6):
        mem = [i for i in range(50) if ids[i] == c]
        assert cnt[c] == len(mem)
        exp = np.mean(V[mem], axis=0) if mem else np.zeros(4)
        np.testing.assert_allclose(mu[c], exp, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------------------
# 6. the generator's recorded index is consistent with its keys
# ---------------------------------------------------------------------------

def test_recorded_codes_are_nearest_encoding_of_generated_keys():
    """Keys = centroid + codewords + small noise: encoding recovers the drawn cluster and codes
    (except the needles, whose keys were replaced)."""
    w = workload("tiny_4k", T=700, C=16, n_recent=50, n_needles=4)
    bt = make_batch(w)
    N = w.n_indexed
    pos = w.n_sink + np.arange(N)
    keys = O.unit_rows(bt.k_cache, bt.block_table[0], 0, pos, w.page_size)
    ids, codes, _ = O.encode_keys(keys, bt.centroids[0, 0], bt.codebooks[0, 0])
    needle = np.zeros(N, bool)
    needle[bt.needle_pos[0, 0] - w.n_sink] = True
    assert np.array_equal(ids[~needle], bt.ids_rec[0, 0, :N][~needle].astype(np.int64))
    agree = (codes[~needle] == bt.codes_rec[0, 0, :N][~needle]).mean()
    assert agree > 0.999
