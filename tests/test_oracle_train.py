"""Pins of the oracle's index training (Lloyd k-means for the coarse centroids, per-subspace
Lloyd k-means on the residuals for the codebooks), checked against closed forms, invariants
and brute force, not against the oracle itself."""
import numpy as np

import oracle as O


def _blobs(rng, k, per, d, spread=100.0, noise=0.01):
    centres = rng.standard_normal((k, d)) * spread
    labels = np.repeat(np.arange(k), per)
    X = centres[labels] + noise * rng.standard_normal((k * per, d))
    return X.astype(np.float32), labels, centres


def test_separated_clusters_are_recovered_in_one_step():
    rng = np.random.default_rng(1)
    X, labels, _ = _blobs(rng, 5, 40, 16)
    init = X[[0, 40, 80, 120, 160]]          # one row of each blob
    a = O.lloyd_assign(X, init)
    assert np.array_equal(a, labels)
    cen = O.lloyd_update(X, a, init)
    for c in range(5):                       # each centre is its blob's mean
        np.testing.assert_allclose(cen[c], X[labels == c].astype(np.float64).mean(0), rtol=0, atol=1e-4)


def test_objective_never_increases():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((300, 8)).astype(np.float32)
    cen = X[rng.choice(300, 12, replace=False)].copy()
    prev = np.inf
    for _ in range(8):
        a = O.lloyd_assign(X, cen)
        obj = O.kmeans_objective(X, cen, a)
        assert obj <= prev * (1 + 1e-6)
        prev = obj
        cen = O.lloyd_update(X, a, cen)


def test_empty_centre_keeps_its_value_and_ties_go_low():
    X = np.array([[0.0, 0.0], [1.0, 0.0]], dtype=np.float32)
    cen = np.array([[0.5, 0.0], [0.5, 0.0], [50.0, 50.0]], dtype=np.float32)   # 0 and 1 tie everywhere
    a = O.lloyd_assign(X, cen)
    assert list(a) == [0, 0]
    new = O.lloyd_update(X, a, cen)
    np.testing.assert_array_equal(new[0], [0.5, 0.0])      # mean of both rows
    np.testing.assert_array_equal(new[1:], cen[1:])         # empty centres unchanged


def test_lloyd_step_matches_brute_force_loops():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((23, 5)).astype(np.float32)
    cen = rng.standard_normal((4, 5)).astype(np.float32)
    a = O.lloyd_assign(X, cen)
    new = O.lloyd_update(X, a, cen)
    for j in range(23):                      # explicit loops, first minimum wins
        best, bi = None, -1
        for c in range(4):
            d = np.float32(sum((float(X[j, t]) - float(cen[c, t])) ** 2 for t in range(5)))
            if best is None or d < best:
                best, bi = d, c
        assert a[j] == bi
    for c in range(4):
        rows = [j for j in range(23) if a[j] == c]
        if rows:
            m = [sum(float(X[j, t]) for j in rows) / len(rows) for t in range(5)]
            np.testing.assert_allclose(new[c], np.float32(m), rtol=0, atol=1e-6)
        else:
            np.testing.assert_array_equal(new[c], cen[c])


def test_noise_free_keys_recover_the_generating_clusters_and_codes():
    """Keys built exactly as centroid + codewords (well-separated centroids and codewords,
    one initial row per cluster and per codeword): training recovers the generating
    cluster of every key and, on the residuals, its generating code in every subspace."""
    rng = np.random.default_rng(4)
    C, M, ncode, dsub, n = 4, 2, 4, 4, 400
    cent = (rng.standard_normal((C, M * dsub)) * 50).astype(np.float32)
    books = (rng.standard_normal((M, ncode, dsub)) * 3).astype(np.float32)
    ids = rng.integers(0, C, n)
    codes = rng.integers(0, ncode, (n, M))
    X = (cent[ids] + books[np.arange(M)[None, :], codes].reshape(n, -1)).astype(np.float32)
    init = [int(np.nonzero(ids == c)[0][0]) for c in range(C)]
    for s in range(M):
        init += [int(np.nonzero(codes[:, s] == m)[0][0]) for m in range(ncode)]
    cen, bks, a = O.train_unit(X, np.array(init), C, coarse_iters=3, pq_iters=3, M=M, ncode=ncode)
    assert np.array_equal(a, ids)
    for c in range(C):                       # each centroid is its cluster's mean key
        np.testing.assert_allclose(cen[c], X[ids == c].astype(np.float64).mean(0), rtol=0, atol=1e-3)
    R = X.astype(np.float64) - cen[a].astype(np.float64)
    for s in range(M):
        got = O.lloyd_assign(R[:, s * dsub:(s + 1) * dsub].astype(np.float32), bks[s])
        assert np.array_equal(got, codes[:, s])


def test_train_unit_shapes_and_determinism():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((500, 128)).astype(np.float32)
    init = rng.choice(500, 8 + 16 * 16, replace=True)
    c1, b1, a1 = O.train_unit(X, init, 8, 2, 2, M=16, ncode=16)
    c2, b2, a2 = O.train_unit(X, init, 8, 2, 2, M=16, ncode=16)
    assert c1.shape == (8, 128) and b1.shape == (16, 16, 8) and a1.shape == (500,)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(b1, b2)


def test_single_centre_is_the_mean_of_all_keys_and_codewords_start_at_seed_residuals():
    """C = 1: one coarse step puts the centroid at the mean of every key (closed form); with no
    codebook step, codeword m of subspace s is the subspace-s residual of its seed key."""
    rng = np.random.default_rng(7)
    X = (rng.standard_normal((50, 16)) * 3).astype(np.float32)
    init = rng.integers(0, 50, size=1 + 2 * 4)
    cen, books, a = O.train_unit(X, init, C=1, coarse_iters=1, pq_iters=0, M=2, ncode=4)
    np.testing.assert_allclose(cen[0], X.astype(np.float64).mean(0), rtol=0, atol=1e-5)
    assert (a == 0).all()
    R = X.astype(np.float64) - cen[0].astype(np.float64)
    for s in range(2):
        for m in range(4):
            np.testing.assert_allclose(books[s, m], R[init[1 + s * 4 + m], 8 * s:8 * s + 8], rtol=0, atol=1e-6)


def test_training_does_not_depend_on_key_order():
    """Lloyd k-means sees a set: permuting the keys (and the seed slots with them) gives the
    same centroids and codebooks, and the assignment permuted alike."""
    rng = np.random.default_rng(8)
    X = rng.standard_normal((120, 16)).astype(np.float32)
    C, M, ncode = 5, 2, 8
    init = rng.choice(120, size=C + M * ncode, replace=True)
    perm = rng.permutation(120)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(120)
    cen1, books1, a1 = O.train_unit(X, init, C, 3, 3, M=M, ncode=ncode)
    cen2, books2, a2 = O.train_unit(X[perm], inv[init], C, 3, 3, M=M, ncode=ncode)
    np.testing.assert_allclose(cen1, cen2, rtol=0, atol=1e-6)
    np.testing.assert_allclose(books1, books2, rtol=0, atol=1e-6)
    assert np.array_equal(a1[perm], a2)
