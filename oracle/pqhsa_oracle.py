"""float64 oracle of one PQ-HSA decode step (and of the index build / append).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke entry and the bench's
CPU-baseline leg, never by the library. It shares no code with the CUDA path.

Source: the rit.work article "pq-hsa-long-context-attention" (PQ-HSA), section
"Как приблизительные оценки возвращают отброшенный контекст" (how approximate
scores return the discarded context). What it states, restated:

* an IVF-PQ index groups the keys into clusters and stores a compressed code per
  key; from it an approximate attention logit is computed for every indexed
  token;
* the same scores do two jobs: the best-scoring tokens (a 1 % read budget in the
  main experiments) are read from the KV cache and attended exactly; every
  other indexed token stays in the shared softmax normalisation through its
  approximate logit;
* the values of those unread tokens are not read: their weights are summed per
  index group and multiplied by that group's mean value;
* the first tokens and a recent window stay exact; the index is built after
  prefill and new tokens are added to it in batches.

Readings where the article is silent (each is also listed in the design notes):

* residual PQ: a key is approximated by centroid_a + concat_s codeword_s[code_s]
  (so the approximate logit is scale * (q . centroid_a + sum_s LUT_s[code_s]));
* every indexed token is scored (every cluster is visited);
* GQA: one selected set per KV head, ranked by the max over the group's query
  heads of the approximate logit; ties go to the smaller position; the ranking
  decision is taken on float32-rounded scores (the kernel's precision);
* k = floor(budget * N) with N the indexed count, computed in float64;
* a cluster's mean value is the mean over all its indexed members;
* nearest-centroid and nearest-codeword decisions compare float32-rounded
  squared distances and break ties to the lower index.

Everything here is computed from its definition in float64, with numpy; no
blocking, fusion or reordering beyond chunking independent rows.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np


# ---------------------------------------------------------------------------
# Input access
# ---------------------------------------------------------------------------

def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    return (np.asarray(bits).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def unit_rows(cache_bits: np.ndarray, block_table_row: np.ndarray, h: int,
              positions: np.ndarray, page_size: int) -> np.ndarray:
    """Rows of KV head h at the given token positions, read through one block-table row.

    cache_bits: [num_pages, Hkv, page_size, D] uint16 (bf16).
    """
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(block_table_row, dtype=np.int64)[positions // page_size]
    return widen_bf16(cache_bits[pages, h, positions % page_size])


# ---------------------------------------------------------------------------
# Approximate logits (IVF coarse term + PQ residual table)
# ---------------------------------------------------------------------------

def pq_lut(q: np.ndarray, codebooks: np.ndarray) -> np.ndarray:
    """LUT[s, m] = sum_d q[s*dsub + d] * codeword[s, m, d] for one query vector.

    q: [D]; codebooks: [M, ncode, dsub]  ->  [M, ncode] float64.
    """
    M, ncode, dsub = codebooks.shape
    qs = np.asarray(q, dtype=np.float64).reshape(M, dsub)
    cb = np.asarray(codebooks, dtype=np.float64)
    return np.einsum("sd,smd->sm", qs, cb)


def approx_logits(qG: np.ndarray, centroids: np.ndarray, codebooks: np.ndarray,
                  codes: np.ndarray, ids: np.ndarray, scale: float) -> np.ndarray:
    """s_hat[g, j] = scale * (q_g . centroid_{ids[j]} + sum_s LUT_g[s, codes[j, s]]).

    qG: [G, D]; centroids: [C, D]; codes: [N, M] uint8; ids: [N]  ->  [G, N] float64.
    """
    qG = np.asarray(qG, dtype=np.float64)
    cent = np.asarray(centroids, dtype=np.float64)
    codes = np.asarray(codes, dtype=np.int64)
    ids = np.asarray(ids, dtype=np.int64)
    G = qG.shape[0]
    M = codebooks.shape[0]
    N = codes.shape[0]
    out = np.empty((G, N), dtype=np.float64)
    for g in range(G):
        lut = pq_lut(qG[g], codebooks)                  # [M, ncode]
        coarse = cent @ qG[g]                           # [C]: q . centroid_c
        resid = np.zeros(N, dtype=np.float64)
        for s in range(M):
            resid += lut[s, codes[:, s]]
        out[g] = float(scale) * (coarse[ids] + resid)
    return out


def decode_k(budget: float, n_indexed: int, k_override: Optional[int] = None) -> int:
    """Number of indexed tokens read exactly: floor(budget * N) in float64, clipped to [0, N]."""
    if k_override is not None and k_override >= 0:
        return int(min(k_override, n_indexed))
    return int(min(n_indexed, max(0, math.floor(float(budget) * float(n_indexed)))))


def select_topk(sigma: np.ndarray, k: int) -> np.ndarray:
    """Indices (into the indexed range) of the k largest scores, returned in ascending order.

    The ranking is taken on float32-rounded scores; equal scores go to the smaller index.
    """
    n = sigma.shape[0]
    k = int(min(k, n))
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    key = np.asarray(sigma, dtype=np.float64).astype(np.float32)
    idx = np.arange(n, dtype=np.int64)
    order = np.lexsort((idx, -key.astype(np.float64)))   # primary: score desc; then index asc
    return np.sort(order[:k])


# ---------------------------------------------------------------------------
# Cluster mean values
# ---------------------------------------------------------------------------

def cluster_means(V: np.ndarray, ids: np.ndarray, C: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """count[c], sum_v[c] and mean_v[c] = sum_v[c] / count[c] (0 for an empty cluster)."""
    V = np.asarray(V, dtype=np.float64)
    ids = np.asarray(ids, dtype=np.int64)
    D = V.shape[1] if V.ndim == 2 else 0
    count = np.bincount(ids, minlength=C).astype(np.int64)[:C]
    sum_v = np.zeros((C, D), dtype=np.float64)
    np.add.at(sum_v, ids, V)
    mean_v = np.zeros((C, D), dtype=np.float64)
    nz = count > 0
    mean_v[nz] = sum_v[nz] / count[nz, None]
    return count, sum_v, mean_v


# ---------------------------------------------------------------------------
# One decode step for one (sequence, KV head) unit
# ---------------------------------------------------------------------------

def dense_unit(qG: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q_g K^T) V for each query head of the group: [G, D]."""
    qG = np.asarray(qG, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros((qG.shape[0], V.shape[1] if V.ndim == 2 else qG.shape[1]))
    s = float(scale) * (qG @ K.T)                        # [G, T]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return (p @ V) / p.sum(axis=1, keepdims=True)


def decode_unit(qG: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                block_table_row: np.ndarray, h: int, seq_len: int, page_size: int,
                centroids: np.ndarray, codebooks: np.ndarray,
                codes: np.ndarray, ids: np.ndarray, n_indexed: int, n_sink: int,
                scale: float, k: int, background: bool = True,
                mean_v: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """One PQ-HSA decode step for the G query heads of one KV head.

    Token sets: sink S = [0, s0), indexed I = [s0, s0 + n_indexed), exact tail
    R = [s0 + n_indexed, T). K = the k selected indexed tokens, U = I minus K.
    Output per query head g, with a common reference M*:

        O_g = (sum_{j in S+K+R} e^{s_gj - M*} v_j + sum_c W_gc mu_c)
              / (sum_{j in S+K+R} e^{s_gj - M*} + sum_{j in U} e^{shat_gj - M*}),
        W_gc = sum_{j in U, a_j = c} e^{shat_gj - M*},

    s_gj = scale * q_g . k_j (exact), shat the approximate logit, mu_c the mean
    value of cluster c over all its indexed members. With background=False the
    unselected tokens get weight 0 (plain top-k sparse attention).
    codes/ids are indexed by slot i <-> position s0 + i.
    """
    qG = np.asarray(qG, dtype=np.float64)
    G, D = qG.shape
    T = int(seq_len)
    s0 = min(int(n_sink), T)
    N = int(n_indexed) if T > s0 else 0
    N = max(0, min(N, T - s0))
    C = centroids.shape[0]

    if N == 0:
        pos = np.arange(T)
        K = unit_rows(k_cache, block_table_row, h, pos, page_size)
        V = unit_rows(v_cache, block_table_row, h, pos, page_size)
        return {"out": dense_unit(qG, K, V, scale), "s_hat": np.zeros((G, 0)),
                "sel": np.zeros(0, dtype=np.int64), "sigma": np.zeros(0)}

    codes_I = np.asarray(codes)[:N]
    ids_I = np.asarray(ids)[:N].astype(np.int64)
    s_hat = approx_logits(qG, centroids, codebooks, codes_I, ids_I, scale)   # [G, N]
    sigma = s_hat.max(axis=0)                                                 # [N]
    k = int(min(max(k, 0), N))
    sel = select_topk(sigma, k)                                               # slots, ascending

    exact_pos = np.concatenate([np.arange(s0), s0 + sel, np.arange(s0 + N, T)]).astype(np.int64)
    Ke = unit_rows(k_cache, block_table_row, h, exact_pos, page_size)
    Ve = unit_rows(v_cache, block_table_row, h, exact_pos, page_size)
    s_exact = float(scale) * (qG @ Ke.T)                                      # [G, |E|]

    unsel = np.ones(N, dtype=bool)
    unsel[sel] = False
    if mean_v is None:
        V_I = unit_rows(v_cache, block_table_row, h, s0 + np.arange(N), page_size)
        _, _, mu = cluster_means(V_I, ids_I, C)
    else:
        mu = np.asarray(mean_v, dtype=np.float64)

    out = np.zeros((G, D), dtype=np.float64)
    for g in range(G):
        su = s_hat[g, unsel] if background else np.zeros(0)
        m_star = -np.inf
        if s_exact.shape[1]:
            m_star = s_exact[g].max()
        if su.size:
            m_star = max(m_star, su.max())
        pe = np.exp(s_exact[g] - m_star)
        num = pe @ Ve
        den = pe.sum()
        if su.size:
            pu = np.exp(su - m_star)
            W = np.bincount(ids_I[unsel], weights=pu, minlength=C)[:C]       # per-cluster weight sums
            num = num + W @ mu
            den = den + pu.sum()
        out[g] = num / den
    return {"out": out, "s_hat": s_hat, "sel": sel, "sigma": sigma}


# ---------------------------------------------------------------------------
# Encoding new keys (nearest centroid, then nearest codeword per subspace)
# ---------------------------------------------------------------------------

def encode_keys(keys: np.ndarray, centroids: np.ndarray, codebooks: np.ndarray,
                chunk: int = 256) -> Tuple[np.ndarray, np.ndarray, Dict[str, np.ndarray]]:
    """ids[j] = argmin_c sum_d (k_jd - c_d)^2; r = k_j - centroid_{ids[j]};
    codes[j, s] = argmin_m sum_{d<dsub} (r_{s*dsub+d} - codeword[s, m, d])^2.

    Distances are evaluated in float64 and compared as float32 (lowest index wins
    ties). Also returns the float64 distances of the winners and runners-up, so a
    caller can recognise near-ties.
    """
    keys = np.asarray(keys, dtype=np.float64)
    cent = np.asarray(centroids, dtype=np.float64)
    cb = np.asarray(codebooks, dtype=np.float64)
    n, D = keys.shape
    M, ncode, dsub = cb.shape
    ids = np.zeros(n, dtype=np.int64)
    codes = np.zeros((n, M), dtype=np.int64)
    gap_c = np.zeros(n)
    gap_m = np.zeros((n, M))
    best_c = np.zeros(n)
    best_m = np.zeros((n, M))
    for a in range(0, n, chunk):
        kk = keys[a:a + chunk]
        d = ((kk[:, None, :] - cent[None, :, :]) ** 2).sum(axis=2)           # [n, C]
        d32 = d.astype(np.float32)
        i = np.argmin(d32, axis=1)
        ids[a:a + chunk] = i
        srt = np.sort(d, axis=1)
        best_c[a:a + chunk] = srt[:, 0]
        gap_c[a:a + chunk] = srt[:, 1] - srt[:, 0] if d.shape[1] > 1 else np.inf
        r = kk - cent[i]                                                     # [n, D]
        rs = r.reshape(-1, M, dsub)
        dm = ((rs[:, :, None, :] - cb[None, :, :, :]) ** 2).sum(axis=3)     # [n, M, ncode]
        codes[a:a + chunk] = np.argmin(dm.astype(np.float32), axis=2)
        srt = np.sort(dm, axis=2)
        best_m[a:a + chunk] = srt[:, :, 0]
        gap_m[a:a + chunk] = srt[:, :, 1] - srt[:, :, 0]
    return ids, codes, {"gap_c": gap_c, "gap_m": gap_m, "best_c": best_c, "best_m": best_m}


# ---------------------------------------------------------------------------
# Index training (the step before the path: the index is built after prefill)
# ---------------------------------------------------------------------------
# The article says the index is built after prefill and groups the keys (IVF) with
# compressed per-key codes (PQ); it does not say how the centroids and codebooks are
# found. Reading: the plain Lloyd k-means iteration, for the coarse centroids on the
# unit's keys and, per subspace, for the codebook on the residuals (key minus its
# centroid). Initial centres are given rows of the training set (the draw is an input).

def lloyd_assign(X: np.ndarray, centres: np.ndarray, chunk: int = 256) -> np.ndarray:
    """a[j] = argmin_c sum_d (X_jd - centre_cd)^2: float64 distances compared as float32,
    ties to the lower index."""
    X = np.asarray(X, dtype=np.float64)
    cen = np.asarray(centres, dtype=np.float64)
    a = np.zeros(X.shape[0], dtype=np.int64)
    for i in range(0, X.shape[0], chunk):
        d = ((X[i:i + chunk, None, :] - cen[None, :, :]) ** 2).sum(axis=2)
        a[i:i + chunk] = np.argmin(d.astype(np.float32), axis=1)   # first minimum = lowest index
    return a


def lloyd_update(X: np.ndarray, a: np.ndarray, centres: np.ndarray) -> np.ndarray:
    """centre_c = mean of the rows assigned to c (float64, rounded to float32); a centre
    with no rows keeps its value."""
    X = np.asarray(X, dtype=np.float64)
    k = centres.shape[0]
    sums = np.zeros((k, X.shape[1]))
    np.add.at(sums, a, X)
    cnt = np.bincount(a, minlength=k)
    out = np.asarray(centres, dtype=np.float64).copy()
    nz = cnt > 0
    out[nz] = sums[nz] / cnt[nz, None]
    return out.astype(np.float32)


def kmeans_objective(X: np.ndarray, centres: np.ndarray, a: np.ndarray) -> float:
    """sum_j |X_j - centre_{a_j}|^2 in float64."""
    X = np.asarray(X, dtype=np.float64)
    return float(((X - np.asarray(centres, dtype=np.float64)[a]) ** 2).sum())


def train_unit(keys: np.ndarray, init_slots: np.ndarray, C: int, coarse_iters: int, pq_iters: int,
               M: int = 16, ncode: int = 256) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Centroids [C, D] and codebooks [M, ncode, D/M] of one unit from its training keys [n, D]
    (float32 values of the bf16 keys).

    Coarse: centres start at rows init_slots[:C]; coarse_iters Lloyd iterations (assign,
    update); then a final assignment gives the residuals r_j = k_j - centroid_{a_j}
    (float32). Codebook s: centres start at the subspace-s residuals of rows
    init_slots[C + s*ncode : C + (s+1)*ncode]; pq_iters Lloyd iterations on the residuals'
    subspace s. Returns (centroids, codebooks, final coarse assignment).
    """
    X = np.asarray(keys, dtype=np.float32)
    init_slots = np.asarray(init_slots, dtype=np.int64)
    cent = X[init_slots[:C]].copy()
    for _ in range(coarse_iters):
        cent = lloyd_update(X, lloyd_assign(X, cent), cent)
    a = lloyd_assign(X, cent)
    R = (X.astype(np.float64) - cent[a].astype(np.float64)).astype(np.float32)
    dsub = X.shape[1] // M
    books = np.empty((M, ncode, dsub), dtype=np.float32)
    for s in range(M):
        Z = R[:, s * dsub:(s + 1) * dsub]
        W = Z[init_slots[C + s * ncode:C + (s + 1) * ncode]].copy()
        for _ in range(pq_iters):
            W = lloyd_update(Z, lloyd_assign(Z, W), W)
        books[s] = W
    return cent, books, a


# ---------------------------------------------------------------------------
# Batch-level wrappers over (sequence, KV head) units
# ---------------------------------------------------------------------------

def _units(B: int, Hkv: int, units: Optional[Iterable[Tuple[int, int]]]) -> List[Tuple[int, int]]:
    return [(b, h) for b in range(B) for h in range(Hkv)] if units is None else list(units)


def oracle_decode(q, k_cache, v_cache, block_table, seq_lens, centroids, codebooks, codes, ids,
                  n_indexed, n_sink: int, scale: float, budget: float = 0.01,
                  k_override: Optional[int] = None, background: bool = True,
                  page_size: int = 16, units=None, mean_v=None) -> Dict[Tuple[int, int], Dict[str, np.ndarray]]:
    """PQ-HSA decode for the chosen units. Returns {(b, h): decode_unit result + 'k'}."""
    B, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    res = {}
    for b, h in _units(B, Hkv, units):
        N = int(n_indexed[b])
        k = decode_k(budget, N, k_override)
        r = decode_unit(q[b, h * G:(h + 1) * G], k_cache, v_cache, block_table[b], h, int(seq_lens[b]),
                        page_size, centroids[b, h], codebooks[b, h], codes[b, h], ids[b, h], N, n_sink,
                        scale, k, background, None if mean_v is None else mean_v[b, h])
        r["k"] = k
        res[(b, h)] = r
    return res


def oracle_dense(q, k_cache, v_cache, block_table, seq_lens, scale: float, page_size: int = 16,
                 units=None) -> Dict[Tuple[int, int], np.ndarray]:
    """Dense softmax attention over all T tokens for the chosen units: {(b, h): [G, D]}."""
    B, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    res = {}
    for b, h in _units(B, Hkv, units):
        pos = np.arange(int(seq_lens[b]))
        K = unit_rows(k_cache, block_table[b], h, pos, page_size)
        V = unit_rows(v_cache, block_table[b], h, pos, page_size)
        res[(b, h)] = dense_unit(q[b, h * G:(h + 1) * G], K, V, scale)
    return res


def oracle_build_means(v_cache, block_table, ids, n_indexed, n_sink: int, C: int,
                       page_size: int = 16, units=None):
    """count / sum_v / mean_v of every cluster over the indexed tokens: {(b, h): (count, sum, mean)}."""
    B, Hkv = ids.shape[0], ids.shape[1]
    res = {}
    for b, h in _units(B, Hkv, units):
        N = int(n_indexed[b])
        V = unit_rows(v_cache, block_table[b], h, n_sink + np.arange(N), page_size)
        res[(b, h)] = cluster_means(V, np.asarray(ids[b, h][:N]).astype(np.int64), C)
    return res


def oracle_append(k_cache, block_table, centroids, codebooks, n_indexed, n_new: int, n_sink: int,
                  page_size: int = 16, units=None):
    """Encode positions [s0 + n_indexed[b], s0 + n_indexed[b] + n_new) of every chosen unit.

    Returns {(b, h): (ids, codes, gaps)} for the new tokens (slots n_indexed[b] ...).
    """
    B, Hkv = centroids.shape[0], centroids.shape[1]
    res = {}
    for b, h in _units(B, Hkv, units):
        pos = n_sink + int(n_indexed[b]) + np.arange(n_new)
        keys = unit_rows(k_cache, block_table[b], h, pos, page_size)
        res[(b, h)] = encode_keys(keys, centroids[b, h], codebooks[b, h])
    return res


def oracle_train(k_cache, block_table, n_sink: int, n_train: int, init_slots, C: int, coarse_iters: int,
                 pq_iters: int, page_size: int = 16, units=None):
    """train_unit on the keys at positions [n_sink, n_sink + n_train) of every (b, h) unit.
    init_slots: [B, Hkv, C + M*ncode] int. Returns {(b, h): (centroids, codebooks, assign)}."""
    B = block_table.shape[0]
    Hkv = k_cache.shape[1]
    out = {}
    for b, h in _units(B, Hkv, units):
        keys = unit_rows(k_cache, block_table[b], h, n_sink + np.arange(n_train), page_size)
        out[(b, h)] = train_unit(keys.astype(np.float32), init_slots[b, h], C, coarse_iters, pq_iters)
    return out
