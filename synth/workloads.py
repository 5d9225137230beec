"""Seeded synthetic PQ-HSA decode workloads.

Shapes and value distributions follow the workloads the PQ-HSA page describes
(rit.work "pq-hsa-long-context-attention": Llama-3.1-8B and Qwen3-30B-A3B
shaped GQA decode at 128K-512K context, 1 % read budget), made concrete as:

* centroids ~ N(0, 1); PQ codewords ~ N(0, 0.3^2) (0.3 is a standard deviation);
* every token picks a uniform cluster a and uniform codes, and its key is
  centroid_a + the concatenated codewords + N(0, 0.02^2) noise, rounded to
  bf16; the cluster id and codes are recorded as drawn;
* values ~ N(0, 1) rounded to bf16; queries ~ N(0, 1) / sqrt(D) in fp32;
* planted needles: needle i of a KV head sits at position
  n_sink + floor((i + 0.5) * N / n_needles) of the indexed range and its key is
  4 * q of query head (i mod G) of that head's group (rounded to bf16). Its
  recorded cluster/codes are those of the key it replaced, so the caller
  re-encodes needle keys before building an index from recorded codes;
* K/V live in a paged bf16 pool [num_pages][Hkv][page_size][D] whose pages
  are handed out through a seeded random permutation (a shuffled block table).

Every random stream is keyed by (workload id, context length, sequence,
KV head, purpose), so any single (sequence, KV head) unit can be regenerated
on its own.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np

# Stream purposes.
_IDX, _TOK, _VAL, _QRY, _PAGES, _TRAIN = 0, 1, 2, 3, 4, 5


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (np.ascontiguousarray(b).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One decode workload. Lengths are per sequence; every sequence has the same length."""

    name: str
    wid: int            # workload id (seed namespace)
    B: int              # sequences
    Hq: int             # query heads
    Hkv: int            # KV heads
    T: int              # context length at the decode step (tokens already in the cache)
    C: int              # IVF clusters per (sequence, KV head)
    n_sink: int         # leading tokens always read exactly
    n_recent: int       # trailing tokens always read exactly (at index build)
    n_needles: int      # planted needle keys per (sequence, KV head)
    D: int = 128
    M: int = 16         # PQ subspaces
    dsub: int = 8       # dims per subspace
    ncode: int = 256    # codewords per subspace
    page_size: int = 16
    budget: float = 0.01
    extra_tokens: int = 0   # tokens generated beyond T (future decode steps)
    append_batch: int = 0   # tokens moved into the index per append (0 = no appends)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def T_cap(self) -> int:
        return self.T + self.extra_tokens

    @property
    def n_indexed(self) -> int:
        """Indexed tokens at build: [n_sink, T - n_recent)."""
        return max(0, self.T - self.n_sink - self.n_recent)

    @property
    def k(self) -> int:
        return int(math.floor(self.budget * self.n_indexed))

    @property
    def pages_per_seq(self) -> int:
        return -(-self.T_cap // self.page_size)

    @property
    def index_cap(self) -> int:
        """Index capacity per unit (every token after the sink could be indexed)."""
        return max(1, self.T_cap - self.n_sink)

    @property
    def units(self) -> int:
        return self.B * self.Hkv

    def scaled(self, **changes) -> "Workload":
        return dataclasses.replace(self, **changes)

    def describe(self) -> Dict[str, object]:
        return {
            "workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv, "D": self.D,
            "T": self.T, "C": self.C, "M": self.M, "dsub": self.dsub, "ncode": self.ncode,
            "n_sink": self.n_sink, "n_recent": self.n_recent, "budget": self.budget,
            "page_size": self.page_size, "n_indexed": self.n_indexed, "k": self.k,
        }


# The five workloads (small reference case; Llama-3.1-8B layer at 128K; context
# sweep; 32-sequence batch at 32K; Qwen3-30B-A3B layer with index appends).
WORKLOADS: Dict[str, Workload] = {
    "tiny_4k": Workload("tiny_4k", 0, B=1, Hq=4, Hkv=1, T=4096, C=64,
                        n_sink=16, n_recent=128, n_needles=8),
    "llama8b_128k": Workload("llama8b_128k", 1, B=1, Hq=32, Hkv=8, T=131072, C=1024,
                             n_sink=16, n_recent=1024, n_needles=64),
    "llama8b_8k": Workload("llama8b_8k", 2, B=1, Hq=32, Hkv=8, T=8192, C=1024,
                           n_sink=16, n_recent=1024, n_needles=64),
    "llama8b_32k": Workload("llama8b_32k", 2, B=1, Hq=32, Hkv=8, T=32768, C=1024,
                            n_sink=16, n_recent=1024, n_needles=64),
    "llama8b_sweep_128k": Workload("llama8b_sweep_128k", 2, B=1, Hq=32, Hkv=8, T=131072, C=1024,
                                   n_sink=16, n_recent=1024, n_needles=64),
    "llama8b_512k": Workload("llama8b_512k", 2, B=1, Hq=32, Hkv=8, T=524288, C=1024,
                             n_sink=16, n_recent=1024, n_needles=64),
    "batch32_32k": Workload("batch32_32k", 3, B=32, Hq=32, Hkv=8, T=32768, C=256,
                            n_sink=16, n_recent=256, n_needles=8),
    "qwen30b_128k_append": Workload("qwen30b_128k_append", 4, B=4, Hq=32, Hkv=4, T=131072, C=1024,
                                    n_sink=16, n_recent=1024, n_needles=8,
                                    extra_tokens=2048, append_batch=512),
}


def train_init_slots(w: Workload, n_train: int, seed: int = 0) -> np.ndarray:
    """Training slots seeding an index's centres, the random draw both sides take as input:
    int32 [B, Hkv, C + M * ncode] uniform in [0, n_train) (centroids first, then the
    codewords of every subspace), per-unit seeded."""
    out = np.empty((w.B, w.Hkv, w.C + w.M * w.ncode), dtype=np.int32)
    for b in range(w.B):
        for h in range(w.Hkv):
            out[b, h] = _rng(w, b, h, _TRAIN, seed).integers(0, n_train, size=out.shape[2])
    return out


def workload(name: str, **changes) -> Workload:
    w = WORKLOADS[name]
    return w.scaled(**changes) if changes else w


def _rng(w: Workload, *key: int) -> np.random.Generator:
    return np.random.default_rng([w.wid, w.T, w.C, *key])


@dataclass
class UnitData:
    """All tokens of one (sequence b, KV head h) unit, positions [0, T_cap)."""

    b: int
    h: int
    k_bits: np.ndarray      # [T_cap, D] uint16 (bf16)
    v_bits: np.ndarray      # [T_cap, D] uint16 (bf16)
    q: np.ndarray           # [G, D] float32, query heads h*G .. h*G+G-1
    centroids: np.ndarray   # [C, D] float32
    codebooks: np.ndarray   # [M, ncode, dsub] float32
    ids_rec: np.ndarray     # [T_cap] uint16, drawn cluster of every token
    codes_rec: np.ndarray   # [T_cap, M] uint8, drawn codes of every token
    needle_pos: np.ndarray  # [n_needles] int64 positions whose keys were replaced


def make_unit(w: Workload, b: int, h: int) -> UnitData:
    D, M, dsub, C, T = w.D, w.M, w.dsub, w.C, w.T_cap
    assert M * dsub == D
    r = _rng(w, b, h, _IDX)
    centroids = r.standard_normal((C, D), dtype=np.float32)
    codebooks = (0.3 * r.standard_normal((M, w.ncode, dsub), dtype=np.float32)).astype(np.float32)

    r = _rng(w, b, h, _TOK)
    ids = r.integers(0, C, size=T, dtype=np.int64)
    codes = r.integers(0, w.ncode, size=(T, M), dtype=np.int64)
    noise = r.standard_normal((T, D), dtype=np.float32)
    # key = centroid + drawn codewords + noise (the generating process, in float32)
    keys = centroids[ids]
    keys += codebooks[np.arange(M)[None, :], codes].reshape(T, D)
    keys += np.float32(0.02) * noise
    del noise

    r = _rng(w, b, h, _QRY)
    q = (r.standard_normal((w.G, D), dtype=np.float32) / np.float32(math.sqrt(D))).astype(np.float32)

    N = w.n_indexed
    if w.n_needles > 0 and N > 0:
        i = np.arange(w.n_needles)
        needle_pos = w.n_sink + np.floor((i + 0.5) * N / w.n_needles).astype(np.int64)
        keys[needle_pos] = np.float32(4.0) * q[i % w.G]
    else:
        needle_pos = np.zeros(0, dtype=np.int64)

    r = _rng(w, b, h, _VAL)
    vals = r.standard_normal((T, D), dtype=np.float32)
    return UnitData(
        b=b, h=h,
        k_bits=f32_to_bf16_bits(keys), v_bits=f32_to_bf16_bits(vals),
        q=q, centroids=centroids, codebooks=codebooks,
        ids_rec=ids.astype(np.uint16), codes_rec=codes.astype(np.uint8),
        needle_pos=needle_pos,
    )


@dataclass
class Batch:
    """Whole-batch buffers in the layouts the library consumes."""

    w: Workload
    q: np.ndarray            # [B, Hq, D] float32
    k_cache: np.ndarray      # [num_pages, Hkv, page_size, D] uint16 (bf16 bits)
    v_cache: np.ndarray      # [num_pages, Hkv, page_size, D] uint16
    block_table: np.ndarray  # [B, max_pages] int32
    seq_lens: np.ndarray     # [B] int32 (= T)
    centroids: np.ndarray    # [B, Hkv, C, D] float32
    codebooks: np.ndarray    # [B, Hkv, M, ncode, dsub] float32
    ids_rec: np.ndarray      # [B, Hkv, cap] uint16; slot i <-> position n_sink + i
    codes_rec: np.ndarray    # [B, Hkv, cap, M] uint8
    needle_pos: np.ndarray   # [B, Hkv, n_needles] int64
    n_indexed: np.ndarray    # [B] int32 (at build)

    @property
    def num_pages(self) -> int:
        return self.k_cache.shape[0]


def make_batch(w: Workload, units: Optional[List[UnitData]] = None) -> Batch:
    B, Hkv, D, P = w.B, w.Hkv, w.D, w.page_size
    pps = w.pages_per_seq
    num_pages = B * pps
    perm = _rng(w, _PAGES).permutation(num_pages).astype(np.int32)
    block_table = perm.reshape(B, pps).copy()
    k_cache = np.zeros((num_pages, Hkv, P, D), dtype=np.uint16)
    v_cache = np.zeros((num_pages, Hkv, P, D), dtype=np.uint16)
    q = np.zeros((B, w.Hq, D), dtype=np.float32)
    cap = w.index_cap
    centroids = np.zeros((B, Hkv, w.C, D), dtype=np.float32)
    codebooks = np.zeros((B, Hkv, w.M, w.ncode, w.dsub), dtype=np.float32)
    ids_rec = np.zeros((B, Hkv, cap), dtype=np.uint16)
    codes_rec = np.zeros((B, Hkv, cap, w.M), dtype=np.uint8)
    needle_pos = np.zeros((B, Hkv, w.n_needles if w.n_indexed > 0 else 0), dtype=np.int64)
    Tpad = pps * P
    it = iter(units) if units is not None else None
    for b in range(B):
        pages = block_table[b]
        for h in range(Hkv):
            u = next(it) if it is not None else make_unit(w, b, h)
            kb = np.zeros((Tpad, D), dtype=np.uint16)
            vb = np.zeros((Tpad, D), dtype=np.uint16)
            kb[: w.T_cap] = u.k_bits
            vb[: w.T_cap] = u.v_bits
            k_cache[pages, h] = kb.reshape(pps, P, D)
            v_cache[pages, h] = vb.reshape(pps, P, D)
            q[b, h * w.G:(h + 1) * w.G] = u.q
            centroids[b, h] = u.centroids
            codebooks[b, h] = u.codebooks
            ids_rec[b, h] = u.ids_rec[w.n_sink: w.n_sink + cap]
            codes_rec[b, h] = u.codes_rec[w.n_sink: w.n_sink + cap]
            needle_pos[b, h] = u.needle_pos
    return Batch(
        w=w, q=q, k_cache=k_cache, v_cache=v_cache, block_table=block_table,
        seq_lens=np.full(B, w.T, dtype=np.int32), centroids=centroids, codebooks=codebooks,
        ids_rec=ids_rec, codes_rec=codes_rec, needle_pos=needle_pos,
        n_indexed=np.full(B, w.n_indexed, dtype=np.int32),
    )
