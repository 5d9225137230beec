"""Test helpers: run the CUDA library and the oracle on the same generated inputs and compare.

The oracle is used here only as the reference; the library never sees it.
"""
from __future__ import annotations

import math
from typing import Dict, Tuple

import numpy as np

import oracle as O
from synth import Batch

# Tolerances of the method's GPU/oracle agreement.
LOGIT_RTOL = 1e-4          # approximate logits: per (sequence, query head) row, relative to the row max
NEAR_TIE = 1e-5            # selection differences allowed only within this distance of the k-th score
OUT_TOL = 2e-3             # attention output: max-abs <= OUT_TOL * max|V|
DENSE_TOL = 1e-4           # dense decode: max-abs <= DENSE_TOL * max|V|


def reference_codes(bt: Batch) -> Tuple[np.ndarray, np.ndarray]:
    """Recorded codes/ids, with every planted needle re-encoded by the oracle's encoder."""
    w = bt.w
    codes = bt.codes_rec.copy()
    ids = bt.ids_rec.copy()
    for b in range(w.B):
        for h in range(w.Hkv):
            pos = bt.needle_pos[b, h]
            if pos.size == 0:
                continue
            keys = O.unit_rows(bt.k_cache, bt.block_table[b], h, pos, w.page_size)
            ii, cc, _ = O.encode_keys(keys, bt.centroids[b, h], bt.codebooks[b, h])
            slots = pos - w.n_sink
            ids[b, h, slots] = ii.astype(np.uint16)
            codes[b, h, slots] = cc.astype(np.uint8)
    return codes, ids


def max_abs_v(bt: Batch) -> float:
    return float(np.abs(O.widen_bf16(bt.v_cache)).max())


def compare_logits(gpu: np.ndarray, orc: np.ndarray) -> float:
    """Worst per-row error relative to the row's max |logit| (floored at 1e-3)."""
    worst = 0.0
    for g in range(orc.shape[0]):
        denom = max(float(np.abs(orc[g]).max()), 1e-3) if orc.shape[1] else 1.0
        err = float(np.abs(gpu[g].astype(np.float64) - orc[g]).max()) if orc.shape[1] else 0.0
        worst = max(worst, err / denom)
    return worst


def compare_selection(gpu_sel_pos: np.ndarray, orc: Dict, n_sink: int) -> Dict[str, int]:
    """Selection sets must agree except for near-ties at the oracle's k-th score."""
    k = orc["k"]
    orc_slots = set(int(x) for x in orc["sel"])
    gpu_slots = set(int(x) - n_sink for x in gpu_sel_pos)
    assert len(gpu_slots) == len(gpu_sel_pos) == k, (len(gpu_slots), len(gpu_sel_pos), k)
    diff = orc_slots ^ gpu_slots
    if diff:
        sig = orc["sigma"]
        tau = np.sort(sig.astype(np.float32).astype(np.float64))[::-1][k - 1]
        bad = [j for j in diff if abs(sig[j] - tau) >= NEAR_TIE]
        assert not bad, f"selection differs beyond near-ties: {sorted(bad)[:10]} (tau={tau})"
    return {"k": k, "excused": len(diff)}


def assert_sorted_positions(sel: np.ndarray):
    assert np.all(np.diff(sel) > 0), "selected positions not strictly ascending"


def scale_for(D: int = 128) -> float:
    return float(np.float32(1.0 / math.sqrt(D)))
