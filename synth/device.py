"""Copy generated workloads into torch tensors (device memory plumbing, no arithmetic)."""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from .workloads import Batch


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def kv_tensors(bt: Batch, device) -> Dict[str, object]:
    """Arguments of PagedKV(...) for a generated batch."""
    return dict(
        k_cache=bf16_tensor(bt.k_cache, device),
        v_cache=bf16_tensor(bt.v_cache, device),
        block_table=torch.from_numpy(bt.block_table).to(device),
        seq_lens=torch.from_numpy(bt.seq_lens.copy()).to(device),
        seq_lens_host=torch.from_numpy(bt.seq_lens.copy()),
        Hq=bt.w.Hq,
    )


def index_tensors(bt: Batch, device, codes: Optional[np.ndarray] = None, ids: Optional[np.ndarray] = None,
                  n_indexed: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Arguments of PQIndex(...): the batch's centroids/codebooks and the given (or recorded) codes/ids."""
    w = bt.w
    codes = bt.codes_rec if codes is None else codes
    ids = bt.ids_rec if ids is None else ids
    n_indexed = bt.n_indexed if n_indexed is None else n_indexed
    f32 = dict(device=device, dtype=torch.float32)
    return dict(
        centroids=torch.from_numpy(bt.centroids).to(device),
        codebooks=torch.from_numpy(bt.codebooks).to(device),
        codes=torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).to(device),
        ids=torch.from_numpy(np.ascontiguousarray(ids, dtype=np.uint16).view(np.int16)).to(device),
        sum_v=torch.zeros(w.B, w.Hkv, w.C, w.D, **f32),
        mean_v=torch.zeros(w.B, w.Hkv, w.C, w.D, **f32),
        count=torch.zeros(w.B, w.Hkv, w.C, device=device, dtype=torch.int32),
        n_indexed=torch.from_numpy(np.ascontiguousarray(n_indexed, dtype=np.int32)).to(device),
        n_indexed_host=torch.from_numpy(np.array(n_indexed, dtype=np.int32)),
        n_sink=w.n_sink,
    )
