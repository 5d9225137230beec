"""The bench's algorithmic bytes per step (the HBM-rate denominators) against the per-unit
formula written out term by term for each workload's shape (no GPU needed)."""
import pytest

import bench
from synth import workload


def _formula(w, k):
    """Per step: PQ codes 16 N, centroids and cluster means 2 x 4 C D (+ 4 C counts),
    codebook 4 x 16 x 256 x 8, LUT 4 G x 16 x 256, exact K+V rows 512 (s0 + R + k),
    q and out 8 G D; dense: every K+V row, 512 T, plus q and out."""
    N = w.n_indexed
    R = w.T - w.n_sink - N
    per_unit = (16 * N + 2 * 4 * w.C * w.D + 4 * w.C + 4 * 16 * 256 * 8 + 4 * w.G * 16 * 256
                + 512 * (w.n_sink + R + k) + 8 * w.G * w.D)
    U = w.B * w.Hkv
    return U * per_unit, U * (512 * w.T + 8 * w.G * w.D)


@pytest.mark.parametrize("name,hsa_mb,dense_mb", [
    ("tiny_4k", 0.42, 2.1),
    ("llama8b_128k", 36.3, 536.9),
    ("llama8b_8k", 15.5, 33.6),
    ("llama8b_32k", 19.7, 134.3),
    ("llama8b_512k", 102.7, 2147.5),
    ("batch32_32k", 330.0, 4296.0),
    ("qwen30b_128k_append", 73.6, 1073.9),
])
def test_step_bytes(name, hsa_mb, dense_mb):
    w = workload(name)
    k = int(w.budget * w.n_indexed)
    hsa, ids, dense, scan = bench.step_bytes(w, w.n_indexed, k)
    want_hsa, want_dense = _formula(w, k)
    assert hsa == want_hsa and dense == want_dense
    assert ids == 2 * w.n_indexed * w.B * w.Hkv
    # the same figures, rounded, as tabulated for the decode workloads (MB = 1e6 bytes)
    assert abs(hsa / 1e6 - hsa_mb) <= 0.05 * max(1.0, hsa_mb / 10)
    assert abs(dense / 1e6 - dense_mb) <= 0.05 * max(1.0, dense_mb / 10)


def test_scan_wavefronts_closed_form():
    """LUT gathers of the scan: 16 look-ups per 32-slot chunk, each 4 wavefronts per 4 heads
    (a conflict-free 128-bit load by 32 lanes is 512 bytes = 4 x 128-byte wavefronts)."""
    assert bench.scan_wavefronts(4, 1) == 64
    assert bench.scan_wavefronts(8, 1) == 128
    assert bench.scan_wavefronts(1, 1) == bench.scan_wavefronts(4, 1)   # heads padded to 4
    assert bench.scan_wavefronts(4, 36374) == 36374 * 64
