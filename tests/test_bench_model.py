"""The bench's overhead-aware crossover model (fixed cost + bytes / bandwidth per method, the
crossover article's procedure) and the measured-crossover interpolation, on synthetic points
whose intercepts, bandwidths and crossing are known in closed form. No GPU needed."""
import math

import numpy as np
import pytest

import bench


def test_fit_recovers_intercept_and_bandwidth_exactly():
    nbytes = [15.5e6, 19.7e6, 36.3e6, 102.7e6]
    t0, bw = 24.7, 856e3                                # µs, bytes per µs
    times = [t0 + b / bw for b in nbytes]
    f0, fbw = bench.fit_overhead_model(nbytes, times)
    assert f0 == pytest.approx(t0, rel=1e-9)
    assert fbw == pytest.approx(bw, rel=1e-9)


def test_fit_is_least_squares_on_noisy_points():
    rng = np.random.default_rng(3)
    x = np.linspace(1e6, 1e8, 9)
    y = 10.0 + x / 2e6 + rng.normal(0, 0.5, size=x.size)
    f0, fbw = bench.fit_overhead_model(x, y)
    slope, icpt = np.polyfit(x, y, 1)                  # independent least-squares routine
    assert f0 == pytest.approx(icpt, rel=1e-9)
    assert 1.0 / fbw == pytest.approx(slope, rel=1e-9)


def test_predicted_crossover_of_two_lines():
    # sparse: 20 µs + 40 B/token at 1 TB/s; dense: 5 µs + 512 B/token at 5 TB/s.
    # crossing: 20 + 40T/1e6 = 5 + 512T/5e6  ->  T = 15 / (0.1024e-3 - 0.04e-3) = 240384.6
    sparse, dense = (20.0, 1e6), (5.0, 5e6)
    bytes_at = lambda T: (40.0 * T, 512.0 * T)
    T = bench.predicted_crossover(sparse, dense, bytes_at, range(1024, 1 << 21, 256))
    exact = 15.0 / (512.0 / 5e6 - 40.0 / 1e6)
    assert T is not None and exact <= T < exact + 256
    assert bench.predicted_crossover(sparse, dense, bytes_at, range(1024, 100000, 256)) is None


def test_measured_crossover_interpolates_between_bracketing_lengths():
    pts = [(8192, 40.0, 20.0), (32768, 45.0, 40.0), (65536, 50.0, 70.0), (131072, 60.0, 125.0)]
    # dense - sparse: -20, -5, +20, +65 -> crossing between 32768 and 65536 at 1/5 of the way
    assert bench.measured_crossover(pts) == pytest.approx(32768 + 0.2 * 32768)
    assert bench.measured_crossover([(8192, 10.0, 20.0), (16384, 12.0, 30.0)]) == 8192.0
    assert bench.measured_crossover([(8192, 30.0, 20.0), (16384, 32.0, 30.0)]) is None
    assert bench.measured_crossover(list(reversed(pts))) == pytest.approx(32768 * 1.2)


def test_oracle_pool_runs_whole_steps_on_worker_processes():
    """The CPU baseline's pool: spawn-started single-threaded workers over the units, the K/V
    pool shared with them; one whole step of the small workload gives the oracle's own output
    for every unit (checked against a direct call in this process)."""
    from synth import make_batch, workload
    w = workload("tiny_4k", Hq=8, Hkv=2)
    bt = make_batch(w)
    pool = bench.OraclePool(bt, w, w.budget, workers=2)
    try:
        assert pool.workers == 2 and len(pool.units) == 2
        assert pool.step() > 0
        assert sorted(pool.pool.map(bench._orc_unit, pool.units)) == pool.units
    finally:
        pool.close()
    us, steps, workers, el = bench.oracle_sample(bt, w, w.budget, seconds=0.0, warmup=0)
    assert us > 0 and steps == 1 and 1 <= workers <= 2


def test_gpus_flag_spawns_replicas_or_refuses_a_mismatch(monkeypatch):
    seen = {}
    monkeypatch.setattr(bench, "spawn_replicas", lambda args, argv: seen.update(n=args.gpus, argv=argv) or 0)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    with pytest.raises(SystemExit) as e:
        bench.main(["--gpus", "2", "--steps", "3"])
    assert e.value.code == 0 and seen == {"n": 2, "argv": ["--gpus", "2", "--steps", "3"]}
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit) as e:
        bench.main(["--gpus", "2"])
    assert "4 ranks" in str(e.value.code)
