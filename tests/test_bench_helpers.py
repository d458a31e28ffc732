"""Host-side pieces of bench.py that need no GPU: the visible-pair count the
variant throughputs divide by, the whole-job throughput formula and the
per-rank workload."""
import importlib.util
import os

import numpy as np
import pytest

import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("seed", range(6))
def test_visible_pairs_counts_the_oracle_mask(bench, seed):
    rng = np.random.default_rng(seed)
    for _ in range(20):
        nq, nk = int(rng.integers(1, 40)), int(rng.integers(1, 40))
        causal = bool(rng.integers(0, 2))
        window = (int(rng.integers(-1, 12)), int(rng.integers(-1, 12)))
        want = int(oracle.visible(np.arange(nq), nq, nk, causal, window).sum())
        assert bench.visible_pairs(nq, nk, causal, window) == want, (nq, nk, causal, window)


def test_visible_pairs_closed_forms(bench):
    n = 4096
    assert bench.visible_pairs(n, n, True) == n * (n + 1) // 2
    assert bench.visible_pairs(n, n, False) == n * n
    # Causal window of w previous keys: rows i >= w see w + 1 keys.
    w = 1024
    assert bench.visible_pairs(n, n, True, (w, 0)) == sum(min(i, w) + 1 for i in range(n))


def test_job_throughput_is_all_ranks_work_over_the_slowest_time(bench):
    # 2 ranks x 10 steps x 1e12 FLOPs in 1 s of the slowest rank -> 20 TFLOP/s.
    assert bench.job_throughput(1e12, 10, 2, 1000.0) == pytest.approx(20.0)
    w = workloads.C5
    flops = w.fwd_flops() + w.bwd_flops()
    assert flops == pytest.approx(14 * w.d * w.B * w.Hq * w.N * w.N / 2)


def test_rank_workload_changes_only_the_seed(bench):
    w = workloads.C5
    r = bench.rank_workload(w, 3)
    assert (r.B, r.Hq, r.Hkv, r.N, r.d, r.causal) == (w.B, w.Hq, w.Hkv, w.N, w.d, w.causal)
    assert r.seed == w.seed + 3
