"""CPU tests of bench.py's host helpers that need no GPU."""

import pytest
from threadpoolctl import threadpool_info

import bench


def test_oracle_threads_limits_blas_and_reports_the_count():
    ctx, cores = bench.oracle_threads(1)
    assert cores == 1
    with ctx:
        pools = threadpool_info()
        assert pools, "no BLAS/OpenMP thread pool found"
        assert all(p["num_threads"] == 1 for p in pools)


def test_oracle_threads_default_is_every_core():
    ctx, cores = bench.oracle_threads(0)
    assert cores == bench.cores_used() >= 1
    with ctx:
        pass


@pytest.mark.parametrize("name,batch,model", [("8b_b1_ctx512", 1, "8b"),
                                              ("1.5b_b1_ctx256", 1, "1.5b"),
                                              ("8b_b16_ctx1024", 16, "8b"),
                                              ("8b_b16_ragged", 16, "8b")])
def test_workload_names(name, batch, model):
    wl = bench.parse_workload(name)
    assert wl["batch"] == batch and wl["model"] == model
    assert len(wl["lengths"]) == batch
