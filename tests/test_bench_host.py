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


def test_oracle_threads_default_reports_the_blas_pool():
    ctx, cores = bench.oracle_threads(0)
    blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
    assert cores == (max(blas) if blas else bench.cores_used()) >= 1
    with ctx:
        pass


def test_reference_arm_under_torchrun_prints_one_line_from_rank0(tmp_path):
    """--impl reference under torchrun: rank 0 times the oracle and prints the
    JSON line, the other rank exits 0 without work."""
    import json
    import os
    import socket
    import subprocess
    import sys

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny_b1_p16",
           "--steps", "2", "--warmup", "3", "--gpus", "2"]
    r = subprocess.run(cmd, cwd=str(tmp_path), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


@pytest.mark.parametrize("name,batch,model", [("8b_b1_ctx512", 1, "8b"),
                                              ("1.5b_b1_ctx256", 1, "1.5b"),
                                              ("8b_b16_ctx1024", 16, "8b"),
                                              ("8b_b16_ragged", 16, "8b")])
def test_workload_names(name, batch, model):
    wl = bench.parse_workload(name)
    assert wl["batch"] == batch and wl["model"] == model
    assert len(wl["lengths"]) == batch


def test_source_digest_ignores_comments_but_not_code():
    """The digest that gates the committed DRAM figures follows the code only:
    comments and whitespace leave it alone, a literal or a token does not."""
    a = 'int f(int x) {  // scale\n  return x * 2; /* two */ }\nconst char *s = "a // b";\n'
    b = 'int f(int x) {\n\n  return x * 2; }\nconst char *s = "a // b"; // the literal\n'
    assert bench.code_text(a) == bench.code_text(b)
    assert bench.code_text(a) != bench.code_text(a.replace("x * 2", "x * 3"))
    assert bench.code_text(a) != bench.code_text(a.replace('"a // b"', '"a //  b"'))
    assert bench.code_text("char c = '/'; int y; /* '\"' */") == bench.code_text("char c = '/'; int y;")
    assert "/*" not in bench.code_text("int y; /* '\"' */")


def test_profiled_traffic_matches_current_sources():
    """The batch-1 summary's digest is that of the current sources, so the
    bench line carries its measured DRAM bytes."""
    t = bench.profiled_traffic("8b_b1_ctx512")
    assert t is not None and t > 15e9
