"""Host logic of multi-process runs, on CPU with the gloo backend: the
max-over-ranks time reduction bench.py applies at N > 1, and the reference
arm's rank rule (rank 0 alone runs and prints)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r took (r + 1) * 1.5 ms: everyone must report the slowest
        got = bench.max_over_ranks((rank + 1) * 1.5, torch.device("cpu"))
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {r: world * 1.5 for r in range(world)}


def test_max_over_ranks_single_process():
    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu")) == 2.5


def test_reference_arm_nonzero_rank_is_silent():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_decode_traffic_tracks_the_captured_source(tmp_path, monkeypatch):
    import bench
    kv = 1_000_000
    cap = bench.DECODE_CAPTURE
    t = bench.decode_traffic(kv, cap["kernel"])
    if t is not None:  # the source is the captured one: traffic scales with the KV bytes
        assert t == pytest.approx(kv * (cap["dram_bytes_read"] + cap["dram_bytes_write"]) /
                                  cap["kv_bytes"])
    # another kernel ran: the capture does not describe it
    assert bench.decode_traffic(kv, "decode_simt") is None
    monkeypatch.setitem(cap, "sha256", "0" * 64)
    assert bench.decode_traffic(kv, cap["kernel"]) is None


def test_reference_arm_rank0_prints_one_contract_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3", "--ref-ctx", "512"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "512 of" in d["config"]["sample"]


def test_bench_e2e_byte_counts_are_assigned_once():
    """The e2e line reports the bytes copied each step; no later measurement
    in the same function may reuse those names for something else."""
    import ast
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    main = next(n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name == "main")
    stores = []

    def visit(node):  # main's own scope: nested functions have their own
        for c in ast.iter_child_nodes(node):
            if isinstance(c, (ast.FunctionDef, ast.Lambda)):
                continue
            if isinstance(c, ast.Name) and isinstance(c.ctx, ast.Store):
                stores.append(c.id)
            visit(c)

    visit(main)
    for name in ("h2d", "d2h", "value", "ms", "kv_bytes", "e2e_ms", "decode_gbs"):
        assert stores.count(name) == 1, name


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_native_arm_refuses_to_run_without_a_gpu():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 1
    assert "needs a CUDA GPU" in r.stderr
    assert r.stdout.strip() == ""
