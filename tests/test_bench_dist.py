"""Host logic of bench.py for N > 1 ranks, on CPU with gloo at world size 2.

The path shards as independent replicas, so the only cross-rank steps are the
barrier around the timed region and the max over ranks of the timed
duration; the reference arm runs on rank 0 alone.
"""

import contextlib
import io
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        w, r, _ = bench.dist_setup()
        assert (w, r) == (world, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(w)
        # each rank "measured" a different duration: everyone must see the slowest
        slowest = bench.max_over_ranks(10.0 + rank, w)
        # the end-to-end figure is whole-job too: slowest rank, all ranks' units and bytes
        e2e = bench.aggregate_e2e({"ms_per_step": 1.0 + rank, "value": 0.0, "unit": "TOPS",
                                   "h2d_bytes_per_step": 100, "d2h_bytes_per_step": 50}, 1e12, w)
        # the reference arm prints one line on rank 0 and nothing elsewhere
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            if rank != 0:
                bench.run_reference(type("A", (), {"warmup": 0, "steps": 1, "cpu_rows": 1})(), w, rank)
        q.put((rank, slowest, out.getvalue(), e2e))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_barrier_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("rank did not finish")
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[1] for g in got] == [11.0, 11.0]
    assert got[1][2] == ""          # rank 1 printed nothing
    for g in got:                   # 2 ranks x 1e12 ops in the slowest rank's 2 ms
        assert g[3]["ms_per_step"] == 2.0 and abs(g[3]["value"] - 1000.0) < 1e-9
        assert g[3]["h2d_bytes_per_step"] == 200 and g[3]["d2h_bytes_per_step"] == 100


def test_reference_arm_prints_one_contract_line_on_rank_zero():
    import json
    sys.path.insert(0, ROOT)
    import bench
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(type("A", (), {"warmup": 0, "steps": 1, "cpu_rows": 16})(), 1, 0)
    lines = [l for l in out.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_value_is_aggregate_units_over_slowest_rank():
    # value = 2*M*N*K*steps*world / slowest time, i.e. per-rank work is fixed (weak scaling)
    sys.path.insert(0, ROOT)
    import bench  # noqa: F401
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert "ops * world / (ms_step * 1e-3)" in src
    assert "max_over_ranks(t[\"total_ms\"], world)" in src


def test_traffic_entries_turn_null_when_their_kernel_sources_change(tmp_path, monkeypatch):
    # a DRAM-traffic figure is reported only while its kernel's sources are the ones profiled
    import json
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "bit_quantized_linear_rotate_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cuh").write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash(["k.cuh"])
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"source_hash": h, "dram_bytes_per_launch": 123, "sources": ["k.cuh"]}}))
    assert bench.load_traffic("k") == 123
    assert bench.load_traffic("missing") is None
    (csrc / "k.cuh").write_text("kernel v2")
    assert bench.load_traffic("k") is None


def test_committed_traffic_entries_are_documented_and_reported_only_while_current():
    import json
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    kernels = [k for k in d if not k.startswith("_")]
    assert kernels
    for k in kernels:
        e = d[k]
        assert os.path.exists(os.path.join(ROOT, e["profile"])), f"{k}: summary {e['profile']} missing"
        assert e["dram_bytes_per_launch"] == e["read"] + e["write"]
        current = e["source_hash"] == bench.kernel_source_hash(e["sources"])
        assert bench.load_traffic(k) == (e["dram_bytes_per_launch"] if current else None)


def test_cpu_baseline_reports_all_cores_and_one_thread():
    sys.path.insert(0, ROOT)
    import bench
    from bit_quantized_linear_rotate_b200 import workloads as WL
    c = bench.cpu_baseline(WL.LINEAR_M8192, rows=16, min_seconds=0.0, max_passes=1)
    assert c["kind"] == "oracle" and c["unit"] == "TOPS" and c["value"] > 0 and c["cores"] >= 1
    assert "16 of 8192 rows" in c["sample"]
    st = c["single_thread"]
    assert st is None or (st["cores"] == 1 and st["value"] > 0)
