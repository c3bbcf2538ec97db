"""bench.py's multi-rank host logic on CPU: two gloo ranks.

Replicas share nothing on the data path; the only cross-rank steps are the
barriers around the timed region and the max over ranks of the elapsed time.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    sys.argv = ["bench.py"]
    import bench
    import torch.distributed as dist
    w, r, local = bench.init_dist(bench.parse())
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    got = bench.reduce_max(10.0 + 5.0 * rank, w)
    bench.barrier(w)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"max": got}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        with open(tmp_path / f"r{r}.json") as f:
            assert json.load(f)["max"] == pytest.approx(15.0)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    bench.barrier(1)


@pytest.mark.timeout(300)
def test_reference_arm_prints_only_on_rank_zero(tmp_path):
    """Under torchrun with two ranks the reference arm prints one line, from rank 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "1",
           "--cpu-seconds", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=280, env=env, cwd=str(tmp_path))
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_traffic_is_reported_only_for_the_current_kernel_sources(tmp_path, monkeypatch):
    """A committed ncu traffic figure is used only while its kernel family's
    sources still hash to the value it was captured on; otherwise the bench
    reports null."""
    sys.path.insert(0, ROOT)
    import bench
    (tmp_path / "profiles").mkdir()
    ent = {"dram_bytes_per_launch": 123, "kernel_hash": bench.kernel_hash("decode")}
    data = {"llama7b-decode": {"decode_fused": ent},
            "llama70b:n16": {"tc_up": {"dram_bytes_per_launch": 456, "kernel_hash": bench.kernel_hash("tc")}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(data))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("decode_fused", "llama7b-decode", 1) == 123
    assert bench.traffic_for("tc_up", "llama70b", 16) == 456
    assert bench.traffic_for("tc_up", "llama70b", 64) is None
    data["llama7b-decode"]["decode_fused"]["kernel_hash"] = "0" * 16
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(data))
    assert bench.traffic_for("decode_fused", "llama7b-decode", 1) is None
    # a tensor-core figure keyed with the decode family's hash does not count
    data["llama70b:n16"]["tc_up"]["kernel_hash"] = bench.kernel_hash("decode")
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(data))
    assert bench.traffic_for("tc_up", "llama70b", 16) is None


def test_kernel_hash_ignores_comments_and_layout():
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) { // add one\n  return x + 1; /* done */ }\n"
    b = "int f(int x)\n{\n    return x + 1;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only('const char* s = "// kept";') == 'const char* s = "// kept";'
    assert bench.code_only("return x + 1;") != bench.code_only("return x + 2;")


def test_bench_bytes_match_the_pinned_oracle_counter():
    """The roofline numerator (bench.algorithmic_bytes and dense_bytes) is the
    oracle's byte counter, which a pin checks against an enumerated read list."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import workloads
    for wl in (workloads.llama7b_decode(0.9), workloads.lopa7b(0.9), workloads.llama70b(4, "lopa", 0.9),
               workloads.llama70b(16, "dense", 0.9), workloads.tiny()):
        w = 2 if wl.dtype == "bf16" else 4
        for union in (0, 1, 1108, wl.d_ff):
            assert bench.algorithmic_bytes(wl, union) == oracle.bytes_moved(
                wl.n, wl.d, wl.d_ff, union, w, w, r=wl.r if wl.gate == "lopa" else 0), (wl.name, union)
        assert bench.dense_bytes(wl) == oracle.dense_bytes(wl.n, wl.d, wl.d_ff, w, w)
