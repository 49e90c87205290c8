"""Host-side logic of bench.py, on the CPU: the multi-rank timing plumbing
(barrier and max over ranks) on two gloo ranks, the reference arm launched
as two ranks, the gating of ncu traffic figures by kernel-source hash, and
the workload table."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench as b
    d = b.Dist()
    d.init("gloo")
    d.barrier()
    # every rank reports its own "time"; all must agree on the largest
    m = d.max(10.0 + 3.5 * rank, "cpu")
    d.barrier()
    d.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": rank, "max": m}, f)


def test_dist_max_over_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [g["max"] for g in got] == [13.5, 13.5]


def test_dist_single_rank_is_identity():
    d = bench.Dist()
    if d.world != 1:
        pytest.skip("run outside a launcher")
    d.init("gloo")
    d.barrier()
    assert d.max(2.25, "cpu") == 2.25
    d.close()


def test_reference_arm_under_two_ranks_prints_one_line():
    """torchrun with 2 ranks: rank 0 times the oracle and prints the JSON
    line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "gemv_4096", "--steps", "3", "--warmup", "3", "--cpu-seconds", "0.3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True
    cores = len(os.sched_getaffinity(0))
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == min(cores, 128)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "gemv_4096"


def test_warmup_below_three_is_rejected():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--warmup", "2"])


def _fake_tree(tmp_path, kernel_text: bytes, profile: str):
    csrc = tmp_path / "bit_weight_quantized_nvq_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_bytes(kernel_text)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "kern_wl.md").write_text(profile)


def test_traffic_is_used_only_for_the_measured_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _fake_tree(tmp_path, b"kernel v1", "placeholder")
    h1 = bench.source_hash("k.cu")
    (tmp_path / "profiles" / "kern_wl.md").write_text(
        f"# summary\n\nsource_hash: {h1}\ndram_bytes_per_launch: 123456\n")
    assert bench.profiled_traffic("kern", "wl", h1) == 123456.0
    # the kernel changed since the counters were taken: no traffic figure
    (tmp_path / "bit_weight_quantized_nvq_b200" / "csrc" / "k.cu").write_bytes(b"kernel v2")
    h2 = bench.source_hash("k.cu")
    assert h2 != h1
    assert bench.profiled_traffic("kern", "wl", h2) is None
    # no summary, or a summary without the bytes line
    assert bench.profiled_traffic("other", "wl", h1) is None
    (tmp_path / "profiles" / "kern_wl.md").write_text(f"source_hash: {h1}\n")
    assert bench.profiled_traffic("kern", "wl", h1) is None


def test_workload_table():
    for name, bound in (("decode_sweep", "hbm"), ("gemv_4096", "hbm"), ("small_batch_m8", "hbm"),
                        ("prefill_m256", "tensor"), ("prefill_m2048", "tensor"),
                        ("stack_decode", "hbm"), ("stack_prefill", "tensor"),
                        ("moe_decode", "hbm"), ("w4a16_decode", "hbm"),
                        ("nvf4_prefill_m2048", "tensor")):
        wk = bench.make_workload(name)
        assert wk.bound == bound, name
        assert wk.config()["workload"] == name
    with pytest.raises(SystemExit):
        bench.make_workload("no_such_workload")


def test_oracle_tasks_split_over_workers_keep_their_units():
    """The all-cores oracle baseline splits each sample's repetitions over
    the pool without losing or double-counting work."""
    wk = bench.make_workload("gemv_4096")
    tasks = wk.oracle_tasks(300)
    (codes, scales, g, x, reps, units), = tasks
    assert reps == 5 and codes.shape[0] == bench.ORACLE_BASE_ROWS      # 300 rows -> 5 x 64
    assert abs(units - 5 * 64 * 4096 * 0.5625 / 1e9) < 1e-12
    parts = bench.split_tasks(tasks, 3)
    assert sum(p[4] for p in parts) == reps
    assert abs(sum(p[5] for p in parts) - units) < 1e-12
    assert abs(bench.run_tasks_serial(parts) - bench.run_tasks_serial(tasks)) < 1e-15


def test_nvf4_oracle_task_runs_the_nvf4_oracle():
    """The NVFP4 x NVFP4 sample runs the oracle's NVFP4 activation quantiser
    and its NVFP4 dot (not the Q8_0 path), and its units are FLOPs."""
    wk = bench.make_workload("nvf4_prefill_m256")
    assert wk.peak_scale == 4.0
    tasks = wk.oracle_tasks(64)
    assert len(tasks) == len(wk.shapes)
    codes, scales, g, x, reps, units = tasks[0]
    assert isinstance(x, tuple) and x[0] == "nvf4" and x[1].shape[0] == 16
    K = wk.shapes[0][0]
    assert abs(units - 2.0 * 16 * K * 64 / 1e12) < 1e-15
    assert bench.oracle_task((codes, scales, g, x, 1, units)) == units
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "source": "test"}
    shapes = [{"K": K, "N": 64, "us_per_launch": 10.0, "amount": 1e9, "weight_copies": 2}]
    r = bench.roofline_entry(wk, shapes, 0.02, peaks)
    assert r["peak"] == 6000.0 and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 100.0) < 1e-9


def test_cpu_baseline_reports_one_core_and_all_cores():
    wk = bench.make_workload("gemv_4096")
    pool = bench.OraclePool()
    try:
        cb = bench.cpu_baseline(wk, 0.2, pool)
    finally:
        pool.close()
    assert cb["cores"] == 1 and cb["kind"] == "oracle" and cb["value"] > 0
    assert cb["all_cores"]["cores"] == pool.cores and cb["all_cores"]["value"] > 0
    assert "64 rows" in cb["sample"]


def test_launch_counts_follow_the_gemm_schedule(monkeypatch):
    """The prefill GEMM adds a fix-up launch exactly when its tiles (128
    tokens x 256 weight rows) do not divide evenly over the CTA pairs; the
    one-token stack is one quantisation plus one persistent launch per 64
    layers."""
    import torch

    class Props:
        multi_processor_count = 148          # 74 CTA pairs

    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda *a: Props())
    # 320 and 1600 tiles over 74 pairs leave a partial wave; 74 tiles do not
    assert bench.gemm_launches(2048, 5120, 5120) == 2
    assert bench.gemm_launches(2048, 25600, 5120) == 2
    assert bench.gemm_launches(256, 9472, 25600) == 1       # 2 x 37 tiles
    assert bench.gemm_launches(128, 256, 128) == 1          # one tile, one stage
    g = bench.GemmWorkload.__new__(bench.GemmWorkload)
    g.M = 2048
    g.cases = [{"K": 5120, "N": 5120}, {"K": 5120, "N": 9472}]
    assert g.launches_per_step() == (2 + 2) + (2 + 1)          # 16 x 37 = 592 tiles: 8 whole waves
    s = bench.StackWorkload.__new__(bench.StackWorkload)
    s.n_layers, s.linears = 64, [("q", 5120, 5120)] * 7
    s.M = 1
    assert s.launches_per_step() == 2
    s.M = 2048
    assert s.launches_per_step() == 64 * (8 + 7 * 2)
