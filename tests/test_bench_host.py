"""Host-side logic of bench.py on the CPU: the multi-rank (replica) reduction under gloo with two
ranks, the whole-job value, the weight-rotation and roofline-bound rules, and the reference
arm's output contract."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(times[rank], world, "cpu")
        dist.barrier()
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    """Each rank gets the slowest rank's time (the bench's timed region is the max over ranks)."""
    world = 2
    times = [3.25, 7.5]
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world, start_method="spawn",
                       join=True)
    assert dict(out) == {0: 7.5, 1: 7.5}


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(1.5, 1) == 1.5


def test_job_value_counts_every_replica():
    # 21.74 TFLOP per step in 18 ms on one GPU, and the same per GPU on 8 replicas
    one = bench.job_value(1, 21.743e12, 18.0)
    assert one == pytest.approx(21.743e12 / 18e-3 / 1e12)
    assert bench.job_value(8, 21.743e12, 18.0) == pytest.approx(8 * one)


def test_rotation_copies_rule():
    l2 = 126 << 20
    assert bench.rotation_copies(3 * l2, 10 << 20, l2) == 1                    # larger than 2x L2
    c = bench.rotation_copies(30 << 20, 28 << 20, l2)                           # 16-token text encoder
    assert c >= 20 and c * (28 << 20) >= 2.2 * l2
    assert bench.rotation_copies(100, 50, l2) == 256                           # tiny: capped


def test_hbm_bound_rule():
    peaks = {"bf16_tflops": 1630.0, "hbm_gbs": 6547.0}                         # ridge ~249 flop/B
    assert bench.is_hbm_bound(2 * 16 * 2560 * 9728, 14.1e6, peaks)               # 16 tokens: 56 flop/B
    assert not bench.is_hbm_bound(2 * 4608 * 3072 * 18432, 213e6, peaks)         # 4608 tokens


def _run_bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=600)


def test_reference_arm_prints_contract_line_on_rank0():
    r = _run_bench(["--impl", "reference", "--workload", "tiny_ternary_g64", "--steps", "1", "--warmup", "3"],
                   {"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "tiny_ternary_g64", "--steps", "1", "--warmup", "3",
                    "--gpus", "2"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def _fake_tree(tmp_path, kernel_text, traffic):
    csrc = tmp_path / "bit_weight_only_w2_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(kernel_text)
    (tmp_path / "include").mkdir()
    (tmp_path / "include" / "lowbit.h").write_text("/* header */\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(traffic))


def test_measured_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    """roofline.traffic is reported only while the CUDA sources hash to the captured ones."""
    _fake_tree(tmp_path, "__global__ void k() {}\n", {})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w": {"dram_bytes_per_launch": 123.0, "source_sha256": h}}))
    assert bench.measured_traffic("w") == 123.0
    assert bench.measured_traffic("other") is None
    (tmp_path / "bit_weight_only_w2_b200" / "csrc" / "k.cu").write_text("__global__ void k() { }\n")
    assert bench.kernel_source_hash() != h
    assert bench.measured_traffic("w") is None          # a changed kernel invalidates the capture


def test_gpus_flag_launches_that_many_ranks():
    """`--gpus 2` outside torchrun starts two ranks itself (torchrun on 127.0.0.1): rank 0 prints the
    one line, with n_gpus equal to the ranks that ran; the other rank prints nothing."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny_ternary_g64", "--steps", "1", "--warmup", "3", "--ref-rows", "4"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["impl"] == "reference"


def test_world_must_match_gpus():
    bench.check_world(2, 2)
    with pytest.raises(SystemExit):
        bench.check_world(4, 2)



def test_traffic_follows_only_its_own_kernels_sources(tmp_path, monkeypatch):
    """A capture of one kernel stays valid when only another kernel's sources change."""
    csrc = tmp_path / "bit_weight_only_w2_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in (*bench.KERNEL_SOURCES["lowbit_gemm_kernel"], *bench.KERNEL_SOURCES["lowbit_smallm_kernel"],
              *bench.SHARED_SOURCES):
        (csrc / f).write_text(f"// {f}\n")
    (tmp_path / "include").mkdir()
    (tmp_path / "include" / "lowbit.h").write_text("/* header */\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash("lowbit_gemm_kernel")
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w": {"dram_bytes_per_launch": 7.0, "source_sha256": h, "kernel": "lowbit_gemm_kernel"}}))
    (csrc / "smallm_kernel.cuh").write_text("// changed\n")
    assert bench.measured_traffic("w") == 7.0
    (csrc / "sm100_ptx.cuh").write_text("// changed\n")          # shared by every kernel
    assert bench.measured_traffic("w") is None
