"""Host-side logic of bench.py that needs no GPU: the replica plumbing over a
two-rank gloo group (the slowest replica sets the job's time), the reference
arm's rank gating, and the bookkeeping that ties the reported DRAM traffic to
the kernel source it was measured on."""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    bench = _bench()
    w, r, local = bench.dist_env()
    dist = bench.dist_init(w, local, backend="gloo")
    try:
        # each replica times its own steps; the job's time is the slowest one
        out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_replicas():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_replica, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_process_needs_no_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    bench = _bench()
    assert bench.dist_env() == (1, 0, 0)
    assert bench.dist_init(1, 0, backend="gloo") is None
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench = _bench()

    class Args:
        seed, steps, warmup, gpus = 0, 1, 1, 2

    assert bench.reference_arm(Args()) == 0  # no oracle work, no line


def test_traffic_is_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    bench = _bench()
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "lmhead_fp8_157184x2560_m1_traffic.txt").write_text(
        f"# comment\nkernel_source_sha256_16 = {h}\ndram_bytes_per_launch = 409988352\n")
    src = tmp_path / "moe_decode_gemv_b200" / "csrc"
    src.mkdir(parents=True)
    for name in ("lmhead_fp8.cu", "common.cuh"):
        with open(os.path.join(ROOT, "moe_decode_gemv_b200", "csrc", name), "rb") as f:
            (src / name).write_bytes(f.read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic() == 409988352.0
    # a comment or a blank line is not a change of the kernel
    (src / "common.cuh").write_bytes((src / "common.cuh").read_bytes() + b"\n// a note, 'quoted'\n/* more */\n")
    assert bench.profiled_traffic() == 409988352.0
    # any change to the code voids the stored counters
    (src / "common.cuh").write_bytes((src / "common.cuh").read_bytes() + b"\nnamespace { int unused_x; }\n")
    assert bench.profiled_traffic() is None


def test_source_code_only_strips_comments_not_literals():
    bench = _bench()
    t = 'int a = 1;  // x\n/* y\n z */ const char* s = "a // b /* c */";\nchar q = \'"\'; char r = \'\\\'\';'
    assert bench.source_code_only(t) == 'int a = 1; const char* s = "a // b /* c */"; char q = \'"\'; char r = \'\\\'\';'


def test_workload_config_names_the_workload():
    bench = _bench()
    cfg = bench.workload_config()
    assert cfg["hidden"] == 2560 and cfg["expert_inter"] == 768 and cfg["experts"] == 512
    assert cfg["top_k"] == 8 and cfg["vocab"] == 157184 and cfg["head_top_k"] == 29 and cfg["M"] == 1
    assert "larger than L2" in cfg["l2"]
    assert bench.UNIT == "us/step"


def test_block_steps_gives_at_least_ten_blocks():
    bench = _bench()
    assert bench.block_steps(2000) == 20
    assert bench.block_steps(200) == 20
    assert bench.block_steps(199) == 19
    assert bench.block_steps(30) == 3
    assert bench.block_steps(3) == 1


def test_measured_peak_is_read_or_falls_back(tmp_path, monkeypatch):
    bench = _bench()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text('{"hbm_gbs": 6558.4, "bf16_tflops": 1590}')
    assert bench.measured_peaks() == (6558.4, "measured")
    f.write_text('{"hbm_gbs": {"value": 6600, "unit": "GB/s"}}')
    assert bench.measured_peaks() == (6600.0, "measured")
    for bad in ('{"bf16_tflops": 1590}', '{"hbm_gbs": null}', '{"hbm_gbs": -1}', "not json"):
        f.write_text(bad)
        peak, kind = bench.measured_peaks()
        assert peak == bench.FALLBACK_HBM_GBS and kind.startswith("fallback (")
