"""The multi-GPU path of bench.py is N independent replicas: the only
cross-rank steps are the barrier and the max-reduction of the per-step time.
Those run here as two gloo ranks on CPU (no GPU), and the reference arm's
non-zero ranks must return without work."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local = 5.0 + 1.25 * rank  # rank 1 is the slower replica
        ms = bench.slowest_rank_ms(local, world)
        e2e = bench.slowest_rank_ms(10.0 - rank, world)  # here rank 0 is the slower one
        dist.barrier()
        out[rank] = (ms, e2e, bench.aggregate_steps_per_s(ms, world))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world = 2
    # the manager process is spawned too: forking a process whose BLAS threads are running can deadlock
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        ms, e2e, value = res[rank]
        assert ms == 6.25 and e2e == 10.0
        assert value == pytest.approx(2 * 1e3 / 6.25)


def test_single_rank_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.slowest_rank_ms(4.0, 1) == 4.0
    assert bench.aggregate_steps_per_s(4.0, 1) == 250.0


def test_reference_arm_other_ranks_exit_without_work():
    class Args:
        steps, warmup, workload = 1, 0, 5

    assert bench.run_reference(Args, rank=1, world=2) == 0


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    """bench.py reports the committed DRAM traffic of a kernel only while the
    kernel's source is byte-identical to the one the capture was taken on."""
    import hashlib

    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (prof / "k_dram_traffic_sd21_base_unet_step_96.md").write_text(
        "summary\n\ntraffic_bytes_per_launch: 1234\nsource: kernel.cu\nsource_sha256: " + digest + "\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k", "sd21_base_unet_step_96") == 1234.0
    assert bench.measured_traffic("k", "other_workload") is None
    src.write_text("// version 2\n")
    assert bench.measured_traffic("k", "sd21_base_unet_step_96") is None
    assert bench.measured_traffic("missing", "sd21_base_unet_step_96") is None


def test_ncu_family_shares_of_the_committed_launch_list():
    """The uninstrumented per-family shares bench.py applies to the headline come
    from the committed ncu launch list of the workload, and cover the whole step."""
    shares = bench.ncu_family_shares("sd21_base_unet_step_96")
    assert set(shares) == {"gemm_tc", "attention", "groupnorm", "other"}
    assert abs(sum(shares.values()) - 1.0) < 0.01
    assert shares["gemm_tc"] > shares["attention"] > shares["groupnorm"]
    assert bench.ncu_family_shares("no_such_workload") == {}


def test_peak_choice_follows_region_length_and_power_cap():
    peaks = {"bf16_tflops": 1674.6, "bf16_tflops_sustained": 1363.4, "hbm_gbs": 6547.5}
    assert bench.choose_peak(peaks, "measured", 0.12, {"reasons": []})[0] == 1674.6
    assert bench.choose_peak(peaks, "measured", 0.12, {"reasons": ["sw_power_cap"]})[0] == 1363.4
    assert bench.choose_peak(peaks, "measured", 1.7, {"reasons": []})[0] == 1363.4


def test_reference_arm_splits_one_pass_into_the_timed_steps():
    """The reference arm's module list covers the whole step in forward order."""
    names = bench.oracle_stage_names(5)
    assert names[0] == "temb" and names[-1] == "out"
    assert sum(n.endswith(".res.0") or n.endswith(".res.1") or n.endswith(".res.2") for n in names) == 22
    assert sum(".attn." in n for n in names) == 16 and "mid.attn.0" in names
