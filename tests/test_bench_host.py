"""Host-side logic of bench.py for N > 1 ranks, on CPU with the gloo backend:
the timed region is the slowest rank's, the value sums every rank's work,
and the reference arm runs on rank 0 only."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 100.0 + 10.0 * rank              # rank r took 100 + 10 r ms
        slowest = bench.max_over_ranks(elapsed)
        q.put((rank, slowest, bench.job_tflops(world, 1e12, slowest / 10)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_timing_is_the_slowest_rank_and_value_sums_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    slowest = 100.0 + 10.0 * (world - 1)
    for rank, s, v in got:
        assert s == slowest
        assert v == pytest.approx(world * 1e12 / (slowest / 10 * 1e-3) / 1e12)


def test_without_a_process_group_the_value_is_local():
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_tflops(1, 4e12, 1000.0) == pytest.approx(4.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_algorithmic_work_formulas():
    # two GEMMs of b x b x d per kept block pair
    assert bench.kept_flops(10, 128, 128) == 4.0 * 128 * 128 * 128 * 10

    class W:
        B, Hq, Hkv, N, d, nb, dtype = 1, 4, 2, 1024, 128, 8, "bf16"
    # Q and K read once (bf16), index lists (k + count) written once
    assert bench.selector_bytes(W, 4) == (4 + 2) * 1024 * 128 * 2 + 4 * 8 * 5 * 4


def test_clock_summary_keeps_the_timed_window():
    import datetime
    base = datetime.datetime(2026, 1, 2, 3, 4, 5)

    def line(dt_ms, mhz, cap="Not Active", thermal="Not Active"):
        ts = (base + datetime.timedelta(milliseconds=dt_ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {mhz}, 1965, 700.5, 0x0, Not Active, {thermal}, Not Active, {cap}\n"

    lines = [line(0, 1200), line(50, 1965), line(100, 1950, cap="Active"), line(150, 1965), line(400, 900,
             thermal="Active")]
    t0 = (base + datetime.timedelta(milliseconds=40)).timestamp()
    t1 = (base + datetime.timedelta(milliseconds=160)).timestamp()
    s = bench.ClockSampler.summarise(lines, (t0, t1))
    assert s["samples"] == 3 and s["in_timed_region"] is True
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    # no sample inside the window: every sample is summarised, and it says so
    s = bench.ClockSampler.summarise(lines, (t1 + 10, t1 + 11))
    assert s["samples"] == 5 and s["in_timed_region"] is False
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert bench.ClockSampler.summarise([], (t0, t1)) is None
    assert bench.ClockSampler.summarise(["garbage\n"], None) is None


def test_clock_sampler_names_the_gpu_by_pci_bus_id(monkeypatch):
    # With CUDA_VISIBLE_DEVICES=3 the process sees that GPU as CUDA device 0,
    # while nvidia-smi's index 0 is another GPU; the bus id names the right one.
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3")

    class Props:
        pci_domain_id, pci_bus_id, pci_device_id = 0, 0x9B, 0
    gid = bench.smi_gpu_id(Props)
    assert gid == "00000000:9B:00.0"
    cmd = bench.ClockSampler(gid).command()
    assert f"--id={gid}" in cmd and "--id=0" not in cmd and "--id=3" not in cmd
    assert any(a.startswith("--query-gpu=") and "pci.bus_id" in a for a in cmd)


def test_step_config_names_the_step_form():
    from block_sparse_attention_ba_b200.workloads import WORKLOADS
    single = bench.step_config(WORKLOADS["sweep_32k"], 0.5, 128, None, 1)
    assert "split" not in single["workload"] and "split_block" not in single
    assert single["workload"].endswith("selector(stats+scores+top-k)+sparse_fwd")
    split = bench.step_config(WORKLOADS["extreme_128k"], 0.5, 512, 77, 1)
    assert split["split_block"] == 77 and "sparse_fwd_merge" in split["workload"]
    assert bench.LAUNCHES_PER_STEP[False] == 4 and bench.LAUNCHES_PER_STEP[True] == 6


def test_attention_kernel_name_follows_the_library_dispatch():
    from block_sparse_attention_ba_b200.workloads import WORKLOADS
    w = WORKLOADS["sweep_32k"]
    assert bench.attention_kernel_name(w) == "attn_tc_kernel"
    assert bench.attention_kernel_name(w.with_(block=64)) == "attn_tc_kernel"
    assert bench.attention_kernel_name(w.with_(block=256)).startswith("attn_tc2_kernel")
    assert bench.attention_kernel_name(w.with_(block=256, d=64)) == "attn_tc_kernel"
    assert bench.attention_kernel_name(w.with_(block=32)) == "attn_simt_kernel"
    assert bench.attention_kernel_name(WORKLOADS["tiny_fp32"]) == "attn_simt_kernel"
