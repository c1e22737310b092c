"""The N > 1 path of bench.py on CPU: two gloo ranks, no GPU.

Decoding needs no collective (every rank decodes its own replica), so the only multi-rank logic is the
timing: each rank's measurement goes through an element-wise max over ranks, and the whole-job value
is N x params per rank / the slowest rank's step time. The reference arm runs on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Rank r reports a step time of 10 + r ms and a best time of 5 - r ms.
        ms, best = bench.max_over_ranks([10.0 + rank, 5.0 - rank], torch.device("cpu"))
        value = bench.weak_scaling_value(world, 6_000_000, ms)
        results[rank] = (ms, best, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_two_gloo_ranks():
    world = 2
    results = mp.get_context("spawn").Manager().dict()  # no fork of this (threaded) process
    mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
    for r in range(world):
        ms, best, value = results[r]
        assert ms == 11.0 and best == 5.0  # every rank sees the slowest rank's numbers
        assert value == pytest.approx(2 * 6_000_000 / 11e-3 / 1e9)


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks([3.5, 1.25], torch.device("cpu")) == [3.5, 1.25]
    assert bench.weak_scaling_value(1, 1_000_000_000, 1000.0) == pytest.approx(1.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    # Ranks other than 0 return before touching the oracle or any data.
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class Args:
        warmup, steps, target_bpp = 3, 2, 4.0

    assert bench.run_reference(Args()) is None


def test_single_tensor_selection_by_label():
    assert len(bench.selected_items("sweep4096")) == 24
    assert [it[0] for it in bench.selected_items("sweep4096", "bf16_6bpp")] == ["gauss4096_bf16_6bpp"]
    fp32 = bench.selected_items("sweep4096", "fp32")
    assert len(fp32) == 8 and all(it[0].startswith("gauss4096_fp32_") for it in fp32)
    assert [it[2] for it in fp32] == [0.5, 1.0, 2.3, 3.0, 5.0, 6.0, 8.0, 11.0]
    assert bench.selected_items("fp8_8192x28672_5bpp", "nothing") == []


def test_committed_traffic_figure_is_consistent():
    """The DRAM traffic per algorithmic byte that the bench line reports: its ratio is the capture's read +
    write bytes over the algorithmic bytes, and it is used only while the kernel source hash matches."""
    import json
    d = json.load(open(bench.os.path.join(bench.ROOT, "profiles", "decode_traffic.json")))
    ratio = (d["dram_bytes_read"] + d["dram_bytes_write"]) / d["algorithmic_bytes"]
    assert abs(ratio - d["dram_bytes_per_algorithmic_byte"]) < 1e-12
    assert 0.5 < ratio < 1.5
    got = bench.committed_traffic()
    assert (got is not None) == (d["kernel_source_sha256_16"] == bench.kernel_source_hash())
