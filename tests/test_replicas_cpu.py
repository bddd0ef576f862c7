"""Replica timing across ranks (bench.py, `--gpus N`): two gloo ranks on the CPU.

The block stack shards by independent sequences, so N GPUs run N replicas with no collective on
the data path; the only cross-rank steps are the barrier and the maximum of the step time. These
tests run that host logic with world_size 2 over gloo (127.0.0.1)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out) -> None:
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        local_ms = 10.0 + 2.0 * rank            # rank 1 is the slow one
        ms_max = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
        value = bench.replicas_throughput(16384, world, ms_max)
        # decode replicas: 8 sequences per rank, rank 1 slower, 0.9 GB streamed per step
        dec = bench.decode_entry(8, 2.0 + rank, 0.9e9, torch.device("cpu"), world, 6525.0)
        out[rank] = (ms_max, value, dec)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_time_is_the_slowest_rank_and_throughput_sums_batches():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for r in (0, 1):
        ms_max, value, dec = out[r]
        assert ms_max == pytest.approx(12.0)
        assert value == pytest.approx(2 * 16384 / 0.012)
        assert dec["ms_per_step"] == pytest.approx(3.0) and dec["replicas"] == 2
        assert dec["value"] == pytest.approx(2 * 8 / 0.003)       # tokens of both replicas
        assert dec["GB/s"] == pytest.approx(0.9e9 / 0.003 / 1e9)  # per GPU
        assert dec["frac_hbm"] == pytest.approx(dec["GB/s"] / 6525.0)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5, torch.device("cpu"), 1) == 7.5
    assert bench.replicas_throughput(1000, 1, 2.0) == pytest.approx(500000.0)
    dec = bench.decode_entry(64, 2.5, 1e9, torch.device("cpu"), 1, 6525.0)
    assert dec["value"] == pytest.approx(64 / 0.0025) and dec["replicas"] == 1


def test_gemm_traffic_tracks_kernel_source(monkeypatch):
    """The traffic figure is reported only for the captured workload and only while the kernel
    source matches the captured one; the profile it cites is committed."""
    import hashlib

    import bench

    src = os.path.join(bench.ROOT, "ternary_weight_matmul_b200", "csrc", "gemm_tc.cuh")
    with open(src, "rb") as fh:
        cur = hashlib.sha256(fh.read()).hexdigest()[:16]
    entry = dict(bench.GEMM_TRAFFIC["prefill-370M"])
    assert os.path.exists(os.path.join(bench.ROOT, entry["profile"]))
    assert 0 < entry["bytes"] < entry["algorithmic"]
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "prefill-370M", dict(entry, sha256=cur))
    assert bench.gemm_traffic("prefill-370M") == entry["bytes"]
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "prefill-370M", dict(entry, sha256="0" * 16))
    assert bench.gemm_traffic("prefill-370M") is None
    assert bench.gemm_traffic("prefill-1.3B") is None


def test_roofline_and_hbm_shares_from_kernel_classes():
    """The roofline of the dominant GEMM and the HBM-kernel figures come from the library's
    per-class launch records: achieved = algorithmic work / device time of the class, frac =
    achieved / peak, share = class time / step time of the attribution pass."""
    import bench

    kern = {"gemm_tc": {"launches": 96, "ms": 8.0, "work": 16.0e12},
            "gemm_simt": {"launches": 0, "ms": 0.0, "work": 0.0},
            "norm_quant": {"launches": 96, "ms": 2.5, "work": 8.0e9},
            "scan": {"launches": 24, "ms": 1.0, "work": 2.0e9},
            "other": {"launches": 1, "ms": 0.01, "work": 3.0e7}}
    r = bench.gemm_roofline(kern, 12.0, 3318.0, "test peak", None)
    assert r["achieved"] == pytest.approx(16.0e12 / 8.0e-3 / 1e12)   # 2000 TOPS
    assert r["frac"] == pytest.approx(2000.0 / 3318.0)
    assert r["avg_launch_us"] == pytest.approx(8.0 / 96 * 1e3)
    assert r["share_of_step"] == pytest.approx(8.0 / 12.0)
    h = bench.hbm_breakdown(kern, 12.0, 6525.0)
    assert set(h) == {"norm_quant", "scan", "other"}          # classes with no launch are left out
    assert h["norm_quant"]["GB/s"] == pytest.approx(8.0e9 / 2.5e-3 / 1e9)
    assert h["scan"]["frac_hbm"] == pytest.approx(2.0e9 / 1.0e-3 / 1e9 / 6525.0)
    assert h["scan"]["share_of_step"] == pytest.approx(1.0 / 12.0)
