"""Host-side logic of bench.py without a GPU: the whole-job throughput
arithmetic and the max-over-ranks timing over a two-rank gloo group."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_step_ops_counts_every_m_and_layer():
    layers = [("a", 256, 512), ("b", 128, 256)]
    assert bench.step_ops([1, 4], layers) == 2.0 * (1 + 4) * (256 * 512 + 128 * 256)


def test_aggregate_is_units_of_all_ranks_over_the_slowest():
    # K timed steps of U units each on W ranks, slowest rank took t seconds
    steps, units, world, t = 20, 1.0e9, 4, 0.5
    assert bench.aggregate(units * steps, world, t) == pytest.approx(units * steps * world / t)


def test_gemm_bytes_matches_the_packed_layout():
    # 6-bit weights are 3 bytes per 4 codes; FP16 scales per group; int8 codes
    M, N, K, gs = 16, 256, 512, 128
    expect = N * K * 3 / 4 + 2 * N * (K // gs) + M * K + 2 * M * (K // gs) + 2 * M * N
    assert bench.gemm_bytes(M, N, K, gs) == expect


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w = bench.dist_init("gloo")
    assert (r, w) == (rank, world)
    try:
        bench.barrier()
        # each rank reports its own elapsed time; every rank must see the max
        t = bench.max_over_ranks(0.25 + 0.5 * rank)
        out.put((rank, t, bench.aggregate(10.0, w, t)))
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in got:
        assert t == pytest.approx(0.75)
        assert v == pytest.approx(10.0 * 2 / 0.75)


def test_single_process_helpers_are_identities():
    assert bench.max_over_ranks(1.5) == 1.5
    bench.barrier()          # no process group: returns without a collective


def test_roofline_picks_the_lower_bound():
    # 4096^2 at M = 1: ~2 ops per byte, far below the ridge -> HBM-bound
    nb = bench.gemm_bytes(1, 4096, 4096)
    bound, frac = bench.roofline(2.0 * 4096 * 4096, nb, 10.0, 6500.0, 3300.0)
    assert bound == "hbm"
    assert abs(frac - (nb / 10e-6 / 1e9) / 6500.0) < 1e-9          # = achieved GB/s / peak GB/s
    # 2048 x 4096 x 4096: hundreds of ops per byte -> tensor-bound
    ops = 2.0 * 2048 * 4096 * 4096
    bound, frac = bench.roofline(ops, bench.gemm_bytes(2048, 4096, 4096), 100.0, 6500.0, 3300.0)
    assert bound == "tensor"
    assert abs(frac - ops / 100e-6 / 1e12 / 3300.0) < 1e-9


def test_headline_workload_is_the_llama2_70b_configuration():
    ms, layers = bench.workload_shapes()
    assert ms == [1, 16, 512, 8192]
    assert [(n, N, K, b) for (n, N, K, b, _) in layers] == [
        ("q", 8192, 8192, 6), ("o", 8192, 8192, 6), ("gate", 28672, 8192, 6),
        ("up", 28672, 8192, 6), ("down", 8192, 28672, 8)]
    # gate and up read the same input; every other layer its own
    assert len({site for (*_, site) in layers}) == 4
    assert "LLaMA-2-70B" in bench.workload_name(ms, layers)


def test_profiled_traffic_follows_the_kernel_source_digest(tmp_path, monkeypatch):
    # the committed summary carries the digest of the sources it was captured
    # with; the bench reports its byte count only while they still match
    text = open(os.path.join(bench.ROOT, bench.TRAFFIC_SUMMARY)).read()
    assert "kernel_src_sha:" in text and "dram_bytes_per_launch:" in text
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    summary = root / bench.TRAFFIC_SUMMARY
    monkeypatch.setattr(bench, "ROOT", str(root))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "00c0ffee")
    assert bench.profiled_traffic() is None                       # no summary
    summary.write_text("kernel_src_sha: 00c0ffee\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic() == 12345
    summary.write_text("kernel_src_sha: deadbeef\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic() is None                       # sources changed
