"""Multi-process host logic of bench.py on CPU: two ranks over gloo (world size 2).

bench.py runs one process per GPU under torchrun; every rank times its own independent problem
(weak scaling), the times are reduced with a MAX all-reduce, and the whole-job value is the units
all ranks processed divided by the slowest rank's time.  These tests run that plumbing as two CPU
processes (spawned, no GPU), with the rendezvous on 127.0.0.1.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None)
    try:
        bench.barrier(w)
        # rank r "took" 10 + 3 r ms for its steps; the job is as slow as its slowest rank
        slowest = bench.max_over_ranks(10.0 + 3.0 * r, w)
        rate = bench.aggregate_rate(w, units_per_step=1000, steps=5, ms=slowest)
        q.put((r, w, dist.get_backend(), slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_times_with_max_and_aggregate_weakly():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for r, (rank, world, backend, slowest, rate) in enumerate(results):
        assert (rank, world, backend) == (r, 2, "gloo")
        assert slowest == 13.0
        # 2 ranks x 1000 units x 5 steps in 13 ms
        assert rate == pytest.approx(2 * 1000 * 5 / 13e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    bench.barrier(1)
    assert bench.aggregate_rate(1, 262144, 2000, 70.0) == pytest.approx(262144 * 2000 / 0.07)


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"])
    # a non-zero rank returns at once, without touching the oracle
    assert bench.reference_arm(args, 2, 1) == 0


def test_search_reference_arm_prints_one_contract_line(capsys):
    """The oracle arm of the search workload: one JSON line with the search metric, its own
    cpu_baseline and e2e (no host-device copies), timed on a bounded sample."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    assert bench.main(["--impl", "reference", "--workload", "search", "--steps", "1", "--warmup", "1"]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["metric"] == "search queries/s" and rec["unit"] == "queries/s"
    assert rec["value"] > 0 and rec["higher_is_better"] is True and rec["dtype"] == "f64"
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["value"] == rec["value"]
    assert rec["e2e"] == {"value": rec["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert rec["config"]["rows"] == 1_000_000 and rec["config"]["k"] == 10


def test_ragged_caches_share_lengths_and_cover_every_block():
    """Every cache of the paged workload maps each sequence's positions to its own distinct, valid
    physical blocks (so no step reads a block twice or outside the cache), and the caches differ
    only in the permutation."""
    import torch

    import bench
    import synth
    cfg = dict(bench.CONFIGS["ragged"])
    lens, table0, nblocks = bench.ragged_layout(cfg, 1102)
    seen_tables = []
    for ci in range(cfg["caches"]):
        tab = bench.cache_block_table(lens, 1102, ci)
        if ci == 0:
            assert torch.equal(tab, table0)
        used = []
        for b, L in enumerate(lens.tolist()):
            k = (L + synth.BLOCK_TOKENS - 1) // synth.BLOCK_TOKENS
            used.extend(tab[b, :k].tolist())
        assert len(used) == nblocks and len(set(used)) == nblocks
        assert min(used) >= 0 and max(used) < nblocks
        seen_tables.append(tab)
    assert not torch.equal(seen_tables[0], seen_tables[1])
