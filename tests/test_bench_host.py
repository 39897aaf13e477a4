"""Host-side logic of bench.py's replica mode, on 2 gloo ranks (CPU only)."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [4.0, 10.0][rank]
        value, ms_max = bench.aggregate_throughput(1e9, ms, world)
        bench.barrier(world)
        q.put((rank, value, ms_max, bench.max_over_ranks(float(rank), world)))
    finally:
        dist.destroy_process_group()


def test_replicas_take_max_over_ranks_and_sum_units():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms_max, mx in res:
        assert ms_max == 10.0                      # the slowest rank's time
        assert value == pytest.approx(2e9 / 10e-3)  # all ranks' units over that time
        assert mx == 1.0


def test_single_rank_is_identity():
    import bench

    value, ms = bench.aggregate_throughput(5e8, 2.0, 1)
    assert ms == 2.0 and value == pytest.approx(5e8 / 2e-3)


def test_measured_traffic_goes_null_when_the_kernel_source_changes(tmp_path):
    import hashlib

    import bench

    csrc = tmp_path / "weight_only_bit_qgemv_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel v1\n")
    digest = hashlib.sha256(b"kernel v1\n").hexdigest()[:16]
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# comment\nwork_a 12345 summary.md k.cu=%s\nwork_b 7 summary.md\n" % digest)
    assert bench.measured_traffic("work_a", str(tmp_path)) == 12345
    assert bench.measured_traffic("work_b", str(tmp_path)) == 7
    assert bench.measured_traffic("missing", str(tmp_path)) is None
    (csrc / "k.cu").write_text("kernel v2\n")
    assert bench.measured_traffic("work_a", str(tmp_path)) is None
    (csrc / "k.cu").unlink()
    assert bench.measured_traffic("work_a", str(tmp_path)) is None


def test_committed_traffic_file_parses():
    import bench

    for workload in ("decoder_block_m1", "lm_head_m1_int8"):
        v = bench.measured_traffic(workload)
        assert v is None or v > 0


def test_reference_arm_prints_the_contract_line_on_rank_zero_only():
    """`bench.py --impl reference`: the oracle on host cores, a bounded sample per step, the
    same metric and config as the GPU arm, zero copy bytes; other ranks print nothing."""
    import types

    import bench

    args = types.SimpleNamespace(steps=2, warmup=3)
    assert bench.run_reference(args, world=2, rank=1, budget_s=1.0) is None
    out = bench.run_reference(args, world=1, rank=0, budget_s=1.0)
    assert out["impl"] == "reference" and out["metric"] == bench.METRIC
    assert out["unit"] == "GB/s" and out["value"] > 0 and out["steps"] == 2 and out["warmup"] == 3
    assert out["config"]["workload"] == "decoder_block_m1"
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"] == {"value": out["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
