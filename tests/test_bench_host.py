"""Host logic of bench.py on the CPU: rank plumbing, max-over-ranks timing and
the replica aggregation, with two gloo ranks (no GPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        w, r, lr = bench.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        bench.init_dist(world, "gloo")
        bench.barrier(world)
        my_ms = [2.0, 3.0][rank]          # rank 1 is the slowest
        mx = bench.reduce_max(my_ms, world)
        val = bench.replica_value(73, world, mx)
        bench.barrier(world)
        dist.destroy_process_group()
        q.put((rank, mx, val))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


def test_two_rank_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    res.sort()
    for rank, mx, val in res:
        assert mx != "error", val
        assert mx == 3.0
        # two replicas of 73 tokens each, timed by the slowest rank
        assert val == pytest.approx(73 * 2 / 3e-3)


def test_single_rank_is_identity():
    assert bench.reduce_max(1.5, 1) == 1.5
    assert bench.replica_value(10, 1, 2.0) == pytest.approx(5000.0)


def test_reference_arm_other_ranks_do_no_work():
    args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert bench.run_reference(args, world=2, rank=1) == 0


def test_cli_rejects_short_warmup():
    with pytest.raises(SystemExit):
        bench.parse(["--warmup", "2"])


def test_reference_arm_times_the_oracle_on_cpu(capsys):
    # the reference arm of the contract: the fp64 oracle on a bounded sample
    import json
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["metric"] == bench.METRIC


def test_default_workload_is_the_405b_block():
    # the N = 1 line is the whole block on the largest single-GPU workload
    args = bench.parse([])
    assert args.workload == "mlp405b"
    assert args.steps >= 1 and args.warmup >= 3
    # about a second of timed work at ~25 ms per step
    assert 20 <= args.steps <= 200
    args = bench.parse(["--workload", "sq4096"])
    assert args.steps >= 1000


def test_reference_and_device_arms_share_the_config():
    # the reference line names the same workload, split, L2 policy and options
    c = bench.workload_config("mlp405b", 8, "pdl+static_weights")
    assert c["name"] == "mlp405b" and c["tp_degree"] == 8 and c["tokens"] == [8192]
    assert "read once per step" in c["l2"] and c["launch_options"] == "pdl+static_weights"
    assert bench.rotation_copies(bench.workload_weight_bytes("sq4096")) == 16
