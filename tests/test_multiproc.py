"""The N > 1 bench path on CPU: two gloo ranks, each with its own independent batch
(weak scaling), time reduced as the max over ranks and work as the sum."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        seed = bench.rank_seed(1, r)
        t_max = bench.max_over_ranks(10.0 + r, device="cpu")
        tok_sum = bench.sum_over_ranks(1000.0 * (r + 1), device="cpu")
        from recurrent_state_memory_b200 import inputs as I
        p = I.make_fwd(1, 8, 1, 32, 32, dtype="bf16", seed=seed)
        out[rank] = (ws, r, local, seed, t_max, tok_sum, bytes(p.q.tobytes()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_helpers():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    a, b = out[0], out[1]
    assert a[0] == b[0] == 2 and (a[1], b[1]) == (0, 1) and (a[2], b[2]) == (0, 1)
    assert a[3] != b[3]                       # independent batches per rank
    assert a[6] != b[6]
    assert a[4] == b[4] == 11.0               # max over ranks
    assert a[5] == b[5] == 3000.0             # whole-job work is the sum


def test_single_process_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.sum_over_ranks(2.0) == 2.0
    assert bench.rank_seed(4, 0) == 4


def test_reference_arm_prints_one_contract_line(capsys):
    """`bench.py --impl reference` (the fp64 oracle timed on the host cores) prints one JSON
    line with the forward metric, impl "reference", an oracle cpu_baseline and an e2e object
    with no host-device traffic; it needs no GPU."""
    import json

    import bench
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "Mtokens/s"
    assert d["value"] > 0 and d["higher_is_better"] and d["steps"] == 1 and d["gpu_launches"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == bench.WORKLOAD
    # the GPU arm builds its config object with the same function from the same workload
    from recurrent_state_memory_b200 import inputs as I
    assert d["config"] == bench.workload_config(bench.WORKLOAD, I.make_config(bench.WORKLOAD))
