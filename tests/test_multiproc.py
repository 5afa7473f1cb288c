"""The N > 1 path of bench.py on CPU: two gloo ranks, each with its own share
of the global batch, combine their timings the way the benchmark does -- the
slowest rank's time and the sum of the ranks' work."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from jagged_attention_recommender_jfa_b200.inputs import make_problem
        p = make_problem("self_bf16", 1 + rank, B=5, max_len=200)
        f_fwd, f_bwd = bench.flops_of(p)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max, flops_all = bench.aggregate_over_ranks(ms, f_fwd + f_bwd, torch.device("cpu"), world)
        lens = torch.tensor(p.q_lens.astype("int64"))
        gathered = [torch.zeros_like(lens) for _ in range(world)]
        dist.all_gather(gathered, lens)
        out[rank] = (ms_max, flops_all, f_fwd + f_bwd,
                     [g.tolist() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    # both ranks report the slowest rank's time and the summed work
    assert r0[0] == r1[0] == 15.0
    assert r0[1] == r1[1] == pytest.approx(r0[2] + r1[2])
    # the ranks ran different batches (independent seeds), and agree on them
    assert r0[3] == r1[3] and r0[3][0] != r0[3][1]
