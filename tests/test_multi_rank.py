"""The batch-sharded multi-GPU path, host side, with two gloo ranks on CPU.

Sequences are independent, so N ranks each verify a batch of their own (seeded
by rank) and exchange nothing on the data path; the job's time is the max over
ranks.  These tests run the ranks' shards through the oracle (no GPU here) and
check the sharding and the timing reduction that bench.py uses."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    import parity
    inp = bench.make_inputs(1, 0, "cpu", rank)              # this rank's shard of the job
    res = parity.oracle_chain(inp, nthreads=2)
    gathered = [None] * world
    dist.all_gather_object(gathered, dict(tokens=res["tokens"], k=res["num_accepted"],
                                          first=inp.target[0, 0, :8].float().numpy()))
    ms = bench.reduce_max_ms(1.0 + rank, world)              # rank r "took" 1 + r ms
    value = bench.job_value(100, world, ms)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, gathered, ms, value))


def test_two_gloo_ranks_shard_the_batch_and_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort(key=lambda t: t[0])
    # every rank sees the same gathered results
    for r in range(world):
        for j in range(world):
            assert np.array_equal(got[r][1][j]["tokens"], got[0][1][j]["tokens"])
    # the shards differ (seeded by rank) ...
    assert not np.array_equal(got[0][1][0]["first"], got[0][1][1]["first"])
    # ... and each equals a single-process run of the same shard
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import bench
    import parity
    for r in range(world):
        ref = parity.oracle_chain(bench.make_inputs(1, 0, "cpu", r), nthreads=2)
        assert np.array_equal(got[0][1][r]["tokens"], ref["tokens"])
        assert np.array_equal(got[0][1][r]["k"], ref["num_accepted"])
    # max over ranks, whole-job rounds/s
    assert all(g[2] == 2.0 for g in got)
    assert all(abs(g[3] - 2 * 100 / 2e-3) < 1e-6 for g in got)



def _vp_rank(rank, world, port, cuts, out):
    """One rank of a vocabulary-parallel chain round: the orchestration of
    spec_verify_chain_vocab_parallel over gloo, with CPU stand-ins for the
    device steps."""
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    from speculative_decoding_verify_temperature_b200 import workloads as wl
    import vp_fakes
    inp = wl.chain_inputs(24, 4, 300, seed=5, device="cpu", target_dtype=__import__("torch").float32,
                          draft_dtype=__import__("torch").float32, zipf=True, temperatures=(0.6, 1.0))
    a, b = cuts[rank], cuts[rank + 1]
    toks, k = sv.spec_verify_chain_vocab_parallel(
        inp.target[:, :, a:b].contiguous(), inp.draft[:, :, a:b].contiguous(), inp.draft_tokens, inp.temperature,
        inp.coins, inp.final_u, vocab_offset=a, V=300, exchange=sv.TorchExchange(), ops=vp_fakes.FakeVpOps())
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, toks.numpy(), k.numpy()))


def test_two_gloo_ranks_vocab_parallel_round_matches_oracle():
    """Two ranks each hold part of every row's vocabulary; the three exchanges
    (all-gather of row statistics, all-gather of residual masses, all-reduce of
    the token) give both ranks the oracle's tokens for the whole rows."""
    world, cuts = 2, [0, 172, 300]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_vp_rank, args=(r, world, port, cuts, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=240) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import sys
    import torch
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity
    from speculative_decoding_verify_temperature_b200 import workloads as wl
    inp = wl.chain_inputs(24, 4, 300, seed=5, device="cpu", target_dtype=torch.float32, draft_dtype=torch.float32,
                          zipf=True, temperatures=(0.6, 1.0))
    o = parity.oracle_chain(inp)
    flags = parity.chain_flags(o, inp.gamma)
    for r in range(world):
        same = (got[r][2] == o["num_accepted"]) & (got[r][1] == o["tokens"]).all(axis=1)
        assert (same | flags).all()
        assert np.array_equal(got[r][1], got[0][1])
