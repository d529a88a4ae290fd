"""World-size-2 (gloo, CPU) check of the data-parallel partition: each rank computes its own
contiguous range of flattened heads -- or, as bench.py's end-to-end leg splits one global batch,
its own range of batch entries -- (here with the CPU oracle standing in for a GPU), and the
gathered shards equal the single-process result exactly: every head is an independent problem,
so there is nothing to exchange but the results.  Also checks the harness's max-over-ranks
timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fwd_bwd_b200.shard import head_range


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_head_range_partition():
    for total in (1, 7, 64, 513):
        for world in (1, 2, 3, 8):
            got = [list(head_range(total, world, r)) for r in range(world)]
            assert sum(got, []) == list(range(total))
            sizes = [len(g) for g in got]
            assert max(sizes) - min(sizes) <= 1


WL = {"heads": dict(B=1, H=5, N=256), "batch": dict(B=3, H=2, N=256)}


def _worker(rank, world, port, out_q, unit):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle.sage_oracle as O
    from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS["llama325m"].replace(**WL[unit])
    if unit == "heads":
        mine = head_range(w.B * w.H, world, rank)
    else:  # contiguous batch entries (bench.py's end-to-end split), as flattened heads
        b = head_range(w.B, world, rank)
        mine = range(b.start * w.H, b.stop * w.H)
    x = make_inputs(w, heads=mine)
    res = O.sage_attention(*(x[n + "_f32"] for n in ("q", "k", "v", "do")), causal=w.causal,
                           qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                           k_block=w.k_block, dtype=w.dtype)
    shards = [None] * world
    dist.all_gather_object(shards, {n: res[n] for n in ("o", "dq", "dk", "dv", "lse")})
    t = torch.tensor([float(rank + 1)])
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    if rank == 0:
        out_q.put(({n: np.concatenate([s[n] for s in shards]) for n in shards[0]},
                   float(t.item())))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("unit", ["heads", "batch"])
def test_two_rank_shards_concatenate_to_single_result(unit):
    import oracle.sage_oracle as O
    from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, unit)) for r in range(2)]
    for p in procs:
        p.start()
    gathered, tmax = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert tmax == 2.0
    w = WORKLOADS["llama325m"].replace(**WL[unit])
    x = make_inputs(w)
    full = O.sage_attention(*(x[n + "_f32"].reshape(-1, w.N, w.d)
                              for n in ("q", "k", "v", "do")), causal=w.causal,
                            qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                            k_block=w.k_block, dtype=w.dtype)
    for n, v in gathered.items():
        np.testing.assert_array_equal(v, full[n])
