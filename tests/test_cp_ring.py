"""Context parallelism on CPU (gloo, world sizes 2 and 3), no GPU: the ring schedule, the
torch.distributed transport (``fwd_bwd_b200.cp.RingComm``) and the ring's dataflow.

The dataflow check runs the schedule and the transport of ``fwd_bwd_b200/cp.py`` with float64
attention in numpy in place of the kernels: the keys travel around the ring, every rank merges
its partial results by log-sum-exp, the dK/dV accumulators travel with the keys and come back
to their owner.  The gathered chunks must equal full-sequence float64 attention (and its
gradients) to rounding, causal and not.  The CUDA pieces themselves are checked on the GPU
(tests/test_gpu_cp.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fwd_bwd_b200.cp import RingComm, schedule


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [True, False])
def test_schedule(world, causal):
    for r in range(world):
        sched = schedule(r, world, causal)
        assert [s for s, _, _ in sched] == list(range(world))
        assert sorted(j for _, j, _ in sched) == list(range(world))  # every chunk once
        assert sched[0] == (0, r, "diag" if causal else "full")  # own chunk first
        for s, j, mode in sched:
            assert j == (r - s) % world
            if causal:
                assert mode == ("diag" if j == r else "full" if j < r else None)
            else:
                assert mode == "full"
        # under a causal mask the computed steps are the first r + 1
        if causal:
            assert [s for s, _, m in sched if m is not None] == list(range(r + 1))


def _attn_rows(q, k, v, tau, mask):
    """float64 softmax attention of q [N,d] over k, v [M,d]: (o, lse, p)."""
    z = tau * q @ k.T
    z = np.where(mask, z, -np.inf)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    return p @ v, (m + np.log(l))[:, 0], p


def _worker(rank, world, port, causal, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    comm = RingComm()
    assert (comm.rank, comm.world) == (rank, world)

    # transport: shift, shift_start / wait, average_
    got = comm.shift([torch.full((3,), float(rank)), torch.full((2, 2), 10.0 + rank)])
    prev = (rank - 1) % world
    assert torch.equal(got[0], torch.full((3,), float(prev)))
    assert torch.equal(got[1], torch.full((2, 2), 10.0 + prev))
    pend = comm.shift_start([torch.arange(4, dtype=torch.float64) + rank])
    assert torch.equal(pend.wait()[0], torch.arange(4, dtype=torch.float64) + prev)
    t = torch.tensor([float(rank), 2.0 * rank])
    comm.average_(t)
    assert torch.allclose(t, torch.tensor([(world - 1) / 2, world - 1.0]))

    # ring dataflow with float64 attention standing in for the kernels
    rng = np.random.default_rng(7)
    N, d, tau = 16, 8, 0.3
    Q, K, V, dO = (rng.standard_normal((world * N, d)) for _ in range(4))
    sl = slice(rank * N, (rank + 1) * N)
    q, k, v, do = Q[sl], K[sl], V[sl], dO[sl]
    rows = np.arange(N)[:, None]

    def visible(mode):
        if mode == "diag":
            return rows >= np.arange(N)[None, :]
        return np.ones((N, N), bool)

    o_acc = lse_acc = None
    payload = [torch.from_numpy(k.copy()), torch.from_numpy(v.copy())]
    for s, j, mode in schedule(rank, world, causal):
        pend = comm.shift_start(payload) if s + 1 < world else None
        if mode is not None:
            o_p, lse_p, _ = _attn_rows(q, payload[0].numpy(), payload[1].numpy(), tau,
                                       visible(mode))
            if o_acc is None:
                o_acc, lse_acc = o_p, lse_p
            else:
                lse_new = np.logaddexp(lse_acc, lse_p)
                o_acc = (np.exp(lse_acc - lse_new)[:, None] * o_acc +
                         np.exp(lse_p - lse_new)[:, None] * o_p)
                lse_acc = lse_new
        if pend is not None:
            payload = pend.wait()
    # backward: dQ local, dK / dV accumulators travel with the keys
    Dv = (do * o_acc).sum(axis=1)
    dq = np.zeros_like(q)
    # as fwd_bwd_b200/cp.py: the keys travel ahead (overlapping the step), the accumulators
    # after the step, and after the last step only they travel, back to their owner
    keys = [torch.from_numpy(k.copy()), torch.from_numpy(v.copy())]
    acc = [torch.zeros(N, d, dtype=torch.float64), torch.zeros(N, d, dtype=torch.float64)]
    for s, j, mode in schedule(rank, world, causal):
        pend = comm.shift_start(keys) if s + 1 < world else None
        if mode is not None:
            kj, vj = keys[0].numpy(), keys[1].numpy()
            z = tau * q @ kj.T
            p = np.where(visible(mode), np.exp(z - lse_acc[:, None]), 0.0)
            dp = do @ vj.T
            ds = p * (dp - Dv[:, None])
            dq += tau * ds @ kj
            acc[0] += torch.from_numpy(tau * ds.T @ q)
            acc[1] += torch.from_numpy(p.T @ do)
        if world > 1:
            acc = comm.shift(acc)
        if pend is not None:
            keys = pend.wait()
    dk, dv = acc[0].numpy(), acc[1].numpy()

    shards = [None] * world
    dist.all_gather_object(shards, dict(o=o_acc, lse=lse_acc, dq=dq, dk=dk, dv=dv))
    if rank == 0:
        out_q.put(({n: np.concatenate([s_[n] for s_ in shards]) for n in shards[0]},
                   (Q, K, V, dO, tau)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_dataflow_gloo(world, causal):
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, out_q))
             for r in range(world)]
    for p in procs:
        p.start()
    got, (Q, K, V, dO, tau) = out_q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    n = Q.shape[0]
    mask = (np.arange(n)[:, None] >= np.arange(n)[None, :]) if causal else np.ones((n, n), bool)
    o, lse, p = _attn_rows(Q, K, V, tau, mask)
    dp = dO @ V.T
    ds = p * (dp - (dO * o).sum(axis=1, keepdims=True))
    ref = dict(o=o, lse=lse, dq=tau * ds @ K, dk=tau * ds.T @ Q, dv=p.T @ dO)
    for name, want in ref.items():
        np.testing.assert_allclose(got[name], want, rtol=1e-11, atol=1e-11, err_msg=name)
