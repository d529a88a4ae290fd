"""Context parallelism: one long sequence split across W ranks, keys passed around a ring.

The sequence of W * N tokens is cut into W contiguous chunks of N tokens; rank r holds tokens
[r N, (r+1) N) of q, k, v and dout for every (batch, head).  Every quantization block of the
method (Q, K, V per block of tokens; P, dS, dO per tile) lies inside one chunk, so the result
is the single-sequence one up to float32 rounding order ("SageBwd: trainable low-bit
attention": the per-block INT8 recipe of the Triton-kernel paragraph, the K-smoothing mean over
the whole sequence).

Forward (``forward``): the K-smoothing mean is the average of the W chunk means (one all-reduce
of a [B, H, d] float32 tensor); each rank quantizes its chunk; the INT8 K and V codes and their
block scales (1 byte per element, half the 16-bit traffic) travel around the ring.  At step s
rank r holds the keys of chunk j = (r - s) mod W and computes its queries against them when any
is visible (``sage_attn_fwd_partial``: the diagonal chunk with the causal mask, earlier chunks
without); the float32 partials are merged by their log-sum-exp (``sage_attn_merge``).  The
transfer of step s+1's keys is issued before step s's kernels, so the two overlap.

Backward (``backward``): the K codes and scales, the raw 16-bit V (for the 16-bit dP product)
and two float32 accumulators for the keys' raw dK and dV travel around the ring; each rank adds
its queries' contribution (``sage_attn_bwd_partial``; dQ accumulates locally), and after W
shifts the accumulators are back with the keys' owner, which applies the RMSNorm backward
(``sage_kv_finalize``).  The keys' transfer overlaps the step's kernels; the accumulators' can
only follow them.

Two transports run the same per-rank code:
  * ``RingComm``: one process per GPU, torch.distributed point-to-point (NCCL on GPUs);
  * ``LocalRing``: W ranks as threads of one process sharing one GPU, for tests and debugging.
    Each thread has its own CUDA stream; hand-offs are device-to-device copies ordered by CUDA
    events (stream dependencies: no kernel spins on another rank's progress).

Every step of the computation runs in libsage's kernels; this module only schedules calls and
moves buffers.  Q-smoothing is not supported here.
"""
from __future__ import annotations

import ctypes
import dataclasses
import threading
from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import ops
from ._lib import SageQBufs, check, lib


def schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, int, Optional[str]]]:
    """(step, key chunk, mode) of every ring step of `rank`: the keys of chunk (rank - step) mod
    world arrive at that step; mode is "diag" (the rank's own chunk under a causal mask),
    "full" (every key visible) or None (every key later than every query: not computed)."""
    out = []
    for s in range(world):
        j = (rank - s) % world
        if j == rank:
            mode = "diag" if causal else "full"
        elif j < rank or not causal:
            mode = "full"
        else:
            mode = None
        out.append((s, j, mode))
    return out


# ---- transports ---------------------------------------------------------------------------
class _Pending:
    def __init__(self, recv, works, finish=None):
        self._recv, self._works, self._finish = recv, works, finish

    def wait(self) -> List[torch.Tensor]:
        for w in self._works:
            w.wait()
        if self._finish is not None:
            return self._finish()
        return self._recv


class RingComm:
    """torch.distributed transport: send to rank + 1, receive from rank - 1 (mod world)."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self._nccl = dist.get_backend(group) == "nccl"

    def _peer(self, r: int) -> int:
        r %= self.world
        return r if self.group is None else dist.get_global_rank(self.group, r)

    def shift_start(self, tensors: Sequence[torch.Tensor]) -> _Pending:
        """Starts sending `tensors` to the next rank and receiving the previous rank's into new
        buffers; ``wait()`` on the result returns them.  The sent tensors must not change
        before then."""
        recv = [torch.empty_like(t) for t in tensors]
        nxt, prv = self._peer(self.rank + 1), self._peer(self.rank - 1)
        if self._nccl:
            # grouped, so that a send and a receive between the same two ranks cannot block
            # each other
            p2p = [dist.P2POp(dist.isend, t, nxt, self.group) for t in tensors]
            p2p += [dist.P2POp(dist.irecv, t, prv, self.group) for t in recv]
            works = dist.batch_isend_irecv(p2p)
        else:
            works = [dist.isend(t, nxt, self.group) for t in tensors]
            works += [dist.irecv(t, prv, self.group) for t in recv]
        return _Pending(recv, works)

    def shift(self, tensors: Sequence[torch.Tensor]) -> List[torch.Tensor]:
        return self.shift_start(tensors).wait()

    def average_(self, t: torch.Tensor) -> None:
        """In-place mean of `t` over the ranks."""
        if self._nccl:
            dist.all_reduce(t, op=dist.ReduceOp.AVG, group=self.group)
        else:  # gloo has no average
            dist.all_reduce(t, group=self.group)
            t.div_(self.world)


class LocalRing:
    """W ranks as threads of this process on one CUDA device.  ``run(fn, args)`` calls
    ``fn(comm_r, *args[r])`` for every rank r, each in its own thread with its own CUDA stream,
    and returns the results in rank order."""

    def __init__(self, world: int, device=None):
        self.world = world
        dev = torch.device("cuda") if device is None else torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self._barrier = threading.Barrier(world)
        self._box: list = [None] * world
        self._done: list = [None] * world

    def run(self, fn, args_per_rank: Sequence[tuple]) -> list:
        lib()  # load the library before the threads start
        self._barrier = threading.Barrier(self.world)  # a fresh one (a failed run breaks it)
        results: list = [None] * self.world
        errors: list = []

        def body(r: int):
            try:
                torch.cuda.set_device(self.device)
                stream = torch.cuda.Stream(self.device)
                with torch.cuda.stream(stream):
                    results[r] = fn(_LocalComm(self, r), *args_per_rank[r])
                stream.synchronize()
            except BaseException as e:  # noqa: BLE001 - re-raised in the caller
                errors.append(e)
                self._barrier.abort()

        threads = [threading.Thread(target=body, args=(r,)) for r in range(self.world)]
        for t in threads:
            t.start()
        for t in threads:
            t.join()
        if errors:
            # the rank that failed first breaks the barrier; the others then see only that
            root = [e for e in errors if not isinstance(e, threading.BrokenBarrierError)]
            raise (root or errors)[0]
        return results


class _LocalComm:
    def __init__(self, ring: LocalRing, rank: int):
        self.ring, self.rank, self.world = ring, rank, ring.world

    def _exchange(self, item, ev=None):
        """Posts `item` with an event of this rank's stream (recorded now unless given); returns
        every rank's post."""
        ring = self.ring
        if ev is None:
            ev = torch.cuda.Event()
            ev.record(torch.cuda.current_stream())
        ring._box[self.rank] = (item, ev)
        ring._barrier.wait()
        posts = list(ring._box)
        ring._barrier.wait()  # every rank has read the box
        return posts

    def shift_start(self, tensors: Sequence[torch.Tensor]) -> _Pending:
        # the tensors are ready now: the next rank's copy must not wait for the kernels this
        # rank enqueues before wait() (as a transfer issued before them would not)
        ev = torch.cuda.Event()
        ev.record(torch.cuda.current_stream())
        tensors = list(tensors)
        return _Pending(None, [], lambda: self._shift(tensors, ev))

    def shift(self, tensors: Sequence[torch.Tensor]) -> List[torch.Tensor]:
        return self._shift(list(tensors), None)

    def _shift(self, tensors, ev) -> List[torch.Tensor]:
        st = torch.cuda.current_stream()
        posts = self._exchange(tensors, ev)
        src, src_ev = posts[(self.rank - 1) % self.world]
        st.wait_event(src_ev)
        recv = [t.clone() for t in src]  # device-to-device copies on this rank's stream
        for t in src:
            # the previous rank may drop these tensors once it returns: the caching allocator
            # then reuses their memory only after this stream's copies have run
            t.record_stream(st)
        self.ring._barrier.wait()  # every copy is recorded before any rank returns
        return recv

    def average_(self, t: torch.Tensor) -> None:
        st = torch.cuda.current_stream()
        posts = self._exchange(t)
        total = torch.zeros_like(t)
        for other, ev in posts:
            st.wait_event(ev)
            total.add_(other)
        done = torch.cuda.Event()
        done.record(st)
        self.ring._done[self.rank] = done
        self.ring._barrier.wait()
        for ev in self.ring._done:  # every rank has read every post
            st.wait_event(ev)
        self.ring._barrier.wait()
        t.copy_(total.div_(self.world))


# ---- per-rank forward and backward ------------------------------------------------------------
@dataclasses.dataclass
class ForwardState:
    """What ``backward`` needs from ``forward`` on the same rank."""

    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    qb: ops.QuantBufs
    cfg: ops.Config
    o: torch.Tensor
    lse: torch.Tensor


def _pair_params(cfg: ops.Config, like: torch.Tensor, mode: str):
    return dataclasses.replace(cfg, causal=(mode == "diag")).params(like)


def _pair_qbufs(qb: ops.QuantBufs, k_codes, k_scale, v_codes=None, v_scale=None) -> SageQBufs:
    """The local queries' views with another chunk's keys (and values)."""
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    return SageQBufs(p(qb.q_codes), p(k_codes), p(qb.v_codes if v_codes is None else v_codes),
                     p(qb.q_scale), p(k_scale), p(qb.v_scale if v_scale is None else v_scale),
                     p(qb.q_inv_rms), p(qb.k_inv_rms), p(qb.k_mean), None, None)


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cfg: ops.Config,
            comm) -> Tuple[torch.Tensor, torch.Tensor, ForwardState]:
    """This rank's chunk of O (q's dtype) and LSE (float32) for the whole sequence's keys."""
    ops._check_inputs(q, k, v)
    if cfg.qsmooth:
        raise ValueError("Q-smoothing is not supported with context parallelism")
    prm = cfg.params(q)
    B, H, N, d = q.shape
    dev = q.device
    stream = ops._stream(dev)
    qb = ops.QuantBufs.empty(tuple(q.shape), cfg, dev)
    st = qb.c_struct()
    if cfg.ksmooth:
        ws, n = ops._workspace(prm, 0, dev)
        check("sage_quant_prologue_part", lib().sage_quant_prologue_part(
            ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
            None if ws is None else ws.data_ptr(), n, 0, stream))
        comm.average_(qb.k_mean)
    check("sage_quant_prologue_part", lib().sage_quant_prologue_part(
        ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st), None, 0,
        1, stream))

    o = torch.empty_like(q)
    o_acc = torch.empty((B, H, N, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    o_part, lse_part = torch.empty_like(o_acc), torch.empty_like(lse)
    sched = schedule(comm.rank, comm.world, cfg.causal)
    last = max(s for s, _, mode in sched if mode is not None)
    payload = [qb.k_codes, qb.k_scale, qb.v_codes, qb.v_scale]
    for s, _, mode in sched:
        # the next chunk's keys are on their way while this one is computed
        pending = comm.shift_start(payload) if s + 1 < comm.world else None
        if mode is not None:
            pp = _pair_params(cfg, q, mode)
            pq = _pair_qbufs(qb, payload[0], payload[1], payload[2], payload[3])
            first = s == 0  # the own chunk goes straight into the accumulator
            dst_o, dst_l = (o_acc, lse) if first else (o_part, lse_part)
            check("sage_attn_fwd_partial", lib().sage_attn_fwd_partial(
                ctypes.byref(pp), ctypes.byref(pq), dst_o.data_ptr(), dst_l.data_ptr(), stream))
            if not first:
                check("sage_attn_merge", lib().sage_attn_merge(
                    ctypes.byref(prm), o_acc.data_ptr(), lse.data_ptr(), o_part.data_ptr(),
                    lse_part.data_ptr(), o.data_ptr() if s == last else None, stream))
        if pending is not None:
            payload = pending.wait()
    if last == 0:  # one chunk only: the accumulator converted to the output type
        check("sage_attn_merge", lib().sage_attn_merge(
            ctypes.byref(prm), o_acc.data_ptr(), lse.data_ptr(), None, None, o.data_ptr(),
            stream))
    return o, lse, ForwardState(q, k, v, qb, cfg, o, lse)


def backward(state: ForwardState, dout: torch.Tensor,
             comm) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """This rank's chunks of dq, dk, dv (the inputs' dtype)."""
    q, k, v, qb, cfg = state.q, state.k, state.v, state.qb, state.cfg
    ops._check_inputs(dout)
    prm = cfg.params(q)
    dev = q.device
    stream = ops._stream(dev)
    ws, n = ops._workspace(prm, 2, dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = qb.c_struct()
    # stage 0: D = rowsum(dO o O), dO codes, the dQ accumulator cleared
    check("sage_attn_bwd_stage", lib().sage_attn_bwd_stage(
        0, ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
        state.o.data_ptr(), state.lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), ws.data_ptr(), n, stream))
    keys = [qb.k_codes, qb.k_scale, v]  # read-only on the way
    acc = [torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(2)]  # dK, dV
    for s, _, mode in schedule(comm.rank, comm.world, cfg.causal):
        # the next chunk's keys are on their way while this one is computed; the accumulators
        # follow once this rank has added to them, and after the last step only they travel,
        # back to their owner
        more = s + 1 < comm.world
        pending = comm.shift_start(keys) if more else None
        if mode is not None:
            pp = _pair_params(cfg, q, mode)
            pq = _pair_qbufs(qb, keys[0], keys[1])
            # the keys' owner computes first (step 0) and stores; later ranks add
            check("sage_attn_bwd_partial", lib().sage_attn_bwd_partial(
                ctypes.byref(pp), keys[2].data_ptr(), ctypes.byref(pq), state.lse.data_ptr(),
                dout.data_ptr(), acc[0].data_ptr(), acc[1].data_ptr(), int(s > 0),
                ws.data_ptr(), n, stream))
        if comm.world > 1:
            acc = comm.shift(acc)
        if pending is not None:
            keys = pending.wait()
    dk_acc, dv_acc = acc
    check("sage_attn_bwd_stage", lib().sage_attn_bwd_stage(
        2, ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
        state.o.data_ptr(), state.lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), ws.data_ptr(), n, stream))
    check("sage_kv_finalize", lib().sage_kv_finalize(
        ctypes.byref(prm), k.data_ptr(), ctypes.byref(st), dk_acc.data_ptr(), dv_acc.data_ptr(),
        dk.data_ptr(), dv.data_ptr(), stream))
    return dq, dk, dv


def forward_backward(q, k, v, dout, cfg: ops.Config, comm):
    """One training step's attention on this rank's chunk: (o, lse, dq, dk, dv)."""
    o, lse, state = forward(q, k, v, cfg, comm)
    dq, dk, dv = backward(state, dout, comm)
    return o, lse, dq, dk, dv
