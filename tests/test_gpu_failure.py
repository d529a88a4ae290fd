"""The kernels' failure path, driven on purpose without a GPU fault.

Every barrier wait in the kernels is bounded; when one runs out, the kernel records
SAGE_ERR_TIMEOUT in the device status word, frees its tensor memory and returns, and kernels
launched afterwards return at once until the host has read (and cleared) the word.  Here a debug
kernel waits on a barrier that nothing arrives on, with a 100 microsecond limit, so the limit
really runs out.  The tests check that the host sees SAGE_ERR_TIMEOUT, that an attention kernel
launched while the word is set leaves its outputs untouched, and that once the word is cleared
the same context runs prologue, forward and backward to oracle parity.
"""
import numpy as np
import pytest
import torch

from fwd_bwd_b200 import _lib, ops
from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

from gpu_helpers import cfg_of, gpu_run, oracle_run, rel_l2, to_device

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout():
    assert ops.device_status() == 0
    ops.wait_timeout_debug(100)
    assert ops.device_status() == _lib.SAGE_ERR_TIMEOUT
    # reading the status cleared it
    assert ops.device_status() == 0


def test_kernels_drain_after_a_timeout_then_recover():
    w = WORKLOADS["tiny"]
    x = make_inputs(w)
    q, k, v = (to_device(x[n], w.dtype) for n in ("q", "k", "v"))
    cfg = cfg_of(w)
    qb = ops.quant_prologue(q, k, v, cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    o = torch.full_like(q, 7.0)
    lse = torch.full(q.shape[:3], 7.0, dtype=torch.float32, device=q.device)
    ops.wait_timeout_debug(100)
    ops.attn_fwd(qb, q, cfg, o=o, lse=lse)  # sees the recorded failure: returns at once
    torch.cuda.synchronize()
    assert ops.device_status() == _lib.SAGE_ERR_TIMEOUT
    assert torch.all(o == 7.0) and torch.all(lse == 7.0)
    # cleared: the same context computes the whole path correctly
    g = gpu_run(w, x)
    ref = oracle_run(w, x)
    BH = w.B * w.H
    for n in ("o", "dq", "dk", "dv"):
        assert rel_l2(g[n].reshape(BH, w.N, w.d), ref[n]) <= 2e-3, n
