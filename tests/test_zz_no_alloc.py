"""The prologue entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a host runtime that owns all device memory through its
own pool, a fixed start-up memory budget, latency-critical threads that must not risk the
synchronization an allocation can cause).  sage_quant_prologue_noalloc serves them by keeping
its K-smoothing scratch in a fixed device array inside the library.  This file checks, through
the C ABI, that two calls in a row give exactly what sage_quant_prologue gives (bit for bit,
the prologue's own tolerance) on different inputs -- so nothing stale from the previous call
leaks through the shared array -- and that a shape needing more scratch than the array holds
is refused before any launch.  It is collected last so that a failure here cannot hide
another test's result.
"""
import ctypes

import numpy as np
import pytest
import torch

from fwd_bwd_b200 import _lib, ops
from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}
FIELDS = ("q_codes", "k_codes", "v_codes", "q_scale", "k_scale", "v_scale", "q_inv_rms",
          "k_inv_rms", "k_mean", "q_mean", "k_bias")


def _dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        TORCH_DT[dtype]).cuda()


def _cfg(w):
    return ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                      k_block=w.k_block, qsmooth=w.qsmooth)


def test_noalloc_prologue_matches_workspace_prologue_twice():
    L = _lib.lib()
    cases = [WORKLOADS["koutlier"].replace(B=2, H=4, N=1024),
             WORKLOADS["llama325m"].replace(B=1, H=3, N=768, seed=7),
             WORKLOADS["qoutlier"].replace(B=1, H=3, N=512)]
    for w in cases:
        x = make_inputs(w)
        q, k, v = (_dev(x[n], w.dtype) for n in ("q", "k", "v"))
        cfg = _cfg(w)
        ref = ops.quant_prologue(q, k, v, cfg)  # existing entry point, caller workspace
        got = ops.QuantBufs.empty(tuple(q.shape), cfg, q.device)
        for f in FIELDS:  # poison the outputs: every byte must be rewritten
            t = getattr(got, f)
            if t is not None:
                t.view(torch.uint8).fill_(0xA5)
        prm = cfg.params(q)
        st = got.c_struct()
        rc = L.sage_quant_prologue_noalloc(ctypes.byref(prm), q.data_ptr(), k.data_ptr(),
                                           v.data_ptr(), ctypes.byref(st),
                                           torch.cuda.current_stream().cuda_stream)
        assert rc == _lib.SAGE_OK, _lib.status_string(rc)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        for f in FIELDS:
            a, b = getattr(got, f), getattr(ref, f)
            assert (a is None) == (b is None)
            if a is not None:
                assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f


def test_noalloc_prologue_refuses_oversized_scratch():
    L = _lib.lib()
    # B*H*(N/64)*d*4 bytes = 64 MiB of column sums > the 32 MiB array: refused, nothing runs
    prm = _lib.SageParams(64, 16, 8192, 128, 1, 1, 1, 1, 128, 64, 0.0, 1e-6)
    qb = _lib.SageQBufs(*([256] * 9))
    rc = L.sage_quant_prologue_noalloc(ctypes.byref(prm), 256, 256, 256, ctypes.byref(qb), None)
    assert rc == _lib.SAGE_ERR_WORKSPACE
