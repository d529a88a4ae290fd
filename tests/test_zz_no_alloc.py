"""The prologue entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a host runtime that owns all device memory through its
own pool, a fixed start-up memory budget, latency-critical threads that must not risk the
synchronization an allocation can cause).  sage_quant_prologue_noalloc serves them by keeping
its K-smoothing scratch in a fixed device array inside the library.  This file checks, through
the C ABI, that two calls in a row give exactly what sage_quant_prologue gives (bit for bit,
the prologue's own tolerance) on different inputs -- so nothing stale from the previous call
leaks through the shared array -- and that a shape needing more scratch than the array holds
is refused before any launch.  It also runs the entry point from a second CUDA driver
context of the caller's own (the kind of host runtime this entry point is for), where the
library's device code and its array live at other addresses, and at the exact size limit.  It
is collected last so that a failure here cannot hide another test's result.
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
             WORKLOADS["qoutlier"].replace(B=1, H=3, N=512),
             # no smoothing: no scratch at all is needed (a null scratch pointer)
             WORKLOADS["koutlier"].replace(B=1, H=2, N=512, ksmooth=False, seed=3)]
    for w in cases:
        x = make_inputs(w)
        q, k, v = (_dev(x[n], w.dtype) for n in ("q", "k", "v"))
        _compare_to_workspace_prologue(L, q, k, v, _cfg(w))


def _compare_to_workspace_prologue(L, q, k, v, cfg):
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
    # one 128-token step past the limit (K- and Q-smoothing: 2 x 2*16*(65664/64)*128*4 bytes)
    prm = _lib.SageParams(2, 16, 65536 + 128, 128, 1, 1, 1, 1, 128, 64, 0.0, 1e-6, 1)
    qb = _lib.SageQBufs(*([256] * 11))
    rc = L.sage_quant_prologue_noalloc(ctypes.byref(prm), 256, 256, 256, ctypes.byref(qb), None)
    assert rc == _lib.SAGE_ERR_WORKSPACE


def test_noalloc_prologue_at_the_size_limit():
    """K- and Q-smoothing at B2 H16 N65536 d128 need exactly 2 x 16 MiB of column sums: the
    whole array, accepted, and still bit-identical to the workspace prologue."""
    from fwd_bwd_b200.inputs import make_inputs_fast

    L = _lib.lib()
    w = WORKLOADS["qoutlier"].replace(B=2, H=16, N=65536)
    assert 2 * w.B * w.H * (w.N // 64) * w.d * 4 == 32 << 20
    x = make_inputs_fast(w, device="cuda")
    _compare_to_workspace_prologue(L, x["q"], x["k"], x["v"], _cfg(w))
    del x
    torch.cuda.empty_cache()


def test_noalloc_prologue_in_a_second_driver_context():
    """A caller's own driver context has its own copy of the library's device code, so the
    array's address differs there; the results must not."""
    from cuda.bindings import driver as drv

    L = _lib.lib()
    w = WORKLOADS["koutlier"].replace(B=1, H=2, N=512, seed=11)
    x = make_inputs(w)
    q, k, v = (_dev(x[n], w.dtype) for n in ("q", "k", "v"))
    cfg = _cfg(w)
    ref = ops.quant_prologue(q, k, v, cfg)
    torch.cuda.synchronize()
    want = {f: getattr(ref, f).cpu().numpy() for f in FIELDS if getattr(ref, f) is not None}

    def ok(res):
        assert res[0] == drv.CUresult.CUDA_SUCCESS, res
        return res[1] if len(res) == 2 else res[1:]

    ok(drv.cuInit(0))
    primary = ok(drv.cuCtxGetCurrent())
    dev = ok(drv.cuDeviceGet(torch.cuda.current_device()))
    ctx = ok(drv.cuCtxCreate(0, dev))  # pushed: current on this thread from here on
    bufs = []
    try:
        def dalloc(nbytes):
            p = ok(drv.cuMemAlloc(max(int(nbytes), 16)))
            bufs.append(p)
            return int(p)

        ins = []
        for n in ("q", "k", "v"):
            h = np.ascontiguousarray(x[n])
            dp = dalloc(h.nbytes)
            ok((drv.cuMemcpyHtoD(dp, h.ctypes.data, h.nbytes)[0], None))
            ins.append(dp)
        ptrs = {f: dalloc(want[f].nbytes) if f in want else None for f in FIELDS}
        st = _lib.SageQBufs(*[ptrs[f] for f in FIELDS])
        prm = cfg.params(q)
        for _ in range(2):  # twice: the second call reuses the context's array
            rc = L.sage_quant_prologue_noalloc(ctypes.byref(prm), *ins, ctypes.byref(st), None)
            assert rc == _lib.SAGE_OK, _lib.status_string(rc)
            ok((drv.cuCtxSynchronize()[0], None))
            assert L.sage_last_device_status(None) == 0
            for f, a in want.items():
                got = np.empty_like(a)
                ok((drv.cuMemcpyDtoH(got.ctypes.data, ptrs[f], got.nbytes)[0], None))
                assert np.array_equal(got.view(np.uint8), a.view(np.uint8)), f
    finally:
        for p in bufs:
            drv.cuMemFree(p)
        drv.cuCtxDestroy(ctx)
        drv.cuCtxSetCurrent(primary)
    torch.cuda.synchronize()
