"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol the
header declares, sizes workspaces, names status codes and rejects bad arguments before any
CUDA call."""
import ctypes
import os
import re

import pytest

from fwd_bwd_b200 import _lib
from fwd_bwd_b200._lib import SageParams, SageQBufs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import fwd_bwd_b200.build as b

    b.build()
    return _lib.lib()


def _declared(header="sage.h"):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) == 19
    fp4 = _declared("sage_nvfp4.h")
    assert fp4 == ["sage_fp4_attn_bwd", "sage_fp4_attn_bwd_stage", "sage_fp4_attn_fwd",
                   "sage_fp4_quant_prologue", "sage_fp4_workspace_bytes"]
    for n in names + fp4:
        assert hasattr(L, n), n


def test_host_pipeline_workspace_and_argument_checks(L):
    p = _params()  # B2 H4 N1024 d128 bf16, ksmooth
    n1 = L.sage_fwd_bwd_host_workspace_bytes(ctypes.byref(p), 1)
    n2 = L.sage_fwd_bwd_host_workspace_bytes(ctypes.byref(p), 2)
    assert n1 > n2 > 0  # two slots of the largest slice: B/1 vs B/2 batch entries
    assert L.sage_fwd_bwd_host_workspace_bytes(ctypes.byref(p), 99) == n2  # capped at B
    assert L.sage_fwd_bwd_host_workspace_bytes(ctypes.byref(p), 0) == 0
    # 16-bit inputs and outputs (8 tensors) dominate each slot
    e = 1 * 4 * 1024 * 128 * 2
    assert n2 >= 2 * 8 * e
    fake = 1 << 20  # never dereferenced: every call below fails its host-side checks
    ten = [fake] * 8
    f = L.sage_fwd_bwd_host
    assert f(ctypes.byref(p), *ten, 0, fake, n2, None, None, None) == _lib.SAGE_ERR_INVALID_ARG
    assert f(ctypes.byref(p), None, *ten[1:], 2, fake, n2, None, None, None) == \
        _lib.SAGE_ERR_INVALID_ARG
    assert f(ctypes.byref(p), *ten, 2, fake, n2 - 1, None, None, None) == _lib.SAGE_ERR_WORKSPACE
    assert f(ctypes.byref(p), *ten, 2, None, n2, None, None, None) == _lib.SAGE_ERR_WORKSPACE
    assert f(ctypes.byref(p), *ten, 2, fake + 8, n2, None, None, None) == _lib.SAGE_ERR_ALIGNMENT
    assert f(ctypes.byref(_params(d=96)), *ten, 2, fake, n2, None, None, None) == \
        _lib.SAGE_ERR_UNSUPPORTED


def test_wait_timeout_argument_checks(L):
    for bad in (0, -5, 1000001):
        assert L.sage_debug_wait_timeout(bad, None) == _lib.SAGE_ERR_INVALID_ARG


def test_mma_peak_argument_checks(L):
    fake = 1 << 20  # never dereferenced: every call below fails its host-side checks
    bad = [(3, 148, 10, fake, 49152), (-1, 148, 10, fake, 49152), (0, 0, 10, fake, 49152),
           (0, 148, 0, fake, 49152), (0, 148, (1 << 26) + 1, fake, 49152),
           (0, 148, 10, None, 49152), (1, 148, 10, fake, 49151)]
    for args in bad:
        assert L.sage_mma_peak(*args, None) == _lib.SAGE_ERR_INVALID_ARG, args
    assert L.sage_mma_peak(2, 148, 10, fake + 4, 49152, None) == _lib.SAGE_ERR_ALIGNMENT


def test_fp4_workspace_and_argument_checks(L):
    from fwd_bwd_b200._lib import SageFp4Bufs

    BH, N, d = 8, 1024, 128
    p = _params()
    assert L.sage_fp4_workspace_bytes(ctypes.byref(p), 0) == 3 * BH * (N // 64) * d * 4 + 256
    assert L.sage_fp4_workspace_bytes(ctypes.byref(p), 1) == 0
    assert L.sage_fp4_workspace_bytes(ctypes.byref(_params(ksmooth=0)), 0) == 256
    assert L.sage_fp4_workspace_bytes(ctypes.byref(_params(qsmooth=1)), 0) == 0
    fake = 1 << 20  # never dereferenced: every call below fails its host-side checks
    fb = SageFp4Bufs(*([fake] * 9 + [None] * 4))
    ws = 3 * BH * (N // 64) * d * 4 + 256
    assert L.sage_fp4_quant_prologue(ctypes.byref(_params(qsmooth=1)), fake, fake,
                                     ctypes.byref(fb), fake, ws, None) == _lib.SAGE_ERR_UNSUPPORTED
    assert L.sage_fp4_quant_prologue(ctypes.byref(_params(d=96)), fake, fake, ctypes.byref(fb),
                                     fake, ws, None) == _lib.SAGE_ERR_UNSUPPORTED
    assert L.sage_fp4_quant_prologue(ctypes.byref(p), None, fake, ctypes.byref(fb), fake, ws,
                                     None) == _lib.SAGE_ERR_INVALID_ARG
    assert L.sage_fp4_quant_prologue(ctypes.byref(p), fake, fake, ctypes.byref(fb), fake, ws - 1,
                                     None) == _lib.SAGE_ERR_WORKSPACE
    assert L.sage_fp4_quant_prologue(ctypes.byref(p), fake + 8, fake, ctypes.byref(fb), fake, ws,
                                     None) == _lib.SAGE_ERR_ALIGNMENT
    # ragged and empty shapes are refused before any launch
    for bad, want in ((dict(N=1000), _lib.SAGE_ERR_UNSUPPORTED),
                      (dict(N=0), _lib.SAGE_ERR_INVALID_ARG),
                      (dict(B=0), _lib.SAGE_ERR_INVALID_ARG),
                      (dict(d=32), _lib.SAGE_ERR_UNSUPPORTED)):
        pb = _params(**bad)
        assert L.sage_fp4_quant_prologue(ctypes.byref(pb), fake, fake, ctypes.byref(fb), fake,
                                         ws, None) == want, bad
        assert L.sage_fp4_attn_fwd(ctypes.byref(pb), ctypes.byref(fb), fake, fake, fake,
                                   None) == want, bad
        assert L.sage_fp4_workspace_bytes(ctypes.byref(pb), 0) == 0
    nosf = SageFp4Bufs(fake, fake, None, fake, fake, fake, fake, fake, fake)
    half_seq = SageFp4Bufs(*([fake] * 9 + [fake, None, None, None]))  # codes without scales
    assert L.sage_fp4_quant_prologue(ctypes.byref(p), fake, fake, ctypes.byref(half_seq), fake,
                                     ws, None) == _lib.SAGE_ERR_INVALID_ARG
    assert L.sage_fp4_attn_fwd(ctypes.byref(p), ctypes.byref(nosf), fake, fake, fake,
                               None) == _lib.SAGE_ERR_INVALID_ARG
    assert L.sage_fp4_attn_fwd(ctypes.byref(p), ctypes.byref(fb), fake, fake + 4, fake,
                               None) == _lib.SAGE_ERR_ALIGNMENT


def test_fp4_backward_workspace_and_argument_checks(L):
    from fwd_bwd_b200._lib import SageFp4Bufs

    BH, N, d = 8, 1024, 128
    p = _params()
    wsb = L.sage_fp4_workspace_bytes(ctypes.byref(p), 2)
    assert wsb == BH * N * 4 + BH * N * d * 4  # D, then the float32 dQ accumulator
    assert L.sage_fp4_workspace_bytes(ctypes.byref(_params(qsmooth=1)), 2) == 0
    fake = 1 << 20  # never dereferenced: every call below fails its host-side checks
    full = SageFp4Bufs(*([fake] * 13))
    noseq = SageFp4Bufs(*([fake] * 9 + [None] * 4))
    noinv = SageFp4Bufs(*([fake] * 6 + [None, None] + [fake] * 5))
    f = L.sage_fp4_attn_bwd

    def call(prm=p, fb=full, ptrs=None, ws=wsb, wsp=fake):
        t = ptrs if ptrs is not None else [fake] * 3
        return f(ctypes.byref(prm), *t, ctypes.byref(fb), fake, fake, fake, fake, fake, fake,
                 wsp, ws, None)

    assert call(fb=noseq) == _lib.SAGE_ERR_INVALID_ARG  # the sequence views are operands
    assert call(fb=noinv) == _lib.SAGE_ERR_INVALID_ARG  # qknorm needs the inverse RMS
    assert call(ptrs=[None, fake, fake]) == _lib.SAGE_ERR_INVALID_ARG
    assert call(ptrs=[fake, fake + 8, fake]) == _lib.SAGE_ERR_ALIGNMENT
    assert call(ws=wsb - 1) == _lib.SAGE_ERR_WORKSPACE
    assert call(wsp=None) == _lib.SAGE_ERR_WORKSPACE
    assert call(prm=_params(qsmooth=1)) == _lib.SAGE_ERR_UNSUPPORTED
    assert call(prm=_params(d=96)) == _lib.SAGE_ERR_UNSUPPORTED
    assert call(prm=_params(N=1000)) == _lib.SAGE_ERR_UNSUPPORTED
    g = L.sage_fp4_attn_bwd_stage
    for stage in (-1, 3):
        assert g(stage, ctypes.byref(p), fake, fake, fake, ctypes.byref(full), fake, fake, fake,
                 fake, fake, fake, fake, wsb, None) == _lib.SAGE_ERR_INVALID_ARG
    assert g(1, ctypes.byref(p), fake, fake, fake, ctypes.byref(noseq), fake, fake, fake, fake,
             fake, fake, fake, wsb, None) == _lib.SAGE_ERR_INVALID_ARG


def _params(**kw):
    p = dict(B=2, H=4, N=1024, d=128, dtype=1, causal=1, qknorm=1, ksmooth=1, q_block=128,
             k_block=64, softmax_scale=0.0, rms_eps=1e-6)
    p.update(kw)
    return SageParams(**p)


def test_workspace_sizes(L):
    p = _params()
    BH, N, d = 8, 1024, 128
    assert L.sage_workspace_bytes(ctypes.byref(p), 0) == BH * (N // 64) * d * 4
    assert L.sage_workspace_bytes(ctypes.byref(p), 1) == 0
    bwd = L.sage_workspace_bytes(ctypes.byref(p), 2)
    assert bwd >= BH * N * (4 + d + 4 * d)
    p0 = _params(ksmooth=0)
    assert L.sage_workspace_bytes(ctypes.byref(p0), 0) == 0
    assert L.sage_workspace_bytes(ctypes.byref(_params(d=96)), 2) == 0
    # Q-smoothing adds Q's column-sum partials beside K's
    pq = _params(qsmooth=1)
    assert L.sage_workspace_bytes(ctypes.byref(pq), 0) == 2 * BH * (N // 64) * d * 4
    pq0 = _params(ksmooth=0, qsmooth=1)
    assert L.sage_workspace_bytes(ctypes.byref(pq0), 0) == BH * (N // 64) * d * 4


def test_status_strings(L):
    for code, name in ((0, "SAGE_OK"), (-1, "SAGE_ERR_INVALID_ARG"), (-6, "SAGE_ERR_TIMEOUT")):
        assert _lib.status_string(code) == name


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), _lib.SAGE_ERR_UNSUPPORTED),
    (dict(N=200), _lib.SAGE_ERR_UNSUPPORTED),
    (dict(k_block=128), _lib.SAGE_ERR_UNSUPPORTED),
    (dict(q_block=32), _lib.SAGE_ERR_UNSUPPORTED),
    (dict(B=0), _lib.SAGE_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.SAGE_ERR_INVALID_ARG),
    (dict(rms_eps=-1.0), _lib.SAGE_ERR_INVALID_ARG),
])
def test_bad_params_rejected_without_launch(L, kw, code):
    p = _params(**kw)
    qb = SageQBufs(*([16] * 9))
    assert L.sage_quant_prologue(ctypes.byref(p), 16, 16, 16, ctypes.byref(qb), 16, 1 << 40,
                                 None) == code
    assert L.sage_attn_fwd(ctypes.byref(p), ctypes.byref(qb), 16, 16, None, 0, None) == code


def test_null_and_misaligned_pointers_rejected(L):
    p = _params()
    qb = SageQBufs(*([16] * 9))
    assert L.sage_quant_prologue(ctypes.byref(p), None, 16, 16, ctypes.byref(qb), 16, 1 << 40,
                                 None) == _lib.SAGE_ERR_INVALID_ARG
    assert L.sage_quant_prologue(ctypes.byref(p), 18, 16, 16, ctypes.byref(qb), 16, 1 << 40,
                                 None) == _lib.SAGE_ERR_ALIGNMENT
    bad = SageQBufs(*([16] * 6 + [None, 16, 16]))  # qknorm needs q_inv_rms
    assert L.sage_attn_fwd(ctypes.byref(p), ctypes.byref(bad), 16, 16, None, 0,
                           None) == _lib.SAGE_ERR_INVALID_ARG
    assert L.sage_quant_prologue(ctypes.byref(p), 16, 16, 16, ctypes.byref(qb), 16, 100,
                                 None) == _lib.SAGE_ERR_WORKSPACE
    assert L.sage_attn_bwd(ctypes.byref(p), 16, 16, 16, ctypes.byref(qb), 16, 16, 16, 16, 16,
                           16, 16, 1, None) == _lib.SAGE_ERR_WORKSPACE


def test_qsmooth_arguments_checked(L):
    qb = SageQBufs(*([16] * 11))
    assert L.sage_attn_fwd(ctypes.byref(_params(qsmooth=2)), ctypes.byref(qb), 16, 16, None, 0,
                           None) == _lib.SAGE_ERR_INVALID_ARG
    p = _params(qsmooth=1)
    no_bias = SageQBufs(*([16] * 10 + [None]))  # Q-smoothing needs k_bias
    assert L.sage_attn_fwd(ctypes.byref(p), ctypes.byref(no_bias), 16, 16, None, 0,
                           None) == _lib.SAGE_ERR_INVALID_ARG
    no_mean = SageQBufs(*([16] * 9 + [None, 16]))  # and q_mean
    assert L.sage_quant_prologue(ctypes.byref(p), 16, 16, 16, ctypes.byref(no_mean), 16,
                                 1 << 40, None) == _lib.SAGE_ERR_INVALID_ARG
    odd = SageQBufs(*([16] * 10 + [20]))  # misaligned k_bias
    assert L.sage_attn_fwd(ctypes.byref(p), ctypes.byref(odd), 16, 16, None, 0,
                           None) == _lib.SAGE_ERR_ALIGNMENT


def test_debug_entry_validation(L):
    assert L.sage_debug_umma_gemm(0, 0, 0, 96, 64, 16, 16, 16, None) == \
        _lib.SAGE_ERR_UNSUPPORTED
    assert L.sage_debug_umma_gemm(1, 1, 0, 64, 64, 16, 16, 16, None) == \
        _lib.SAGE_ERR_UNSUPPORTED
    assert L.sage_debug_umma_gemm(0, 0, 0, 64, 64, None, 16, 16, None) == \
        _lib.SAGE_ERR_INVALID_ARG


def test_context_parallel_entry_argument_checks(L):
    """The context-parallel entry points refuse bad arguments before any launch."""
    from ctypes import byref
    E = _lib
    p, pq = _params(), _params(qsmooth=1)
    qb = SageQBufs(*([16] * 9))
    f = 1 << 20  # never dereferenced
    part = L.sage_quant_prologue_part
    assert part(byref(p), f, f, f, byref(qb), f, 1 << 40, 2, None) == E.SAGE_ERR_INVALID_ARG
    assert part(byref(pq), f, f, f, byref(qb), f, 1 << 40, 0, None) == E.SAGE_ERR_UNSUPPORTED
    assert part(byref(p), None, f, f, byref(qb), f, 1 << 40, 1, None) == E.SAGE_ERR_INVALID_ARG
    assert part(byref(p), f, f, f + 2, byref(qb), f, 1 << 40, 1, None) == E.SAGE_ERR_ALIGNMENT
    assert part(byref(p), f, f, f, byref(qb), f, 100, 0, None) == E.SAGE_ERR_WORKSPACE
    fwd = L.sage_attn_fwd_partial
    assert fwd(byref(pq), byref(qb), f, f, None) == E.SAGE_ERR_UNSUPPORTED
    assert fwd(byref(p), byref(qb), None, f, None) == E.SAGE_ERR_INVALID_ARG
    assert fwd(byref(p), byref(qb), f + 4, f, None) == E.SAGE_ERR_ALIGNMENT
    merge = L.sage_attn_merge
    assert merge(byref(p), None, f, f, f, None, None) == E.SAGE_ERR_INVALID_ARG
    assert merge(byref(p), f, f, None, f, None, None) == E.SAGE_ERR_INVALID_ARG  # o without lse
    assert merge(byref(p), f, f, f, f, f + 8, None) == E.SAGE_ERR_ALIGNMENT
    bwd = L.sage_attn_bwd_partial
    assert bwd(byref(p), f, byref(qb), f, f, f, f, 2, f, 1 << 40, None) == E.SAGE_ERR_INVALID_ARG
    assert bwd(byref(pq), f, byref(qb), f, f, f, f, 0, f, 1 << 40, None) == \
        E.SAGE_ERR_UNSUPPORTED
    assert bwd(byref(p), f, byref(qb), f, f, None, f, 1, f, 1 << 40, None) == \
        E.SAGE_ERR_INVALID_ARG
    assert bwd(byref(p), f, byref(qb), f, f, f, f, 1, f, 100, None) == E.SAGE_ERR_WORKSPACE
    fin = L.sage_kv_finalize
    assert fin(byref(p), None, byref(qb), f, f, f, f, None) == E.SAGE_ERR_INVALID_ARG  # qknorm
    assert fin(byref(p), f, byref(qb), f, f, None, f, None) == E.SAGE_ERR_INVALID_ARG
    assert fin(byref(p), f, byref(qb), f, f, f + 2, f, None) == E.SAGE_ERR_ALIGNMENT
