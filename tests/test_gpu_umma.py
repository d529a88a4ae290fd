"""The tensor-core path in isolation: tcgen05 MMAs from TMA-staged shared memory, exact.

Every operand form the attention kernels use (INT8 K-major and MN-major A and B, 64- and
128-byte swizzles, FP16/BF16 K-major with two swizzle atoms along K) against integer brute
force, and the forward kernel's score product against the oracle's exact integer Qc Kc^T.
"""
import numpy as np
import pytest
import torch

import oracle.sage_oracle as O
from fwd_bwd_b200 import ops
from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

from gpu_helpers import cfg_of, gpu_run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("K", [64, 128])
def test_umma_int8_exact(a_mn, b_mn, N, K):
    g = np.random.default_rng(a_mn * 8 + b_mn * 4 + N + K)
    A = g.integers(-127, 128, (128, K)).astype(np.int8)
    B = g.integers(-127, 128, (K, N)).astype(np.int8)
    ref = A.astype(np.int64) @ B.astype(np.int64)
    a_st = A.T.copy() if a_mn else A
    b_st = B if b_mn else B.T.copy()
    c = ops.umma_gemm_debug(0, torch.from_numpy(a_st).cuda(), torch.from_numpy(b_st).cuda(),
                            bool(a_mn), bool(b_mn), N, K)
    np.testing.assert_array_equal(c.cpu().numpy(), ref)


@pytest.mark.parametrize("kind,dt", [(1, torch.float16), (2, torch.bfloat16)])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("K", [64, 128])
def test_umma_f16(kind, dt, N, K):
    g = torch.Generator().manual_seed(N + K + kind)
    A = torch.randn(128, K, generator=g).to(dt)
    B = torch.randn(N, K, generator=g).to(dt)
    ref = A.double() @ B.double().T
    c = ops.umma_gemm_debug(kind, A.cuda(), B.cuda(), False, False, N, K).cpu().double()
    assert torch.allclose(c, ref, rtol=1e-5, atol=1e-4 * float(ref.abs().max()))


@pytest.mark.parametrize("name,tiles", [("llama325m", [0, 3]), ("sweep8192", [0, 4])])
def test_forward_scores_int32_exact(name, tiles):
    w = WORKLOADS[name].replace(B=1, H=2, N=640)
    x = make_inputs(w)
    res = gpu_run(w, x, backward=False)
    qb, like = res["_qb"], res["_dev"][0]
    ref = O.prologue(*(x[n + "_f32"].reshape(-1, w.N, w.d) for n in ("q", "k", "v")),
                     q_block=w.q_block, k_block=w.k_block, qknorm=w.qknorm, ksmooth=w.ksmooth)
    for bh in range(w.B * w.H):
        qc = ref["q_codes"][bh].astype(np.float64)
        kc = ref["k_codes"][bh].astype(np.float64)
        for t in tiles:
            s = ops.qk_int32_debug(qb, like, cfg_of(w), bh, t).cpu().numpy()
            # the oracle's score product (exact integers) on the same codes
            A = O._scores(qc[t * 128:(t + 1) * 128], np.ones(128), kc, np.ones(w.N), 1.0,
                          False, 0)
            np.testing.assert_array_equal(s, A.astype(np.int64))
