"""Forward / backward parity of the CUDA path against the oracle, on the same seeded inputs.

Gates (element by element over every output):
  * O, dQ, dK, dV: relative L2 error <= 2e-3 against the oracle's quantized recipe;
  * LSE: max |difference| <= 1e-3;
  * cosine similarity >= 0.995 against full-precision (float64) attention.
The sizes span several query/key tiles, a ragged number of 256-query CTA tiles, both head
dims, both 16-bit types, both quantization block sizes for Q, causal and not, every
combination of the QK-norm / K-smoothing flags, and the Q-smoothing variant (score bias and
dK correction) on Q-outlier inputs.
"""
import numpy as np
import pytest

from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

from gpu_helpers import cosine, gpu_run, oracle_run, rel_l2

pytestmark = pytest.mark.gpu

TOL_REL = 2e-3
TOL_LSE = 1e-3
TOL_COS = 0.995

S = WORKLOADS["sweep8192"]
L = WORKLOADS["llama325m"]
K = WORKLOADS["koutlier"]
CASES = {
    "tiny_fp16_d64_noncausal_qb64": WORKLOADS["tiny"],
    "llama_bf16_d64_causal": L.replace(B=1, H=2, N=512),
    "llama_bf16_d64_noncausal": L.replace(B=1, H=2, N=384, causal=False),
    "d128_bf16_causal_ragged": S.replace(B=1, H=2, N=640),
    "d128_fp16_causal_qb64": S.replace(B=1, H=2, N=512, dtype="fp16", q_block=64),
    "d128_bf16_noncausal": S.replace(B=2, H=1, N=384, causal=False),
    "koutlier_on_on": K.replace(B=1, H=2, N=512),
    "koutlier_norm_off": K.replace(B=1, H=2, N=512, qknorm=False),
    "koutlier_smooth_off": K.replace(B=1, H=2, N=512, ksmooth=False),
    "koutlier_off_off": K.replace(B=1, H=2, N=512, qknorm=False, ksmooth=False),
    "small_ds_regime": WORKLOADS["long16k"].replace(H=2, N=1024),
    "single_tile": S.replace(B=1, H=1, N=128),
    "qsmooth_d128_causal": WORKLOADS["qoutlier"].replace(B=1, H=2, N=512),
    "qsmooth_d64_fp16_noncausal_qb64": WORKLOADS["tiny"].replace(q_outlier=True, qsmooth=True),
    "qsmooth_d128_qb64_ksmooth_off": WORKLOADS["qoutlier"].replace(B=1, H=2, N=384, q_block=64,
                                                                  ksmooth=False),
    "qsmooth_d64_causal_norm_off": L.replace(B=1, H=2, N=512, qknorm=False, q_outlier=True,
                                             qsmooth=True),
}


@pytest.fixture(scope="module")
def results():
    return {}


def _run(case, results):
    if case not in results:
        w = CASES[case]
        x = make_inputs(w)
        results[case] = (w, gpu_run(w, x), oracle_run(w, x), oracle_run(w, x, quant=False))
    return results[case]


@pytest.mark.parametrize("case", sorted(CASES))
def test_forward_matches_oracle(case, results):
    w, g, o, _ = _run(case, results)
    BH = w.B * w.H
    assert rel_l2(g["o"].reshape(BH, w.N, w.d), o["o"]) <= TOL_REL
    assert np.abs(g["lse"].reshape(BH, w.N) - o["lse"]).max() <= TOL_LSE


@pytest.mark.parametrize("case", sorted(CASES))
def test_backward_matches_oracle(case, results):
    w, g, o, _ = _run(case, results)
    BH = w.B * w.H
    for n in ("dq", "dk", "dv"):
        err = rel_l2(g[n].reshape(BH, w.N, w.d), o[n])
        assert err <= TOL_REL, (n, err)


@pytest.mark.parametrize("case", sorted(CASES))
def test_cosine_vs_full_precision(case, results):
    """cosine >= 0.995 vs float64 attention for the recipe as specified (K-smoothing on).

    The K-smoothing ablation on K-outlier inputs (smoothing off) is where the page reports the
    recipe degrading; there the GPU must reproduce the oracle's own (lower) cosine.
    """
    w, g, o, x = _run(case, results)
    BH = w.B * w.H
    for n in ("o", "dq", "dk", "dv"):
        c = cosine(g[n].reshape(BH, w.N, w.d), x[n])
        if w.ksmooth or not w.k_outlier:
            assert c >= TOL_COS, (n, c)
        else:
            assert abs(c - cosine(o[n], x[n])) <= 1e-3, (n, c)


def test_k_smoothing_ablation_trend(results):
    """With channel outliers in K, turning K-smoothing off lowers the dQ cosine vs float64
    (K-smoothing paragraph and ablation of the SageBwd page), on the GPU as in the oracle."""
    for norm in ("on", "off"):
        on_case = "koutlier_on_on" if norm == "on" else "koutlier_norm_off"
        off_case = "koutlier_smooth_off" if norm == "on" else "koutlier_off_off"
        cs = {}
        for case in (on_case, off_case):
            w, g, _, x = _run(case, results)
            cs[case] = cosine(g["dq"].reshape(w.B * w.H, w.N, w.d), x["dq"])
        assert cs[on_case] > cs[off_case] + 0.01, cs
