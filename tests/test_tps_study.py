"""The tokens-per-step study's full-precision reference against the oracle's X mode, and a small
GPU run of the study itself."""
import numpy as np
import pytest
import torch

import oracle.sage_oracle as O
from fwd_bwd_b200 import ops
from fwd_bwd_b200.inputs import WORKLOADS, make_study_inputs
from fwd_bwd_b200.tps_study import full_precision_grads, measure


@pytest.mark.parametrize("causal,qknorm,ksmooth", [(True, True, True), (False, True, False),
                                                   (True, False, True)])
def test_full_precision_reference_matches_oracle_xmode(causal, qknorm, ksmooth):
    w = WORKLOADS["tiny"].replace(B=2, H=2, N=128, d=64, causal=causal, qknorm=qknorm,
                                  ksmooth=ksmooth, dtype="bf16")
    x = make_study_inputs(w, seed=3)
    cfg = ops.Config(causal=causal, qknorm=qknorm, ksmooth=ksmooth, q_block=64, k_block=64)
    o, dq, dk, dv = full_precision_grads(x["q"], x["k"], x["v"], x["do"], cfg)
    f = {n: x[n].float().numpy().reshape(-1, w.N, w.d) for n in ("q", "k", "v", "do")}
    ref = O.sage_attention(f["q"], f["k"], f["v"], f["do"], causal=causal, qknorm=qknorm,
                           ksmooth=ksmooth, q_block=64, k_block=64, dtype="bf16", quant=False,
                           round_outputs=False)
    for a, name in ((o, "o"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        a = a.numpy().reshape(ref[name].shape)
        err = np.linalg.norm(a - ref[name]) / np.linalg.norm(ref[name])
        assert err < 1e-12, (name, err)


def test_study_inputs_share_structure_across_seeds():
    w = WORKLOADS["tiny"].replace(B=1, H=1, N=4096, d=64, dtype="bf16")
    a, b = make_study_inputs(w, 1), make_study_inputs(w, 2)
    assert not torch.equal(a["k"], b["k"])
    ma, mb = a["k"].float().mean(dim=(0, 1, 2)), b["k"].float().mean(dim=(0, 1, 2))
    assert (ma - mb).abs().max() < 0.2 and ma.abs().max() > 10.0  # shared outlier channels


@pytest.mark.gpu
def test_study_runs_on_gpu():
    w = WORKLOADS["sweep8192"].replace(N=256, H=2)
    res = measure(w, [1, 2], [0, 1, 2])
    assert len(res["rows"]) == 2
    for row in res["rows"]:
        for t in ("dq", "dk"):
            r = row[t]
            assert np.isfinite(r["bias"]) and r["snoise"] > 0 and r["qnoise"] >= 0
            # the INT8 recipe stays close to full precision in the batch average
            assert r["bias"] < 0.1 * r["signal"] + 3 * r["bias_stderr"] + 1e-12
