"""The host-buffer entry point sage_fwd_bwd_host (batch slices streamed through copy / compute /
copy streams inside the C library) gives the same results as the device-resident path: O, dK,
dV bit for bit (each head's arithmetic is independent of how the batch is sliced), dQ up to the
order of its float32 reductions.  Two calls in a row reuse one workspace and stream set."""
import numpy as np
import pytest
import torch

from fwd_bwd_b200 import ops
from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

from gpu_helpers import TORCH_DT, cfg_of

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,chunks", [("llama325m", 3), ("sweep8192", 2), ("qoutlier", 2)])
def test_host_pipeline_matches_device_path(name, chunks):
    w = WORKLOADS[name].replace(B=5, H=2, N=512)
    x = make_inputs(w)
    dt = TORCH_DT[w.dtype]
    host = [torch.from_numpy(x[n].view(np.int16)).view(dt).pin_memory()
            for n in ("q", "k", "v", "do")]
    cfg = cfg_of(w)
    pipe = ops.HostPipeline(host[0], cfg, chunks)
    for _ in range(2):
        o_h, dq_h, dk_h, dv_h = ops.fwd_bwd_host(*host, cfg, pipeline=pipe)
    q, k, v, do = (t.cuda() for t in host)
    qb = ops.quant_prologue(q, k, v, cfg)
    o, lse = ops.attn_fwd(qb, q, cfg)
    dq, dk, dv = ops.attn_bwd(q, k, v, qb, o, lse, do, cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for a, b in ((o_h, o), (dk_h, dk), (dv_h, dv)):
        assert torch.equal(a, b.cpu())
    diff = (dq_h.float() - dq.cpu().float()).norm() / dq.cpu().float().norm()
    assert diff < 1e-2 * 2 ** -7  # at most bf16 rounding flips from atomic order
