"""FwdBwdPipeline: several fwd + bwd steps from pinned host buffers with the
copies overlapped across steps give the same results as one call at a time."""
import pytest
import torch

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


def test_pipeline_matches_direct_calls():
    import attention_attn_fwd_10_b200 as attn

    ws = [workloads.small(B=1, H_q=4, H_kv=2, S_q=640, S_k=640, D=128, causal=True, seed=s, backward=True)
          for s in (1, 2, 3)]
    w = ws[0]
    pipe = attn.FwdBwdPipeline(w.B, w.S_q, w.S_k, w.H_q, w.H_kv, w.D, causal=True, scale=w.scale, depth=2)
    inputs, outs = [], []
    for wi in ws:
        x = workloads.make_inputs(wi)
        inputs.append(x)
        h = [x[n].pin_memory() for n in ("q", "k", "v", "do")]
        out = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in
               (("o", h[0]), ("dq", h[0]), ("dk", h[1]), ("dv", h[2]))}
        out["lse"] = torch.empty((w.B, w.H_q, w.S_q), dtype=torch.float32).pin_memory()
        pipe.submit(*h, out)
        outs.append(out)
    pipe.synchronize()
    assert attn.device_status() == 0
    for x, out in zip(inputs, outs):
        q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
        o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
        dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
        assert torch.equal(out["o"], o.cpu()) and torch.equal(out["lse"], lse.cpu())
        assert torch.equal(out["dk"], dk.cpu()) and torch.equal(out["dv"], dv.cpu())
        # dQ sums in fp32 in whatever order the key tiles finish: compare within the gradient bound
        parity.check_grad(parity.to_np(out["dq"]), parity.to_np(dq.cpu()).astype("float64"), "pipeline dq")
