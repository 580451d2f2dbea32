"""One process, two devices: the forward and the backward run on device 0 and
then on device 1.  The kernels' shared-memory opt-in and the library's device
symbols are per device (per context); a library that set them up only on the
first device would fail the second device's launches.  Skipped with fewer than
two devices."""
import pytest
import torch

import workloads
from oracle import reference as ref
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two devices")
def test_forward_backward_on_two_devices_in_turn():
    import attention_attn_fwd_10_b200 as attn

    w = workloads.small(B=1, H_q=2, S_q=300, S_k=300, D=128, causal=True, seed=5, backward=True)
    x = workloads.make_inputs(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    g_ref = ref.backward(x["q"], x["k"], x["v"], x["do"], True, w.scale)
    for d in (0, 1):
        dev = torch.device("cuda", d)
        q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
        o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
        grads = attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
        torch.cuda.synchronize(dev)
        with torch.cuda.device(dev):
            assert attn.device_status() == 0
        parity.check_o(o, o_ref, f"device {d}")
        parity.check_lse(lse, lse_ref, f"device {d}")
        for name, g, gr in zip(("dq", "dk", "dv"), grads, g_ref):
            parity.check_grad(g, gr, f"device {d} {name}")
