"""Failure detection: every internal wait of the kernels is bounded.

With the wait limit lowered to 1 ns, any wait that is not satisfied within a
few polls gives up: the kernel raises its CTA abort flag, drains its in-flight
copies and MMAs, releases tensor memory and records ATTN_ERR_DEVICE_TIMEOUT in
the device status word -- no trap, no hang.  The test then restores the
default limit and checks that the same context still computes correct results.
"""
import pytest
import torch

import workloads
from oracle import reference as ref
from tests import parity

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # ATTN_ERR_DEVICE_TIMEOUT


def test_timeouts_are_reported_and_the_context_stays_usable():
    import attention_attn_fwd_10_b200 as attn

    w = workloads.small(B=1, H_q=4, S_q=2048, S_k=2048, D=128, causal=True, seed=12, backward=True)
    x = workloads.make_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    assert attn.device_status() == 0
    attn.set_wait_limit_ns(1)
    try:
        o, lse = attn.fwd(q, k, v, causal=True)
        st_fwd = attn.device_status()
        attn.bwd(q, k, v, o, lse, do, causal=True)
        st_bwd = attn.device_status()
        attn.bwd(q, k, v, o, lse, do, causal=True, cta_mode=2)  # the CTA-pair kernel's abort paths
        st_pairs = attn.device_status()
    finally:
        attn.set_wait_limit_ns(0)  # back to the default limit
    assert st_fwd == TIMEOUT and st_bwd == TIMEOUT and st_pairs == TIMEOUT
    # the context is intact: a normal run is correct and reports no error
    o, lse = attn.fwd(q, k, v, causal=True)
    dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=True)
    pairs = attn.bwd(q, k, v, o, lse, do, causal=True, cta_mode=2)
    assert attn.device_status() == 0
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o, o_ref)
    parity.check_lse(lse, lse_ref)
    g_ref = ref.backward(x["q"], x["k"], x["v"], x["do"], True, w.scale)
    for g, gp, gr in zip((dq, dk, dv), pairs, g_ref):
        parity.check_grad(g, gr)
        parity.check_grad(gp, gr)
