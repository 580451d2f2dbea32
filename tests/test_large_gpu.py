"""The largest sequence lengths the tests reach: 131072 tokens in one (batch,
head).  The forward is checked on sampled rows against the oracle (each output row
depends only on its own query row); the backward on the rows of one sampled query
block per end and on identities that hold at any size."""
import numpy as np
import pytest
import torch

import workloads
from oracle import reference as ref
from tests import parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

S_LONG = 131072


def _attn():
    import attention_attn_fwd_10_b200 as attn

    return attn


def _rows(S):
    return [0, 1, 127, 128, 4095, S // 2 - 1, S // 2, S - 129, S - 128, S - 2, S - 1]


@pytest.mark.parametrize("causal", [True, False])
def test_forward_131072_tokens(causal):
    w = workloads.small(B=1, H_q=2, H_kv=1, S_q=S_LONG, S_k=S_LONG, D=128, causal=causal, seed=77)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = _attn().fwd(q, k, v, causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    o_c, lse_c = o.cpu(), lse.cpu()
    rows = _rows(S_LONG)
    for h in (0, 1):
        o_ref, lse_ref = ref.forward_rows(x["q"], x["k"], x["v"], causal, w.scale, 0, h, rows)
        parity.check_o(o_c[0, rows, h, :], o_ref, f"{w.name} h={h}")
        parity.check_lse(lse_c[0, h, rows], lse_ref, f"{w.name} h={h}")
    assert torch.isfinite(o_c.float()).all() and torch.isfinite(lse_c).all()


def test_backward_65536_tokens_invariants():
    S = 65536
    w = workloads.small(B=1, H_q=2, H_kv=1, S_q=S, S_k=S, D=128, causal=True, seed=78, backward=True)
    x = workloads.make_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _attn().fwd(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = _attn().bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    for g in (dq, dk, dv):
        assert torch.isfinite(g.float()).all()
    # sum over keys of dK is 0 (softmax rows sum to one); sum over keys of dV = sum over queries of dO
    dk64 = dk.double()
    assert dk64.sum(dim=1).abs().max() <= 3e-2 * dk64.abs().max() * S ** 0.5
    sum_dv = dv.double().sum(dim=1)
    sum_do = x["do"].double().sum(dim=1).view(1, 2, 1, 128).sum(dim=1).cuda()
    assert (sum_dv - sum_do).abs().max() <= 3e-2 * sum_do.abs().max()
    # dQ rows of the first query block see keys 0..63 only: the oracle on that prefix gives them exactly
    n = 64
    g_ref = ref.backward(x["q"][:, :n], x["k"][:, :n], x["v"][:, :n], x["do"][:, :n], True, w.scale)
    parity.check_grad(parity.to_np(dq[:, :n].cpu()), g_ref[0], "dq first block")
