"""GPU split-KV forward (attn_fwd_split) vs the fp64 oracle, through the C ABI.

The split forward computes the same O and lse as the plain forward: each key
range yields (O_s, lse_s) and the ranges are merged by the log-sum-exp identity,
so the oracle is the ordinary fp64 forward and the tolerances are the forward's."""
import numpy as np
import pytest
import torch

import workloads
from oracle import reference as ref
from tests import parity

pytestmark = pytest.mark.gpu


def _attn():
    import attention_attn_fwd_10_b200 as attn

    return attn


def _run(w, num_splits):
    x = workloads.make_inputs(w)
    q, k, v = (x[n].to("cuda") for n in ("q", "k", "v"))
    o, lse = _attn().fwd_split(q, k, v, causal=w.causal, scale=w.scale, num_splits=num_splits)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    return x, o, lse


@pytest.mark.parametrize("S_q,S_k", [(1, 129), (1, 4096), (3, 1000), (64, 2048), (300, 1500), (1, 1)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("num_splits", [0, 2, 7, 128])
def test_decode_shapes(S_q, S_k, causal, num_splits):
    w = workloads.small(B=2, H_q=4, H_kv=1, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q * 31 + S_k)
    x, o, lse = _run(w, num_splits)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_head_dim_64(causal):
    w = workloads.small(B=1, H_q=8, H_kv=2, S_q=5, S_k=3000, D=64, causal=causal, seed=5)
    x, o, lse = _run(w, 0)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


def test_rows_that_see_no_key():
    # causal, S_q > S_k: the first S_q - S_k rows see no key (O = 0, lse = -inf) in every range
    w = workloads.small(B=1, H_q=2, S_q=700, S_k=300, D=128, causal=True, seed=9)
    x, o, lse = _run(w, 3)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)
    assert torch.all(lse[:, :, : 700 - 300].cpu() == -np.inf)
    assert torch.all(o[:, : 700 - 300].float().cpu() == 0)


def test_one_split_is_the_plain_forward():
    w = workloads.small(B=1, H_q=4, S_q=200, S_k=900, D=128, causal=True, seed=13)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].to("cuda") for n in ("q", "k", "v"))
    o1, l1 = _attn().fwd_split(q, k, v, causal=True, scale=w.scale, num_splits=1)
    o2, l2 = _attn().fwd(q, k, v, causal=True, scale=w.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_decode_sampled_heads():
    # one query row per head against 32768 keys (a decoding step with a long context, GQA 4:1)
    w = workloads.small(B=1, H_q=32, H_kv=8, S_q=1, S_k=32768, D=128, causal=True, seed=17)
    x, o, lse = _run(w, 0)
    assert _attn().fwd_split_count(1, 32, 8, 1, 32768, True) > 1
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


def test_deterministic():
    w = workloads.small(B=1, H_q=4, H_kv=2, S_q=2, S_k=5000, D=128, causal=False, seed=19)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].to("cuda") for n in ("q", "k", "v"))
    o1, l1 = _attn().fwd_split(q, k, v, scale=w.scale, num_splits=9)
    o2, l2 = _attn().fwd_split(q, k, v, scale=w.scale, num_splits=9)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
