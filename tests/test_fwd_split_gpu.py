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


# Decode shapes with at most 8 query rows per kv group (G query heads x S_q queries):
# the packed tile's real rows sit in its first warp and the other softmax warps skip
# their work, and few output rows take the row-parallel merge.  Ragged key counts
# around the 128-key blocks and ranges, causal rows that end at different keys, every
# range count, both head dims.
@pytest.mark.parametrize("H_q,H_kv,S_q", [(1, 1, 1), (2, 1, 1), (8, 2, 1), (4, 1, 2), (8, 1, 1), (5, 1, 1),
                                          (3, 3, 2), (1, 1, 8)])
@pytest.mark.parametrize("S_k", [1, 31, 33, 129, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_decode_few_rows(H_q, H_kv, S_q, S_k, causal):
    w = workloads.small(B=2, H_q=H_q, H_kv=H_kv, S_q=S_q, S_k=S_k, D=128, causal=causal,
                        seed=H_q * 7 + S_q * 3 + S_k)
    for n in (0, 1, 3):
        x, o, lse = _run(w, n)
        o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
        parity.check_o(o, o_ref, f"{w.name} splits={n}")
        parity.check_lse(lse, lse_ref, f"{w.name} splits={n}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("num_splits", [0, 1, 5, 128])
def test_decode_few_rows_head_dim_64(causal, num_splits):
    w = workloads.small(B=3, H_q=8, H_kv=2, S_q=2, S_k=2500, D=64, causal=causal, seed=23)
    x, o, lse = _run(w, num_splits)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


def test_decode_few_rows_that_see_no_key():
    # causal with S_q > S_k and one head: rows 0..S_q-S_k-1 see no key in any range
    w = workloads.small(B=1, H_q=1, S_q=8, S_k=3, D=128, causal=True, seed=29)
    x, o, lse = _run(w, 2)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)
    assert torch.all(lse[:, :, :5].cpu() == -np.inf)
    assert torch.all(o[:, :5].float().cpu() == 0)


def test_decode_few_rows_deterministic():
    w = workloads.small(B=2, H_q=32, H_kv=8, S_q=1, S_k=8192, D=128, causal=True, seed=31)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].to("cuda") for n in ("q", "k", "v"))
    o1, l1 = _attn().fwd_split(q, k, v, causal=True, scale=w.scale)
    o2, l2 = _attn().fwd_split(q, k, v, causal=True, scale=w.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o1, o_ref, w.name)
    parity.check_lse(l1, lse_ref, w.name)
