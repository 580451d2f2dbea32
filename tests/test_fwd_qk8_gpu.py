"""GPU forward with 8-bit (e4m3) Q and K vs the fp64 oracle on the same e4m3 values.

The kernel computes S = Q K^T on the tensor cores' 8-bit path with fp32
accumulation; the oracle takes the e4m3 values of q and k (converted exactly to
fp64).  Everything after S is as in the bf16 forward, so are the tolerances."""
import pytest
import torch

import workloads
from oracle import reference as ref
from tests import parity

pytestmark = pytest.mark.gpu


def _run(w, **kw):
    import attention_attn_fwd_10_b200 as attn

    x = workloads.make_inputs(w)
    q8 = x["q"].to(torch.float8_e4m3fn)
    k8 = x["k"].to(torch.float8_e4m3fn)
    o, lse = attn.fwd_qk8(q8.cuda(), k8.cuda(), x["v"].cuda(), causal=w.causal, scale=w.scale, **kw)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    # the oracle sees exactly the e4m3 values (fp8 -> fp32 is exact)
    return q8.float(), k8.float(), x, o, lse


@pytest.mark.parametrize("S_q,S_k", [(1, 1), (17, 17), (128, 128), (129, 129), (300, 300), (64, 500), (500, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_small_shapes(S_q, S_k, causal):
    w = workloads.small(B=2, H_q=2, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q * 13 + S_k)
    q, k, x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(q, k, x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("H_q,H_kv,S", [(4, 1, 400), (8, 2, 40)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa(H_q, H_kv, S, causal):
    w = workloads.small(B=1, H_q=H_q, H_kv=H_kv, S_q=S, S_k=S, D=128, causal=causal, seed=5)
    q, k, x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(q, k, x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("poly", [0, 8])
def test_causal_config_sampled(poly):
    w = workloads.FWD_CAUSAL
    q, k, x, o, lse = _run(w, poly_exp_every=poly)
    o_c, lse_c = o.cpu(), lse.cpu()
    rows = [0, 1, 127, 128, 255, 4095, 8190, 8191]
    for (b, h) in [(0, 0), (1, 15)]:
        o_ref, lse_ref = ref.forward_rows(q, k, x["v"], True, w.scale, b, h, rows)
        parity.check_o(o_c[b, rows, h, :], o_ref, f"{w.name} b={b} h={h}")
        parity.check_lse(lse_c[b, h, rows], lse_ref, f"{w.name} b={b} h={h}")
    assert torch.isfinite(o_c.float()).all() and torch.isfinite(lse_c).all()


@pytest.mark.parametrize("S_q,S_k,H_q,H_kv", [(1, 4096, 32, 8), (16, 3000, 8, 2), (100, 1000, 4, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_split_kv_decode_shapes(S_q, S_k, H_q, H_kv, causal):
    import attention_attn_fwd_10_b200 as attn

    w = workloads.small(B=2, H_q=H_q, H_kv=H_kv, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q + S_k)
    x = workloads.make_inputs(w)
    q8, k8 = x["q"].to(torch.float8_e4m3fn), x["k"].to(torch.float8_e4m3fn)
    o, lse = attn.fwd_split(q8.cuda(), k8.cuda(), x["v"].cuda(), causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    o_ref, lse_ref = ref.forward(q8.float(), k8.float(), x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


def test_last_wave_in_halves():
    # 152 non-causal units on 148 SMs: the last 4 run in the second launch as the dual
    # stream (with 8-bit Q/K its V ring keeps two stages); every row of the heads that
    # hold them and of the first against the oracle
    w = workloads.small(B=1, H_q=38, S_q=1024, S_k=1024, D=128, causal=False, seed=11)
    q, k, x, o, lse = _run(w)
    o_c, lse_c = o.cpu(), lse.cpu()
    rows = list(range(w.S_q))
    for h in (0, 34, 35, 36, 37):
        o_ref, lse_ref = ref.forward_rows(q, k, x["v"], False, w.scale, 0, h, rows)
        parity.check_o(o_c[0, rows, h, :], o_ref, f"{w.name} h={h}")
        parity.check_lse(lse_c[0, h, rows], lse_ref, f"{w.name} h={h}")
