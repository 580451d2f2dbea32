"""GPU forward with 8-bit (e4m3) Q, K and V (attn_fwd_qkv8) vs the fp64 oracle.

The caller's quantisation of q, k and v is the input: the oracle takes exactly
those e4m3 values (fp8 -> fp32 is exact).  Inside, the kernel rounds the softmax
weights p = 2^(c s - m) <= 2^tau to e4m3 before O += P V, while the row sums
(and lse) use the unrounded p.  That rounding is the only approximation beyond
the bf16 forward's, and it bounds the O error per element:
    |O - O_ref|_ij <= 2^-4 sum_k P_ik |v_kj|          (e4m3 keeps 3 mantissa bits:
                                                       relative rounding error <= 2^-4)
                    + 2^-10 sum_k |v_kj| / L_i        (weights in e4m3's subnormal range:
                                                       absolute error <= 2^-10; the kernel's
                                                       row sum l >= L_i = sum_k e^(s_ik - max s_i))
                    + ulp_bf16(O_ref)/2 + 1e-3        (output rounding; fp32 terms and the
                                                       exponentials' approximation)
The first term is the oracle's forward applied to |V|.  lse keeps the forward's
1e-3 bound."""
import numpy as np
import pytest
import torch

import workloads
from oracle import reference as ref
from tests import parity

pytestmark = pytest.mark.gpu


def _run(w, **kw):
    import attention_attn_fwd_10_b200 as attn

    x = workloads.make_inputs(w)
    q8, k8, v8 = (x[n].to(torch.float8_e4m3fn) for n in ("q", "k", "v"))
    o, lse = attn.fwd_qk8(q8.cuda(), k8.cuda(), v8.cuda(), causal=w.causal, scale=w.scale, **kw)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    return q8.float(), k8.float(), v8.float(), x, o, lse


def _subnormal_term(q, k, v, causal, scale, b, h, rows):
    """2^-10 * sum over visible keys of |v_kj| / L_i for the given rows of (b, h)."""
    qf, kf, vf = (ref.to_f64(t) for t in (q, k, v))
    g = h // (qf.shape[2] // kf.shape[2])
    s = scale * (qf[b, rows, h, :] @ kf[b, :, g, :].T)
    vis = ref.visible(qf.shape[1], kf.shape[1], causal, rows)
    s = np.where(vis, s, -np.inf)
    smax = s.max(axis=1)
    ok = np.isfinite(smax)
    L = np.where(ok, np.exp(s - np.where(ok, smax, 0.0)[:, None]).sum(axis=1), 1.0)
    sumabs = vis.astype(np.float64) @ np.abs(vf[b, :, g, :])
    return np.where(ok[:, None], 2.0 ** -10 * sumabs / L[:, None], 0.0)


def _check(w, q, k, v, o, lse, heads=None, rows=None):
    o_np, lse_np = parity.to_np(o), parity.to_np(lse)
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H_q)]
    worst = 0.0
    for (b, h) in heads:
        r = np.arange(w.S_q) if rows is None else np.asarray(rows)
        o_ref, lse_ref = ref.forward_rows(q, k, v, w.causal, w.scale, b, h, r)
        o_abs, _ = ref.forward_rows(q, k, v.abs(), w.causal, w.scale, b, h, r)
        bound = (2.0 ** -4 * o_abs + _subnormal_term(q, k, v, w.causal, w.scale, b, h, r)
                 + parity.ulp_bf16(o_ref) / 2 + 1e-3)
        got = o_np[b, r, h, :]
        assert np.all(np.isfinite(got))
        err = np.abs(got - o_ref)
        assert np.all(err <= bound), f"{w.name} b={b} h={h}: error {err.max():.3e} above the e4m3 bound"
        parity.check_lse(lse_np[b, h, r], lse_ref, f"{w.name} b={b} h={h}")
        worst = max(worst, float((err / bound).max()))
    return worst


@pytest.mark.parametrize("S_q,S_k", [(1, 1), (17, 17), (128, 128), (129, 129), (300, 300), (64, 500), (500, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_small_shapes(S_q, S_k, causal):
    w = workloads.small(B=2, H_q=2, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q * 17 + S_k)
    q, k, v, x, o, lse = _run(w)
    _check(w, q, k, v, o, lse)


@pytest.mark.parametrize("H_q,H_kv,S", [(4, 1, 400), (8, 2, 40)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa(H_q, H_kv, S, causal):
    w = workloads.small(B=1, H_q=H_q, H_kv=H_kv, S_q=S, S_k=S, D=128, causal=causal, seed=6)
    q, k, v, x, o, lse = _run(w)
    _check(w, q, k, v, o, lse)


@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_rescale_threshold_spiky_keys(tau):
    w = workloads.small(B=1, H_q=2, S_q=1024, S_k=1024, D=128, causal=True, seed=5, spiky_keys=True)
    q, k, v, x, o, lse = _run(w, rescale_threshold=tau)
    _check(w, q, k, v, o, lse)


def test_causal_config_sampled_rows():
    w = workloads.FWD_CAUSAL
    q, k, v, x, o, lse = _run(w)
    rows = sorted(set(range(0, 256)) | set(range(w.S_q - 256, w.S_q)) | {4095, 4096})
    _check(w, q, k, v, o, lse, heads=[(0, 0), (1, 15)], rows=rows)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_error_against_unquantised_inputs_is_reported_scale():
    # Against the oracle on the unquantised bf16 inputs the error also carries the
    # caller's quantisation of q, k and v, which no per-element bound covers
    # (rounding q and k moves every score).  This checks the relative Frobenius error
    # stays at the few-percent scale that 3-bit mantissas give on N(0,1) data.
    w = workloads.small(B=1, H_q=4, S_q=1024, S_k=1024, D=128, causal=True, seed=8)
    q, k, v, x, o, lse = _run(w)
    o_ref, _ = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    rel = np.linalg.norm(parity.to_np(o) - o_ref) / np.linalg.norm(o_ref)
    assert rel < 0.15, rel


def test_last_wave_in_halves():
    # 152 non-causal units on 148 SMs: the last 4 run in the second launch as the dual
    # stream with e4m3 P and V; every row of the heads that hold them and of the first
    w = workloads.small(B=1, H_q=38, S_q=1024, S_k=1024, D=128, causal=False, seed=12)
    q, k, v, x, o, lse = _run(w)
    _check(w, q, k, v, o, lse, heads=[(0, 0), (0, 34), (0, 35), (0, 36), (0, 37)])
