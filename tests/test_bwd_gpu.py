"""GPU backward vs the fp64 oracle, through the C ABI.  The GPU backward consumes
the GPU forward's O and lse; the oracle recomputes its own fp64 P."""
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


# main-pass kernels at head dim 128: 1 = one CTA per key tile (the default), 2 = CTA pairs
CTA_MODES = [1, 2]


def _gpu_fwd_bwd(x, causal, scale, cta_mode=0):
    attn = _attn()
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=causal, scale=scale, cta_mode=cta_mode)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    return dq, dk, dv


def _check(w, x, grads, groups=None, batches=None):
    ref_g = ref.backward(x["q"], x["k"], x["v"], x["do"], w.causal, w.scale, groups=groups, batches=batches)
    G = w.H_q // w.H_kv
    for name, g, gr in zip(("dq", "dk", "dv"), grads, ref_g):
        g = parity.to_np(g)
        if groups is not None:
            bs = batches if batches is not None else range(w.B)
            sel_q = [h for grp in groups for h in range(grp * G, (grp + 1) * G)]
            idx = (list(bs), slice(None), sel_q if name == "dq" else list(groups), slice(None))
            g = g[np.ix_(idx[0], range(g.shape[1]), idx[2], range(g.shape[3]))]
            gr = gr[np.ix_(idx[0], range(gr.shape[1]), idx[2], range(gr.shape[3]))]
        parity.check_grad(g, gr, f"{w.name} {name}")


@pytest.mark.parametrize("S_q,S_k", [(1, 1), (17, 17), (64, 64), (127, 127), (128, 128), (129, 129),
                                     (200, 200), (300, 300), (100, 260), (260, 100)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cta_mode", CTA_MODES)
def test_small_shapes(S_q, S_k, causal, cta_mode):
    w = workloads.small(B=2, H_q=2, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q * 7 + S_k, backward=True)
    x = workloads.make_inputs(w)
    _check(w, x, _gpu_fwd_bwd(x, causal, w.scale, cta_mode))


@pytest.mark.parametrize("H_q,H_kv", [(4, 1), (8, 2), (6, 3)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cta_mode", CTA_MODES)
def test_gqa(H_q, H_kv, causal, cta_mode):
    w = workloads.small(B=1, H_q=H_q, H_kv=H_kv, S_q=384, S_k=384, D=128, causal=causal, seed=21, backward=True)
    x = workloads.make_inputs(w)
    _check(w, x, _gpu_fwd_bwd(x, causal, w.scale, cta_mode))


@pytest.mark.parametrize("cta_mode", CTA_MODES)
def test_medium_causal(cta_mode):
    w = workloads.small(B=1, H_q=2, S_q=1536, S_k=1536, D=128, causal=True, seed=33, backward=True)
    x = workloads.make_inputs(w)
    _check(w, x, _gpu_fwd_bwd(x, True, w.scale, cta_mode))


@pytest.mark.parametrize("S_q,S_k", [(300, 300), (1536, 1536), (200, 712), (712, 200)])
@pytest.mark.parametrize("causal", [False, True])
def test_cta_pairs_match_one_cta_per_tile(S_q, S_k, causal):
    """The two main-pass kernels compute the same sums in different orders: dK, dV
    agree to rounding of their fp32 accumulations, dQ to the order of its parts."""
    w = workloads.small(B=1, H_q=4, H_kv=2, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=5 + S_k, backward=True)
    x = workloads.make_inputs(w)
    one = _gpu_fwd_bwd(x, causal, w.scale, 1)
    two = _gpu_fwd_bwd(x, causal, w.scale, 2)
    for name, a, b_ in zip(("dq", "dk", "dv"), one, two):
        a, b_ = a.float(), b_.float()
        tol = 2 ** -7 * a.abs().amax() + 1e-6
        assert (a - b_).abs().max() <= tol, f"{name}: pairs and single CTAs disagree"


def test_cta_mode_arguments():
    attn = _attn()
    w = workloads.small(B=1, H_q=2, S_q=64, S_k=64, D=64, causal=False, seed=1, backward=True)
    x = workloads.make_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v)
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        attn.bwd(q, k, v, o, lse, do, cta_mode=2)  # pairs need head dim 128
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        attn.bwd(q, k, v, o, lse, do, cta_mode=3)


# (batch, kv head) groups of the backward workload checked whole against the oracle:
# the first and the last, and two in between (in the other batch entry)
BWD_GROUPS = [(0, 0), (0, 9), (1, 6), (1, 15)]


def _check_groups(w, x, grads, ref_by_group, what):
    for (b, g), ref_g in zip(BWD_GROUPS, ref_by_group):
        for name, gg, gr in zip(("dq", "dk", "dv"), grads, ref_g):
            gg = parity.to_np(gg[b:b + 1, :, g:g + 1])
            parity.check_grad(gg, gr, f"{w.name} {what} b={b} h_kv={g} {name}")


def test_backward_config_groups_both_modes_and_invariants():
    w = workloads.BWD_CAUSAL
    assert w.H_q == w.H_kv  # one query head per group: dq rows of group g are head g
    x = workloads.make_inputs(w)
    attn = _attn()
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
    runs = {(det, mode): attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale, deterministic=det,
                                  cta_mode=mode)
            for det in (False, True) for mode in CTA_MODES}
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    ref_by_group = [[a[b:b + 1, :, g:g + 1].copy()
                     for a in ref.backward(x["q"], x["k"], x["v"], x["do"], True, w.scale, groups=[g], batches=[b])]
                    for (b, g) in BWD_GROUPS]
    for (det, mode), grads in runs.items():
        _check_groups(w, x, grads, ref_by_group, ("deterministic" if det else "default") + f" cta_mode={mode}")
    # properties at full size: sum over keys of dK is 0; sum over keys of dV = sum over queries of dO
    dq, dk, dv = runs[(False, 2)]
    dk64 = dk.double()
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all() and torch.isfinite(dv.float()).all()
    assert dk64.sum(dim=1).abs().max() <= 3e-2 * dk64.abs().max() * w.S_k ** 0.5
    sum_dv = dv.double().sum(dim=1)
    sum_do = x["do"].double().sum(dim=1).cuda()
    assert (sum_dv - sum_do).abs().max() <= 3e-2 * sum_do.abs().max()


@pytest.mark.parametrize("S_q,S_k", [(1, 1), (64, 64), (129, 129), (300, 300), (100, 260)])
@pytest.mark.parametrize("causal", [False, True])
def test_head_dim_64(S_q, S_k, causal):
    w = workloads.small(B=2, H_q=4, H_kv=2, S_q=S_q, S_k=S_k, D=64, causal=causal, seed=S_q + 3 * S_k,
                        backward=True)
    x = workloads.make_inputs(w)
    _check(w, x, _gpu_fwd_bwd(x, causal, w.scale))


def test_unsupported_head_dim_is_rejected():
    attn = _attn()
    q = torch.zeros(1, 8, 1, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        attn.bwd(q, q, q, q, torch.zeros(1, 1, 8, device="cuda"), q)


def _bwd_twice(w, deterministic, cta_mode=0):
    attn = _attn()
    x = workloads.make_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v, causal=w.causal, scale=w.scale)
    runs = [attn.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, deterministic=deterministic,
                     cta_mode=cta_mode)
            for _ in range(2)]
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    return x, runs


@pytest.mark.parametrize("S_q,S_k,causal,H_q,H_kv", [(1536, 1536, True, 4, 2), (1536, 1536, False, 2, 2),
                                                    (100, 900, True, 4, 1), (900, 100, True, 2, 2),
                                                    (333, 333, False, 6, 3)])
@pytest.mark.parametrize("cta_mode", CTA_MODES)
def test_deterministic_mode(S_q, S_k, causal, H_q, H_kv, cta_mode):
    w = workloads.small(B=2, H_q=H_q, H_kv=H_kv, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q + S_k,
                        backward=True)
    x, (g1, g2) = _bwd_twice(w, True, cta_mode)
    for a, b_ in zip(g1, g2):
        assert torch.equal(a, b_), "deterministic backward differs between runs"
    _check(w, x, g1)


def test_deterministic_mode_head_dim_64():
    w = workloads.small(B=1, H_q=4, H_kv=2, S_q=700, S_k=700, D=64, causal=True, seed=3, backward=True)
    x, (g1, g2) = _bwd_twice(w, True)
    for a, b_ in zip(g1, g2):
        assert torch.equal(a, b_)
    _check(w, x, g1)


def test_deterministic_mode_backward_config_repeats_bitwise():
    w = workloads.BWD_CAUSAL
    x, (g1, g2) = _bwd_twice(w, True)
    for a, b_ in zip(g1, g2):
        assert torch.equal(a, b_)
