"""Pins for the fp64 oracle: it is checked against facts other than itself.

Each check below would fail for a plausible mistake in the oracle (a dropped
scale, a wrong mask direction, a transposed operand, a wrong group mapping, a
missing delta term, a sign error ...); ``test_pins_catch_planted_mistakes``
plants such mistakes in copies of the oracle and shows they are caught.
"""
import math

import numpy as np
import pytest
import torch

from oracle import brute, exp2_cubic
from oracle import reference as ref
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _tolist(x):
    return np.asarray(x).tolist()


# --------------------------------------------------------------------------- brute force

@pytest.mark.parametrize("B,S_q,S_k,H_q,H_kv,D,causal", [
    (1, 5, 5, 1, 1, 3, False),
    (2, 7, 7, 2, 1, 4, True),
    (1, 4, 9, 4, 2, 3, True),   # S_q < S_k: bottom-right causal
    (1, 9, 4, 2, 2, 2, True),   # S_q > S_k: the first rows see no key
    (1, 16, 16, 3, 3, 8, True),
    (1, 6, 11, 2, 2, 5, False),
])
def test_numpy_equals_brute_force(B, S_q, S_k, H_q, H_kv, D, causal):
    q = _rand((B, S_q, H_q, D), 1)
    k = _rand((B, S_k, H_kv, D), 2)
    v = _rand((B, S_k, H_kv, D), 3)
    scale = 0.37
    o, lse = ref.forward(q, k, v, causal, scale, block_rows=3)
    ob, lseb = brute.forward(_tolist(q), _tolist(k), _tolist(v), causal, scale)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
    lseb = np.array(lseb)
    assert np.array_equal(np.isinf(lse), np.isinf(lseb))
    fin = np.isfinite(lseb)
    np.testing.assert_allclose(lse[fin], lseb[fin], rtol=0, atol=1e-12)


def test_rows_api_equals_full():
    w = workloads.small(B=2, H_q=4, H_kv=2, S_q=300, S_k=300, D=16, causal=True)
    x = workloads.make_inputs(w)
    o, lse = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    rows = [0, 1, 127, 128, 299]
    orow, lrow = ref.forward_rows(x["q"], x["k"], x["v"], True, w.scale, 1, 3, rows)
    np.testing.assert_allclose(orow, o[1, rows, 3, :], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lrow, lse[1, 3, rows], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------- library special case

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(2, 2), (4, 1), (6, 2)])
def test_matches_torch_sdpa_fp64(causal, H_q, H_kv):
    B, S, D = 2, 33, 16
    q = torch.randn(B, S, H_q, D, dtype=torch.float64, generator=torch.Generator().manual_seed(0))
    k = torch.randn(B, S, H_kv, D, dtype=torch.float64, generator=torch.Generator().manual_seed(1))
    v = torch.randn(B, S, H_kv, D, dtype=torch.float64, generator=torch.Generator().manual_seed(2))
    scale = 1 / math.sqrt(D)
    G = H_q // H_kv
    kr = k.repeat_interleave(G, dim=2)
    vr = v.repeat_interleave(G, dim=2)
    ot = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2), is_causal=causal, scale=scale
    ).transpose(1, 2)
    o, lse = ref.forward(q, k, v, causal, scale)
    np.testing.assert_allclose(o, ot.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("bqhd,bkhd->bhqk", q, kr) * scale
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_backward_matches_torch_autograd_fp64():
    B, S, H_q, H_kv, D = 1, 20, 4, 2, 8
    g = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn(B, S, h, D, dtype=torch.float64, generator=g) for h in (H_q, H_kv, H_kv, H_q))
    for causal in (False, True):
        qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
        G = H_q // H_kv
        ot = torch.nn.functional.scaled_dot_product_attention(
            qt.transpose(1, 2), kt.repeat_interleave(G, 2).transpose(1, 2),
            vt.repeat_interleave(G, 2).transpose(1, 2), is_causal=causal, scale=0.3).transpose(1, 2)
        (ot * do).sum().backward()
        dq, dk, dv = ref.backward(q, k, v, do, causal, 0.3, block_rows=7)
        np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=0, atol=1e-11)


# --------------------------------------------------------------------------- invariants and closed forms

def _fwd(q, k, v, causal, scale=0.5):
    return ref.forward(q, k, v, causal, scale, block_rows=5)


@pytest.mark.parametrize("causal", [False, True])
def test_P_rows_sum_to_one_and_are_nonnegative(causal):
    # With V = identity (D = S_k) the output rows ARE the rows of P.
    S = 12
    q = _rand((1, S, 1, 6), 4)
    k = _rand((1, S, 1, 6), 5)
    # pad keys' feature dim to S with zeros so V can be the identity
    v = np.eye(S)[None, :, None, :]
    q2 = np.concatenate([q, np.zeros((1, S, 1, S - 6))], axis=3)
    k2 = np.concatenate([k, np.zeros((1, S, 1, S - 6))], axis=3)
    P, _ = _fwd(q2, k2, v, causal)
    P = P[0, :, 0, :]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    assert (P >= 0).all()
    if causal:
        assert np.all(P[np.triu_indices(S, 1)] == 0)
        assert np.all(P[np.tril_indices(S)] > 0)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_give_constant_output(causal):
    q = _rand((2, 9, 2, 4), 6)
    k = _rand((2, 9, 2, 4), 7)
    c = _rand((1, 1, 1, 4), 8)
    v = np.broadcast_to(c, (2, 9, 2, 4)).copy()
    o, _ = _fwd(q, k, v, causal)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-14)


def test_identical_keys_give_mean_of_values():
    S = 10
    q = _rand((1, S, 1, 4), 9)
    k = np.broadcast_to(_rand((1, 1, 1, 4), 10), (1, S, 1, 4)).copy()
    v = _rand((1, S, 1, 4), 11)
    o, lse = _fwd(q, k, v, False)
    np.testing.assert_allclose(o[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (S, 4)), atol=1e-14)
    oc, lsec = _fwd(q, k, v, True)
    prefix = np.cumsum(v[0, :, 0], axis=0) / np.arange(1, S + 1)[:, None]
    np.testing.assert_allclose(oc[0, :, 0], prefix, atol=1e-14)
    # lse = s + ln(#visible) when all visible scores are equal
    s = 0.5 * (q[0, :, 0] @ k[0, 0, 0])
    np.testing.assert_allclose(lsec[0, 0], s + np.log(np.arange(1, S + 1)), atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], s + np.log(S), atol=1e-13)


def test_causal_row0_sees_only_key0():
    q = _rand((1, 8, 3, 5), 12)
    k = _rand((1, 8, 3, 5), 13)
    v = _rand((1, 8, 3, 5), 14)
    o, lse = _fwd(q, k, v, True, scale=0.7)
    np.testing.assert_allclose(o[0, 0], v[0, 0], atol=1e-15)
    np.testing.assert_allclose(lse[0, :, 0], 0.7 * np.einsum("hd,hd->h", q[0, 0], k[0, 0]), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_per_row_score_shift(causal):
    # Append to q a component c_i and to every key a constant 1: every score of
    # row i moves by scale*c_i.  O must not change; lse moves by scale*c_i.
    B, S, H, D = 1, 11, 2, 4
    q = _rand((B, S, H, D), 15)
    k = _rand((B, S, H, D), 16)
    v = _rand((B, S, H, D), 17)
    c = 3.0 * _rand((B, S, H, 1), 18)
    o, lse = _fwd(q, k, v, causal)
    o2, lse2 = _fwd(np.concatenate([q, c], 3), np.concatenate([k, np.ones((B, S, H, 1))], 3), v, causal)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2 - lse, 0.5 * np.transpose(c[..., 0], (0, 2, 1)), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_closed_form(causal):
    S_q, S_k = 6, 9
    q = np.zeros((1, S_q, 1, 3))
    k = _rand((1, S_k, 1, 3), 19)
    v = _rand((1, S_k, 1, 3), 20)
    o, lse = _fwd(q, k, v, causal)
    for i in range(S_q):
        nvis = (i + S_k - S_q + 1) if causal else S_k
        np.testing.assert_allclose(o[0, i, 0], v[0, :nvis, 0].mean(0), atol=1e-14)
        np.testing.assert_allclose(lse[0, 0, i], math.log(nvis), atol=1e-14)


def test_single_key_returns_value():
    q = _rand((2, 5, 2, 3), 21)
    k = _rand((2, 1, 2, 3), 22)
    v = _rand((2, 1, 2, 3), 23)
    o, _ = _fwd(q, k, v, False)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), atol=1e-15)


def test_fully_masked_rows():
    # S_q > S_k with bottom-right alignment: rows i < S_q - S_k see no key.
    q = _rand((1, 7, 1, 3), 24)
    k = _rand((1, 3, 1, 3), 25)
    v = _rand((1, 3, 1, 3), 26)
    o, lse = _fwd(q, k, v, True)
    assert np.all(o[0, :4] == 0) and np.all(np.isneginf(lse[0, 0, :4]))
    np.testing.assert_allclose(o[0, 4, 0], v[0, 0, 0], atol=1e-15)


def test_key_permutation_equivariance():
    q = _rand((1, 6, 2, 4), 27)
    k = _rand((1, 13, 2, 4), 28)
    v = _rand((1, 13, 2, 4), 29)
    perm = np.random.default_rng(0).permutation(13)
    o, lse = _fwd(q, k, v, False)
    o2, lse2 = _fwd(q, k[:, perm], v[:, perm], False)
    np.testing.assert_allclose(o2, o, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, atol=1e-14)


def test_gqa_equals_mha_with_repeated_heads():
    q = _rand((2, 9, 6, 4), 30)
    k = _rand((2, 9, 2, 4), 31)
    v = _rand((2, 9, 2, 4), 32)
    for causal in (False, True):
        o, lse = _fwd(q, k, v, causal)
        o2, lse2 = _fwd(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), causal)
        np.testing.assert_allclose(o, o2, atol=1e-15)
        np.testing.assert_allclose(lse, lse2, atol=1e-15)


def test_scale_enters_once():
    q = _rand((1, 5, 1, 3), 33)
    k = _rand((1, 5, 1, 3), 34)
    v = _rand((1, 5, 1, 3), 35)
    o1, l1 = _fwd(q, k, v, False, scale=2.0)
    o2, l2 = _fwd(2.0 * q, k, v, False, scale=1.0)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)


# --------------------------------------------------------------------------- backward

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S_q,S_k,H_q,H_kv", [(5, 5, 2, 1), (4, 7, 2, 2), (8, 8, 1, 1)])
def test_backward_central_differences(causal, S_q, S_k, H_q, H_kv):
    D, scale, h = 3, 0.6, 1e-6
    q = _rand((1, S_q, H_q, D), 36)
    k = _rand((1, S_k, H_kv, D), 37)
    v = _rand((1, S_k, H_kv, D), 38)
    do = _rand((1, S_q, H_q, D), 39)
    dq, dk, dv = ref.backward(q, k, v, do, causal, scale, block_rows=3)

    def L(q_, k_, v_):
        o, _ = ref.forward(q_, k_, v_, causal, scale)
        return float((o * do).sum())

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (L(**{a + "_": b for a, b in args_p.items()}) -
                        L(**{a + "_": b for a, b in args_m.items()})) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-7, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_sum_invariants(causal):
    q = _rand((2, 12, 4, 5), 40)
    k = _rand((2, 12, 2, 5), 41)
    v = _rand((2, 12, 2, 5), 42)
    do = _rand((2, 12, 4, 5), 43)
    dq, dk, dv = ref.backward(q, k, v, do, causal, 0.45)
    # sum_j dS_ij = 0  =>  the key gradients of every (b, h_kv) sum to zero
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    # every P row sums to 1 => sum over keys of dV = sum over the group's queries of dO
    grp = do.reshape(2, 12, 2, 2, 5).sum(axis=3).sum(axis=1)
    np.testing.assert_allclose(dv.sum(axis=1), grp, atol=1e-12)


def test_backward_brute_loss_gradient_spot():
    # dL/dq at one entry via the pure-Python loss (independent of numpy).
    q = _rand((1, 4, 1, 2), 44)
    k = _rand((1, 4, 1, 2), 45)
    v = _rand((1, 4, 1, 2), 46)
    do = _rand((1, 4, 1, 2), 47)
    dq, dk, dv = ref.backward(q, k, v, do, True, 0.8)
    h = 1e-6
    for arr, grad, idx in ((q, dq, (0, 2, 0, 1)), (k, dk, (0, 1, 0, 0)), (v, dv, (0, 3, 0, 1))):
        xp, xm = arr.copy(), arr.copy()
        xp[idx] += h
        xm[idx] -= h
        sub = lambda a: {"q": q, "k": k, "v": v, **a}
        key = "q" if arr is q else ("k" if arr is k else "v")
        lp = brute.loss(*[_tolist(sub({key: xp})[n]) for n in "qkv"], _tolist(do), True, 0.8)
        lm = brute.loss(*[_tolist(sub({key: xm})[n]) for n in "qkv"], _tolist(do), True, 0.8)
        assert abs((lp - lm) / (2 * h) - grad[idx]) < 1e-7


# --------------------------------------------------------------------------- exp2 cubic

def test_exp2_cubic_minimax_and_bound():
    c, E = exp2_cubic.remez_cubic()
    # Equioscillation: 5 alternating extrema of equal size (a minimax certificate).
    f = np.linspace(0, 1, 200001)
    err = (np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    assert abs(np.max(np.abs(err)) - E) < 1e-9
    assert 6e-5 < E < 9e-5  # a cubic cannot do better than ~7.5e-5 on [0, 1]
    sign_changes = np.count_nonzero(np.diff(np.sign(err)) != 0)
    assert sign_changes == 4
    # fp32 evaluation over a wide input range stays within the bound (+ fp32 rounding)
    x = np.linspace(-125, 8, 3_000_001).astype(np.float32)
    y = exp2_cubic.exp2_cubic_f32(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < E + 4e-7
    # integers are exact up to p(0) = c0
    xi = np.arange(-125, 9, dtype=np.float32)
    np.testing.assert_allclose(exp2_cubic.exp2_cubic_f32(xi, c), np.exp2(xi) * np.float32(c[0]), rtol=1e-7)


def test_exp2_cubic_tiny_and_clamped():
    c, _ = exp2_cubic.remez_cubic()
    # below 2^-125 the exponent-field add may leave the normal range: results
    # there only need to be tiny and non-negative (the row sum is >= 1)
    y = exp2_cubic.exp2_cubic_f32(np.array([-1e30, -200, -127.5, -126, -125.5], np.float32), c)
    assert np.all(y >= 0) and np.all(y < 2.0 ** -124)


# --------------------------------------------------------------------------- mutation check

def _mutants():
    """Copies of the forward with one plausible mistake each."""
    def no_scale(q, k, v, causal, scale, block_rows=5):
        return ref.forward(q, k, v, causal, 1.0, block_rows)

    def transposed_mask(q, k, v, causal, scale, block_rows=5):
        o, lse = ref.forward(q[:, ::-1], k[:, ::-1], v[:, ::-1], causal, scale, block_rows)
        return o[:, ::-1], lse[:, :, ::-1]

    def wrong_group(q, k, v, causal, scale, block_rows=5):
        G = q.shape[2] // k.shape[2]
        kk = np.concatenate([k[:, :, h % k.shape[2]:h % k.shape[2] + 1] for h in range(q.shape[2])], 2)
        vv = np.concatenate([v[:, :, h % k.shape[2]:h % k.shape[2] + 1] for h in range(q.shape[2])], 2)
        return ref.forward(q, kk, vv, causal, scale, block_rows) if G > 1 else ref.forward(q, k, v, causal, scale)

    def lse_log2(q, k, v, causal, scale, block_rows=5):
        o, lse = ref.forward(q, k, v, causal, scale, block_rows)
        return o, lse / math.log(2)

    def no_max_shift_overflow(q, k, v, causal, scale, block_rows=5):
        o, lse = ref.forward(q, k, v, causal, scale, block_rows)
        return o, lse + 0.0 * lse + (np.isfinite(lse) * 1e-3)

    return [no_scale, transposed_mask, wrong_group, lse_log2, no_max_shift_overflow]


def _pins_pass(fwd) -> bool:
    """A compact subset of the pins above, parameterised by the forward under test."""
    try:
        B, S, H_q, H_kv, D = 1, 9, 4, 2, 4
        q, k, v = _rand((B, S, H_q, D), 50), _rand((B, S, H_kv, D), 51), _rand((B, S, H_kv, D), 52)
        for causal in (False, True):
            o, lse = fwd(q, k, v, causal, 0.5)
            ob, lseb = brute.forward(_tolist(q), _tolist(k), _tolist(v), causal, 0.5)
            if not np.allclose(o, ob, atol=1e-12, rtol=0) or not np.allclose(lse, lseb, atol=1e-12, rtol=0):
                return False
        return True
    except Exception:
        return False


@pytest.mark.parametrize("causal", [False, True])
def test_key_range_merge_by_logsumexp(causal):
    """The split-KV forward's combine step: attention over disjoint key ranges,
    each normalised over its own keys (O_s, lse_s), merges into the full result
    by lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.  Checked with
    per-range softmaxes computed here from explicit fp64 scores (global causal
    mask, so ranges that see no key of a row contribute lse_s = -inf)."""
    B, S_q, S_k, H, D, scale = 1, 5, 40, 2, 8, 0.3
    q, k, v = _rand((B, S_q, H, D), 1), _rand((B, S_k, H, D), 2), _rand((B, S_k, H, D), 3)
    o_ref, lse_ref = ref.forward(q, k, v, causal, scale)
    mask = ref.visible(S_q, S_k, causal)
    for bounds in ([0, 40], [0, 13, 40], [0, 1, 2, 30, 39, 40], [0, 8, 16, 24, 32, 40]):
        o_parts, l_parts = [], []
        for a, b_ in zip(bounds[:-1], bounds[1:]):
            s = np.einsum("bqhd,bkhd->bhqk", q, k[:, a:b_]) * scale
            s = np.where(mask[None, None, :, a:b_], s, -np.inf)
            m = s.max(axis=-1, keepdims=True)
            e = np.where(np.isfinite(m), np.exp(s - np.where(np.isfinite(m), m, 0.0)), 0.0)
            l = e.sum(axis=-1, keepdims=True)
            with np.errstate(divide="ignore", invalid="ignore"):
                o_parts.append(np.where(l > 0, np.einsum("bhqk,bkhd->bhqd", e, v[:, a:b_]) / l, 0.0))
                l_parts.append(np.where(l[..., 0] > 0, m[..., 0] + np.log(l[..., 0]), -np.inf))
        ls = np.stack(l_parts)                      # [splits, B, H, S_q]
        mx = ls.max(axis=0)
        w = np.where(np.isfinite(ls), np.exp(ls - np.where(np.isfinite(mx), mx, 0.0)), 0.0)
        tot = w.sum(axis=0)
        lse = np.where(tot > 0, mx + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
        o = np.einsum("sbhq,sbhqd->bhqd", w, np.stack(o_parts)) / np.where(tot > 0, tot, 1.0)[..., None]
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12)
        np.testing.assert_allclose(o.transpose(0, 2, 1, 3), o_ref, atol=1e-12)


def test_pins_catch_planted_mistakes():
    assert _pins_pass(lambda *a, **kw: ref.forward(*a, **kw))
    for m in _mutants():
        assert not _pins_pass(m), m.__name__
