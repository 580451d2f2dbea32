"""GPU forward vs the fp64 oracle, through the C ABI (ctypes binding), on seeded inputs."""
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


def _run(w, **kw):
    x = workloads.make_inputs(w)
    dev = "cuda"
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o, lse = _attn().fwd(q, k, v, causal=w.causal, scale=w.scale, **kw)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    return x, o, lse


def test_tiny_config_full():
    w = workloads.TINY
    x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], w.causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("S_q,S_k", [(1, 1), (17, 17), (127, 127), (128, 128), (129, 129), (255, 255),
                                     (300, 300), (64, 200), (200, 64), (1, 333), (333, 1)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_small_shapes(S_q, S_k, causal, D):
    w = workloads.small(B=2, H_q=2, S_q=S_q, S_k=S_k, D=D, causal=causal, seed=S_q * 1000 + S_k)
    x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("H_q,H_kv", [(4, 1), (8, 2), (6, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa(H_q, H_kv, causal):
    w = workloads.small(B=1, H_q=H_q, H_kv=H_kv, S_q=400, S_k=400, D=128, causal=causal, seed=11)
    x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("tau", [0.0, 8.0, 16.0])
@pytest.mark.parametrize("poly", [0, 4, 8])
def test_rescale_threshold_and_poly_fraction(tau, poly):
    w = workloads.small(B=1, H_q=2, S_q=1024, S_k=1024, D=128, causal=True, seed=5, spiky_keys=True)
    x, o, lse = _run(w, rescale_threshold=tau, poly_exp_every=poly)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o, o_ref, f"{w.name} tau={tau} poly={poly}", v_absmax=float(x["v"].float().abs().max()))
    parity.check_lse(lse, lse_ref, f"{w.name} tau={tau} poly={poly}")


def test_noncausal_config_full():
    w = workloads.FWD_NONCAUSAL
    x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], w.causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


def _sampled(w, o, lse, x, heads, rows_of):
    """Check the rows rows_of(b, h) of every listed (b, h) against the oracle, row by row
    (each output row depends only on its own query row and the keys)."""
    o_c, lse_c = o.cpu(), lse.cpu()
    vmax = float(x["v"].float().abs().max()) if w.spiky_keys else None
    for (b, h) in heads:
        rows = rows_of(b, h)
        o_ref, lse_ref = ref.forward_rows(x["q"], x["k"], x["v"], w.causal, w.scale, b, h, rows)
        parity.check_o(o_c[b, rows, h, :], o_ref, f"{w.name} b={b} h={h}", v_absmax=vmax)
        parity.check_lse(lse_c[b, h, rows], lse_ref, f"{w.name} b={b} h={h}")
    assert torch.isfinite(o_c.float()).all() and torch.isfinite(lse_c).all()


def _unit_rows(S, n_random=64, seed=0):
    """Rows of one head to check: its whole first and last 256-row work unit (the
    longest and shortest causal units, and the diagonal blocks of both), plus
    n_random rows drawn uniformly from the rest."""
    def rows_of(b, h):
        g = np.random.default_rng(seed + 1000 * b + h)
        ends = set(range(0, min(256, S))) | set(range(max(0, S - 256), S))
        rest = np.setdiff1d(np.arange(S), np.fromiter(ends, dtype=np.int64))
        pick = g.choice(rest, min(n_random, len(rest)), replace=False).tolist() if len(rest) else []
        return sorted(ends | set(pick))
    return rows_of


def _all_heads(w):
    return [(b, h) for b in range(w.B) for h in range(w.H_q)]


@pytest.mark.parametrize("w", [workloads.FWD_CAUSAL, workloads.FWD_CAUSAL_SPIKY], ids=lambda w: w.name)
def test_causal_config_every_head(w):
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    x, o, lse = _run(w, rescale_count=cnt)
    _sampled(w, o, lse, x, _all_heads(w), _unit_rows(w.S_q))
    if w.spiky_keys:
        assert int(cnt.item()) > 0  # the spiky keys exercise the rescale path


def test_gqa_long_config_every_head():
    w = workloads.FWD_CAUSAL_GQA
    x, o, lse = _run(w)
    # every query head: the four of each kv group share one key/value head
    _sampled(w, o, lse, x, _all_heads(w), _unit_rows(w.S_q))


def test_deterministic_and_overwrites_poison():
    w = workloads.small(B=2, H_q=4, S_q=700, S_k=700, D=128, causal=True, seed=3)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1 = torch.full_like(q, float("nan"))
    l1 = torch.full((2, 4, 700), float("nan"), device="cuda")
    _attn().fwd(q, k, v, causal=True, out=o1, lse=l1)
    o2, l2 = _attn().fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o1.float()).all() and torch.isfinite(l1).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_output_at_16_byte_offset(causal, D):
    # O at a 16- but not 32-byte aligned address (the contract asks for 16; the
    # non-causal epilogue then writes with 16-byte stores instead of 256-bit ones): the
    # result equals the one written to an aligned O, and matches the oracle
    w = workloads.small(B=1, H_q=2, S_q=300, S_k=300, D=D, causal=causal, seed=31)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o_al, lse_al = _attn().fwd(q, k, v, causal=causal, scale=w.scale)
    assert o_al.data_ptr() % 32 == 0
    buf = torch.full((q.numel() + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    o = buf[8:].view(q.shape)
    assert o.data_ptr() % 32 == 16
    lse = torch.full_like(lse_al, float("nan"))
    _attn().fwd(q, k, v, causal=causal, scale=w.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    assert torch.equal(o, o_al) and torch.equal(lse, lse_al)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)


def test_host_buffers_round_trip():
    w = workloads.small(B=1, H_q=2, S_q=300, S_k=300, D=64, causal=False, seed=9)
    x = workloads.make_inputs(w)
    o, lse = _attn().fwd(x["q"].pin_memory(), x["k"].pin_memory(), x["v"].pin_memory(), causal=False)
    assert not o.is_cuda
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], False, w.scale)
    parity.check_o(o, o_ref)
    parity.check_lse(lse, lse_ref)


@pytest.mark.parametrize("S_q,S_k", [(1, 300), (17, 17), (64, 500), (100, 100), (128, 1000)])
@pytest.mark.parametrize("H_q,H_kv", [(4, 2), (8, 2), (16, 2), (64, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_packed_query_heads(S_q, S_k, H_q, H_kv, causal):
    # S_q <= 128 with a power-of-two group: the group's query heads share a tile
    w = workloads.small(B=2, H_q=H_q, H_kv=H_kv, S_q=S_q, S_k=S_k, D=128, causal=causal, seed=S_q + H_q)
    x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], causal, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


def test_packed_query_heads_d64():
    w = workloads.small(B=1, H_q=8, H_kv=1, S_q=33, S_k=700, D=64, causal=True, seed=4)
    x, o, lse = _run(w)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], True, w.scale)
    parity.check_o(o, o_ref, w.name)
    parity.check_lse(lse, lse_ref, w.name)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H_q,H_kv,S,D", [(8, 16, 16, 640, 128), (4, 12, 4, 1000, 64), (2, 40, 8, 2304, 128)])
def test_persistent_ctas_match_one_cta_per_unit(B, H_q, H_kv, S, D, causal):
    # more work units than SMs: persistent CTAs take over the units of CTAs that have not
    # started (several units each, of different lengths when causal).  Each unit's
    # arithmetic is the same either way, so the results are bitwise equal (unless the
    # last wave went to the second launch, whose units split their keys between two
    # tiles: then every row only matches the oracle); and they match the oracle.
    w = workloads.small(B=B, H_q=H_q, H_kv=H_kv, S_q=S, S_k=S, D=D, causal=causal, seed=B * S + H_q)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = _attn().fwd(q, k, v, causal=causal, scale=w.scale, persistent=True)
    o2, l2 = _attn().fwd(q, k, v, causal=causal, scale=w.scale, persistent=False)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    if not _last_wave_split(B, H_q, S, causal):
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_c, l_c = o1.cpu(), l1.cpu()
    for (b, h) in [(0, 0), (B - 1, H_q - 1), (B // 2, H_q // 2)]:
        rows = sorted(set(range(0, min(S, 300))) | set(range(max(0, S - 300), S)))
        o_ref, lse_ref = ref.forward_rows(x["q"], x["k"], x["v"], causal, w.scale, b, h, rows)
        parity.check_o(o_c[b, rows, h, :], o_ref, f"{w.name} b={b} h={h}")
        parity.check_lse(l_c[b, h, rows], lse_ref, f"{w.name} b={b} h={h}")


def _last_wave_split(B, H_q, S, causal, sms=148):
    """Whether the persistent forward sends its last wave of work units (256 query
    rows of one head each) to the second launch: non-causal, more units than SMs,
    and a last wave of at most half the SMs."""
    units = -(-S // 256) * B * H_q
    r = units % sms
    return (not causal) and units > sms and 0 < r <= sms // 2


@pytest.mark.parametrize("B,H_q,H_kv,S,D", [(1, 20, 20, 2048, 128), (1, 38, 38, 1024, 128), (4, 12, 4, 1000, 64)])
def test_last_wave_in_halves(B, H_q, H_kv, S, D):
    # the last units of the grid run in the second launch, each as two CTAs on 128 rows
    # whose tiles split the keys; those units are the last (batch, head) pairs' (the grid
    # lists heads in groups of 8): every row of the last heads and of the first against
    # the oracle
    assert _last_wave_split(B, H_q, S, False)
    w = workloads.small(B=B, H_q=H_q, H_kv=H_kv, S_q=S, S_k=S, D=D, causal=False, seed=S + H_q)
    x = workloads.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = _attn().fwd(q, k, v, causal=False, scale=w.scale, persistent=True)
    torch.cuda.synchronize()
    assert _attn().device_status() == 0
    o_c, l_c = o.cpu(), lse.cpu()
    rows = list(range(S))
    for b in sorted({0, B - 1}):
        for h in sorted({0, H_q - 4, H_q - 3, H_q - 2, H_q - 1}):
            o_ref, lse_ref = ref.forward_rows(x["q"], x["k"], x["v"], False, w.scale, b, h, rows)
            parity.check_o(o_c[b, rows, h, :], o_ref, f"{w.name} b={b} h={h}")
            parity.check_lse(l_c[b, h, rows], lse_ref, f"{w.name} b={b} h={h}")
