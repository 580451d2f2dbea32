"""Plain fp64 numpy oracle for exact scaled-dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``): the product never calls this.

What it follows
---------------
* The computation itself -- S = scale * Q K^T, an optional causal mask,
  P = softmax(S) row-wise, O = P V, plus the row log-sum-exp -- is the
  "attention kernel" the pages analyse as GEMM plus softmax exponentials
  (AI Infra series ch. 6, "GPU performance engineering (II)", section 1,
  quoting the FlashAttention-4 paper).  FlashAttention-4's online softmax,
  conditional rescaling and software exponential (same article, section 7,
  items 1-2) are exact reformulations of this plain softmax up to rounding,
  so the oracle is the plain definition: a naive two-pass softmax over an
  explicit P matrix, in fp64, with no tiling or fusion.
* The backward recomputes P (same article, section 5, "recomputation") and
  applies the analytic softmax Jacobian:
      dP = dO V^T,  delta_i = sum_j P_ij dP_ij,  dS = P o (dP - delta),
      dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO,
  with dK/dV of a shared (grouped) key/value head summed over its query heads.

Readings where the pages are silent (each stated once here):
* layout BSHD contiguous, D innermost; lse natural-log, shape [B, H_q, S_q];
* causal alignment bottom-right: key j is visible to query i iff
  j <= i + (S_k - S_q)  (identical to top-left when S_q == S_k);
* a row with no visible key has O = 0 and lse = -inf (and zero gradients);
* grouped-query attention: query head h reads key/value head h // (H_q / H_kv).

Numbers: inputs are the bf16 tensors both sides share, upcast exactly to fp64;
everything here is fp64.
"""
from __future__ import annotations

import numpy as np


def to_f64(x) -> np.ndarray:
    """Exact upcast of a (CPU) torch tensor or array to a float64 ndarray."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only for the dtype conversion of torch inputs

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def visible(S_q: int, S_k: int, causal: bool, rows=None) -> np.ndarray:
    """Boolean [len(rows), S_k] mask: True where key j is visible to query i."""
    rows = np.arange(S_q) if rows is None else np.asarray(rows)
    if not causal:
        return np.ones((len(rows), S_k), dtype=bool)
    j = np.arange(S_k)[None, :]
    return j <= (rows[:, None] + (S_k - S_q))


def _softmax_rows(s: np.ndarray):
    """Naive two-pass softmax of score rows (fp64). Returns (P, m, l).

    Pass 1: m_i = max_j s_ij.  Pass 2: p_ij = exp(s_ij - m_i), l_i = sum_j p_ij,
    P = p / l.  Rows whose scores are all -inf (nothing visible) give P = 0,
    m = -inf, l = 0.
    """
    m = s.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])  # exp(-inf) = 0 for masked entries
    l = p.sum(axis=1)
    l_safe = np.where(empty, 1.0, l)
    P = p / l_safe[:, None]
    P[empty] = 0.0
    return P, m, l


def _scores(qh: np.ndarray, kh: np.ndarray, scale: float, causal: bool, rows, S_q: int):
    s = scale * (qh @ kh.T)
    if causal:
        s = np.where(visible(S_q, kh.shape[0], True, rows), s, -np.inf)
    return s


def forward(q, k, v, causal: bool, scale: float, block_rows: int = 512):
    """O = softmax(scale Q K^T [+ mask]) V and lse, all heads, fp64.

    q [B,S_q,H_q,D], k/v [B,S_k,H_kv,D] -> o [B,S_q,H_q,D], lse [B,H_q,S_q].
    The explicit P matrix is formed block_rows query rows at a time only to
    bound memory; each row is computed independently of the others.
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, S_q, H_q, D = q.shape
    _, S_k, H_kv, _ = k.shape
    assert H_q % H_kv == 0
    G = H_q // H_kv
    o = np.zeros((B, S_q, H_q, v.shape[3]))
    lse = np.full((B, H_q, S_q), -np.inf)
    for b in range(B):
        for h in range(H_q):
            g = h // G
            kh, vh = k[b, :, g, :], v[b, :, g, :]
            for r0 in range(0, S_q, block_rows):
                rows = np.arange(r0, min(S_q, r0 + block_rows))
                s = _scores(q[b, rows, h, :], kh, scale, causal, rows, S_q)
                P, m, l = _softmax_rows(s)
                o[b, rows, h, :] = P @ vh
                with np.errstate(divide="ignore"):
                    lse[b, h, rows] = np.where(np.isfinite(m), m + np.log(np.where(l > 0, l, 1.0)),
                                               -np.inf)
    return o, lse


def forward_rows(q, k, v, causal: bool, scale: float, b: int, h: int, rows):
    """The forward for selected query rows of one (batch, query head) only.

    Used to check full-size outputs on a sample: each output row depends only
    on its own query row and all keys, so it can be computed alone.
    Returns (o_rows [n, D], lse_rows [n]).
    """
    rows = np.asarray(rows)
    H_q, H_kv = q.shape[2], k.shape[2]
    g = h // (H_q // H_kv)
    S_q = q.shape[1]
    idx = rows
    if hasattr(q, "detach"):
        import torch  # local: indexing a torch input with the row list

        idx = torch.as_tensor(rows)
    qh = to_f64(q[b, idx, h, :])
    kh = to_f64(k[b, :, g, :])
    vh = to_f64(v[b, :, g, :])
    s = _scores(qh, kh, scale, causal, rows, S_q)
    P, m, l = _softmax_rows(s)
    with np.errstate(divide="ignore"):
        lse = np.where(np.isfinite(m), m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return P @ vh, lse


def backward(q, k, v, do, causal: bool, scale: float, block_rows: int = 512, groups=None, batches=None):
    """Analytic gradients (dQ, dK, dV) of L = sum(dO o O) in fp64.

    P is recomputed from Q and K here (the oracle never takes the GPU's O or
    lse).  ``groups``/``batches`` restrict the work to some (b, h_kv) pairs
    (all their query heads); outputs outside them stay zero.
    """
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    B, S_q, H_q, D = q.shape
    _, S_k, H_kv, _ = k.shape
    G = H_q // H_kv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in (range(B) if batches is None else batches):
        for g in (range(H_kv) if groups is None else groups):
            kh, vh = k[b, :, g, :], v[b, :, g, :]
            for h in range(g * G, (g + 1) * G):
                for r0 in range(0, S_q, block_rows):
                    rows = np.arange(r0, min(S_q, r0 + block_rows))
                    qh, doh = q[b, rows, h, :], do[b, rows, h, :]
                    s = _scores(qh, kh, scale, causal, rows, S_q)
                    P, _, _ = _softmax_rows(s)
                    dP = doh @ vh.T
                    delta = (P * dP).sum(axis=1)
                    dS = P * (dP - delta[:, None])
                    dq[b, rows, h, :] = scale * (dS @ kh)
                    dk[b, :, g, :] += scale * (dS.T @ qh)
                    dv[b, :, g, :] += P.T @ doh
    return dq, dk, dv


def flops_fwd(B, H_q, S_q, S_k, D, causal) -> float:
    """FLOP convention for the forward: 4 B H S_q S_k D, halved when causal."""
    f = 4.0 * B * H_q * S_q * S_k * D
    return f / 2 if causal else f
