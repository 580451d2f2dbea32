"""Pure-Python brute-force attention for tiny shapes -- TEST INFRASTRUCTURE ONLY.

A second, independent statement of the same definition as ``reference``
(nested loops, ``math.exp``, no numpy), used to pin the numpy oracle on
shapes with S <= 16.  Same readings: BSHD layout, bottom-right causal
alignment, H_q/H_kv contiguous query-head groups, natural-log lse.
"""
from __future__ import annotations

import math


def forward(q, k, v, causal, scale):
    """q/k/v nested lists [B][S][H][D] of floats -> (o [B][S_q][H_q][D], lse [B][H_q][S_q])."""
    B, S_q, H_q, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    S_k, H_kv = len(k[0]), len(k[0][0])
    G = H_q // H_kv
    o = [[[[0.0] * D for _ in range(H_q)] for _ in range(S_q)] for _ in range(B)]
    lse = [[[float("-inf")] * S_q for _ in range(H_q)] for _ in range(B)]
    for b in range(B):
        for h in range(H_q):
            g = h // G
            for i in range(S_q):
                scores = []
                for j in range(S_k):
                    if causal and j > i + (S_k - S_q):
                        continue
                    dot = 0.0
                    for d in range(D):
                        dot += q[b][i][h][d] * k[b][j][g][d]
                    scores.append((j, scale * dot))
                if not scores:
                    continue
                m = max(s for _, s in scores)
                w = [(j, math.exp(s - m)) for j, s in scores]
                l = sum(e for _, e in w)
                for d in range(D):
                    o[b][i][h][d] = sum(e * v[b][j][g][d] for j, e in w) / l
                lse[b][h][i] = m + math.log(l)
    return o, lse


def loss(q, k, v, do, causal, scale):
    """L = sum over all outputs of dO * O (the scalar whose gradients the backward returns)."""
    o, _ = forward(q, k, v, causal, scale)
    total = 0.0
    for b in range(len(o)):
        for i in range(len(o[0])):
            for h in range(len(o[0][0])):
                for d in range(len(o[0][0][0])):
                    total += do[b][i][h][d] * o[b][i][h][d]
    return total
