"""Seeded synthetic workloads for exact attention (shapes and input recipes only).

This module holds no attention arithmetic.  It is the one place that both the
CUDA path's tests/benchmark and the fp64 oracle draw their inputs from, so the
two sides see bit-identical bf16 tensors.

Layout (both sides): BSHD, contiguous, D innermost --
  q, o, dO : [B, S_q, H_q, D]
  k, v     : [B, S_k, H_kv, D]
  lse      : [B, H_q, S_q]   (fp32 on the GPU, fp64 in the oracle)

Recipe: values are standard normal fp32 drawn from a CPU ``torch.Generator``
seeded with ``1000 + index`` of the workload, then rounded to bf16
(round-to-nearest-even).  The "spiky keys" variant multiplies round(1% * S_k)
key rows of every (b, h_kv) by 8 after rounding (exact: a power of two); the
rows are drawn without replacement from a second generator seeded with
``seed + 100``.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    S_q: int
    S_k: int
    D: int
    causal: bool
    seed: int
    spiky_keys: bool = False  # 1% of K rows scaled by 8
    backward: bool = False     # needs dO as well

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def fwd_flops(self) -> float:
        """Forward FLOP convention: 4*B*H_q*S_q*S_k*D, halved for causal."""
        f = 4.0 * self.B * self.H_q * self.S_q * self.S_k * self.D
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Backward FLOP convention: 2.5x the forward's."""
        return 2.5 * self.fwd_flops()

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the measurements and parity tests are quoted on.
TINY = Workload("tiny_fwd_B1_H2_S256_D64", 1, 2, 2, 256, 256, 64, False, 1000)
FWD_NONCAUSAL = Workload("fwd_B4_H16_S2048_D128", 4, 16, 16, 2048, 2048, 128, False, 1001)
FWD_CAUSAL = Workload("fwd_causal_B2_H16_S8192_D128", 2, 16, 16, 8192, 8192, 128, True, 1002)
FWD_CAUSAL_SPIKY = FWD_CAUSAL.replace(name="fwd_causal_spikyK_B2_H16_S8192_D128", spiky_keys=True)
FWD_CAUSAL_GQA = Workload("fwd_causal_gqa_B1_Hq32_Hkv8_S32768_D128", 1, 32, 8, 32768, 32768, 128, True, 1003)
BWD_CAUSAL = Workload("bwd_causal_B2_H16_S8192_D128", 2, 16, 16, 8192, 8192, 128, True, 1004, backward=True)

ALL = [TINY, FWD_NONCAUSAL, FWD_CAUSAL, FWD_CAUSAL_SPIKY, FWD_CAUSAL_GQA, BWD_CAUSAL]


def _randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(w: Workload, seed: int | None = None, with_do: bool | None = None) -> dict:
    """Return CPU bf16 tensors q, k, v (and dO when the workload needs it)."""
    seed = w.seed if seed is None else seed
    with_do = w.backward if with_do is None else with_do
    gen = torch.Generator().manual_seed(seed)
    q = _randn_bf16((w.B, w.S_q, w.H_q, w.D), gen)
    k = _randn_bf16((w.B, w.S_k, w.H_kv, w.D), gen)
    v = _randn_bf16((w.B, w.S_k, w.H_kv, w.D), gen)
    out = {"q": q, "k": k, "v": v}
    if with_do:
        out["do"] = _randn_bf16((w.B, w.S_q, w.H_q, w.D), gen)
    if w.spiky_keys:
        out["k"] = spike_key_rows(k, seed + 100)
    return out


def spike_rows(S_k: int, B: int, H_kv: int, seed: int) -> torch.Tensor:
    """Indices [B, H_kv, n] of the key rows that get scaled by 8 (n = round(0.01*S_k))."""
    n = max(1, int(round(0.01 * S_k)))
    gen = torch.Generator().manual_seed(seed)
    idx = torch.empty((B, H_kv, n), dtype=torch.long)
    for b in range(B):
        for h in range(H_kv):
            idx[b, h] = torch.randperm(S_k, generator=gen)[:n]
    return idx


def spike_key_rows(k: torch.Tensor, seed: int) -> torch.Tensor:
    B, S_k, H_kv, _ = k.shape
    idx = spike_rows(S_k, B, H_kv, seed)
    k = k.clone()
    for b in range(B):
        for h in range(H_kv):
            k[b, idx[b, h], h, :] = k[b, idx[b, h], h, :] * 8  # power of two: exact in bf16
    return k


def small(B=1, H_q=2, H_kv=None, S_q=256, S_k=None, D=64, causal=False, seed=7, backward=False,
          spiky_keys=False) -> Workload:
    """An ad-hoc small workload for parity/edge-case tests."""
    H_kv = H_q if H_kv is None else H_kv
    S_k = S_q if S_k is None else S_k
    name = f"small_B{B}_Hq{H_q}_Hkv{H_kv}_Sq{S_q}_Sk{S_k}_D{D}_{'causal' if causal else 'full'}"
    return Workload(name, B, H_q, H_kv, S_q, S_k, D, causal, seed, spiky_keys=spiky_keys,
                    backward=backward)
