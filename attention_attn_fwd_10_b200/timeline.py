"""Per-block clock64 timeline of one CTA, from the timeline build of the library.

    python -m attention_attn_fwd_10_b200.timeline fwd [--cta 0 300] [--S 8192]
    python -m attention_attn_fwd_10_b200.timeline bwd [--cta 0 40] [--deterministic]
    python -m attention_attn_fwd_10_b200.timeline bwd_pairs [--cta 0 40] [--deterministic]
    python -m attention_attn_fwd_10_b200.timeline decode [--cta 0] [--S 32768]

Builds libattn_timeline.so if needed (the same sources with -DATTN_TIMELINE), loads
it instead of libattn.so, runs on N(0, 1) inputs the causal B2 H16 S D128 forward (one
CTA per work unit), the backward main pass (one CTA per key tile, or `bwd_pairs`: CTA
pairs, whose even CTA holds the MMA issuer), or (`decode`) the split-KV forward of one
query row per head of B1 H32/8 against S keys, and prints, for each selected CTA,
the first and last blocks' event times (SM clocks from the CTA's start) and the
median of each step between events over the steady-state blocks.  The events are
listed in include/attn_timeline.h.  A measurement aid: nothing in the package uses
it.
"""
from __future__ import annotations

import argparse
import ctypes
import math

import numpy as np

from . import _abi, build as _build

N_EVENTS, N_BLOCKS = 16, 256

FWD_NAMES = {0: "A S ready", 1: "B S ready", 2: "A max done", 3: "B max done", 4: "A P pub", 5: "B P pub",
             6: "PV_A iss", 7: "PV_B iss", 8: "S_A iss", 9: "S_B iss", 10: "V ready", 15: "V load iss"}
# (label, from event, to event, block shift of the second event); events 8/9 of block
# j are the issue of S_t(j), which follows PV_t(j - 1)
FWD_STEPS = [("S_A ready -> row max done", 0, 2, 0), ("row max done -> P_A published", 2, 4, 0),
             ("P_A published -> PV_A issued", 4, 6, 0), ("PV_A(j) issued -> S_A(j+1) issued", 6, 8, 1),
             ("S_A issued -> S_A ready", 8, 0, 0), ("S_A ready -> S_B ready (same j)", 0, 1, 0),
             ("V load issued -> V ready at the issuer", 15, 10, 0),
             ("period: S_A(j) ready -> S_A(j+1) ready", 0, 0, 1)]
BWD_NAMES = {0: "S/dP iss", 1: "S ready", 2: "dS pub", 3: "dS seen", 4: "dV/dK iss", 5: "dQ iss",
             6: "dQ ready", 7: "staged", 8: "red iss", 9: "red done", 10: "turn"}
BWD_STEPS = [("S^T/dP^T issued -> S^T ready at the softmax", 0, 1, 0), ("S^T ready -> dS^T published", 1, 2, 0),
             ("dS^T published -> seen by the issuer", 2, 3, 0), ("dS^T seen -> dV/dK issued", 3, 4, 0),
             ("dV/dK issued -> dQ^T issued", 4, 5, 0), ("dQ^T issued -> ready at staging", 5, 6, 0),
             ("dQ^T ready -> tile staged", 6, 7, 0), ("staged -> reduce-add issued", 7, 8, 0),
             ("reduce-add issued -> source read (fixed order: done)", 8, 9, 0),
             ("staged -> turn received (fixed order)", 7, 10, 0),
             ("period: S^T ready(i) -> S^T ready(i+1)", 1, 1, 1)]
PAIR_NAMES = {**BWD_NAMES, 11: "dS sent", 12: "dS both", 13: "peer half"}
PAIR_STEPS = BWD_STEPS[:2] + [("dS^T published -> half sent to the other CTA", 2, 11, 0),
                              ("dS^T published -> dQ^T inputs ready at the issuer", 2, 12, 0),
                              ("S^T ready -> dS^T half sent", 1, 11, 0),
                              ("S^T ready -> the other CTA's half landed (odd CTA)", 1, 13, 0)] + BWD_STEPS[2:]


def _load_timeline_lib() -> ctypes.CDLL:
    path = _build.build(timeline=True)
    lib = _abi.load(path)  # the package's calls go through this library from now on
    if not hasattr(lib, "attn_timeline_read"):
        raise RuntimeError(f"{path} has no timeline (built without -DATTN_TIMELINE)")
    lib.attn_timeline_read.restype = ctypes.c_int
    lib.attn_timeline_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return lib


def _read(lib, next_cta: int) -> tuple[np.ndarray, int]:
    ev = np.zeros((N_EVENTS, N_BLOCKS), dtype=np.int64)
    t0 = ctypes.c_longlong(0)
    code = lib.attn_timeline_read(ev.ctypes.data, ctypes.addressof(t0), next_cta)
    _abi.check(code, "attn_timeline_read")
    return ev, int(t0.value)


def _report(ev: np.ndarray, t0: int, names: dict, steps: list, out=print) -> None:
    cols = sorted(names)
    n = int(max((ev[e] > 0).sum() for e in cols))
    out("    j " + " ".join(f"{names[e][:10]:>10s}" for e in cols))
    for i in list(range(min(n, 6))) + list(range(max(6, n - 3), n)):
        out(f"  {i:3d} " + " ".join(f"{int(ev[e, i] - t0) if ev[e, i] else -1:10d}" for e in cols))
    for label, a, b, sh in steps:
        na = int((ev[a] > 0).sum())
        # steady state: skip the first 4 blocks (pipeline fill) and the last 2 (drain)
        d = [ev[b, i + sh] - ev[a, i] for i in range(min(4, na), na - 2) if i + sh < N_BLOCKS and ev[b, i + sh]]
        out(f"  {label:48s} median {float(np.median(d)) if d else float('nan'):8.0f} clk  ({len(d)} blocks)")


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("pass_", choices=("fwd", "bwd", "bwd_pairs", "decode"), metavar="fwd|bwd|bwd_pairs|decode")
    ap.add_argument("--cta", type=int, nargs="+", default=None, help="CTA indices to record (blockIdx.x)")
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--S", type=int, default=8192)
    ap.add_argument("--deterministic", action="store_true", help="bwd: the fixed-order dQ instance")
    args = ap.parse_args(argv)

    lib = _load_timeline_lib()
    import torch

    from . import bwd as attn_bwd, fwd as attn_fwd

    torch.manual_seed(1)
    dev = torch.device("cuda", torch.cuda.current_device())
    B, H, S, D = args.B, args.H, args.S, 128
    scale = 1.0 / math.sqrt(D)
    ctas = args.cta if args.cta is not None else [0, 40]
    if args.pass_ == "decode":
        from . import fwd_split as attn_fwd_split

        B, H = 1, 32
        S = args.S if args.S != 8192 else 32768
        q = torch.randn(B, 1, H, D, device=dev).to(torch.bfloat16)
        k, v = (torch.randn(B, S, 8, D, device=dev).to(torch.bfloat16) for _ in range(2))
        o, lse = attn_fwd_split(q, k, v, causal=True, scale=scale)
        run = lambda: attn_fwd_split(q, k, v, causal=True, scale=scale, out=o, lse=lse)  # noqa: E731
        names, steps = FWD_NAMES, FWD_STEPS
    else:
        q, k, v = (torch.randn(B, S, H, D, device=dev).to(torch.bfloat16) for _ in range(3))
        o, lse = attn_fwd(q, k, v, causal=True, scale=scale, persistent=False)
    if args.pass_ == "fwd":
        run = lambda: attn_fwd(q, k, v, causal=True, scale=scale, out=o, lse=lse, persistent=False)  # noqa: E731
        names, steps = FWD_NAMES, FWD_STEPS
    elif args.pass_ in ("bwd", "bwd_pairs"):
        do = torch.randn(B, S, H, D, device=dev).to(torch.bfloat16)
        mode = 1 if args.pass_ == "bwd" else 2
        run = lambda: attn_bwd(q, k, v, o, lse, do, causal=True, scale=scale, cta_mode=mode,  # noqa: E731
                               deterministic=args.deterministic)
        names, steps = (BWD_NAMES, BWD_STEPS) if mode == 1 else (PAIR_NAMES, PAIR_STEPS)
    for cta in ctas:
        _read(lib, cta)
        for _ in range(3):  # warm-up calls, recorded and discarded
            run()
        _read(lib, cta)
        run()
        ev, t0 = _read(lib, -1)
        print(f"{args.pass_} causal B{B} H{H} S{S} D{D}, CTA {cta} (SM clocks from the CTA's start)")
        _report(ev, t0, names, steps)
    status = _abi.load().attn_device_status(None)
    _abi.check(status, "device status")


if __name__ == "__main__":
    main()
