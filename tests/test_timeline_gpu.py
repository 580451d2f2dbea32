"""The timeline build records without changing results: the forward (with a CTA
selected for recording) and the backward main pass of libattn_timeline.so give
bitwise the outputs of libattn.so on the same inputs (the backward in its fixed dQ
order), and the recorded forward events are in pipeline order.  Each library runs
in its own process (the package loads one library per process)."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
from attention_attn_fwd_10_b200 import _abi, build
timeline = sys.argv[2] == "1"
lib = _abi.load(build.build(timeline=timeline))
import torch
import attention_attn_fwd_10_b200 as attn
g = torch.Generator().manual_seed(5)
B, S, H, D = 1, 1024, 4, 128
q, k, v, do = (torch.randn(B, S, H, D, generator=g).to(torch.bfloat16).cuda() for _ in range(4))
if timeline:
    lib.attn_timeline_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    ev = np.zeros((16, 256), dtype=np.int64); t0 = ctypes.c_longlong(0)
    assert lib.attn_timeline_read(ev.ctypes.data, ctypes.addressof(t0), 1) == 0
o, lse = attn.fwd(q, k, v, causal=True, persistent=False)
if timeline:  # the forward's events of CTA 1; the backward records nothing
    assert lib.attn_timeline_read(ev.ctypes.data, ctypes.addressof(t0), -1) == 0
dq, dk, dv = attn.bwd(q, k, v, o, lse, do, causal=True, deterministic=True, cta_mode=1)  # fixed dQ order
torch.cuda.synchronize()
assert attn.device_status() == 0
out = {n: t.float().cpu().numpy() for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
if timeline:
    out["ev"] = ev
np.savez(sys.argv[3], **out)
"""


def _run(timeline: bool, path: str):
    subprocess.run([sys.executable, "-c", CHILD, ROOT, "1" if timeline else "0", path], check=True, timeout=600)
    return np.load(path)


def test_timeline_build_changes_no_result(tmp_path):
    ref = _run(False, str(tmp_path / "ref.npz"))
    tl = _run(True, str(tmp_path / "tl.npz"))
    for n in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(ref[n], tl[n], equal_nan=True), n
    ev = tl["ev"]
    # CTA 1 of the forward recorded its blocks: for each, tile A's S ready, row max
    # done and P published, in that order
    n = int((ev[0] > 0).sum())
    assert n > 0
    assert np.all(ev[0, :n] <= ev[2, :n]) and np.all(ev[2, :n] <= ev[4, :n])
