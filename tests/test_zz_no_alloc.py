"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some integrations call this library where no allocation is possible -- under a
framework's memory pool they may not grow, from a plug-in or callback that has
no allocator handle, or on a latency path that must never reach cudaMalloc.
For them attn_bwd_noalloc takes its scratch from a fixed buffer built into the
library instead of a caller-provided workspace.  This test calls it through
the C ABI twice in a row on the same inputs (the second call must not see the
first call's leftovers in the shared buffer) and compares both results with
the workspace-based attn_bwd, within the gradient tolerance of the parity
tests.  The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import workloads
from oracle import reference as oracle_ref
from tests import parity

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20  # the fixed buffer's size, as include/attn.h states


def test_noalloc_backward_matches_workspace_backward_on_two_calls():
    import attention_attn_fwd_10_b200 as attn
    from attention_attn_fwd_10_b200 import _abi

    lib = _abi.load()
    w = workloads.small(B=1, H_q=4, H_kv=2, S_q=1000, S_k=1000, D=128, causal=True, seed=77, backward=True)
    assert lib.attn_bwd_workspace_size(w.B, w.H_q, w.S_q, w.D) <= SCRATCH_BYTES
    x = workloads.make_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.fwd(q, k, v, causal=True, scale=w.scale)
    ref = attn.bwd(q, k, v, o, lse, do, causal=True, scale=w.scale)  # caller-provided workspace
    torch.cuda.synchronize()
    ref = [parity.to_np(g) for g in ref]
    exact = oracle_ref.backward(x["q"], x["k"], x["v"], x["do"], True, w.scale)  # fp64 oracle
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rc = lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  w.B, w.H_q, w.H_kv, w.S_q, w.S_k, w.D, 1, ctypes.c_float(w.scale), stream)
        assert rc == 0, _abi.status_string(rc)
        assert lib.attn_device_status(stream) == 0
        for name, g, r, e in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, exact):
            parity.check_grad(g, r, f"noalloc {name} vs attn_bwd")
            parity.check_grad(g, e, f"noalloc {name} vs the oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    from attention_attn_fwd_10_b200 import _abi

    lib = _abi.load()
    w = workloads.BWD_CAUSAL  # needs ~130 MiB of scratch
    assert lib.attn_bwd_workspace_size(w.B, w.H_q, w.S_q, w.D) > SCRATCH_BYTES
    p = [16] * 9
    rc = lib.attn_bwd_noalloc(*p, w.B, w.H_q, w.H_kv, w.S_q, w.S_k, w.D, 1, ctypes.c_float(w.scale), None)
    assert rc == 6 and "SCRATCH_TOO_SMALL" in _abi.status_string(rc)
