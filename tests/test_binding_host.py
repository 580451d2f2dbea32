"""Host-side logic of the Python binding that needs no GPU: every tensor of a
call must live on one CUDA device (the library runs its kernels on the current
device and reads operands with TMA, which must never be handed another GPU's
memory), and a given stream must belong to that device."""
import types

import pytest
import torch

import attention_attn_fwd_10_b200 as attn


def _fake(device: str):
    return types.SimpleNamespace(is_cuda=device.startswith("cuda"), device=torch.device(device))


def test_one_device_is_accepted():
    assert attn._device_of(_fake("cuda:1"), _fake("cuda:1"), None) == torch.device("cuda:1")


def test_mixed_devices_are_rejected():
    with pytest.raises(ValueError, match="different devices"):
        attn._device_of(_fake("cuda:0"), _fake("cuda:1"))


def test_host_tensor_among_device_tensors_is_rejected():
    with pytest.raises(ValueError, match="CUDA tensor"):
        attn._device_of(_fake("cuda:0"), _fake("cpu"))


def test_stream_of_another_device_is_rejected():
    stream = types.SimpleNamespace(device=torch.device("cuda:1"), cuda_stream=1234)
    with pytest.raises(ValueError, match="stream is on"):
        attn._stream_ptr(stream, torch.device("cuda:0"))
    assert attn._stream_ptr(stream, torch.device("cuda:1")) == 1234


def test_timeline_report_medians():
    """The timeline tool's step medians: event b of block i + shift minus event a of
    block i over the steady-state blocks (the first 4 and the last 2 are skipped)."""
    import numpy as np

    from attention_attn_fwd_10_b200 import timeline

    n = 12
    ev = np.zeros((timeline.N_EVENTS, timeline.N_BLOCKS), dtype=np.int64)
    for i in range(n):
        ev[0, i] = 1000 + 3000 * i  # S ready, period 3000
        ev[2, i] = ev[0, i] + 500   # row max 500 later
    lines = []
    timeline._report(ev, 0, {0: "S", 2: "max"}, [("max", 0, 2, 0), ("period", 0, 0, 1)], out=lines.append)
    med = {ln.split()[0]: float(ln.split("median")[1].split()[0]) for ln in lines if "median" in ln}
    assert med == {"max": 500.0, "period": 3000.0}
