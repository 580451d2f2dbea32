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
