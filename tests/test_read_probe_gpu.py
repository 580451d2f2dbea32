"""attn_read_probe, the plain-read yardstick the bench puts beside the decode line:
it reads every byte it is given (its fold of a planted word reaches the sink) and
leaves the device status clean."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_read_probe_reads_its_input():
    import attention_attn_fwd_10_b200 as attn

    lib = attn.load()
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    # one 16-byte word: a single thread folds it, and the fold equals the probe's marker
    one = torch.tensor([0x9E3779B9 - (1 << 32), 0, 0, 0], dtype=torch.int64).to(torch.int32).cuda()
    assert lib.attn_read_probe(one.data_ptr(), 16, sink.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert sink.item() == 1
    # a large zero buffer folds to 0: the sink is untouched
    big = torch.zeros(64 << 20, dtype=torch.int32, device="cuda")
    assert lib.attn_read_probe(big.data_ptr(), big.numel() * 4, sink.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert sink.item() == 1
    assert attn.device_status() == 0
