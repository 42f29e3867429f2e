"""The read-only stream probe that gives the select's second roofline
denominator: it must read every word of its buffer (the XOR it returns equals
the host's) and refuse buffers it cannot stream."""

import numpy as np
import pytest
import torch

from coreset_attention_approximation_b200 import wildcat


@pytest.mark.gpu
@pytest.mark.parametrize("words", [4, 4 * 1001, 1 << 26])
def test_read_probe_reads_every_word(words):
    g = torch.Generator(device="cuda").manual_seed(words)
    buf = torch.randint(-(2 ** 31), 2 ** 31 - 1, (words,), dtype=torch.int32, device="cuda", generator=g)
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    wildcat.read_probe(buf, sink)
    torch.cuda.synchronize()
    expect = np.bitwise_xor.reduce(buf.cpu().numpy().view(np.uint32))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(expect)


@pytest.mark.gpu
def test_read_probe_refuses_misaligned_or_ragged_buffers():
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(wildcat.WildcatError):
        wildcat.read_probe(buf[1:5], sink)      # 4-byte offset
    with pytest.raises(wildcat.WildcatError):
        wildcat.read_probe(buf[:3], sink)       # 12 bytes
