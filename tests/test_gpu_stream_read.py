"""gq_stream_read: the streaming-read calibration kernel reads every byte once.

Its result (the XOR of all 32-bit words) is checked against numpy, for sizes
that leave a ragged remainder after the four-loads-per-thread main loop, and
its argument checks against the header's rules.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_gemv_q4_b200 as m
    return m


@pytest.mark.parametrize("nbytes", [16, 48, 4096 + 16, 1 << 20, 25362432, 24305664 + 160])
def test_xor_of_every_word(gq, nbytes):
    rng = np.random.default_rng(nbytes)
    host = rng.integers(0, 256, size=nbytes, dtype=np.uint8)
    buf = torch.from_numpy(host).cuda()
    sink = gq.gq_stream_read(buf)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.view(np.uint32))
    assert int(sink.item()) & 0xFFFFFFFF == int(want)


def test_accumulates_into_sink(gq):
    host = np.arange(64, dtype=np.uint32)
    buf = torch.from_numpy(host.view(np.uint8).copy()).cuda()
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    gq.gq_stream_read(buf, sink)
    gq.gq_stream_read(buf, sink)  # the fold of the same bytes twice cancels
    torch.cuda.synchronize()
    assert int(sink.item()) == 0


def test_argument_checks(gq):
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(gq.GQError) as e:
        gq.gq_stream_read(buf[:40], sink)  # not a multiple of 16 bytes
    assert e.value.status == 2
    with pytest.raises(gq.GQError) as e:
        gq.gq_stream_read(buf[8:8 + 32], sink)  # not 16-byte aligned
    assert e.value.status == 3
    assert int(gq.gq_stream_read(buf[:0], sink).item()) == 0  # empty: nothing launched
