"""md_stream_read: the read-bandwidth diagnostic runs, folds without writing
the sink for ordinary data, and refuses misaligned or ragged buffers."""
import pytest

import medusa_draft_heads_b200 as md

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_stream_read_runs_and_leaves_sink():
    buf = torch.arange(1 << 22, dtype=torch.int32, device="cuda")     # values < 2^22 never fold to the marker
    sink = torch.full((1,), -5, dtype=torch.int32, device="cuda")
    md.stream_read(buf, sink)
    torch.cuda.synchronize()
    assert int(sink.item()) == -5
    assert md.device_status() == 0


def test_stream_read_refuses_bad_sizes():
    buf = torch.zeros(9, dtype=torch.int32, device="cuda")            # 36 bytes: not a multiple of 16
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(md.MedusaError):
        md.stream_read(buf, sink)
    with pytest.raises(md.MedusaError):
        md.stream_read(buf[1:5], sink)                                  # 16 bytes at a 4-byte offset
