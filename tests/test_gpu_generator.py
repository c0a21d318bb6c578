"""The device twin of the seeded generator gives the host generator's bits."""
import numpy as np
import pytest

from seeded_inputs import device, gen

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,start,sigma", [(1, 0, 1.0), (1000, 0, 0.02), (1 << 20, 12345, 0.02),
                                           (4097, (1 << 33) + 7, 3.0)])
def test_device_bf16_and_f32_draws_match_host(n, start, sigma):
    key = gen.stream_key(3, "Wv")
    tb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    device.fill_normal(tb, 3, "Wv", sigma, start=start)
    tf = torch.empty(n, dtype=torch.float32, device="cuda")
    device.fill_normal(tf, 3, "Wv", sigma, start=start)
    idx = np.arange(start, start + n, dtype=np.uint64)
    hb = gen.normal_bf16_at(key, idx, sigma)
    hf = gen.normal_f32_at(key, idx, sigma)
    assert np.array_equal(tb.cpu().view(torch.int16).numpy().view(np.uint16), hb)
    assert np.array_equal(tf.cpu().numpy().view(np.uint32), hf.view(np.uint32))


def test_device_planting_matches_host():
    from seeded_inputs import synth
    from oracle import tree as ot
    from seeded_inputs.workloads import TREE_ACCEPT
    parent, _, _ = ot.spec_from_tuples(ot.select_tree((10, 10, 10, 10), TREE_ACCEPT, 16))
    tokens = synth.synthetic_tree_tokens(4, 3, parent, 5000)
    host = synth.planted_logits(4, parent, tokens, 5000, TREE_ACCEPT, sigma=3.0, bump=3.0)
    dev = synth.planted_logits_device(4, parent, tokens, 5000, TREE_ACCEPT, sigma=3.0, bump=3.0)
    assert np.array_equal(dev.cpu().numpy().view(np.uint32), host.view(np.uint32))
