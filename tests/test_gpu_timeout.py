"""The bounded device-side waits: with a 0 ns limit every wait that does not succeed
at once gives up, the kernel records MOE_ETIMEOUT, drains its own copies and MMAs,
frees TMEM and returns; the host reads the status and the context stays usable."""
import pytest
import torch

import moe_synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [0, 1], ids=["in_out", "packed"])
def test_timeout_is_reported_and_context_survives(layout):
    import mixture_experts_softmax_b200 as m
    inp = moe_synth.make_inputs("tiny", device="cpu", T=256)
    layer = parity.to_dev(inp.layers[0])
    x = inp.x.cuda()
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == 0
    m.check(m.moe_set_weight_layout(h, layout))
    if layout == m.MOE_LAYOUT_PACKED:
        layer = m.pack_layer(h, layer)
    try:
        ref = torch.empty_like(x)
        m.check(m.moe_forward(h, 256, x, *m.layer_args(layer), ref))
        m.check(m.moe_sync_status(h))

        m.check(m.moe_set_timeout(h, 0))
        seen = []
        for _ in range(3):
            out = torch.empty_like(x)
            m.check(m.moe_forward(h, 256, x, *m.layer_args(layer), out))
            seen.append(m.moe_sync_status(h))
        assert m.MOE_ETIMEOUT in seen
        assert set(seen) <= {m.MOE_OK, m.MOE_ETIMEOUT}

        m.check(m.moe_set_timeout(h, 2_000_000_000))
        out = torch.empty_like(x)
        m.check(m.moe_forward(h, 256, x, *m.layer_args(layer), out))
        assert m.moe_sync_status(h) == m.MOE_OK
        assert torch.equal(out, ref)
    finally:
        m.moe_destroy(h)
