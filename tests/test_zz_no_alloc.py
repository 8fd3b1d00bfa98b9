"""moe_route_noalloc: the layer's routing (router + dispatch) for callers that cannot
allocate device memory -- code inside a device-memory arena sized once up front, or
inside a framework that owns the allocator.  Its dispatch scratch is a static device
array, so the call allocates nothing.

Checked here, through the C ABI, on two calls in a row: the same expert indices,
gates, expert offsets and grouped order as the full layer (moe_forward, read back
with moe_get_routing) on the same inputs, and no change in free device memory.
This file is collected last so that a failure here never hides another test."""
import numpy as np
import pytest
import torch

import moe_synth
from tests import parity

pytestmark = pytest.mark.gpu


def _routing_via_forward(m, layer, x):
    T, d = x.shape
    rc, h = m.moe_create(d, layer["wl"].shape[2], 8, 2)
    m.check(rc)
    try:
        run = parity.Run(h, x, layer)
    finally:
        m.moe_destroy(h)
    return run


def test_route_noalloc_matches_forward_twice():
    import mixture_experts_softmax_b200 as m
    dev = torch.device("cuda", 0)
    inp = moe_synth.make_inputs("tiny", device="cpu", T=1500)
    layer = parity.to_dev(inp.layers[0], dev)
    cases = [inp.x[:1500].to(dev), inp.x[100:421].to(dev)]     # two calls in a row, different T
    refs = [_routing_via_forward(m, layer, x) for x in cases]
    outs = []
    for x in cases:
        T = x.shape[0]
        outs.append(dict(idx=torch.empty((T, 2), dtype=torch.int32, device=dev),
                         gate=torch.empty((T, 2), dtype=torch.float32, device=dev),
                         offsets=torch.empty(9, dtype=torch.int32, device=dev),
                         perm=torch.empty(2 * T, dtype=torch.int32, device=dev)))
    torch.cuda.synchronize(dev)
    # the first call on a device looks up the scratch address; free memory must not move after it
    x, o = cases[0], outs[0]
    m.check(m.moe_route_noalloc(x.shape[0], x.shape[1], x, layer["router_w"], None,
                                o["idx"], o["gate"], o["offsets"], o["perm"]), "moe_route_noalloc")
    torch.cuda.synchronize(dev)
    free_before = torch.cuda.mem_get_info(dev)[0]
    x, o = cases[1], outs[1]
    m.check(m.moe_route_noalloc(x.shape[0], x.shape[1], x, layer["router_w"], None,
                                o["idx"], o["gate"], o["offsets"], o["perm"]), "moe_route_noalloc")
    torch.cuda.synchronize(dev)
    assert torch.cuda.mem_get_info(dev)[0] == free_before
    for o, ref in zip(outs, refs):
        assert np.array_equal(o["idx"].cpu().numpy(), ref.idx_h)
        np.testing.assert_allclose(o["gate"].cpu().numpy(), ref.gate_h, rtol=parity.GATE_RTOL, atol=1e-7)
        assert np.array_equal(o["offsets"].cpu().numpy(), ref.offsets_h)
        assert np.array_equal(o["perm"].cpu().numpy(), ref.perm_h)


def test_route_noalloc_rejects_oversize():
    import mixture_experts_softmax_b200 as m
    A = 1 << 20   # aligned dummy addresses: the size check comes before any use
    assert m.moe_route_noalloc(m.MOE_NOALLOC_MAX_TOKENS + 1, 256, A, A, None, A, A, A, A, 0) == m.MOE_EINVAL
