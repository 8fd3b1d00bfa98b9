"""moe_route_noalloc: the layer's routing (router + dispatch) for callers that cannot
allocate device memory -- code inside a device-memory arena sized once up front, or
inside a framework that owns the allocator.  Its dispatch scratch is a static device
array, so the call allocates nothing.

Checked here, through the C ABI, on calls in a row with different token counts (the
one-block-per-token router up to 256 tokens and the four-tokens-per-warp router above):
the same expert indices, gates, expert offsets and grouped order as the full layer
(moe_forward, read back with moe_get_routing) where both run the same router kernel,
agreement with the fp64 oracle outside near ties at every size, and no change in free
device memory.  This file is collected last so that a failure here never hides another
test."""
import types

import numpy as np
import pytest
import torch

import moe_synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

SIZES = [1500, 321, 8, 32, 200]   # > 256: four tokens per warp; <= 256: one block per token


def _routing_via_forward(m, layer, x):
    T, d = x.shape
    rc, h = m.moe_create(d, layer["wl"].shape[2], 8, 2)
    m.check(rc)
    try:
        run = parity.Run(h, x, layer)
    finally:
        m.moe_destroy(h)
    return run


def test_route_noalloc_matches_forward_and_oracle():
    import mixture_experts_softmax_b200 as m
    dev = torch.device("cuda", 0)
    inp = moe_synth.make_inputs("tiny", device="cpu", T=1500)
    layer = parity.to_dev(inp.layers[0], dev)
    starts = {1500: 0, 321: 100, 8: 7, 32: 900, 200: 1234}
    cases = [inp.x[starts[T]:starts[T] + T] for T in SIZES]
    outs = []
    for x in cases:
        T = x.shape[0]
        outs.append(dict(idx=torch.empty((T, 2), dtype=torch.int32, device=dev),
                         gate=torch.empty((T, 2), dtype=torch.float32, device=dev),
                         offsets=torch.empty(9, dtype=torch.int32, device=dev),
                         perm=torch.empty(2 * T, dtype=torch.int32, device=dev)))
    xs = [x.to(dev) for x in cases]
    # the full layer's routing of the two large batches (the same router kernel as the entry point)
    refs = [_routing_via_forward(m, layer, x) for x in xs[:2]]
    torch.cuda.synchronize(dev)

    def call(x, o):
        m.check(m.moe_route_noalloc(x.shape[0], x.shape[1], x, layer["router_w"], None,
                                    o["idx"], o["gate"], o["offsets"], o["perm"]), "moe_route_noalloc")

    # the first call on a device looks up the scratch address; free memory must not move after it
    call(xs[0], outs[0])
    torch.cuda.synchronize(dev)
    free_before = torch.cuda.mem_get_info(dev)[0]
    for x, o in zip(xs[1:], outs[1:]):
        call(x, o)
    torch.cuda.synchronize(dev)
    assert torch.cuda.mem_get_info(dev)[0] == free_before
    for o, ref in zip(outs, refs):
        assert np.array_equal(o["idx"].cpu().numpy(), ref.idx_h)
        np.testing.assert_allclose(o["gate"].cpu().numpy(), ref.gate_h, rtol=parity.GATE_RTOL, atol=1e-7)
        assert np.array_equal(o["offsets"].cpu().numpy(), ref.offsets_h)
        assert np.array_equal(o["perm"].cpu().numpy(), ref.perm_h)
    # every call against the oracle: bit-exact experts and grouping outside near ties
    for x, o in zip(cases, outs):
        got = types.SimpleNamespace(idx_h=o["idx"].cpu().numpy(), gate_h=o["gate"].cpu().numpy(),
                                    offsets_h=o["offsets"].cpu().numpy(), perm_h=o["perm"].cpu().numpy())
        parity.check_routing(got, oracle.route(x, inp.layers[0]["router_w"]), 8)


def test_route_noalloc_rejects_oversize():
    import mixture_experts_softmax_b200 as m
    A = 1 << 20   # aligned dummy addresses: the size check comes before any use
    assert m.moe_route_noalloc(m.MOE_NOALLOC_MAX_TOKENS + 1, 256, A, A, None, A, A, A, A, 0) == m.MOE_EINVAL
