"""Expert parallelism through the C ABI on one GPU: W ranks' handles, each holding its E/W
experts, driven from one process (mixture_experts_softmax_b200.ep.forward_local: the
ranks' steps run one after another, the exchanges are local all-to-alls), so every
kernel of the multi-rank path runs without any rank waiting for another.  Every rank's
output is compared with the fp64 oracle on its own tokens, routing bit-exact outside
near ties, in both weight layouts, at the tiny shape (W = 2, 4, 8; uneven, small and
masked batches) and at the Grok-1 shape (W = 8: one expert per rank, decode batches).
"""
import types

import numpy as np
import pytest
import torch

import moe_synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def _check_rank(rk, out, x_cpu, layer_cpu, mask=None):
    import mixture_experts_softmax_b200 as m
    T = x_cpu.shape[0]
    if T == 0:
        return
    rb = parity.read_routing(rk.layer.h, T)
    run = types.SimpleNamespace(out_h=out.cpu(), **vars(rb))
    ref = oracle.route(x_cpu, layer_cpu["router_w"])
    if mask is None:
        near = parity.check_routing(run, ref, 8)
        parity.check_output(run, layer_cpu, x_cpu, range(T), near)
        return
    pad = mask.numpy() == 0
    assert (rb.idx_h[pad] == -1).all() and torch.all(run.out_h[torch.from_numpy(pad)] == 0)
    near = oracle.near_ties(ref["probs"], parity.NEAR_TIE) & ~pad
    ok = ~pad & ~near
    assert np.array_equal(rb.idx_h[ok], ref["idx"][ok])
    real = np.nonzero(~pad & ~near)[0].tolist()
    parity.check_output(run, layer_cpu, x_cpu, real, near)


@pytest.mark.parametrize("packed", [True, False], ids=["packed", "in_out"])
@pytest.mark.parametrize("world", [2, 4, 8])
def test_ep_tiny_matches_oracle(world, packed):
    from mixture_experts_softmax_b200 import ep
    import mixture_experts_softmax_b200 as m
    layer_cpu = moe_synth.make_inputs("tiny", device="cpu").layers[0]
    full = parity.to_dev(layer_cpu)
    sizes = [37, 5, 300, 1, 64, 17, 0, 128][:world]
    ranks = [ep.EPRank(256, 512, world, r, ep.slice_experts(full, *ep.expert_range(8, world, r)), packed=packed)
             for r in range(world)]
    try:
        xs = [moe_synth.draw_tokens(T, 256, moe_synth.generator(200 + r, "cpu"), "cpu") for r, T in enumerate(sizes)]
        mask = None
        if world == 2:   # rank 0's batch has padding tokens
            g = torch.Generator().manual_seed(5)
            mask = (torch.rand(sizes[0], generator=g) > 0.3).to(torch.uint8)
            mask_dev = mask.cuda()
            m.check(m.moe_set_padding_mask(ranks[0].layer.h, mask_dev))
        outs = [torch.empty((T, 256), dtype=torch.bfloat16, device="cuda") for T in sizes]
        ep.forward_local(ranks, [x.cuda() for x in xs], outs)
        for r, rk in enumerate(ranks):
            m.check(m.moe_sync_status(rk.layer.h))
            _check_rank(rk, outs[r], xs[r], layer_cpu, mask if r == 0 else None)
    finally:
        for rk in ranks:
            rk.close()


def test_ep_grok_decode_one_expert_per_rank():
    """Grok-1 shape, W = 8 (one expert per rank, the pages' 8-way layout), 8 decode tokens per
    rank; the packed layout."""
    from mixture_experts_softmax_b200 import ep
    import mixture_experts_softmax_b200 as m
    inp = moe_synth.make_inputs("decode", device="cuda")
    full = inp.layers[0]
    layer_cpu = parity.to_cpu(full)
    W = 8
    ranks = [ep.EPRank(6144, 32768, W, r, ep.slice_experts(full, *ep.expert_range(8, W, r)), packed=True)
             for r in range(W)]
    del inp, full
    torch.cuda.empty_cache()
    try:
        xs = [moe_synth.draw_tokens(8, 6144, moe_synth.generator(300 + r, "cuda"), "cuda") for r in range(W)]
        outs = [torch.empty_like(x) for x in xs]
        ep.forward_local(ranks, xs, outs)
        for r, rk in enumerate(ranks):
            m.check(m.moe_sync_status(rk.layer.h))
            _check_rank(rk, outs[r], xs[r].cpu(), layer_cpu)
    finally:
        for rk in ranks:
            rk.close()
        torch.cuda.empty_cache()
