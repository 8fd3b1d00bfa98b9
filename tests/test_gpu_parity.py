"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Small shapes are compared on every token and span several tiles, ragged tails
and every tile width the library picks; the Grok-1-shape workloads (decode T=8,
prefill T=8192, skewed T=4096, four stacked residual blocks T=32) are compared
on all tokens where the oracle is cheap and on seeded token samples otherwise,
in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import moe_synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import mixture_experts_softmax_b200 as m
    return m


@pytest.fixture(scope="module")
def tiny_inputs():
    inp = moe_synth.make_inputs("tiny", device="cpu", T=1024)
    return inp


LAYOUTS = [0, 1]   # MOE_LAYOUT_IN_OUT (weights through shared memory), MOE_LAYOUT_PACKED (packed tiles, through TMEM)


@pytest.fixture(scope="module", params=LAYOUTS, ids=["in_out", "packed"])
def tiny_handle(m, request, tiny_inputs):
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == 0
    m.check(m.moe_set_weight_layout(h, request.param))
    dev = parity.to_dev(tiny_inputs.layers[0])
    if request.param == m.MOE_LAYOUT_PACKED:
        dev = m.pack_layer(h, dev)
    yield h, dev, request.param
    m.moe_destroy(h)


def _run_tiny(m, hl, inp, T, bias=None, x=None):
    h, dev, _ = hl
    layer_cpu = inp.layers[0]
    x_cpu = inp.x[:T] if x is None else x
    run = parity.Run(h, x_cpu.cuda(), dev, None if bias is None else bias.cuda())
    ref = oracle.route(x_cpu, layer_cpu["router_w"], bias)
    near = parity.check_routing(run, ref, 8)
    return run, layer_cpu, x_cpu, near


@pytest.mark.parametrize("T", [64, 1, 3, 16, 17, 32, 33, 65, 127, 300, 1000])
def test_tiny_all_tokens(m, tiny_inputs, tiny_handle, T):
    run, layer, x, near = _run_tiny(m, tiny_handle, tiny_inputs, T)
    parity.check_output(run, layer, x, range(T), near)


def test_tiny_zero_input_is_exact_zero(m, tiny_inputs, tiny_handle):
    x0 = torch.zeros(40, 256, dtype=torch.bfloat16)
    run, layer, x, near = _run_tiny(m, tiny_handle, tiny_inputs, 40, x=x0)
    assert (run.out_h == 0).all()
    assert (run.idx_h == [[0, 1]] * 40).all()


def test_tiny_all_routes_to_one_expert(m, tiny_inputs, tiny_handle):
    """+100 on expert 3: every token sends slot 0 there; skew and empty experts."""
    bias = torch.tensor([0, 0, 0, 100.0, 0, 0, 0, 0])
    run, layer, x, near = _run_tiny(m, tiny_handle, tiny_inputs, 300, bias=bias)
    assert (run.idx_h[:, 0] == 3).all()
    parity.check_output(run, layer, x, range(300), near, bias_cpu=bias)


@pytest.mark.parametrize("T", [13, 16, 32])
def test_tiny_small_batch_one_expert_full_tile(m, tiny_inputs, tiny_handle, T):
    """Small batches with +100 on expert 3: that expert's tile holds all T routes (a full
    16- or 32-row tile at T = 16, 32; a ragged one at 13), the other experts share the
    second picks; covers the up-projection's own row gather at every fill level."""
    bias = torch.tensor([0, 0, 0, 100.0, 0, 0, 0, 0])
    run, layer, x, near = _run_tiny(m, tiny_handle, tiny_inputs, T, bias=bias)
    assert (run.idx_h[:, 0] == 3).all()
    parity.check_output(run, layer, x, range(T), near, bias_cpu=bias)


def test_tiny_only_two_experts_used(m, tiny_inputs, tiny_handle):
    bias = torch.tensor([0, 0, 0, 0, 0, 60.0, 0, 50.0])
    run, layer, x, near = _run_tiny(m, tiny_handle, tiny_inputs, 200, bias=bias)
    assert set(np.unique(run.idx_h).tolist()) == {5, 7}
    assert run.offsets_h.tolist() == [0, 0, 0, 0, 0, 0, 200, 200, 400]
    parity.check_output(run, layer, x, range(200), near, bias_cpu=bias)


def test_tiny_deterministic(m, tiny_inputs, tiny_handle):
    a, *_ = _run_tiny(m, tiny_handle, tiny_inputs, 1000)
    b, *_ = _run_tiny(m, tiny_handle, tiny_inputs, 1000)
    assert torch.equal(a.out_h, b.out_h)
    assert np.array_equal(a.perm_h, b.perm_h)


def test_tiny_token_permutation(m, tiny_inputs, tiny_handle):
    """Permuting the tokens permutes the outputs (bit-exactly: no cross-token arithmetic)."""
    T = 300
    P = torch.randperm(T, generator=torch.Generator().manual_seed(9))
    a, *_ = _run_tiny(m, tiny_handle, tiny_inputs, T)
    b, *_ = _run_tiny(m, tiny_handle, tiny_inputs, T, x=tiny_inputs.x[:T][P])
    assert torch.equal(b.out_h, a.out_h[P])


@pytest.mark.parametrize("T", [100, 8, 32])
def test_forward_host_matches_device_path(m, tiny_inputs, tiny_handle, T):
    """Host buffers give the device path's result bit for bit.  For T <= 32 the staged input
    already is the routed-rows buffer the packed up-projection reads, so nothing is copied."""
    h, layer, _ = tiny_handle
    m.check(m.moe_set_router_bias(h, None))    # the handle is shared: no state from earlier tests
    m.check(m.moe_set_padding_mask(h, None))
    x_host = tiny_inputs.x[:T].clone().pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()
    m.check(m.moe_forward_host(h, T, x_host, *m.layer_args(layer), out_host))
    m.check(m.moe_sync_status(h))
    run = parity.Run(h, x_host.cuda(), layer)
    assert torch.equal(out_host, run.out_h)


def test_host_overlap_matches_serial(m, tiny_inputs, tiny_handle):
    """moe_set_host_overlap: calls alternating between two staging slots, input copies on the
    handle's copy stream, give the serial path's results bit for bit.  The chain feeds each
    call's host output to the next call as its input (the copy in must wait for it), changes
    T on the way (the slots grow) and ends on a small batch (the staged input is copied into
    the routed-rows buffer)."""
    h, layer, _ = tiny_handle
    m.check(m.moe_set_router_bias(h, None))
    m.check(m.moe_set_padding_mask(h, None))
    sizes = [100, 100, 300, 300, 8]
    x0 = tiny_inputs.x[:300].clone().pin_memory()

    def chain():
        outs = [torch.empty((T, 256), dtype=torch.bfloat16).pin_memory() for T in sizes]
        src = x0
        for i, (T, out) in enumerate(zip(sizes, outs)):
            m.check(m.moe_forward_host(h, T, src, *m.layer_args(layer), out))
            nxt = sizes[i + 1] if i + 1 < len(sizes) else 0
            src = out if 0 < nxt <= T else x0    # the next call reads this output where it fits
        m.check(m.moe_sync_status(h))
        return outs

    serial = chain()
    try:
        m.check(m.moe_set_host_overlap(h, 1))
        overlapped = chain()
        again = chain()
    finally:
        m.check(m.moe_set_host_overlap(h, 0))
    for a, b, c in zip(serial, overlapped, again):
        assert torch.equal(a, b) and torch.equal(a, c)


def test_host_overlap_streams_and_pageable_memory(m, tiny_inputs, tiny_handle):
    """Host overlap across a change of stream between calls (the handle waits for the previous
    stream) and with pageable host buffers (the copies are then synchronous): the serial
    path's results, bit for bit."""
    h, layer, _ = tiny_handle
    m.check(m.moe_set_router_bias(h, None))
    m.check(m.moe_set_padding_mask(h, None))
    T = 200
    x_pinned = tiny_inputs.x[:T].clone().pin_memory()
    x_pageable = tiny_inputs.x[:T].clone()
    ref = torch.empty_like(x_pinned).pin_memory()
    m.check(m.moe_forward_host(h, T, x_pinned, *m.layer_args(layer), ref))
    m.check(m.moe_sync_status(h))
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    try:
        m.check(m.moe_set_host_overlap(h, 1))
        for i, (x, st) in enumerate(((x_pinned, s1), (x_pageable, s2), (x_pinned, s2), (x_pageable, s1))):
            out = torch.empty_like(x_pinned).pin_memory() if i % 2 == 0 else torch.empty_like(x_pageable)
            m.check(m.moe_forward_host(h, T, x, *m.layer_args(layer), out, st))
            outs.append((out, st))
        for out, st in outs:
            st.synchronize()
        m.check(m.moe_sync_status(h))
    finally:
        m.check(m.moe_set_host_overlap(h, 0))
    for out, _ in outs:
        assert torch.equal(out, ref)


def test_host_wait_orders_the_output_copies(m, tiny_inputs, tiny_handle):
    """With host overlap on, the output copies run on a stream of the handle: after moe_host_wait on
    the caller's stream and a synchronisation of that stream alone (no moe_sync_status), every
    output holds the serial path's result, bit for bit.  A serial call afterwards into the same host
    buffer lands after the overlapped call's copy."""
    h, layer, _ = tiny_handle
    m.check(m.moe_set_router_bias(h, None))
    m.check(m.moe_set_padding_mask(h, None))
    T = 300
    xs = [tiny_inputs.x[i * 8:i * 8 + T].clone().pin_memory() for i in range(4)]
    refs = []
    for x in xs:
        r = torch.empty_like(x).pin_memory()
        m.check(m.moe_forward_host(h, T, x, *m.layer_args(layer), r))
        refs.append(r)
    m.check(m.moe_sync_status(h))
    st = torch.cuda.Stream()
    outs = [torch.empty_like(x).pin_memory() for x in xs]
    try:
        m.check(m.moe_set_host_overlap(h, 1))
        for x, out in zip(xs, outs):
            m.check(m.moe_forward_host(h, T, x, *m.layer_args(layer), out, st))
        m.check(m.moe_host_wait(h, st))
        st.synchronize()
        for out, ref in zip(outs, refs):
            assert torch.equal(out, ref)
        # an overlapped call, then a serial one writing the same host buffer: the serial result wins
        m.check(m.moe_forward_host(h, T, xs[0], *m.layer_args(layer), outs[1], st))
        m.check(m.moe_set_host_overlap(h, 0))
        m.check(m.moe_forward_host(h, T, xs[1], *m.layer_args(layer), outs[1], st))
        m.check(m.moe_sync_status(h, st))
        assert torch.equal(outs[1], refs[1])
    finally:
        m.check(m.moe_set_host_overlap(h, 0))
        m.check(m.moe_sync_status(h))


def test_kernel_times_reported(m, tiny_inputs, tiny_handle):
    h, layer, _ = tiny_handle
    x = tiny_inputs.x[:64].cuda()
    out = torch.empty_like(x)
    m.check(m.moe_set_profiling(h, True))
    for _ in range(3):
        m.check(m.moe_forward(h, 64, x, *m.layer_args(layer), out))
    rc, times = m.moe_get_kernel_times(h)
    m.check(m.moe_set_profiling(h, False))
    assert rc == 0
    for k in ("router", "dispatch", "gather", "up_proj", "down_proj", "combine"):
        assert times[k][1] == 3 and times[k][0] > 0


def test_small_batch_routing_is_one_launch(m, tiny_inputs, tiny_handle):
    """T <= 32 runs router, dispatch and gather as one launch (kernel id 7)."""
    h, layer, _ = tiny_handle
    x = tiny_inputs.x[:8].cuda()
    out = torch.empty_like(x)
    m.check(m.moe_set_profiling(h, True))
    for _ in range(3):
        m.check(m.moe_forward(h, 8, x, *m.layer_args(layer), out))
    rc, times = m.moe_get_kernel_times(h)
    m.check(m.moe_set_profiling(h, False))
    assert rc == 0
    assert times["route_small"][1] == 3 and times["route_small"][0] > 0
    for k in ("router", "dispatch", "gather"):
        assert times[k][1] == 0


@pytest.mark.parametrize("T", [8, 64, 300])
def test_tiny_residual_block(m, tiny_inputs, tiny_handle, T):
    """moe_block_forward on the tiny layer with non-unit RMSNorm gains, checked on the GPU's own
    MoE input (parity.check_block).  T=8 normalises inside the small-batch routing launch,
    T=64 inside the one-block-per-token router, T=300 inside the four-tokens-per-warp router:
    no separate pre-norm launch in any of them."""
    h, layer, _ = tiny_handle
    layer_cpu = parity.to_cpu(tiny_inputs.layers[0])
    g = torch.Generator().manual_seed(11)
    gam = {k: (0.5 + torch.rand(256, generator=g)).to(torch.bfloat16) for k in ("pre", "post")}
    h_in = tiny_inputs.x[:T].clone()
    h_dev = h_in.cuda().contiguous()
    m.check(m.moe_set_router_bias(h, None))
    m.check(m.moe_set_padding_mask(h, None))
    m.check(m.moe_set_profiling(h, True))
    m.moe_get_kernel_times(h)
    m.check(m.moe_block_forward(h, T, h_dev, gam["pre"].cuda(), gam["post"].cuda(), 1e-5, *m.layer_args(layer)))
    rc, times = m.moe_get_kernel_times(h)
    m.check(m.moe_set_profiling(h, False))
    assert rc == 0 and times["prenorm"][1] == 0
    parity.check_block(h, T, h_in, h_dev, layer_cpu, gam["pre"], gam["post"], 1e-5)


def _padding_mask(T, seed):
    g = torch.Generator().manual_seed(seed)
    mask = (torch.rand(T, generator=g) > 0.3).to(torch.uint8)
    mask[0], mask[-1] = 1, 0          # at least one real and one padding token
    return mask


@pytest.mark.parametrize("T", [8, 64, 300])
def test_padding_mask(m, tiny_inputs, tiny_handle, T):
    """Padding tokens (mask 0) are routed nowhere: experts -1, gates 0, no dispatched
    route, output row 0; real tokens match the oracle as without a mask."""
    h, layer, _ = tiny_handle
    layer_cpu = tiny_inputs.layers[0]
    x_cpu = tiny_inputs.x[:T]
    mask = _padding_mask(T, 40 + T)
    pad = mask.numpy() == 0
    mask_dev = mask.cuda()
    m.check(m.moe_set_padding_mask(h, mask_dev))
    try:
        run = parity.Run(h, x_cpu.cuda(), layer)
    finally:
        m.check(m.moe_set_padding_mask(h, None))
    ref = oracle.route(x_cpu, layer_cpu["router_w"])
    near = oracle.near_ties(ref["probs"], parity.NEAR_TIE) & ~pad
    assert (run.idx_h[pad] == -1).all() and np.all(run.gate_h[pad] == 0.0)
    ok = ~pad & ~near
    assert np.array_equal(run.idx_h[ok], ref["idx"][ok])
    np.testing.assert_allclose(run.gate_h[ok], ref["gate"][ok], rtol=parity.GATE_RTOL, atol=1e-7)
    merged = np.where(near[:, None], run.idx_h, np.where(pad[:, None], -1, ref["idx"]))
    counts, offsets, perm = oracle.dispatch(merged, 8)
    assert np.array_equal(run.offsets_h, offsets)
    assert offsets[-1] == 2 * int((~pad).sum())
    assert np.array_equal(run.perm_h[:offsets[-1]], perm[:offsets[-1]])
    assert torch.all(run.out_h[torch.from_numpy(pad)] == 0)
    real = np.nonzero(~pad)[0].tolist()
    forced = np.array([run.idx_h[t] if near[t] else (-1, -1) for t in real], dtype=np.int32)
    out, _, _ = oracle.forward(layer_cpu, x_cpu, tokens=real, mask=mask.numpy())
    for s_, t in enumerate(real):
        if near[t]:
            o, _, _ = oracle.forward(layer_cpu, x_cpu, tokens=[t], forced_idx=[forced[s_]])
            out[s_] = o[0]
    got = run.out_h[real].to(torch.float64).numpy()
    assert np.abs(got - out).max() <= parity.OUT_RTOL * np.abs(out).max()


def test_padding_mask_residual_block(m, tiny_inputs, tiny_handle):
    """moe_block_forward leaves a padding token's residual row unchanged (bit for bit)."""
    h, layer, _ = tiny_handle
    T = 8
    mask = _padding_mask(T, 77)
    pad = torch.from_numpy(mask.numpy() == 0)
    h_in = tiny_inputs.x[:T].clone()
    h_dev = h_in.cuda().contiguous()
    ones = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    m.check(m.moe_set_padding_mask(h, mask.cuda()))
    try:
        m.check(m.moe_block_forward(h, T, h_dev, ones, ones, 1e-5, *m.layer_args(layer)))
        m.check(m.moe_sync_status(h))
    finally:
        m.check(m.moe_set_padding_mask(h, None))
    got = h_dev.cpu()
    assert torch.equal(got[pad], h_in[pad])
    assert not torch.equal(got[~pad], h_in[~pad])


@pytest.mark.parametrize("T", [8, 64, 300])
def test_block_scales(m, tiny_inputs, tiny_handle, T):
    """Per-block weight scales (one per 128 input rows and output channel): the packed layout
    dequantises bf16(w * s) before the MMA and matches the oracle; the API layout refuses."""
    h, _, layout = tiny_handle
    layer_cpu = moe_synth.block_scales(tiny_inputs.layers[0], 128, torch.Generator().manual_seed(33))
    dev = parity.to_dev(layer_cpu)
    x_cpu = tiny_inputs.x[:T]
    m.check(m.moe_set_scale_block(h, 128))
    try:
        if layout != m.MOE_LAYOUT_PACKED:
            out = torch.empty((T, 256), dtype=torch.bfloat16, device="cuda")
            assert m.moe_forward(h, T, x_cpu.cuda(), *m.layer_args(dev), out) == m.MOE_EUNSUPPORTED
            return
        run = parity.Run(h, x_cpu.cuda(), m.pack_layer(h, dev))
    finally:
        m.check(m.moe_set_scale_block(h, 0))
    ref = oracle.route(x_cpu, layer_cpu["router_w"])
    near = parity.check_routing(run, ref, 8)
    parity.check_output(run, layer_cpu, x_cpu, range(T), near)


@pytest.mark.parametrize("T,mode", [(65, 1), (300, 2), (1000, 2), (1, 3), (8, 3), (17, 3), (32, 3)])
def test_cta_pairs_match_single_cta(m, tiny_inputs, tiny_handle, T, mode):
    """The GEMMs of 128-route plans on CTA pairs (the default for the packed layout) and on one
    CTA per tile give the same bits (these sizes have no last-wave pieces), and both match the
    oracle; the API layout ignores the switch."""
    h, layer, layout = tiny_handle
    m.check(m.moe_set_router_bias(h, None))
    m.check(m.moe_set_padding_mask(h, None))
    x = tiny_inputs.x[:T].cuda()
    try:
        m.check(m.moe_set_cta_pairs(h, m.MOE_PAIRS_OFF))
        single = parity.Run(h, x, layer)
        m.check(m.moe_set_cta_pairs(h, mode))
        paired = parity.Run(h, x, layer)
    finally:
        m.check(m.moe_set_cta_pairs(h, m.MOE_PAIRS_LARGE_DOWN))
    assert torch.equal(paired.out_h, single.out_h)
    ref = oracle.route(tiny_inputs.x[:T], tiny_inputs.layers[0]["router_w"])
    near = parity.check_routing(paired, ref, 8)
    parity.check_output(paired, tiny_inputs.layers[0], tiny_inputs.x[:T], range(T), near)


def _packed_bytes(wt):
    """The packed bytes of int8 values wt [..., K] (K contiguous, the input elements of one output
    feature): every four values w0..w3 become the bytes s2|m0, s0|m2, s3|m1, s1|m3, where mi = |wi|
    and si = 0x80 for a negative wi."""
    wi = wt.to(torch.int16).reshape(*wt.shape[:-1], -1, 4)
    m = wi.abs()
    sg = (wi < 0).to(torch.int16) * 0x80
    out = torch.stack([sg[..., 2] | m[..., 0], sg[..., 0] | m[..., 2], sg[..., 3] | m[..., 1], sg[..., 1] | m[..., 3]],
                      dim=-1)
    return out.reshape(wt.shape).to(torch.uint8)


def test_pack_weight_layout(m, tiny_handle):
    """moe_pack_weight transposes each expert and stores every value of [-127, 127] as a sign and a
    magnitude, four values to a word with crossed signs; a tensor holding -128 is refused with
    MOE_ERANGE."""
    h, _, _ = tiny_handle
    g = torch.Generator(device="cuda").manual_seed(3)
    for which, shape in ((0, (8, 256, 512)), (1, (8, 512, 256))):
        w = torch.randint(-127, 128, shape, generator=g, device="cuda", dtype=torch.int8)
        p = torch.empty((shape[0], shape[2], shape[1]), dtype=torch.int8, device="cuda")
        m.check(m.moe_pack_weight(h, w, p, which))
        torch.cuda.synchronize()
        assert torch.equal(p.view(torch.uint8), _packed_bytes(w.transpose(1, 2)))
        # a rank's share of the experts: exactly its bytes are read and written
        part = w[2:5].contiguous()
        guard = torch.full((4, shape[2], shape[1]), 7, dtype=torch.int8, device="cuda")
        m.check(m.moe_pack_weight_n(h, part, guard, which, 3))
        torch.cuda.synchronize()
        assert torch.equal(guard[:3].view(torch.uint8), _packed_bytes(part.transpose(1, 2)))
        assert bool((guard[3] == 7).all())
        # one -128 anywhere: no packed form
        w.view(-1)[12345] = -128
        assert m.moe_pack_weight(h, w, p, which) == m.MOE_ERANGE
        # and the range flag does not outlive the call
        w.view(-1)[12345] = -127
        m.check(m.moe_pack_weight(h, w, p, which))


@pytest.mark.parametrize("T", [8, 300])
def test_every_weight_byte(m, tiny_handle, tiny_inputs, T):
    """Weights taking every int8 value the layout holds equally often: all 256 in the [E, in, out]
    layout, -128 included (the synthetic draws stop at -127), and the 255 values of [-127, 127] in
    the packed layout (-128 has no packed form: test_pack_weight_layout).  Each layout's
    converters turn every value into its exact bf16 operand.  One value converted wrongly moves
    the outputs by about a fifth of their spread, far above the tolerance."""
    h, _, layout = tiny_handle
    g = torch.Generator().manual_seed(77)
    layer_cpu = dict(tiny_inputs.layers[0])
    lo = -127 if layout == m.MOE_LAYOUT_PACKED else -128
    for key in ("wl", "wv", "w1"):
        shape = layer_cpu[key].shape
        n = layer_cpu[key].numel()
        vals = (torch.arange(n) % (128 - lo) + lo).to(torch.int8)
        layer_cpu[key] = vals[torch.randperm(n, generator=g)].view(shape).contiguous()
    dev = parity.to_dev(layer_cpu)
    if layout == m.MOE_LAYOUT_PACKED:
        dev = m.pack_layer(h, dev)
    x_cpu = tiny_inputs.x[:T]
    run = parity.Run(h, x_cpu.cuda(), dev)
    near = parity.check_routing(run, oracle.route(x_cpu, layer_cpu["router_w"]), 8)
    parity.check_output(run, layer_cpu, x_cpu, parity.sample_tokens(run, T, 64), near)


@pytest.mark.parametrize("e", [-24, 24])
@pytest.mark.parametrize("T", [8, 300])
def test_activation_scale(m, tiny_handle, tiny_inputs, T, e):
    """Activations 2^e times the synthetic draws (router weight 2^-e times, so the routing is
    the same): the packed path keeps its operands at fixed power-of-two scales, so tiny and large
    activations keep their relative accuracy (H, about quadratic in x, spans 2^-50 .. 2^50 here).
    Without the scaled B operands the down-projection's sums at e = -24 (about 2^-170 before the
    epilogue's factor) would underflow to zero."""
    h, _, layout = tiny_handle
    layer_cpu = dict(tiny_inputs.layers[0])
    layer_cpu["router_w"] = layer_cpu["router_w"] * 2.0 ** -e
    x_cpu = (tiny_inputs.x[:T].float() * 2.0 ** e).to(torch.bfloat16)
    dev = parity.to_dev(layer_cpu)
    if layout == m.MOE_LAYOUT_PACKED:
        dev = m.pack_layer(h, dev)
    run = parity.Run(h, x_cpu.cuda(), dev)
    near = parity.check_routing(run, oracle.route(x_cpu, layer_cpu["router_w"]), 8)
    parity.check_output(run, layer_cpu, x_cpu, parity.sample_tokens(run, T, 64), near)


def test_tiny_maximum_token_count(m, tiny_handle):
    h, _, layout = tiny_handle
    T = m.MOE_MAX_TOKENS
    inp = moe_synth.make_inputs("tiny", device="cuda", T=T)
    layer = inp.layers[0]
    run = parity.Run(h, inp.x, m.pack_layer(h, layer) if layout == m.MOE_LAYOUT_PACKED else layer)
    layer_cpu = parity.to_cpu(layer)
    x_cpu = inp.x.cpu()
    ref = oracle.route(x_cpu, layer_cpu["router_w"])
    near = parity.check_routing(run, ref, 8)
    toks = parity.sample_tokens(run, T, 256)
    parity.check_output(run, layer_cpu, x_cpu, toks, near)


# ---- Grok-1 shape ---------------------------------------------------------------

@pytest.fixture(scope="module")
def grok_layer():
    """One Grok-1-shape layer (seed 0), on the GPU and on the host."""
    inp = moe_synth.make_inputs("decode", device="cuda")
    layer = inp.layers[0]
    cpu = parity.to_cpu(layer)
    yield layer, cpu
    del layer
    torch.cuda.empty_cache()


@pytest.fixture(scope="module", params=LAYOUTS, ids=["in_out", "packed"])
def grok_handle(m, request, grok_layer):
    rc, h = m.moe_create(6144, 32768, 8, 2)
    assert rc == 0
    m.check(m.moe_set_weight_layout(h, request.param))
    layer = grok_layer[0]
    if request.param == m.MOE_LAYOUT_PACKED:
        layer = m.pack_layer(h, layer)
    yield h, layer, request.param
    m.moe_destroy(h)
    del layer
    torch.cuda.empty_cache()


def test_decode_T8_all_tokens(m, grok_handle, grok_layer):
    grok_handle, layer, _ = grok_handle
    _, layer_cpu = grok_layer
    inp = moe_synth.make_inputs("decode", device="cuda")   # same seed: x drawn after the same weights
    x = inp.x
    del inp
    run = parity.Run(grok_handle, x, layer)
    x_cpu = x.cpu()
    ref = oracle.route(x_cpu, layer_cpu["router_w"])
    near = parity.check_routing(run, ref, 8)
    parity.check_output(run, layer_cpu, x_cpu, range(8), near)


def test_decode_T8_rerun_bit_identical(m, grok_handle):
    """Decode T=8: the packed layout cuts the up-projection's last wave of tiles into K pieces
    (1792 tiles on 148 CTAs) whose partial sums are added in piece order, and the
    down-projection splits K 8 ways; two runs on the same inputs give the same bits."""
    h, layer, _ = grok_handle
    g = moe_synth.generator(31, "cuda")
    x = moe_synth.draw_tokens(8, 6144, g, "cuda")
    m.check(m.moe_set_router_bias(h, None))
    a = parity.Run(h, x, layer)
    b = parity.Run(h, x, layer)
    assert torch.equal(a.out_h, b.out_h)
    assert np.array_equal(a.perm_h, b.perm_h) and np.array_equal(a.gate_h, b.gate_h)


@pytest.mark.parametrize("T,mode", [(2048, 2), (8, 3), (32, 3)])
def test_grok_cta_pairs_match_single_cta(m, grok_handle, grok_layer, T, mode):
    """Grok-1 shape: T = 2048 (every expert several 128-route tiles) and the decode sizes
    T = 8, 32 (32-route pair tiles, K-split down-projection, last-wave pieces, rows gathered
    by the up-projection): CTA pairs and single CTAs agree (each path cuts its own last wave
    into K pieces, so the bits may differ there), and the pairs match the oracle."""
    h, layer, layout = grok_handle
    _, layer_cpu = grok_layer
    if layout != m.MOE_LAYOUT_PACKED:
        pytest.skip("CTA pairs serve the packed layout")
    g = moe_synth.generator(41, "cuda")
    x = moe_synth.draw_tokens(T, 6144, g, "cuda")
    m.check(m.moe_set_router_bias(h, None))
    try:
        m.check(m.moe_set_cta_pairs(h, m.MOE_PAIRS_OFF))
        single = parity.Run(h, x, layer)
        m.check(m.moe_set_cta_pairs(h, mode))
        paired = parity.Run(h, x, layer)
        again = parity.Run(h, x, layer)   # the same mode again: bit for bit
    finally:
        m.check(m.moe_set_cta_pairs(h, m.MOE_PAIRS_LARGE_DOWN))
    assert torch.equal(again.out_h, paired.out_h)
    a, b = paired.out_h.to(torch.float64), single.out_h.to(torch.float64)
    assert (a - b).abs().max() <= 2e-3 * b.abs().max()
    x_cpu = x.cpu()
    ref = oracle.route(x_cpu, layer_cpu["router_w"])
    near = parity.check_routing(paired, ref, 8)
    parity.check_output(paired, layer_cpu, x_cpu, parity.sample_tokens(paired, T, 32), near)


@pytest.mark.parametrize("name,T", [("prefill", 8192), ("skewed", 4096)])
def test_large_T_sampled(m, grok_handle, grok_layer, name, T):
    grok_handle, layer, _ = grok_handle
    _, layer_cpu = grok_layer
    w = moe_synth.WORKLOADS[name]
    g = moe_synth.generator(w.seed + 17, "cuda")
    x = moe_synth.draw_tokens(T, w.d, g, "cuda")
    bias = None if w.bias is None else torch.tensor(w.bias, dtype=torch.float32)
    run = parity.Run(grok_handle, x, layer, None if bias is None else bias.cuda())
    x_cpu = x.cpu()
    ref = oracle.route(x_cpu, layer_cpu["router_w"], bias)
    near = parity.check_routing(run, ref, 8)
    if name == "skewed":
        share0 = (run.idx_h == 0).sum() / run.idx_h.size
        assert share0 > 0.4
    toks = parity.sample_tokens(run, T, 64)
    parity.check_output(run, layer_cpu, x_cpu, toks, near, bias_cpu=bias)


@pytest.mark.parametrize("pairs", [False, True], ids=["single_cta", "cta_pairs"])
def test_wide_tiles_odd_segments_and_pieces(m, grok_handle, grok_layer, pairs):
    """+100 on experts 0 and 1: both take all T = 1664 routes, 13 segments of 128 each, so the
    down-projection's 256-route tiles end on an odd 128-route tile, with 2 K-splits.  One CTA
    per tile: 2 experts * 48 * 7 * 2 = 1344 tiles on 148 CTAs, the last wave of 12 tiles cut
    into 12 pieces each.  CTA pairs: the odd segment's tile still runs N = 256 and its epilogue
    stops at the segment's own rows."""
    h, layer, _ = grok_handle
    _, layer_cpu = grok_layer
    T = 1664
    rc, bn, splits = m.moe_plan(h, T)
    assert (rc, bn, splits) == (0, 128, 2)
    g = moe_synth.generator(23, "cuda")
    x = moe_synth.draw_tokens(T, 6144, g, "cuda")
    bias = torch.tensor([100.0, 100.0, 0, 0, 0, 0, 0, 0])
    m.check(m.moe_set_cta_pairs(h, m.MOE_PAIRS_LARGE_DOWN if pairs else m.MOE_PAIRS_OFF))
    try:
        run = parity.Run(h, x, layer, bias.cuda())
        again = parity.Run(h, x, layer, bias.cuda())     # a fixed summation order: same bits
    finally:
        m.check(m.moe_set_cta_pairs(h, m.MOE_PAIRS_LARGE_DOWN))
    assert torch.equal(again.out_h, run.out_h)
    assert run.offsets_h.tolist() == [0, T, 2 * T] + [2 * T] * 6
    x_cpu = x.cpu()
    ref = oracle.route(x_cpu, layer_cpu["router_w"], bias)
    near = parity.check_routing(run, ref, 8)
    toks = parity.sample_tokens(run, T, 48)
    parity.check_output(run, layer_cpu, x_cpu, toks, near, bias_cpu=bias)


def test_stacked_blocks_per_block(m, grok_handle):
    """Four residual blocks, T=32: each block on the GPU is fed the oracle's residual
    stream (bf16) so that every block is compared on identical inputs, and is checked on
    its own MoE input (parity.check_block)."""
    grok_handle, _, layout = grok_handle
    w = moe_synth.WORKLOADS["stacked"]
    inp = moe_synth.make_inputs("stacked", device="cuda")
    layers_dev = inp.layers
    if layout == m.MOE_LAYOUT_PACKED:
        layers_dev = [m.pack_layer(grok_handle, l) for l in inp.layers]
    layers_cpu = [parity.to_cpu(l) for l in inp.layers]
    gam_cpu = [{k: v.cpu() for k, v in g.items()} for g in inp.gammas]
    chain = oracle.block_chain(layers_cpu, gam_cpu, inp.x.cpu(), eps=w.eps)
    m.check(m.moe_set_router_bias(grok_handle, None))
    m.check(m.moe_set_padding_mask(grok_handle, None))
    for b in range(w.blocks):
        h_in = torch.from_numpy(oracle.f64_to_bf16_bits(chain[b]["h_in"]).view(np.int16)).view(torch.bfloat16)
        h_dev = h_in.cuda().contiguous()
        m.check(m.moe_block_forward(grok_handle, w.T, h_dev, inp.gammas[b]["pre"], inp.gammas[b]["post"], w.eps,
                                    *m.layer_args(layers_dev[b])))
        parity.check_block(grok_handle, w.T, h_in, h_dev, layers_cpu[b], gam_cpu[b]["pre"], gam_cpu[b]["post"],
                           w.eps)
