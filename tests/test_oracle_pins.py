"""Pins of the fp64 CPU oracle against facts fixed outside the oracle itself.

Each test ties one part of the oracle to something it cannot agree with by
construction: a library routine (numpy float64 matmul, math.erf, torch's bf16
rounding), a brute-force search, a closed form, or an invariant of the
mathematics.  A plausible slip in the oracle (a transposed weight, a scale on the
wrong axis, gates renormalised or swapped, a wrong tie rule, a token index
mix-up) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_synth
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def tiny():
    return moe_synth.make_inputs("tiny", device="cpu")


def _np_layer(layer):
    """float64 dequantised weights of every expert, from torch tensors."""
    f = lambda t: t.to(torch.float64).numpy()
    return dict(
        Wl=f(layer["wl"]) * f(layer["sl"])[:, None, :],   # [E,d,F] * scale per output channel
        Wv=f(layer["wv"]) * f(layer["sv"])[:, None, :],
        W1=f(layer["w1"]) * f(layer["s1"])[:, None, :],   # [E,F,d]
    )


def _erf_gelu(a):
    v = np.vectorize(lambda z: 0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0))))
    return v(a)


def _dense_ffn(npl, e, x64):
    """numpy reference of one expert (library matmuls, erf GELU)."""
    a = x64 @ npl["Wl"][e]
    v = x64 @ npl["Wv"][e]
    return (_erf_gelu(a) * v) @ npl["W1"][e]


# ---- page facts and number formats -------------------------------------------

def test_shape_facts_from_pages():
    facts = json.load(open(os.path.join(GOLDEN, "grok1_moe_facts.json")))
    assert oracle.ffn_size(facts["emb_size"]["value"], facts["widening_factor"]["value"]) == \
        facts["d_expert"]["value"]
    assert facts["num_selected_experts"]["value"] == moe_synth.GROK_K
    assert facts["num_experts"]["value"] == moe_synth.GROK_E
    assert facts["emb_size"]["value"] == moe_synth.GROK_D
    assert facts["d_expert"]["value"] == moe_synth.GROK_F
    # the rounding-up-to-8 branch of the rule
    assert oracle.ffn_size(100, 8) == 536          # int(800)*2//3 = 533 -> 536
    assert oracle.ffn_size(96, 8) == 512           # already a multiple of 8


def test_round_bf16_matches_torch():
    g = torch.Generator().manual_seed(7)
    v = torch.randn(20000, generator=g, dtype=torch.float32) * 10.0 ** torch.randint(-6, 6, (20000,), generator=g)
    # exact halfway cases (ties go to even)
    halves = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(2.0 + 2.0 ** -7), 3.0 * 2.0 ** -9], dtype=torch.float32)
    v = torch.cat([v, halves])
    ref = v.to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(v.to(torch.float64).numpy())
    assert np.array_equal(ref, got)


def test_int8_times_bf16_scale_is_exact_in_fp32():
    """Dequantisation w*s is exact in fp32 and fp64 (8-bit integer x 8-bit significand),
    so a kernel may keep the scale out of the K-sum and apply it in fp32."""
    g = torch.Generator().manual_seed(3)
    w = torch.arange(-127, 128, dtype=torch.int32)
    s = (torch.randn(4096, generator=g) / (127 * 78.4)).to(torch.bfloat16)
    p64 = w.to(torch.float64)[:, None] * s.to(torch.float64)[None, :]
    p32 = w.to(torch.float32)[:, None] * s.to(torch.float32)[None, :]
    assert torch.equal(p64, p32.to(torch.float64))
    # and int8 -> bf16 is lossless
    assert torch.equal(w.to(torch.bfloat16).to(torch.int32), w)


def test_gelu_tanh_form():
    xs = np.linspace(-8, 8, 3201)
    g = np.array([oracle.gelu(x, 0) for x in xs])
    gm = np.array([oracle.gelu(-x, 0) for x in xs])
    # x*Phi~(x) with Phi~(x) + Phi~(-x) = 1  =>  gelu(x) - gelu(-x) = x
    assert np.max(np.abs(g - gm - xs)) < 1e-14
    assert oracle.gelu(0.0, 0) == 0.0
    # close to the exact GELU (math.erf) everywhere, and equal to it in the tails
    exact = _erf_gelu(xs)
    dev = np.abs(g - exact)
    assert dev.max() < 1e-3
    assert dev[np.abs(xs) > 6].max() < 1e-8
    # slope 1/2 at the origin
    assert abs(oracle.gelu(1e-6, 0) / 1e-6 - 0.5) < 1e-6


def test_gelu_tanh_form_is_torch_tanh_gelu():
    """The oracle's default GELU is torch's tanh-approximate GELU (a library routine written
    independently of the oracle's C): a wrong 0.044715 or sqrt(2/pi) fails here."""
    xs = torch.linspace(-9, 9, 4001, dtype=torch.float64)
    xs = torch.cat([xs, torch.tensor([-1e-3, 1e-3, 0.3, -2.7, 5.5, 1e-8], dtype=torch.float64)])
    ref = torch.nn.functional.gelu(xs, approximate="tanh").numpy()
    got = np.array([oracle.gelu(float(x), 0) for x in xs])
    assert np.max(np.abs(got - ref)) <= 1e-15 * np.maximum(1.0, np.abs(ref)).max()


def test_gelu_erf_form_is_erf():
    for x in (-3.0, -0.7, 0.1, 1.0, 2.5):
        assert oracle.gelu(x, 1) == pytest.approx(0.5 * x * (1 + math.erf(x / math.sqrt(2))), rel=1e-15)


# ---- router ------------------------------------------------------------------

def _np_logits(x_bf16, router_w, bias=None):
    x64 = x_bf16.to(torch.float64).numpy()
    L = (x64 @ router_w.to(torch.float64).numpy()).astype(np.float32)
    if bias is not None:
        L = (L + bias.numpy()).astype(np.float32)
    return L


def test_route_brute_force_pairs(tiny):
    layer = tiny.layers[0]
    r = oracle.route(tiny.x, layer["router_w"])
    L = _np_logits(tiny.x, layer["router_w"])
    # fp32 logits: exact sum rounded once; numpy's float64 sum may differ in the last
    # fp64 bits, which can move the fp32 rounding by at most one ulp
    assert np.all(np.abs(r["logits"] - L) <= np.spacing(np.abs(L)))
    E = L.shape[1]
    for t in range(L.shape[0]):
        p = np.exp(L[t].astype(np.float64) - L[t].max())
        p /= p.sum()
        assert abs(r["probs"][t].sum() - 1.0) < 1e-15
        best = max(itertools.combinations(range(E), 2), key=lambda ab: p[ab[0]] + p[ab[1]])
        a, b = sorted(best, key=lambda e: (-p[e], e))
        assert (r["idx"][t] == [a, b]).all(), t
        assert r["gate"][t][0] == pytest.approx(p[a], rel=1e-12)
        assert r["gate"][t][1] == pytest.approx(p[b], rel=1e-12)
        assert r["gate"][t][0] >= r["gate"][t][1]


def test_route_tie_rule_and_zero_input():
    d, E = 64, 8
    x = torch.zeros(3, d, dtype=torch.bfloat16)
    w = torch.randn(d, E)
    r = oracle.route(x, w)
    assert (r["idx"] == [[0, 1]] * 3).all()            # all equal -> lowest indices
    assert np.allclose(r["gate"], 1.0 / 8, rtol=0, atol=1e-16)
    bias = torch.tensor([0, 2, 2, 0, 5, 5, 0, 0], dtype=torch.float32)
    r = oracle.route(x, w, bias)
    assert (r["idx"] == [[4, 5]] * 3).all()            # tie at the top: lower index first
    bias = torch.tensor([0, 2, 2, 0, 5, 1, 0, 0], dtype=torch.float32)
    r = oracle.route(x, w, bias)
    assert (r["idx"] == [[4, 1]] * 3).all()            # tie for second place


# ---- dispatch ----------------------------------------------------------------

def test_dispatch_brute_force():
    g = torch.Generator().manual_seed(11)
    for T in (0, 1, 7, 300):
        E = 8
        idx = np.zeros((T, 2), np.int32)
        for t in range(T):
            idx[t] = torch.randperm(E, generator=g)[:2].numpy()
        counts, offsets, perm = oracle.dispatch(idx, E)
        groups = [[2 * t + j for t in range(T) for j in range(2) if idx[t, j] == e] for e in range(E)]
        assert counts.tolist() == [len(gr) for gr in groups]
        assert offsets.tolist() == [0] + list(np.cumsum([len(gr) for gr in groups]))
        assert perm.tolist() == [r for gr in groups for r in gr]


def test_dispatch_skips_padding_routes():
    """Expert id -1 (a padding token) is not dispatched: brute-force grouping of the rest."""
    g = torch.Generator().manual_seed(12)
    E, T = 8, 200
    idx = np.zeros((T, 2), np.int32)
    for t in range(T):
        idx[t] = torch.randperm(E, generator=g)[:2].numpy()
    pad = (torch.rand(T, generator=g) < 0.3).numpy()
    idx[pad] = -1
    counts, offsets, perm = oracle.dispatch(idx, E)
    groups = [[2 * t + j for t in range(T) for j in range(2) if idx[t, j] == e] for e in range(E)]
    assert counts.tolist() == [len(gr) for gr in groups]
    assert offsets[-1] == 2 * int((~pad).sum())
    assert perm[:offsets[-1]].tolist() == [r for gr in groups for r in gr]


# ---- expert FFN and the layer -------------------------------------------------

def test_expert_ffn_matches_numpy(tiny):
    layer = tiny.layers[0]
    npl = _np_layer(layer)
    x64 = tiny.x.to(torch.float64).numpy()
    for e, t in [(0, 0), (3, 5), (7, 63)]:
        y = oracle.expert_ffn(x64[t], layer, e, gelu_kind=1)
        ref = _dense_ffn(npl, e, x64[t])
        assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_expert_ffn_tanh_gelu_matches_numpy(tiny):
    """The default (tanh) GELU branch of the expert FFN against numpy float64 matmuls with
    torch's tanh-approximate GELU."""
    layer = tiny.layers[0]
    npl = _np_layer(layer)
    x64 = tiny.x.to(torch.float64).numpy()
    tanh_gelu = lambda a: torch.nn.functional.gelu(torch.from_numpy(a), approximate="tanh").numpy()
    for e, t in [(1, 2), (6, 33)]:
        y = oracle.expert_ffn(x64[t], layer, e)          # gelu_kind 0: the tanh form
        ref = (tanh_gelu(x64[t] @ npl["Wl"][e]) * (x64[t] @ npl["Wv"][e])) @ npl["W1"][e]
        assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_forward_rejects_inconsistent_shapes(tiny):
    """A layer whose weights were transposed to another layout (or whose scales belong to
    another matrix) is refused instead of being read as a layer of another width."""
    layer = tiny.layers[0]
    packed = dict(layer)
    packed["wl"] = layer["wl"].transpose(1, 2).contiguous()
    packed["wv"] = layer["wv"].transpose(1, 2).contiguous()
    packed["w1"] = layer["w1"].transpose(1, 2).contiguous()
    with pytest.raises(ValueError):
        oracle.forward(packed, tiny.x, tokens=[0])
    with pytest.raises(ValueError):
        oracle.expert_ffn(tiny.x[0].to(torch.float64).numpy(), packed, 0)
    swapped = dict(layer)
    swapped["s1"] = layer["sl"]
    with pytest.raises(ValueError):
        oracle.forward(swapped, tiny.x, tokens=[0])
    wrong_router = dict(layer)
    wrong_router["router_w"] = layer["router_w"].t().contiguous()
    with pytest.raises(ValueError):
        oracle.forward(wrong_router, tiny.x, tokens=[0])
    assert oracle.check_layer(layer, 256) == (8, 256, 512, 0)


def test_forced_expert_reduces_to_dense_ffn(tiny):
    layer = tiny.layers[0]
    npl = _np_layer(layer)
    x64 = tiny.x.to(torch.float64).numpy()
    toks = [0, 9, 40]
    for a in (0, 5):
        bias = torch.zeros(8)
        bias[a] = 100.0
        out, idx, gate = oracle.forward(layer, tiny.x, bias=bias, tokens=toks, gelu_kind=1)
        assert (idx[:, 0] == a).all()
        assert np.all(gate[:, 0] >= 1 - 1e-15)
        for s, t in enumerate(toks):
            ref = _dense_ffn(npl, a, x64[t])
            assert np.max(np.abs(out[s] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_two_equal_experts_average(tiny):
    """Zero router weight and +100 on experts 2 and 6: an exact tie, so the lower
    index takes slot 0 and each gate is 1/2 (the other six are ~e^-100)."""
    layer = dict(tiny.layers[0])
    layer["router_w"] = torch.zeros_like(layer["router_w"])
    npl = _np_layer(layer)
    x64 = tiny.x.to(torch.float64).numpy()
    bias = torch.zeros(8)
    bias[2] = bias[6] = 100.0
    out, idx, gate = oracle.forward(layer, tiny.x, bias=bias, tokens=[3, 17], gelu_kind=1)
    assert (idx == [[2, 6], [2, 6]]).all()
    for s, t in enumerate([3, 17]):
        ref = 0.5 * (_dense_ffn(npl, 2, x64[t]) + _dense_ffn(npl, 6, x64[t]))
        assert np.max(np.abs(out[s] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_closed_form_gates_not_renormalised(tiny):
    """router_w = 0 and bias = (ln 4, ln 2, 0, ...) give p = (1/3, 1/6, 1/12, ...):
    the output is FFN_0/3 + FFN_1/6 (renormalised gates would give 2/3 and 1/3)."""
    layer = dict(tiny.layers[0])
    layer["router_w"] = torch.zeros_like(layer["router_w"])
    npl = _np_layer(layer)
    x64 = tiny.x.to(torch.float64).numpy()
    bias = torch.tensor([math.log(4), math.log(2), 0, 0, 0, 0, 0, 0], dtype=torch.float32)
    out, idx, gate = oracle.forward(layer, tiny.x, bias=bias, tokens=[1, 2], gelu_kind=1)
    assert (idx == [[0, 1], [0, 1]]).all()
    assert gate[0] == pytest.approx([1 / 3, 1 / 6], rel=1e-7)
    for s, t in enumerate([1, 2]):
        ref = _dense_ffn(npl, 0, x64[t]) / 3 + _dense_ffn(npl, 1, x64[t]) / 6
        assert np.max(np.abs(out[s] - ref)) <= 1e-6 * np.max(np.abs(ref))


def test_token_permutation_invariance(tiny):
    layer = tiny.layers[0]
    g = torch.Generator().manual_seed(5)
    P = torch.randperm(tiny.x.shape[0], generator=g)
    out, idx, gate = oracle.forward(layer, tiny.x)
    out_p, idx_p, gate_p = oracle.forward(layer, tiny.x[P])
    assert np.array_equal(out_p, out[P.numpy()])
    assert np.array_equal(idx_p, idx[P.numpy()])
    assert np.array_equal(gate_p, gate[P.numpy()])
    # a token's result does not depend on which other tokens are in the batch
    sub, _, _ = oracle.forward(layer, tiny.x, tokens=[5, 60])
    assert np.array_equal(sub, out[[5, 60]])


def test_zero_input_gives_zero_output(tiny):
    layer = tiny.layers[0]
    x0 = torch.zeros(4, tiny.x.shape[1], dtype=torch.bfloat16)
    out, idx, gate = oracle.forward(layer, x0)
    assert np.all(out == 0.0)
    assert (idx == [[0, 1]] * 4).all()
    assert np.all(gate == 0.125)


def test_padding_mask_routes_nothing(tiny):
    """Padding tokens get output 0, experts -1, gates 0; every real token's result is
    bit-identical to the unmasked layer's (tokens are independent)."""
    layer = tiny.layers[0]
    g = torch.Generator().manual_seed(8)
    mask = (torch.rand(tiny.x.shape[0], generator=g) > 0.3).numpy()
    out, idx, gate = oracle.forward(layer, tiny.x)
    out_m, idx_m, gate_m = oracle.forward(layer, tiny.x, mask=mask)
    assert np.array_equal(out_m[mask], out[mask])
    assert np.array_equal(idx_m[mask], idx[mask]) and np.array_equal(gate_m[mask], gate[mask])
    assert np.all(out_m[~mask] == 0.0) and (idx_m[~mask] == -1).all() and np.all(gate_m[~mask] == 0.0)
    out_0, idx_0, _ = oracle.forward(layer, tiny.x[:5], mask=np.zeros(5, np.uint8))
    assert np.all(out_0 == 0.0) and (idx_0 == -1).all()
    # in the residual block a padding row passes through unchanged
    gam = {"pre": torch.ones(tiny.x.shape[1], dtype=torch.bfloat16),
           "post": torch.ones(tiny.x.shape[1], dtype=torch.bfloat16)}
    blk = oracle.block_chain([layer], [gam], tiny.x[:16], mask=mask[:16])[0]
    assert np.array_equal(blk["h_out"][~mask[:16]], blk["h_in"][~mask[:16]])


def test_block_scales_match_numpy(tiny):
    """Per-block scales ([E, in/kb, out]): the oracle's expert FFN equals numpy float64
    matmuls on weights dequantised with np.repeat of the scale rows over their blocks."""
    layer = moe_synth.block_scales(tiny.layers[0], 128, torch.Generator().manual_seed(21))
    assert oracle.scale_block(layer) == 128
    f = lambda t: t.to(torch.float64).numpy()
    rep = lambda sc, n: np.repeat(f(sc), n, axis=1)        # [E, in/kb, out] -> [E, in, out]
    Wl = f(layer["wl"]) * rep(layer["sl"], 128)
    Wv = f(layer["wv"]) * rep(layer["sv"], 128)
    W1 = f(layer["w1"]) * rep(layer["s1"], 128)
    x64 = tiny.x[:3].to(torch.float64).numpy()
    for e in (0, 5):
        for t in range(3):
            y = oracle.expert_ffn(x64[t], layer, e, gelu_kind=1)
            ref = (_erf_gelu(x64[t] @ Wl[e]) * (x64[t] @ Wv[e])) @ W1[e]
            np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_block_scales_equal_rows_reduce_to_channel_scales(tiny):
    """Block scales whose rows are all the per-channel scale give the per-channel layer bit for bit."""
    layer = tiny.layers[0]
    E, d, F = layer["wl"].shape
    blk = dict(layer)
    blk["sl"] = layer["sl"][:, None, :].expand(E, d // 128, F).contiguous()
    blk["sv"] = layer["sv"][:, None, :].expand(E, d // 128, F).contiguous()
    blk["s1"] = layer["s1"][:, None, :].expand(E, F // 128, d).contiguous()
    out, idx, _ = oracle.forward(layer, tiny.x[:16])
    out_b, idx_b, _ = oracle.forward(blk, tiny.x[:16])
    assert np.array_equal(out, out_b) and np.array_equal(idx, idx_b)


def test_linear_in_output_scale(tiny):
    layer = dict(tiny.layers[0])
    out, _, _ = oracle.forward(layer, tiny.x, tokens=[0, 1, 2])
    layer["s1"] = (layer["s1"].to(torch.float32) * 2).to(torch.bfloat16)   # exact in bf16
    out2, _, _ = oracle.forward(layer, tiny.x, tokens=[0, 1, 2])
    assert np.array_equal(out2, 2 * out)


def test_forced_idx_override(tiny):
    layer = tiny.layers[0]
    out, idx, gate = oracle.forward(layer, tiny.x, tokens=[4], forced_idx=[[6, 1]])
    r = oracle.route(tiny.x[4:5], layer["router_w"])
    assert (idx == [[6, 1]]).all()
    assert gate[0].tolist() == [r["probs"][0][6], r["probs"][0][1]]


# ---- RMSNorm and the stacked blocks -------------------------------------------

def test_rmsnorm_properties():
    g = torch.Generator().manual_seed(2)
    z = (torch.randn(5, 256, generator=g, dtype=torch.float64) * 3).numpy()
    y = oracle.rmsnorm(z, None, eps=0.0)
    assert np.allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-14)
    assert np.allclose(oracle.rmsnorm(7.5 * z, None, eps=0.0), y, rtol=1e-13)
    gamma = torch.full((256,), 2.0, dtype=torch.bfloat16)
    assert np.allclose(oracle.rmsnorm(z, gamma, eps=0.0), 2 * y, rtol=1e-14)
    # eps enters inside the root: a zero row stays zero, a tiny row is damped
    assert np.all(oracle.rmsnorm(np.zeros((1, 256)), None, eps=1e-5) == 0)


def test_rmsnorm_constant_row_closed_form():
    """A constant row c normalises to c / sqrt(c^2 + eps) (times the gain): this fixes where
    eps enters (inside the root, added to the mean square).  With c = 1e-3 and eps = 1e-5
    the reading c / (|c| + eps) would give 0.99 instead of 0.3015."""
    d = 256
    gamma = torch.full((d,), 1.5, dtype=torch.bfloat16)
    for c, eps in ((1e-3, 1e-5), (0.25, 1e-5), (-3.0, 0.5), (2.0, 0.0)):
        z = np.full((2, d), c)
        got = oracle.rmsnorm(z, None, eps=eps)
        want = c / math.sqrt(c * c + eps)
        np.testing.assert_allclose(got, want, rtol=1e-15, atol=0)
        np.testing.assert_allclose(oracle.rmsnorm(z, gamma, eps=eps), 1.5 * want, rtol=1e-15, atol=0)


def _stack(seed=3, T=6):
    w = moe_synth.Workload("tiny_stack", T=T, d=256, F=512, blocks=1, seed=seed)
    inp = moe_synth.make_inputs(w, device="cpu")
    g = torch.Generator().manual_seed(seed + 50)
    # non-unit, non-uniform gains, so that a gain applied before its norm changes the result
    gam = [{k: (0.5 + torch.rand(256, generator=g)).to(torch.bfloat16) for k in ("pre", "post")}]
    return inp, gam


def _times2(t):
    return (t.to(torch.float32) * 2).to(t.dtype)   # exact in bf16 (power of two)


def test_block_chain_pre_norm_is_applied():
    """Scaling the residual stream by 2 leaves u = bf16(RMSNorm(h) * g_pre) and the routing
    unchanged bit for bit when eps = 0; a chain that skipped the pre-norm would route 2h."""
    inp, gam = _stack()
    a = oracle.block_chain(inp.layers, gam, inp.x, eps=0.0)[0]
    b = oracle.block_chain(inp.layers, gam, _times2(inp.x), eps=0.0)[0]
    assert np.array_equal(a["u"], b["u"])
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["gate"], b["gate"])
    assert np.array_equal(a["delta"], b["delta"])
    assert not np.array_equal(a["u"], a["h_in"])


def test_block_chain_pre_gain_after_the_norm():
    """Doubling g_pre doubles u exactly (the gain multiplies the normalised row); a gain
    applied before the norm would cancel out and leave u unchanged."""
    inp, gam = _stack()
    a = oracle.block_chain(inp.layers, gam, inp.x, eps=1e-5)[0]
    gam2 = [{"pre": _times2(gam[0]["pre"]), "post": gam[0]["post"]}]
    b = oracle.block_chain(inp.layers, gam2, inp.x, eps=1e-5)[0]
    assert np.array_equal(b["u"], 2 * a["u"])


def test_block_chain_post_norm_is_applied():
    """Scaling every linear_1 scale by 2 doubles the MoE output y exactly, and with eps = 0
    the post-norm cancels it: the block's contribution and h_out are unchanged bit for bit.
    A chain without the post-norm would add 2y instead of y."""
    inp, gam = _stack()
    a = oracle.block_chain(inp.layers, gam, inp.x, eps=0.0)[0]
    layer2 = dict(inp.layers[0])
    layer2["s1"] = _times2(layer2["s1"])
    b = oracle.block_chain([layer2], gam, inp.x, eps=0.0)[0]
    assert np.array_equal(b["y"], 2 * a["y"])
    assert np.array_equal(b["delta"], a["delta"])
    assert np.array_equal(b["h_out"], a["h_out"])


def test_block_chain_post_gain_after_the_norm():
    """Doubling g_post doubles the contribution exactly; a gain applied before the post-norm
    would cancel out."""
    inp, gam = _stack()
    a = oracle.block_chain(inp.layers, gam, inp.x, eps=1e-5)[0]
    gam2 = [{"pre": gam[0]["pre"], "post": _times2(gam[0]["post"])}]
    b = oracle.block_chain(inp.layers, gam2, inp.x, eps=1e-5)[0]
    assert np.array_equal(b["delta"], 2 * a["delta"])
    assert not np.array_equal(b["h_out"], a["h_out"])


def test_block_chain_residual_add():
    """linear_1 scales 0: y = 0, RMSNorm(0) = 0 (eps > 0), so h_out equals h_in exactly; a
    chain that dropped the residual add would return 0.  With real scales, h_out is the
    bf16 rounding of h_in + delta."""
    inp, gam = _stack()
    layer0 = dict(inp.layers[0])
    layer0["s1"] = torch.zeros_like(layer0["s1"])
    z = oracle.block_chain([layer0], gam, inp.x, eps=1e-5)[0]
    assert np.all(z["y"] == 0) and np.all(z["delta"] == 0)
    assert np.array_equal(z["h_out"], z["h_in"])
    a = oracle.block_chain(inp.layers, gam, inp.x, eps=1e-5)[0]
    assert np.array_equal(a["h_out"], torch.from_numpy(a["h_in"] + a["delta"]).to(torch.bfloat16)
                          .to(torch.float64).numpy())


def test_block_chain_rows_are_independent(tiny):
    w = moe_synth.Workload("tiny_stack", T=6, d=256, F=512, blocks=2)
    inp = moe_synth.make_inputs(w, device="cpu")
    full = oracle.block_chain(inp.layers, inp.gammas, inp.x, eps=w.eps)
    part = oracle.block_chain(inp.layers, inp.gammas, inp.x, eps=w.eps, tokens=[1, 4])
    for b in range(2):
        assert np.array_equal(part[b]["h_out"], full[b]["h_out"][[1, 4]])
        # the residual stream is bf16: rounding to bf16 changes nothing
        assert np.array_equal(oracle.round_bf16(full[b]["h_out"]), full[b]["h_out"])


def test_near_tie_detection():
    p = np.array([[0.4, 0.4 - 5e-7, 0.1, 0.1 - 5e-7, 0, 0, 0, 0],
                  [0.5, 0.3, 0.3 - 2e-7, 0, 0, 0, 0, 0],
                  [0.5, 0.3, 0.1, 0.1, 0, 0, 0, 0]])
    assert oracle.near_ties(p).tolist() == [True, True, False]


# ---- regression anchor written by tests/golden/make_golden.py ------------------

def test_tiny_regression_anchor(tiny):
    path = os.path.join(GOLDEN, "tiny_oracle_anchor.json")
    ref = json.load(open(path))
    wl = tiny.layers[0]["wl"]
    if int(wl.to(torch.int64).sum()) != ref["input_checksum"]["wl_sum"]:
        pytest.skip("torch's CPU random stream differs from the one the anchor was written with")
    out, idx, gate = oracle.forward(tiny.layers[0], tiny.x, tokens=ref["tokens"])
    assert idx.tolist() == ref["idx"]
    np.testing.assert_allclose(out[:, :16], np.array(ref["out_head"]), rtol=1e-12, atol=0)
