"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same seeded inputs.

Criteria (from the layer's contract):
  * expert indices, their order, the grouped offsets and the grouped order are
    bit-exact, except on tokens whose top-3 softmax probabilities have a gap
    below 1e-6 (near ties), where either pick is a correct top-2;
  * the output satisfies  max|gpu - oracle| <= 1e-2 * max|oracle|  over the
    compared tokens; for near-tie tokens the oracle is evaluated with the experts
    the GPU picked.

The residual block adds its own bf16 rounding of the MoE input u = RMSNorm(h):
the GPU forms it in fp32, the oracle in fp64, so one element in a few hundred lies
close enough to a bf16 rounding midpoint to round the other way.  The block is
therefore checked in three steps (check_block): the GPU's u (read back with
moe_get_block_input) against the oracle's u, one bf16 step allowed only where the
exact value lies within fp32 error of a midpoint; the GPU's routing against the
oracle's routing OF THE GPU'S u, under the rule above; and the block's output
against the oracle's exact h + RMSNorm(MoE(u); g_post) on that u, before its bf16
store, within 1e-2 of the largest contribution.
"""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_softmax_b200 as moe
import oracle

OUT_RTOL = 1e-2          # max|gpu - oracle| <= OUT_RTOL * max|oracle|
NEAR_TIE = 1e-6          # prob gap below which either selection is correct
GATE_RTOL = 2e-5         # fp32 softmax vs fp64 softmax of the same fp32 logits
U_RTOL = 1e-5            # fp32 RMSNorm of a bf16 row: relative error bound of the unrounded u


def to_dev(layer: dict, device="cuda"):
    return {k: v.to(device) for k, v in layer.items()}


def to_cpu(layer: dict):
    return {k: v.cpu() for k, v in layer.items()}


class Run:
    """One forward through the C ABI plus the routing the library reports."""

    def __init__(self, h, x_dev, layer_dev, bias_dev=None, T=None):
        T = x_dev.shape[0] if T is None else T
        E = layer_dev["router_w"].shape[1]
        self.out = torch.empty_like(x_dev)
        moe.check(moe.moe_set_router_bias(h, bias_dev))
        moe.check(moe.moe_forward(h, T, x_dev, *moe.layer_args(layer_dev), self.out), "moe_forward")
        self.idx = torch.empty((T, 2), dtype=torch.int32, device=x_dev.device)
        self.gate = torch.empty((T, 2), dtype=torch.float32, device=x_dev.device)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=x_dev.device)
        self.perm = torch.empty(2 * T, dtype=torch.int32, device=x_dev.device)
        moe.check(moe.moe_get_routing(h, self.idx, self.gate, self.offsets, self.perm))
        moe.check(moe.moe_sync_status(h), "device status")
        self.out_h = self.out.cpu()
        self.idx_h = self.idx.cpu().numpy()
        self.gate_h = self.gate.cpu().numpy()
        self.offsets_h = self.offsets.cpu().numpy()
        self.perm_h = self.perm.cpu().numpy()


def check_routing(run: Run, ref: dict, E: int):
    """Bit-exact routing and dispatch outside near ties; returns the near-tie mask."""
    near = oracle.near_ties(ref["probs"], NEAR_TIE)
    ok = ~near
    mism = np.nonzero((run.idx_h != ref["idx"]).any(axis=1) & ok)[0]
    assert mism.size == 0, f"expert choice differs on tokens {mism[:10]}"
    np.testing.assert_allclose(run.gate_h[ok], ref["gate"][ok], rtol=GATE_RTOL, atol=1e-7)
    assert (run.gate_h[:, 0] >= run.gate_h[:, 1]).all()
    # the grouping must be the stable grouping of the chosen experts (the oracle's
    # choice everywhere except near ties, where the GPU's own choice is valid)
    merged = np.where(near[:, None], run.idx_h, ref["idx"])
    counts, offsets, perm = oracle.dispatch(merged, E)
    assert np.array_equal(run.offsets_h, offsets)
    assert np.array_equal(run.perm_h, perm)
    return near


def sample_tokens(run: Run, T: int, n: int, seed: int = 1234):
    """n seeded tokens plus the first and last grouped row of every expert."""
    must = []
    off = run.offsets_h
    for e in range(len(off) - 1):
        if off[e + 1] > off[e]:
            must += [int(run.perm_h[off[e]]) // 2, int(run.perm_h[off[e + 1] - 1]) // 2]
    from moe_synth import token_sample
    return token_sample(T, n, seed=seed, must_include=must)


def check_output(run: Run, layer_cpu: dict, x_cpu, tokens, near, bias_cpu=None, nthreads=0):
    tokens = list(tokens)
    forced = np.array([run.idx_h[t] if near[t] else (-1, -1) for t in tokens], dtype=np.int32)
    need_forced = any(near[t] for t in tokens)
    ref, ridx, _ = oracle.forward(layer_cpu, x_cpu, bias=bias_cpu, tokens=tokens, nthreads=nthreads)
    if need_forced:
        for s, t in enumerate(tokens):
            if near[t]:
                o, _, _ = oracle.forward(layer_cpu, x_cpu, bias=bias_cpu, tokens=[t],
                                         forced_idx=[run.idx_h[t]], nthreads=nthreads)
                ref[s] = o[0]
    got = run.out_h[tokens].to(torch.float64).numpy()
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    assert np.isfinite(got).all()
    assert err <= OUT_RTOL * scale, f"max|gpu-oracle| = {err:.3e} > {OUT_RTOL} * {scale:.3e}"
    return err / max(scale, 1e-300)



def read_routing(h, T: int, E: int = 8, device="cuda"):
    """The routing of the handle's last forward, on the host (fields as in Run)."""
    import types
    idx = torch.empty((T, 2), dtype=torch.int32, device=device)
    gate = torch.empty((T, 2), dtype=torch.float32, device=device)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=device)
    perm = torch.empty(2 * T, dtype=torch.int32, device=device)
    moe.check(moe.moe_get_routing(h, idx, gate, offsets, perm))
    moe.check(moe.moe_sync_status(h), "device status")
    return types.SimpleNamespace(idx_h=idx.cpu().numpy(), gate_h=gate.cpu().numpy(),
                                 offsets_h=offsets.cpu().numpy(), perm_h=perm.cpu().numpy())


def check_block_input(u_gpu: np.ndarray, u_exact: np.ndarray, u_round: np.ndarray):
    """The GPU's bf16 u equals the oracle's bf16 rounding of the exact fp64 u, except where
    it is the rounding of a value within U_RTOL (relative) of the exact one: a one-step
    difference next to a rounding midpoint.  Returns the number of such elements."""
    diff = u_gpu != u_round
    if diff.any():
        a, x = u_gpu[diff], u_exact[diff]
        lo, hi = oracle.round_bf16(x * (1 - U_RTOL)), oracle.round_bf16(x * (1 + U_RTOL))
        bad = ~((a == lo) | (a == hi))
        assert not bad.any(), (f"{int(bad.sum())} elements of u differ from the oracle beyond rounding: "
                               f"gpu {a[bad][:4]}, exact {x[bad][:4]}")
        assert diff.mean() < 1e-2, f"{diff.mean():.2%} of u rounds differently"
    return int(diff.sum())


def check_block(h, T: int, h_in_bits, h_out_dev, layer_cpu: dict, g_pre, g_post, eps: float, E: int = 8):
    """One moe_block_forward (already run on h_in_bits, bf16 [T, d], leaving h_out_dev) against
    the oracle, in the three steps of the module docstring.  Returns (u differences, near-tie
    tokens, max|gpu - oracle| / max contribution)."""
    d = h_in_bits.shape[1]
    u_dev = torch.empty((T, d), dtype=torch.bfloat16, device=h_out_dev.device)
    moe.check(moe.moe_get_block_input(h, u_dev), "moe_get_block_input")
    rb = read_routing(h, T, E, h_out_dev.device)
    gam = {"pre": g_pre.cpu(), "post": g_post.cpu()}
    chain = oracle.block_chain([layer_cpu], [gam], h_in_bits.cpu(), eps=eps)[0]
    u_cpu = u_dev.cpu()
    nflip = check_block_input(u_cpu.to(torch.float64).numpy(), chain["u_exact"], chain["u"])
    ref = oracle.route(u_cpu, layer_cpu["router_w"])
    near = check_routing(rb, ref, E)
    y, _, _ = oracle.forward(layer_cpu, u_cpu)
    for t in np.nonzero(near)[0]:
        o, _, _ = oracle.forward(layer_cpu, u_cpu, tokens=[int(t)], forced_idx=[rb.idx_h[t]])
        y[t] = o[0]
    delta = oracle.rmsnorm(y, gam["post"], eps)
    exact = chain["h_in"] + delta
    got = h_out_dev.cpu().to(torch.float64).numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - exact).max()
    scale = np.abs(delta).max()
    assert err <= OUT_RTOL * scale, f"max|gpu - oracle| = {err:.3e} > {OUT_RTOL} * {scale:.3e}"
    return nflip, int(near.sum()), err / scale
