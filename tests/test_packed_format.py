"""The packed weight layout's arithmetic, on the host (no GPU needed).

The packed layout stores every four consecutive input elements w0..w3 of an output feature as the
bytes  s2|m0, s0|m2, s3|m1, s1|m3  (mi = |wi|, si = 0x80 for a negative wi), and the GEMMs' converters
read a word two ways: masked with 0x807F807F it is the bf16 pair (w0, w1) with zero exponent fields,
and with the bytes of each 16-bit half swapped first, the pair (w2, w3); per-block scales use the
exact form (q & 0x807F807F | 0x43004300) - (q & 0x80008000 | 0x43004300) instead.  These tests build
the words from the documented byte layout, apply the same integer steps in numpy and read the
results as bf16 through torch (an implementation of bf16 independent of the CUDA path): every int8
value but -128 must come out as exactly w * 2^-133, or as w itself in the exact form.  The GPU tests
(test_pack_weight_layout, test_every_weight_byte) check the CUDA pack kernel and converters against
the same layout and against the oracle."""
import numpy as np
import torch

MASK = np.uint32(0x807F807F)


def packed_words(w):
    """int8 values w [n, 4] -> the packed 32-bit words (documented byte layout)."""
    w = w.astype(np.int32)
    m = np.abs(w)
    s = (w < 0).astype(np.int32) * 0x80
    b = [s[:, 2] | m[:, 0], s[:, 0] | m[:, 2], s[:, 3] | m[:, 1], s[:, 1] | m[:, 3]]
    return (b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24).astype(np.uint32)


def swap_halves(q):
    """prmt q, q, 0x2301: the two bytes of each 16-bit half exchanged."""
    return ((q >> np.uint32(8)) & np.uint32(0x00FF00FF)) | ((q << np.uint32(8)) & np.uint32(0xFF00FF00))


def bf16_pair(q):
    """A 32-bit word as its two bf16 halves (low half first), in float64."""
    halves = np.stack([q & np.uint32(0xFFFF), q >> np.uint32(16)], axis=1).astype(np.int32)
    t = torch.from_numpy(halves.astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def all_quads():
    """Every value of [-127, 127] in every one of the four positions of a word."""
    v = np.arange(-127, 128)
    rng = np.random.default_rng(5)
    cols = [np.roll(v, 17 * k) for k in range(4)]
    quads = np.stack(cols, axis=1)
    return np.concatenate([quads, rng.integers(-127, 128, size=(4096, 4))]).astype(np.int8)


def test_mask_and_swap_give_the_weights_times_2_to_the_minus_133():
    w = all_quads()
    q = packed_words(w)
    lo = bf16_pair(q & MASK)                  # (w0, w1)
    hi = bf16_pair(swap_halves(q) & MASK)     # (w2, w3)
    got = np.concatenate([lo, hi], axis=1)
    want = w[:, [0, 1, 2, 3]].astype(np.float64) * 2.0 ** -133
    assert np.array_equal(got, want)
    # zero exponent fields: these operands are bf16 numbers below the normal range
    assert np.all(np.abs(got) < 2.0 ** -126)


def test_exact_form_gives_the_weights():
    w = all_quads()
    q = packed_words(w)
    for word, cols in ((q, [0, 1]), (swap_halves(q), [2, 3])):
        a = (word & MASK) | np.uint32(0x43004300)
        b = (word & np.uint32(0x80008000)) | np.uint32(0x43004300)
        ta = torch.from_numpy(np.stack([a & np.uint32(0xFFFF), a >> np.uint32(16)], 1).astype(np.int32)
                              .astype(np.int16)).view(torch.bfloat16)
        tb = torch.from_numpy(np.stack([b & np.uint32(0xFFFF), b >> np.uint32(16)], 1).astype(np.int32)
                              .astype(np.int16)).view(torch.bfloat16)
        diff = (ta - tb).to(torch.float64).numpy()   # a bf16 subtraction, rounded to bf16
        assert np.array_equal(diff, w[:, cols].astype(np.float64))


def test_minus_128_has_no_packed_form():
    """-128 would need an 8-bit magnitude: its packed byte collides with the form of 0."""
    w = np.array([[-128, 0, 0, 0]], dtype=np.int8)
    q = packed_words(w)
    assert bf16_pair(q & MASK)[0, 0] == 0.0
