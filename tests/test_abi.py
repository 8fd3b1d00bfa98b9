"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/moe.h declares, and rejects invalid arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    import mixture_experts_softmax_b200 as m
    return m


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports(m):
    assert declared_symbols() == sorted(m.EXPORTS)


def declared_parameters():
    """name -> the kinds of its parameters in include/moe.h: 'p' pointer (moe_handle included), 'i' int
    (int, int32_t), 'f' float, 'l' long long."""
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "moe.h")).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(([^)]*)\)", src):
        kinds = []
        for prm in (q.strip() for q in params.split(",")):
            if prm in ("", "void"):
                continue
            if "*" in prm or prm.startswith("moe_handle"):
                kinds.append("p")
            elif prm.startswith("long long"):
                kinds.append("l")
            elif prm.startswith("float"):
                kinds.append("f")
            else:
                assert prm.split()[0] in ("int", "int32_t"), prm
                kinds.append("i")
        out[name] = kinds
    return out


def test_binding_signatures_follow_the_header(m):
    """Every ctypes signature the binding sets has the header's parameter count and kinds, so a call
    through the binding passes each argument in the width the library reads."""
    def kind(t):
        if t is ctypes.c_int:
            return "i"
        if t is ctypes.c_float:
            return "f"
        if t is ctypes.c_longlong:
            return "l"
        return "p"   # c_void_p and POINTER(...)
    lib = m.lib()
    declared = declared_parameters()
    assert sorted(declared) == sorted(m.EXPORTS)
    for name, kinds in declared.items():
        got = [kind(t) for t in getattr(lib, name).argtypes]
        assert got == kinds, (name, got, kinds)


def test_library_exports_every_declared_symbol(m):
    lib = ctypes.CDLL(m.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_library_needs_no_cuda_shared_library(m):
    # the CUDA runtime is linked statically; libcuda is reached through the runtime at first use
    import subprocess
    out = subprocess.run(["ldd", m.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out and "libcuda.so" not in out


def test_strerror_and_version(m):
    assert m.moe_strerror(0) == "ok"
    for code in (m.MOE_EINVAL, m.MOE_EUNSUPPORTED, m.MOE_ENOMEM, m.MOE_ECUDA, m.MOE_ETIMEOUT, m.MOE_ENODEV,
                 m.MOE_ERANGE):
        assert m.moe_strerror(code) not in ("ok", "unknown status code")
    assert m.moe_strerror(12345) == "unknown status code"
    assert m.moe_version() >= 100


def test_create_validation(m):
    assert m.moe_create(0, 512, 8, 2)[0] == m.MOE_EINVAL
    assert m.moe_create(256, 512, 8, 9)[0] == m.MOE_EINVAL          # k > E
    assert m.moe_create(256, 512, 4, 2)[0] == m.MOE_EUNSUPPORTED    # E != 8
    assert m.moe_create(256, 512, 8, 1)[0] == m.MOE_EUNSUPPORTED    # k != 2
    assert m.moe_create(200, 512, 8, 2)[0] == m.MOE_EUNSUPPORTED    # d % 128
    assert m.moe_create(256, 500, 8, 2)[0] == m.MOE_EUNSUPPORTED    # ffn % 128
    rc, h = m.moe_create(6144, 32768, 8, 2)
    assert rc == m.MOE_OK and h
    assert m.moe_destroy(h) == m.MOE_OK
    assert m.moe_destroy(None) == m.MOE_OK


def test_plan(m):
    rc, h = m.moe_create(6144, 32768, 8, 2)
    try:
        assert m.moe_plan(h, 8)[:2] == (0, 16)
        assert m.moe_plan(h, 32)[:2] == (0, 32)
        assert m.moe_plan(h, 64)[:2] == (0, 64)
        assert m.moe_plan(h, 8192)[:2] == (0, 128)
        assert m.moe_plan(h, 8)[2] == 8          # decode: the down-projection splits K
        assert m.moe_plan(h, 8192)[2] == 1       # prefill: enough tiles without splitting
        assert m.moe_plan(h, 1664) == (0, 128, 2)   # the plan test_wide_tiles_odd_segments_and_pieces needs
        assert m.moe_plan(h, -1)[0] == m.MOE_EINVAL
    finally:
        m.moe_destroy(h)


def test_forward_argument_checks_on_host(m):
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == 0
    A = 1 << 20                       # fake, 16-byte aligned addresses: never dereferenced
    good = [A, A + 0x1000, A + 0x2000, A + 0x3000, A + 0x4000, A + 0x5000, A + 0x6000]
    x, out = A + 0x100000, A + 0x200000
    try:
        assert m.moe_forward(h, -1, x, *good, out, 0) == m.MOE_EINVAL
        assert m.moe_forward(h, m.MOE_MAX_TOKENS + 1, x, *good, out, 0) == m.MOE_EINVAL
        assert m.moe_forward(h, 0, x, *good, out, 0) == m.MOE_OK              # empty input: no-op
        assert m.moe_forward(h, 4, None, *good, out, 0) == m.MOE_EINVAL
        assert m.moe_forward(h, 4, x, *good, None, 0) == m.MOE_EINVAL
        assert m.moe_forward(h, 4, x + 2, *good, out, 0) == m.MOE_EINVAL      # misaligned
        for i in range(7):
            bad = list(good)
            bad[i] = None
            assert m.moe_forward(h, 4, x, *bad, out, 0) == m.MOE_EINVAL
            bad[i] = good[i] + 8
            assert m.moe_forward(h, 4, x, *bad, out, 0) == m.MOE_EINVAL
        assert m.moe_forward(h, 4, x, *good, x + 16, 0) == m.MOE_EINVAL      # out overlaps x
        assert m.moe_forward(None, 4, x, *good, out, 0) == m.MOE_EINVAL
        assert m.moe_block_forward(h, 4, None, x, x, 1e-5, *good, 0) == m.MOE_EINVAL
        assert m.moe_block_forward(h, 4, out, x, x, -1.0, *good, 0) == m.MOE_EINVAL
        assert m.moe_forward_host(h, 4, None, *good, out, 0) == m.MOE_EINVAL
        assert m.moe_get_routing(h) == m.MOE_EINVAL                             # no forward yet
        assert m.moe_set_timeout(h, -5) == m.MOE_EINVAL
        assert m.moe_set_router_bias(h, A + 4) == m.MOE_EINVAL
    finally:
        m.moe_destroy(h)


def test_setter_argument_checks(m):
    """Handle settings are validated on the host; they need no GPU."""
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == 0
    try:
        assert m.moe_set_scale_block(None, 0) == m.MOE_EINVAL
        assert m.moe_set_scale_block(h, 64) == m.MOE_EUNSUPPORTED
        assert m.moe_set_scale_block(h, 128) == m.MOE_OK
        assert m.moe_set_scale_block(h, 0) == m.MOE_OK
        assert m.moe_set_padding_mask(None, None) == m.MOE_EINVAL
        assert m.moe_set_padding_mask(h, (1 << 20) + 3) == m.MOE_OK     # kept, not dereferenced here
        assert m.moe_set_padding_mask(h, None) == m.MOE_OK
    finally:
        m.moe_destroy(h)


def test_forward_without_gpu_reports_no_device(m):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc, h = m.moe_create(256, 512, 8, 2)
    A = 1 << 20
    good = [A + i * 0x1000 for i in range(7)]
    try:
        assert m.moe_forward(h, 4, A + 0x100000, *good, A + 0x200000, 0) == m.MOE_ENODEV
    finally:
        m.moe_destroy(h)



def test_block_input_needs_a_block_forward(m):
    """moe_get_block_input before any forward (here: a handle that never ran) is refused on the host."""
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == m.MOE_OK
    try:
        assert m.moe_get_block_input(h, 1 << 20, 0) == m.MOE_EINVAL
        assert m.moe_get_block_input(None, 1 << 20, 0) == m.MOE_EINVAL
    finally:
        m.moe_destroy(h)


def test_pack_weight_n_checks_the_expert_count(m):
    """An expert-parallel rank packs its own experts: the count must lie in 1 .. E (checked on
    the host before any device work)."""
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == m.MOE_OK
    try:
        A, B = 1 << 20, 1 << 30   # aligned, far apart: the count check comes first
        assert m.moe_pack_weight_n(h, A, B, 0, 0, 0) == m.MOE_EINVAL
        assert m.moe_pack_weight_n(h, A, B, 0, 9, 0) == m.MOE_EINVAL
        assert m.moe_pack_weight_n(h, A, B, 2, 4, 0) == m.MOE_EINVAL
    finally:
        m.moe_destroy(h)


def test_cta_pairs_modes(m):
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == m.MOE_OK
    try:
        for mode in (m.MOE_PAIRS_OFF, m.MOE_PAIRS_LARGE_DOWN, m.MOE_PAIRS_LARGE, m.MOE_PAIRS_ALL):
            assert m.moe_set_cta_pairs(h, mode) == m.MOE_OK
        assert m.moe_set_cta_pairs(h, 4) == m.MOE_EINVAL
        assert m.moe_set_cta_pairs(h, -1) == m.MOE_EINVAL
        assert m.moe_set_cta_pairs(None, 1) == m.MOE_EINVAL
    finally:
        m.moe_destroy(h)


def test_host_overlap_switch(m):
    rc, h = m.moe_create(256, 512, 8, 2)
    assert rc == m.MOE_OK
    try:
        assert m.moe_set_host_overlap(h, 1) == m.MOE_OK
        assert m.moe_set_host_overlap(h, 0) == m.MOE_OK
        assert m.moe_set_host_overlap(h, 2) == m.MOE_EINVAL
        assert m.moe_set_host_overlap(None, 1) == m.MOE_EINVAL
        # nothing in flight: nothing to wait for (no CUDA call is made)
        assert m.moe_host_wait(h, None) == m.MOE_OK
        assert m.moe_host_wait(None, None) == m.MOE_EINVAL
    finally:
        m.moe_destroy(h)
