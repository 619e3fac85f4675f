"""The C-ABI library loads, exports every entry point include/moe.h declares,
and rejects bad arguments on the host before touching a device.

No test here launches a kernel: every call below fails an argument check
that runs before any CUDA call, so these run on a machine without a GPU.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    from mixture_experts_layer_33_b200 import build
    build.build()
    from mixture_experts_layer_33_b200 import moe
    return moe


def _declared():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"MOE_API\s+[^;(]*?\b(moe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_eight_layer_calls():
    names = _declared()
    for n in ("moe_router", "moe_select_topk", "moe_select_expert_choice", "moe_core_set_vote",
              "moe_dispatch", "moe_grouped_mlp", "moe_combine", "moe_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(m):
    lib = ctypes.CDLL(m.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert sorted(_declared()) == sorted(m.ENTRY_POINTS)


def test_status_strings(m):
    for code in range(7):
        assert m.status_string(code).startswith("MOE_")
    assert m.status_string(1234) == "unknown moe_status"


def _cfg(m, **kw):
    from mixture_experts_layer_33_b200 import inputs as gen
    name = kw.pop("name", "ditmoe_xl")
    return m.make_config(gen.workload(name, **kw))


def test_workspace_size_and_assignments(m):
    c = _cfg(m)
    assert m.num_assignments(c) == 8192 * 2
    ws = m.workspace_size(c)
    assert ws % 256 == 0
    # x_perm + H + H_sh + Y + Y_sh dominate: at least their algorithmic size.
    na, d, h, T = 16384, 1152, 4608, 8192
    assert ws >= na * d * 2 + na * h * 2 + T * 2 * h * 2 + na * d * 4 + T * d * 4
    c3 = _cfg(m, name="ecdit")
    assert m.num_assignments(c3) == 64 * 32 * 8
    c4 = _cfg(m, name="des_vote")
    assert m.num_assignments(c4) == 32 * 8


@pytest.mark.parametrize("field,value", [
    ("d", 12), ("E", 0), ("k", 0), ("k", 9), ("dtype", 7), ("routing", 9), ("T", -1),
])
def test_bad_config_rejected(m, field, value):
    c = _cfg(m)
    setattr(c, field, value)
    n = ctypes.c_size_t()
    assert m.LIB.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) == 1


def test_unsupported_sizes(m):
    c = _cfg(m)
    c.E = 200
    n = ctypes.c_size_t()
    assert m.LIB.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) == 2


def test_expert_kinds_must_follow_heavy_ids(m):
    c = _cfg(m, name="mmoe")
    c.expert_kind[3] = m.ZERO  # a zero-computation kind inside the heavy range
    n = ctypes.c_size_t()
    assert m.LIB.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)) == 1


def test_forward_rejects_before_launch(m):
    c = _cfg(m)
    fake = 1 << 20  # never dereferenced: every call below fails a host check first
    args = [ctypes.byref(c), fake, fake, None, fake, None, fake, fake, fake, fake, None, fake,
            None, None]
    # workspace too small
    assert m.LIB.moe_forward(*args, fake, 256, None) == 3
    # misaligned workspace
    assert m.LIB.moe_forward(*args, fake + 8, 1 << 40, None) == 1
    # missing expert weights
    bad = list(args)
    bad[6] = None
    assert m.LIB.moe_forward(*bad, fake, 1 << 40, None) == 1
    # misaligned activation
    bad = list(args)
    bad[1] = fake + 2
    assert m.LIB.moe_forward(*bad, fake, 1 << 40, None) == 1


def test_entry_points_reject_bad_sizes(m):
    fake = 1 << 20
    assert m.LIB.moe_router(fake, fake, None, None, 0.0, 4, 64, 300, 1, fake, fake, 0, 0,
                            None, None, None) == 2
    assert m.LIB.moe_router(fake, fake, None, None, 0.0, 4, 64, 8, 1, fake, fake, 9, 0,
                            fake, fake, None) == 1
    assert m.LIB.moe_select_topk(fake, fake, 4, 8, 0, 0, fake, fake, None) == 1
    assert m.LIB.moe_select_expert_choice(fake, 100, 8, 64, 2, fake, fake, None) == 1
    assert m.LIB.moe_select_expert_choice(fake, 128, 8, 64, 65, fake, fake, None) == 1
    assert m.LIB.moe_core_set_vote(fake, 32, 64, 8, 4, fake, fake, fake, fake, None) == 1
    assert m.LIB.moe_core_set_vote(fake, 32, 300, 8, 32, fake, fake, fake, fake, None) == 2


def test_barrier_wait_hook_checks_its_arguments(m):
    # host-side checks only; valid values just set the hook (no launch)
    assert m.LIB.moe_test_set_barrier_wait(2_000_000_001, 0) == 1  # MOE_ERR_INVALID_ARG
    assert m.LIB.moe_test_set_barrier_wait(0, -1) == 1
    assert m.LIB.moe_test_set_barrier_wait(0, 1025) == 1
    assert m.LIB.moe_test_set_barrier_wait(1000, 1) == 0
    assert m.LIB.moe_test_set_barrier_wait(0, 0) == 0


def test_debug_build_exports_the_same_symbols_and_says_so(m):
    """The MOE_DEBUG variant exports every declared entry point and reports
    itself through moe_build_flags; the regular build does not."""
    from mixture_experts_layer_33_b200 import build
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(dbg, name), name
    dbg.moe_build_flags.restype = ctypes.c_int
    assert dbg.moe_build_flags() & m.BUILD_DEBUG
    assert not m.build_flags() & m.BUILD_DEBUG
