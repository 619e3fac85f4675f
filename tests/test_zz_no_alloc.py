"""moe_dispatch_noalloc, the dispatch for callers that cannot allocate.

Some callers cannot allocate device memory (a host framework that owns all
device memory and forbids allocation outside its pool, or a path that
cannot afford cudaMalloc's implicit synchronisation), so they cannot pass
the workspace moe_dispatch needs. moe_dispatch_noalloc keeps that scratch in
a fixed library-owned device array instead. These tests call it through the
C ABI and check that two calls in a row give exactly what moe_dispatch
gives and what the oracle's dispatch gives (dispatch is integer and copy
work, so the tolerance is zero); that a large configuration followed by a
smaller one with another expert count still matches (every call shares the
array, so a histogram left by the earlier call must not leak into the
later one); and that a configuration too large for the array is refused.

This file is named to be collected last; it passes alone in a fresh
process and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_33_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def _moe():
    from mixture_experts_layer_33_b200 import moe
    return moe


def _selection(m, cfg, inp):
    """The GPU's own routing for cfg, through the library's entry points."""
    c = m.make_config(cfg)
    na = m.num_assignments(c)
    T, E = cfg["T"], cfg["E"]
    logits = torch.empty(T, E, device="cuda")
    probs = torch.empty(T, E, device="cuda")
    sel = torch.empty(na, dtype=torch.int32, device="cuda")
    w = torch.empty(na, device="cuda")
    topk = cfg["routing"] == "token_topk"
    m.router(inp["x"], inp["W_r"], logits, probs, bias=inp["logit_bias"], z_prev=inp["z_prev"],
             z_prev_scale=cfg["gate_residual_scale"], k=cfg["k"] if topk else 0,
             idx=sel if topk else None, w=w if topk else None)
    if cfg["routing"] == "expert_choice":
        m.select_expert_choice(probs, cfg["group_size"], cfg["capacity"], sel, w)
    return c, sel


def _outputs(m, c, cfg, poison):
    na = m.num_assignments(c)
    ec = cfg["routing"] == "expert_choice"
    T, d = cfg["T"], cfg["d"]
    t = {
        "offsets": torch.full((c.n_heavy + 1,), poison, dtype=torch.int32, device="cuda"),
        "perm": torch.full((na,), poison, dtype=torch.int32, device="cuda"),
        "row_of": torch.full((na,), poison, dtype=torch.int32, device="cuda"),
        "x_perm": torch.full((na, d), float(poison), device="cuda").to(torch.bfloat16),
        "tok_ptr": torch.full((T + 1,), poison, dtype=torch.int32, device="cuda") if ec else None,
        "tok_assign": torch.full((na,), poison, dtype=torch.int32, device="cuda") if ec else None,
        "status": torch.zeros(1, dtype=torch.int32, device="cuda"),
    }
    return t


def _check_against_oracle(m, c, cfg, sel, got):
    """offsets, perm and row_of (and the expert-choice token lists) against
    the oracle's dispatch of the same selection; x_perm rows against x."""
    na = m.num_assignments(c)
    s = sel.cpu().numpy()
    if cfg["routing"] == "expert_choice":
        G = cfg["T"] // cfg["group_size"]
        a_tok = s.astype(np.int64)
        a_exp = np.tile(np.repeat(np.arange(cfg["E"]), cfg["capacity"]), G)
    else:
        a_tok = np.arange(na) // cfg["k"]
        a_exp = s.astype(np.int64)
    off, perm, row_of, tptr, tass = oracle.dispatch(a_tok, a_exp, cfg["E_heavy"], cfg["T"])
    n_rows = int(off[-1])
    np.testing.assert_array_equal(got["offsets"].cpu().numpy(), off)
    np.testing.assert_array_equal(got["perm"].cpu().numpy()[:n_rows], perm)
    np.testing.assert_array_equal(got["row_of"].cpu().numpy(), row_of)
    if got["tok_ptr"] is not None:
        np.testing.assert_array_equal(got["tok_ptr"].cpu().numpy(), tptr)
        np.testing.assert_array_equal(got["tok_assign"].cpu().numpy(), tass)
    return n_rows


CASES = [
    ("token_choice", "ditmoe_xl", dict(T=600, d=256, h=512, h_shared=256)),
    # 12 groups x 16 experts x C = 8: 1536 assignments, two dispatch blocks
    ("expert_choice", "ecdit", dict(T=12 * 64, group_size=64, d=256, E=16, h=512, capacity=8)),
    ("expert_choice_one_block", "ecdit", dict(T=6 * 64, group_size=64, d=256, E=16, h=512,
                                              capacity=8)),
    ("zero_compute", "mmoe", dict(T=600, d=256, h=512, h_shared=256)),
]


@pytest.mark.parametrize("label,name,over", CASES, ids=[c[0] for c in CASES])
def test_noalloc_dispatch_matches_workspace_dispatch_twice(label, name, over):
    m = _moe()
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    c, sel = _selection(m, cfg, inp)

    ref = _outputs(m, c, cfg, poison=-3)
    ws = m.alloc_workspace(c)
    m.dispatch(c, sel, inp["x"], ref["x_perm"], ref["offsets"], ref["perm"], ref["row_of"],
               ref["tok_ptr"], ref["tok_assign"], ref["status"], ws)
    torch.cuda.synchronize()
    n_rows = int(ref["offsets"][-1].item())

    for call in range(2):
        got = _outputs(m, c, cfg, poison=-7 - call)
        m.dispatch_noalloc(c, sel, inp["x"], got["x_perm"], got["offsets"], got["perm"],
                           got["row_of"], got["tok_ptr"], got["tok_assign"], got["status"])
        torch.cuda.synchronize()
        assert int(got["status"].item()) == 0
        assert torch.equal(got["offsets"], ref["offsets"]), call
        assert torch.equal(got["perm"][:n_rows], ref["perm"][:n_rows]), call
        assert torch.equal(got["row_of"], ref["row_of"]), call
        assert torch.equal(got["x_perm"][:n_rows], ref["x_perm"][:n_rows]), call
        if got["tok_ptr"] is not None:
            assert torch.equal(got["tok_ptr"], ref["tok_ptr"]), call
            assert torch.equal(got["tok_assign"], ref["tok_assign"]), call
        assert _check_against_oracle(m, c, cfg, sel, got) == n_rows
        assert torch.equal(got["x_perm"][:n_rows], inp["x"][got["perm"][:n_rows].long()])


def test_noalloc_dispatch_large_then_small_configuration():
    """A large call (65536 assignments: 64 blocks x 64 heavy experts of
    histograms) fills much of the shared array; the smaller call after it,
    with 16 heavy experts and three blocks, must match moe_dispatch and the
    oracle exactly, as must the large one."""
    m = _moe()
    seq = [gen.workload("ditmoe_xl", T=8192, d=128, E=64, k=8, h=128, n_shared=0),
           gen.workload("mmoe", T=1200, d=128, h=256, h_shared=128),
           gen.workload("ditmoe_xl", T=8192, d=128, E=64, k=8, h=128, n_shared=0)]
    for i, cfg in enumerate(seq):
        inp = gen.make_inputs(cfg, "cuda")
        c, sel = _selection(m, cfg, inp)
        ref = _outputs(m, c, cfg, poison=-3)
        ws = m.alloc_workspace(c)
        m.dispatch(c, sel, inp["x"], ref["x_perm"], ref["offsets"], ref["perm"], ref["row_of"],
                   ref["tok_ptr"], ref["tok_assign"], ref["status"], ws)
        got = _outputs(m, c, cfg, poison=-9)
        m.dispatch_noalloc(c, sel, inp["x"], got["x_perm"], got["offsets"], got["perm"],
                           got["row_of"], got["tok_ptr"], got["tok_assign"], got["status"])
        torch.cuda.synchronize()
        assert int(got["status"].item()) == 0, i
        n_rows = _check_against_oracle(m, c, cfg, sel, got)
        assert torch.equal(got["offsets"], ref["offsets"]), i
        assert torch.equal(got["perm"][:n_rows], ref["perm"][:n_rows]), i
        assert torch.equal(got["row_of"], ref["row_of"]), i
        assert torch.equal(got["x_perm"][:n_rows], ref["x_perm"][:n_rows]), i


def test_noalloc_dispatch_rejects_configurations_beyond_its_scratch():
    m = _moe()
    # 65536 tokens x top-8 over 128 experts need 512 blocks x 128 experts x 4 B
    # = 256 KiB of histograms, which just fits; 1024 tokens more add eight
    # blocks, more than the array holds.
    cfg = gen.workload("ditmoe_xl", T=65536 + 1024, d=256, E=128, k=8, h=256, n_shared=0)
    c = m.make_config(cfg)
    fake = 1 << 20  # never dereferenced: the size check comes first
    code = m.LIB.moe_dispatch_noalloc(ctypes.byref(c), fake, None, None, fake, fake, fake,
                                      None, None, None, None)
    assert code == 2  # MOE_ERR_UNSUPPORTED
    with pytest.raises(RuntimeError, match="library-owned array"):
        m.dispatch_noalloc(c, torch.empty(1, dtype=torch.int32, device="cuda"), None, None,
                           torch.empty(129, dtype=torch.int32, device="cuda"),
                           torch.empty(1, dtype=torch.int32, device="cuda"),
                           torch.empty(1, dtype=torch.int32, device="cuda"), None, None, None)
