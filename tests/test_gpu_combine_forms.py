"""The combine's two work splits agree bit for bit, and both match the oracle.

`moe_combine` gives each warp a whole token when there are enough tokens
to occupy every resident warp, and otherwise one 256-feature chunk of a
token (the token's slot metadata then read once per chunk). Both sum each
feature in the same fp32 order (residual, shared output, expert rows in
slot order) and round once, so a prefix of the tokens run alone (chunk
items) must reproduce the same rows of the full call (whole-token items)
byte for byte. The inputs are synthetic combine operands from a seeded
generator: expert ids over every expert kind, dropped rows (row_of = -1),
out-of-range ids, tokens with nothing to sum, expert choice with a varying
number of experts per token, a model width whose last 256-feature chunk is
ragged, and fp32.
"""

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_33_b200 import inputs as gen

from parity_helpers import moe, normwise

pytestmark = pytest.mark.gpu

HEAVY, IDENTITY, ZERO, CONST = gen.HEAVY, gen.IDENTITY, gen.ZERO, gen.CONST


def _token_choice_operands(cfg, gen_t, drop):
    T, k, E, d = cfg["T"], cfg["k"], cfg["E"], cfg["d"]
    sel = torch.randint(0, E, (T * k,), generator=gen_t, dtype=torch.int32)
    bad = torch.rand(T * k, generator=gen_t) < 0.03  # ids the combine must skip
    sel[bad] = torch.where(torch.rand(T * k, generator=gen_t) < 0.5, -1, E).to(torch.int32)[bad]
    row_of = torch.randperm(T * k, generator=gen_t).to(torch.int32)
    row_of[torch.rand(T * k, generator=gen_t) < drop] = -1
    # tokens 5..9: every slot dropped (nothing but the residual, or nothing)
    row_of[5 * k:10 * k] = -1
    sel[5 * k:10 * k] = 0  # expert 0 is heavy in every case here
    a_tok = np.repeat(np.arange(T), k)
    return sel, row_of, None, None, a_tok, T * k


def _expert_choice_operands(cfg, gen_t, drop):
    T, E, S, C = cfg["T"], cfg["E"], cfg["group_size"], cfg["capacity"]
    G = T // S
    per_tok = [[] for _ in range(T)]
    for e in range(E):
        for g in range(G):
            pick = torch.randperm(S, generator=gen_t)[:C].sort().values.numpy() + g * S
            for c, t in enumerate(pick):
                per_tok[int(t)].append(e * G * C + g * C + c)
    tok_assign = np.concatenate([np.sort(np.asarray(p, np.int64)) for p in per_tok]).astype(np.int32)
    tok_ptr = np.concatenate([[0], np.cumsum([len(p) for p in per_tok])]).astype(np.int32)
    n = E * G * C
    row_of = torch.arange(n, dtype=torch.int32)
    row_of[torch.rand(n, generator=gen_t) < drop] = -1
    sel = torch.zeros(n, dtype=torch.int32)  # not read by expert choice
    return sel, row_of, torch.from_numpy(tok_ptr), torch.from_numpy(tok_assign), None, n


CASES = [
    # token choice over heavy, identity, zero and constant experts, shared output
    ("mmoe_kinds", "mmoe", dict(T=2400, d=256, h=256, h_shared=128), 512, True, True),
    # width 1160: the last 256-feature chunk holds 136 features; k = 3,
    # no residual and no shared output (tokens with every slot dropped sum nothing)
    ("ragged_width_no_residual", "ditmoe_xl", dict(T=1500, d=1160, E=8, k=3, h=256, n_shared=0),
     700, False, False),
    # expert choice: 0..16 experts per token
    ("expert_choice", "ecdit", dict(T=4096, group_size=128, d=512, E=16, h=256, capacity=16),
     512, True, False),
    # fp32, 64 features: one partial chunk per warp
    ("fp32", "tiny_fp32", dict(T=4096, n_shared=1, h_shared=64), 1000, True, True),
    # model width 2048 (eight chunks per lane), expert choice with 32 experts
    ("ec_width_2048", "ecdit", dict(T=1280, group_size=128, d=2048, E=32, h=256, capacity=8),
     256, True, False),
]


@pytest.mark.parametrize("label,name,over,T0,with_res,with_sh", CASES, ids=[c[0] for c in CASES])
def test_combine_forms_agree_bitwise(label, name, over, T0, with_res, with_sh):
    m = moe()
    cfg = gen.workload(name, **over)
    T, d, E = cfg["T"], cfg["d"], cfg["E"]
    dt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    g = torch.Generator().manual_seed(1000 + len(label))
    ec = cfg["routing"] == "expert_choice"
    sel, row_of, tok_ptr, tok_assign, a_tok, n_assign = (
        _expert_choice_operands if ec else _token_choice_operands)(cfg, g, drop=0.1)
    w = torch.rand(n_assign, generator=g)
    kinds = cfg["kinds"]
    n_const = sum(1 for kd in kinds if kd == CONST)
    x = torch.randn(T, d, generator=g).to(dt)
    res = torch.randn(T, d, generator=g).to(dt) if with_res else None
    y_sh = torch.randn(T, d, generator=g).to(dt) if with_sh else None
    y_perm = torch.randn(n_assign, d, generator=g).to(dt)
    cv = torch.randn(max(n_const, 1), d, generator=g).to(dt) if n_const else None
    dev = lambda t: None if t is None else t.cuda()
    args = [dev(t) for t in (y_perm, y_sh, sel, w, row_of, tok_ptr, tok_assign, x, cv, res)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    c_full = m.make_config(cfg)
    y_full = torch.full((T, d), 7.0, dtype=dt, device="cuda")
    m.combine(c_full, *args, y_full, status)
    c_pre = m.make_config(gen.workload(name, **dict(over, T=T0)))
    y_pre = torch.full((T0, d), 7.0, dtype=dt, device="cuda")
    m.combine(c_pre, *args, y_pre, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ib = torch.int16 if dt == torch.bfloat16 else torch.int32
    assert torch.equal(y_full[:T0].view(ib), y_pre.view(ib))

    # both against the oracle's combine (fp64) on the same operands
    f64 = lambda t: None if t is None else t.double().numpy()
    yp, xs, cvs = f64(y_perm), f64(x), f64(cv)
    sel_np, row_np, w_np = sel.numpy(), row_of.numpy(), w.numpy()
    cidx = np.cumsum([kd == CONST for kd in kinds]) - 1

    def expert_out(a):
        asg = int(tok_assign.numpy()[a]) if ec else int(a)
        e = (asg // cfg["capacity"]) % E if ec else int(sel_np[asg])
        if not 0 <= e < E:
            return np.zeros(d)
        if kinds[e] == HEAVY:
            return yp[row_np[asg]] if row_np[asg] >= 0 else np.zeros(d)
        if kinds[e] == IDENTITY:
            return xs[a_tok_slots[a]]
        if kinds[e] == CONST:
            return cvs[cidx[e]]
        return np.zeros(d)

    # the oracle walks slots: slot a of token a_tok_slots[a], weight w of its assignment
    if ec:
        a_tok_slots = np.repeat(np.arange(T), np.diff(tok_ptr.numpy()))
        a_w = w_np[tok_assign.numpy()]
    else:
        a_tok_slots = a_tok
        a_w = w_np
    tokens = np.arange(T)
    ref = oracle.combine(tokens, a_tok_slots, None, a_w, expert_out,
                         residual=f64(res), shared_out=f64(y_sh))
    # one rounding of an fp32 sum: 2^-9 relative in bf16, ~1e-7 in fp32
    tol = 2.0 ** -8 if dt == torch.bfloat16 else 1e-5
    assert normwise(y_full.double().cpu().numpy(), ref) <= tol
