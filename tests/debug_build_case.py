"""Run by tests/test_gpu_debug_build.py in a process of its own with
MOE_DEBUG=1, so that the binding loads the MOE_DEBUG build of the library
(libmoe_debug.so). Not collected by pytest (no test_ prefix).

1. The debug build computes what the regular one does: two small layers
   against the oracle.
2. Its range checks catch corrupt indices handed to the standalone entry
   points without faulting: row offsets that run backwards or past the
   rows (moe_grouped_mlp), a row past the expert outputs (moe_combine), an
   expert-choice token list entry out of range. Each sets
   MOE_DEV_BAD_INDEX; the combine's output then equals the output with the
   bad slot dropped, byte for byte; a clean call afterwards leaves the
   status at 0.

These corrupt inputs are handed only to a library that reports the
MOE_DEBUG build; the regular build trusts these arrays.
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_33_b200 import inputs as gen  # noqa: E402
from tests import parity_helpers as H  # noqa: E402


def layer_parity(name, over):
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    assert out["status"] == 0, out["status"]
    sel = H.selection_of(cfg, out)
    ref = H.oracle_selection_from_gpu(cfg, out)
    key = "tok" if cfg["routing"] == "expert_choice" else "idx"
    np.testing.assert_array_equal(sel[key], ref[key])
    err = H.normwise(out["y"], H.oracle_layer(cfg, H.host(inp), ref))
    assert err <= H.Y_TOL[cfg["dtype"]], err
    return err


def staged(m, cfg, inp):
    """Router, selection and dispatch through the entry points."""
    c = m.make_config(cfg)
    na = m.num_assignments(c)
    T, E, d = cfg["T"], cfg["E"], cfg["d"]
    r = cfg["routing"]
    logits = torch.empty(T, E, device="cuda")
    probs = torch.empty(T, E, device="cuda")
    sel = torch.empty(na, dtype=torch.int32, device="cuda")
    w = torch.empty(na, device="cuda")
    m.router(inp["x"], inp["W_r"], logits, probs, bias=inp["logit_bias"], z_prev=inp["z_prev"],
             z_prev_scale=cfg["gate_residual_scale"], k=cfg["k"] if r == "token_topk" else 0,
             idx=sel if r == "token_topk" else None, w=w if r == "token_topk" else None)
    if r == "expert_choice":
        m.select_expert_choice(probs, cfg["group_size"], cfg["capacity"], sel, w)
    ws = m.alloc_workspace(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.n_heavy + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(na, dtype=torch.int32, device="cuda")
    row_of = torch.empty(na, dtype=torch.int32, device="cuda")
    ec = r == "expert_choice"
    tok_ptr = torch.empty(T + 1, dtype=torch.int32, device="cuda") if ec else None
    tok_assign = torch.empty(na, dtype=torch.int32, device="cuda") if ec else None
    x_perm = torch.empty(na, d, dtype=inp["x"].dtype, device="cuda")
    m.dispatch(c, sel, inp["x"], x_perm, offsets, perm, row_of, tok_ptr, tok_assign, st, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return c, ws, sel, w, offsets, row_of, tok_ptr, tok_assign, x_perm


def corrupt_offsets(m):
    cfg = gen.workload("mmoe", T=600, d=256, h=512, h_shared=256)
    inp = gen.make_inputs(cfg, "cuda")
    c, ws, sel, w, offsets, row_of, _, _, x_perm = staged(m, cfg, inp)
    na = m.num_assignments(c)
    y_perm = torch.zeros(na, cfg["d"], dtype=torch.bfloat16, device="cuda")
    y_sh = torch.empty(cfg["T"], cfg["d"], dtype=torch.bfloat16, device="cuda")
    bad = offsets.clone()
    bad[3] = bad[4] + 50           # group 3 runs backwards
    bad[-1] = na + 1000            # the last group runs past the rows
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.grouped_mlp(c, x_perm, bad, inp["W1"], inp["W2"], inp["x"], inp["Ws1"], inp["Ws2"],
                  y_perm, y_sh, st, ws)
    torch.cuda.synchronize()
    flagged = int(st.item())
    assert flagged & m.DEV_BAD_INDEX, flagged
    st.zero_()
    m.grouped_mlp(c, x_perm, offsets, inp["W1"], inp["W2"], inp["x"], inp["Ws1"], inp["Ws2"],
                  y_perm, y_sh, st, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return flagged


def corrupt_rows(m):
    cfg = gen.workload("mmoe", T=600, d=256, h=512, h_shared=256)
    inp = gen.make_inputs(cfg, "cuda")
    c, ws, sel, w, offsets, row_of, _, _, x_perm = staged(m, cfg, inp)
    na = m.num_assignments(c)
    y_perm = torch.empty(na, cfg["d"], dtype=torch.bfloat16, device="cuda")
    y_sh = torch.empty(cfg["T"], cfg["d"], dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.grouped_mlp(c, x_perm, offsets, inp["W1"], inp["W2"], inp["x"], inp["Ws1"], inp["Ws2"],
                  y_perm, y_sh, st, ws)
    slot = int(torch.nonzero(row_of >= 0)[5].item())  # a slot with a heavy row
    bad, dropped = row_of.clone(), row_of.clone()
    bad[slot] = na + 10 ** 6
    dropped[slot] = -1
    outs = []
    for rows in (bad, dropped):
        y = torch.empty_like(inp["x"])
        st.zero_()
        m.combine(c, y_perm, y_sh, sel, w, rows, None, None, inp["x"], inp["const_vecs"],
                  inp["x"], y, st)
        torch.cuda.synchronize()
        outs.append((y, int(st.item())))
    assert outs[0][1] & m.DEV_BAD_INDEX, outs[0][1]
    assert outs[1][1] == 0
    assert torch.equal(outs[0][0], outs[1][0])  # the bad slot contributes nothing
    return outs[0][1]


def corrupt_token_list(m):
    cfg = gen.workload("ecdit", T=6 * 64, group_size=64, d=256, E=16, h=512, capacity=8)
    inp = gen.make_inputs(cfg, "cuda")
    c, ws, sel, w, offsets, row_of, tok_ptr, tok_assign, x_perm = staged(m, cfg, inp)
    na = m.num_assignments(c)
    y_perm = torch.zeros(na, cfg["d"], dtype=torch.bfloat16, device="cuda")
    bad_assign = tok_assign.clone()
    bad_assign[7] = na + 12345
    bad_ptr = tok_ptr.clone()
    bad_ptr[-1] = na + 99          # the last token's list runs past the assignments
    flags = []
    for tp, ta in ((tok_ptr, bad_assign), (bad_ptr, tok_assign)):
        y = torch.empty_like(inp["x"])
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        m.combine(c, y_perm, None, sel, w, row_of, tp, ta, inp["x"], None, inp["x"], y, st)
        torch.cuda.synchronize()
        flags.append(int(st.item()))
    assert all(f & m.DEV_BAD_INDEX for f in flags), flags
    return flags


def main():
    from mixture_experts_layer_33_b200 import moe as m
    if not (m.build_flags() & m.BUILD_DEBUG) or not m.LIB_PATH.endswith("libmoe_debug.so"):
        raise SystemExit("not the MOE_DEBUG build: refusing to hand it corrupt indices")
    res = {"lib": os.path.basename(m.LIB_PATH)}
    res["parity_mmoe"] = layer_parity("mmoe", dict(T=600, d=256, h=512, h_shared=256))
    res["parity_ecdit"] = layer_parity("ecdit", dict(T=6 * 64, group_size=64, d=256, E=16,
                                                     h=512, capacity=8))
    res["offsets_flag"] = corrupt_offsets(m)
    res["rows_flag"] = corrupt_rows(m)
    res["token_list_flags"] = corrupt_token_list(m)
    print("DEBUG_BUILD_CASE " + json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
