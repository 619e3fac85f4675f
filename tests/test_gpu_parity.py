"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases run the whole oracle and span several 128-row tiles with
ragged tails; the full workloads compare the router and every selection
index in full and the layer output on a seeded sample of tokens (the
oracle computes each sampled token's output exactly). Selection, dispatch
and core-set indices must be bit-identical with the oracle fed the GPU's
own fp32 logits/affinities; the router within 1e-4, the layer within 2e-2
(bf16) or 1e-4 (fp32), all normwise relative.
"""

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_33_b200 import inputs as gen
from tests import parity_helpers as H

pytestmark = pytest.mark.gpu

SMALL = [
    ("tiny_fp32", {}),
    ("ditmoe_xl", dict(T=600, d=256, h=512, h_shared=256)),
    ("ecdit", dict(T=6 * 64, group_size=64, d=256, E=16, h=512, capacity=8)),
    ("des_vote", dict(d=256, h=256)),
    ("mmoe", dict(T=600, d=256, h=512, h_shared=256)),
    ("mmoe_skewed", dict(T=600, d=256, h=512, h_shared=256)),
    ("mmoe_constmix", dict(T=600, d=256, h=512, h_shared=256)),
]
# Groups averaging >= 256 rows: the grouped GEMM runs on two-SM (M=256) tiles.
PAIR = [
    ("ditmoe_xl", dict(T=2048, d=256, h=512, h_shared=256)),
    ("ecdit", dict(T=32 * 128, group_size=128, d=256, E=8, h=512, capacity=32)),
    ("des_vote", dict(T=1024, d=256, E=16, k=4, h=256, M_core=8)),
]
FULL = ["tiny_fp32", "ditmoe_xl", "ecdit", "des_vote", "mmoe", "mmoe_skewed", "mmoe_late",
        "mmoe_constmix", "des_seq", "des_vanilla"]


def _check_router(cfg, hin, out):
    z_ref = oracle.router_logits(hin["x"], hin["W_r"], hin["logit_bias"], hin["z_prev"],
                                 cfg["gate_residual_scale"])
    assert H.normwise(out["logits"], z_ref) <= H.ROUTER_TOL
    A = out["probs"].astype(np.float64)
    assert np.all(A >= 0)
    assert np.max(np.abs(A.sum(axis=1) - 1.0)) <= H.ROWSUM_TOL
    assert H.normwise(A, oracle.softmax_rows(z_ref)) <= H.ROUTER_TOL
    return z_ref


def _check_selection(cfg, out):
    gpu = H.selection_of(cfg, out)
    ref = H.oracle_selection_from_gpu(cfg, out)
    key = "tok" if cfg["routing"] == "expert_choice" else "idx"
    np.testing.assert_array_equal(gpu[key], ref[key])
    if cfg.get("renorm"):
        # fp32 w / sum(w) against the same division in fp64: a few ulps.
        np.testing.assert_allclose(gpu["w"].astype(np.float64), ref["w"], rtol=1e-6, atol=0)
    else:
        np.testing.assert_array_equal(gpu["w"].astype(np.float64), ref["w"])
    if cfg["routing"] == "des_vote":
        np.testing.assert_array_equal(out["votes"], ref["votes"])
        np.testing.assert_array_equal(out["core"][:cfg["M_core"]], ref["core"])
    if cfg["routing"] == "des_seq":
        nc = len(ref["core"])
        np.testing.assert_array_equal(out["core"][:nc], ref["core"])
        assert np.all(out["core"][nc:] == -1)
    a_tok, a_exp, _ = oracle.assignments_from_selection(cfg, gpu)
    offsets, *_ = oracle.dispatch(a_tok, a_exp, cfg["E_heavy"], cfg["T"])
    np.testing.assert_array_equal(out["offsets"], offsets)
    return gpu


@pytest.mark.parametrize("name,over", SMALL, ids=[s[0] for s in SMALL])
def test_layer_small_full_oracle(name, over):
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    assert out["status"] == 0
    hin = H.host(inp)
    _check_router(cfg, hin, out)
    sel = _check_selection(cfg, out)
    H.log_errors(f"small/{name}", *H.check_layer_outputs(cfg, inp, hin, sel, out))


@pytest.mark.parametrize("name,over", PAIR, ids=[p[0] for p in PAIR])
def test_layer_two_sm_tiles_full_oracle(name, over):
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    assert out["status"] == 0
    hin = H.host(inp)
    _check_router(cfg, hin, out)
    sel = _check_selection(cfg, out)
    H.log_errors(f"pair/{name}", *H.check_layer_outputs(cfg, inp, hin, sel, out))


@pytest.mark.parametrize("name", FULL)
def test_layer_full_size_sampled(name):
    cfg = gen.workload(name)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    assert out["status"] == 0
    hin = H.host(inp)
    _check_router(cfg, hin, out)
    sel = _check_selection(cfg, out)
    rng = np.random.default_rng(1234)
    T = cfg["T"]
    tokens = np.sort(rng.choice(T, size=min(T, 192), replace=False))
    tokens[-1] = T - 1  # include the ragged end of the last tile
    H.log_errors(f"full/{name}", *H.check_layer_outputs(cfg, inp, hin, sel, out, tokens=tokens))


@pytest.mark.parametrize("name", ["ditmoe_xl", "mmoe"])
def test_independent_routing_flips_are_near_ties(name):
    # The oracle routes from its own fp64 logits; any set that differs from
    # the GPU's must be a near tie of the ranking key.
    cfg = gen.workload(name)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    hin = H.host(inp)
    z_ref = oracle.router_logits(hin["x"], hin["W_r"], hin["logit_bias"], hin["z_prev"],
                                 cfg["gate_residual_scale"])
    idx_ref = oracle.topk_token_choice(z_ref, cfg["k"])
    idx_gpu = out["sel"].reshape(cfg["T"], cfg["k"])
    scale = np.max(np.abs(z_ref))
    for s in np.nonzero(np.any(np.sort(idx_ref, 1) != np.sort(idx_gpu, 1), axis=1))[0]:
        kth_ref = z_ref[s, idx_ref[s, -1]]
        gpu_min = z_ref[s, idx_gpu[s]].min()
        assert abs(kth_ref - gpu_min) <= 1e-5 * scale


def _z_ref(cfg, hin):
    return oracle.router_logits(hin["x"], hin["W_r"], hin["logit_bias"], hin["z_prev"],
                                cfg["gate_residual_scale"])


def _log_affinity(z):
    """log A = z - logsumexp(z) per token, in fp64: the ranking key of A."""
    m = z.max(axis=1, keepdims=True)
    return z - (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))


def test_independent_routing_flips_are_near_ties_expert_choice():
    """Expert choice from the oracle's own fp64 affinities: any (group,
    expert) whose chosen token set differs from the GPU's must differ only
    at a near tie of the key at the C-th place (ranked on log A, so the gap
    is measured like the logits' error)."""
    cfg = gen.workload("ecdit")
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    hin = H.host(inp)
    z = _z_ref(cfg, hin)
    la = _log_affinity(z)
    tok_ref, _ = oracle.expert_choice(np.exp(la), cfg["group_size"], cfg["capacity"])
    S, E, C = cfg["group_size"], cfg["E"], cfg["capacity"]
    G = cfg["T"] // S
    tok_gpu = out["sel"].reshape(G, E, C)
    scale = np.max(np.abs(z))
    flips = 0
    for g in range(G):
        for e in range(E):
            if np.array_equal(tok_ref[g, e], tok_gpu[g, e]):
                continue
            flips += 1
            key = la[g * S:(g + 1) * S, e]
            cth_ref = np.sort(key)[::-1][C - 1]  # the oracle's boundary key
            gpu_min = key[tok_gpu[g, e] - g * S].min()
            assert abs(cth_ref - gpu_min) <= 1e-5 * scale, (g, e)
    H.log_errors(f"independent_routing/ecdit/flipped_sets={flips}", 0.0, 0.0)


def test_independent_routing_flips_are_near_ties_des_vote():
    """DES-Vote from the oracle's own fp64 probabilities, one decision at a
    time, each fed the GPU's earlier decisions: (i) every token's top-K on
    log P, (iii) the core set from the votes the oracle tallies in fp64
    over the GPU's top-K sets, (iv) the re-route over the GPU's core set.
    Every difference must be a near tie of its key."""
    cfg = gen.workload("des_vote")
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    hin = H.host(inp)
    z = _z_ref(cfg, hin)
    la = _log_affinity(z)
    P = np.exp(la)
    T, M, K, Mc = cfg["T"], cfg["E"], cfg["k"], cfg["M_core"]
    scale = np.max(np.abs(z))
    # (i) per-token top-K, the GPU's from its own fp32 probabilities
    P_gpu = out["probs"].astype(np.float64)
    top_gpu = oracle.topk_token_choice(P_gpu, K)
    top_ref = oracle.topk_token_choice(la, K)
    for n in range(T):
        if set(top_gpu[n]) != set(top_ref[n]):
            assert abs(la[n, top_ref[n, -1]] - la[n, top_gpu[n]].min()) <= 1e-5 * scale, n
    # (iii) the core set: fp64 votes over the GPU's top-K sets
    V = np.zeros(M)
    for n in range(T):
        V[top_gpu[n]] += P[n, top_gpu[n]]
    core_gpu = out["core"][:Mc]
    order = sorted(range(M), key=lambda e: (-V[e], e))
    core_ref = np.sort(order[:Mc])
    if not np.array_equal(core_ref, core_gpu):
        vth = V[order[Mc - 1]]
        assert abs(vth - V[core_gpu].min()) <= 1e-5 * V.max()
    # (iv) the re-route over the GPU's core set
    idx_gpu = out["sel"].reshape(T, K)
    for n in range(T):
        keys = la[n, core_gpu]
        ref = core_gpu[np.argsort(-keys, kind="stable")[:K]]
        if set(ref) != set(idx_gpu[n]):
            assert abs(la[n, ref[-1]] - la[n, idx_gpu[n]].min()) <= 1e-5 * scale, n


STAGEWISE = SMALL[1:5] + [("ditmoe_xl_2sm", PAIR[0][1])]


@pytest.mark.parametrize("name,over", STAGEWISE, ids=[s[0] for s in STAGEWISE])
def test_stagewise_entry_points(name, over):
    """Each entry point alone: router -> select -> dispatch -> grouped MLP -> combine."""
    m = H.moe()
    cfg = gen.workload(name.replace("_2sm", ""), **over)
    inp = gen.make_inputs(cfg, "cuda")
    hin = H.host(inp)
    c = m.make_config(cfg)
    na = m.num_assignments(c)
    T, E, d = cfg["T"], cfg["E"], cfg["d"]
    dev = "cuda"
    logits = torch.empty(T, E, device=dev)
    probs = torch.empty(T, E, device=dev)
    sel = torch.empty(na, dtype=torch.int32, device=dev)
    w = torch.empty(na, device=dev)
    r = cfg["routing"]
    m.router(inp["x"], inp["W_r"], logits, probs, bias=inp["logit_bias"], z_prev=inp["z_prev"],
             z_prev_scale=cfg["gate_residual_scale"], k=cfg["k"] if r == "token_topk" else 0,
             idx=sel if r == "token_topk" else None, w=w if r == "token_topk" else None)
    if r == "expert_choice":
        m.select_expert_choice(probs, cfg["group_size"], cfg["capacity"], sel, w)
        torch.cuda.synchronize()
        # the entry point's own outputs, against the oracle on the GPU's probabilities
        ref_tok, ref_w = oracle.expert_choice(probs.cpu().numpy().astype(np.float64),
                                              cfg["group_size"], cfg["capacity"])
        np.testing.assert_array_equal(sel.cpu().numpy().reshape(ref_tok.shape), ref_tok)
        np.testing.assert_array_equal(w.cpu().numpy().reshape(ref_w.shape).astype(np.float64),
                                      ref_w)
    elif r == "des_vote":
        votes = torch.empty(E, dtype=torch.int64, device=dev)
        core = torch.empty(cfg["M_core"], dtype=torch.int32, device=dev)
        m.core_set_vote(probs, cfg["k"], cfg["M_core"], votes, core, sel, w)
        torch.cuda.synchronize()
        ref_votes, ref_core, ref_idx, ref_w = oracle.des_vote(
            probs.cpu().numpy().astype(np.float64), cfg["k"], cfg["M_core"])
        np.testing.assert_array_equal(votes.cpu().numpy(), ref_votes)
        np.testing.assert_array_equal(core.cpu().numpy(), ref_core)
        np.testing.assert_array_equal(sel.cpu().numpy().reshape(ref_idx.shape), ref_idx)
        np.testing.assert_array_equal(w.cpu().numpy().reshape(ref_w.shape).astype(np.float64),
                                      ref_w)
    else:
        # the standalone selection must agree with the fused one bit for bit
        sel2 = torch.empty_like(sel)
        w2 = torch.empty_like(w)
        m.select_topk(logits, probs, cfg["k"], sel2, w2)
        torch.cuda.synchronize()
        assert torch.equal(sel, sel2) and torch.equal(w, w2)
    ws = m.alloc_workspace(c, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets = torch.empty(c.n_heavy + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(na, dtype=torch.int32, device=dev)
    row_of = torch.empty(na, dtype=torch.int32, device=dev)
    tok_ptr = torch.empty(T + 1, dtype=torch.int32, device=dev) if r == "expert_choice" else None
    tok_assign = torch.empty(na, dtype=torch.int32, device=dev) if r == "expert_choice" else None
    x_perm = torch.empty(na, d, dtype=inp["x"].dtype, device=dev)
    m.dispatch(c, sel, inp["x"], x_perm, offsets, perm, row_of, tok_ptr, tok_assign, status, ws)
    torch.cuda.synchronize()
    out = {"logits": logits.cpu().numpy(), "probs": probs.cpu().numpy(),
           "sel": sel.cpu().numpy(), "w": w.cpu().numpy()}
    gsel = H.selection_of(cfg, out)
    a_tok, a_exp, _ = oracle.assignments_from_selection(cfg, gsel)
    o_off, o_perm, o_row, o_tptr, o_tass = oracle.dispatch(a_tok, a_exp, cfg["E_heavy"], T)
    n_rows = int(o_off[-1])
    np.testing.assert_array_equal(offsets.cpu().numpy(), o_off)
    np.testing.assert_array_equal(perm.cpu().numpy()[:n_rows], o_perm)
    np.testing.assert_array_equal(row_of.cpu().numpy(), o_row)
    if r == "expert_choice":
        np.testing.assert_array_equal(tok_ptr.cpu().numpy(), o_tptr)
        np.testing.assert_array_equal(tok_assign.cpu().numpy(), o_tass)
    assert torch.equal(x_perm[:n_rows], inp["x"][perm[:n_rows].long()])

    y_perm = torch.empty(na, d, dtype=inp["x"].dtype, device=dev)
    y_sh = torch.empty(T, d, dtype=inp["x"].dtype, device=dev) if cfg["n_shared"] else None
    m.grouped_mlp(c, x_perm, offsets, inp["W1"], inp["W2"], inp["x"], inp["Ws1"], inp["Ws2"],
                  y_perm, y_sh, status, ws)
    torch.cuda.synchronize()
    yp = gen.to_numpy_f32(y_perm)[:n_rows]
    ref_rows = np.empty_like(yp, dtype=np.float64)
    for e in range(cfg["E_heavy"]):
        lo, hi = o_off[e], o_off[e + 1]
        if hi > lo:
            ref_rows[lo:hi] = oracle.heavy_expert(cfg["act"], hin["x"][o_perm[lo:hi]],
                                                  hin["W1"][e], hin["W2"][e], cfg["h"])
    assert H.normwise(yp, ref_rows) <= H.Y_TOL[cfg["dtype"]]
    if y_sh is not None:
        ref_sh = oracle.mlp_gelu(hin["x"], hin["Ws1"], hin["Ws2"])
        assert H.normwise(gen.to_numpy_f32(y_sh), ref_sh) <= H.Y_TOL[cfg["dtype"]]

    y = torch.empty_like(inp["x"])
    m.combine(c, y_perm, y_sh, sel, w, row_of, tok_ptr, tok_assign, inp["x"],
              inp["const_vecs"], inp["x"], y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    y_ref = H.oracle_layer(cfg, hin, gsel)
    assert H.normwise(gen.to_numpy_f32(y), y_ref) <= H.Y_TOL[cfg["dtype"]]


def _sample_rows(lo, hi, n, rng):
    """n rows of [lo, hi): the first and last (ragged tile end) and a seeded draw."""
    if hi - lo <= n:
        return np.arange(lo, hi)
    mid = rng.choice(np.arange(lo + 1, hi - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[lo, hi - 1], mid]))


@pytest.mark.parametrize("name", ["ditmoe_xl", "ecdit", "mmoe"])
def test_grouped_mlp_full_shape_sampled(name):
    """moe_grouped_mlp alone at the full workload shape (the launch shapes
    the layer uses: wide CTA-pair down projections at K = 4608 / 8192 / 9216,
    the one-SM up projections), without the residual: sampled rows of four
    experts' outputs against the oracle's expert MLP, and the shared
    expert's output on sampled tokens."""
    m = H.moe()
    cfg = gen.workload(name)
    inp = gen.make_inputs(cfg, "cuda")
    c = m.make_config(cfg)
    na = m.num_assignments(c)
    T, E, d = cfg["T"], cfg["E"], cfg["d"]
    dev = "cuda"
    r = cfg["routing"]
    logits = torch.empty(T, E, device=dev)
    probs = torch.empty(T, E, device=dev)
    sel = torch.empty(na, dtype=torch.int32, device=dev)
    w = torch.empty(na, device=dev)
    m.router(inp["x"], inp["W_r"], logits, probs, bias=inp["logit_bias"], z_prev=inp["z_prev"],
             z_prev_scale=cfg["gate_residual_scale"], k=cfg["k"] if r == "token_topk" else 0,
             idx=sel if r == "token_topk" else None, w=w if r == "token_topk" else None)
    if r == "expert_choice":
        m.select_expert_choice(probs, cfg["group_size"], cfg["capacity"], sel, w)
    ws = m.alloc_workspace(c, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets = torch.empty(c.n_heavy + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(na, dtype=torch.int32, device=dev)
    row_of = torch.empty(na, dtype=torch.int32, device=dev)
    ec = r == "expert_choice"
    tok_ptr = torch.empty(T + 1, dtype=torch.int32, device=dev) if ec else None
    tok_assign = torch.empty(na, dtype=torch.int32, device=dev) if ec else None
    x_perm = torch.empty(na, d, dtype=inp["x"].dtype, device=dev)
    m.dispatch(c, sel, inp["x"], x_perm, offsets, perm, row_of, tok_ptr, tok_assign, status, ws)
    y_perm = torch.empty(na, d, dtype=inp["x"].dtype, device=dev)
    y_sh = torch.empty(T, d, dtype=inp["x"].dtype, device=dev) if cfg["n_shared"] else None
    m.grouped_mlp(c, x_perm, offsets, inp["W1"], inp["W2"], inp["x"], inp["Ws1"], inp["Ws2"],
                  y_perm, y_sh, status, ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    off = offsets.cpu().numpy()
    pm = perm.cpu().numpy()
    x_h = gen.to_numpy_f32(inp["x"])
    rng = np.random.default_rng(99)
    # four experts: the first, the last and the two with the most / fewest rows
    cnt = np.diff(off)
    live = np.nonzero(cnt > 0)[0]
    experts = sorted({int(live[0]), int(live[-1]), int(live[np.argmax(cnt[live])]),
                      int(live[np.argmin(cnt[live])])})
    for e in experts:
        rows = _sample_rows(int(off[e]), int(off[e + 1]), 64, rng)
        W1e = gen.to_numpy_f32(inp["W1"][e])
        W2e = gen.to_numpy_f32(inp["W2"][e])
        ref = oracle.heavy_expert(cfg["act"], x_h[pm[rows]], W1e, W2e, cfg["h"])
        got = gen.to_numpy_f32(y_perm[torch.as_tensor(rows, device=dev).long()])
        err = H.normwise(got, ref)
        H.log_errors(f"grouped_mlp/{name}/expert{e}", err, err)
        assert err <= H.Y_TOL[cfg["dtype"]], (e, err)
    if y_sh is not None:
        tokens = _sample_rows(0, T, 128, rng)
        ref = oracle.mlp_gelu(x_h[tokens], gen.to_numpy_f32(inp["Ws1"]),
                              gen.to_numpy_f32(inp["Ws2"]))
        got = gen.to_numpy_f32(y_sh[torch.as_tensor(tokens, device=dev).long()])
        err = H.normwise(got, ref)
        H.log_errors(f"grouped_mlp/{name}/shared", err, err)
        assert err <= H.Y_TOL[cfg["dtype"]], err


# ---------------------------------------------------------------- edge cases
EDGE = [
    ("empty", "ditmoe_xl", dict(T=0, d=256, h=512, h_shared=256)),
    ("one_token", "ditmoe_xl", dict(T=1, d=256, h=512, h_shared=256)),
    ("single_expert", "ditmoe_xl", dict(T=300, d=128, E=1, k=1, h=256, n_shared=0)),
    ("k_equals_E", "ditmoe_xl", dict(T=130, d=128, E=4, k=4, h=256, n_shared=0)),
    ("E_128", "ditmoe_xl", dict(T=257, d=128, E=128, k=8, h=128, n_shared=0)),
    # widths off the 256 grid: GEMM1 N = 640 (128-wide tiles, GELU) next to
    # the shared N = 768, GEMM2 N = 384 (192-wide tiles); ragged tokens
    ("gemm_off_grid_widths", "ditmoe_xl", dict(T=777, d=384, h=640, h_shared=384)),
    # down projections with K >= 2048 and enough tiles to take the CTA-pair
    # tiles with two MMAs per k-step: 256 x 384 tiles (N = 768, shared
    # K = 4096 before routed K = 2048, ragged groups) and 256 x 512 tiles
    # (N = 1024, expert choice)
    ("gemm2_pair_two_mma_384", "ditmoe_xl", dict(T=3000, d=768, h=2048, h_shared=2048)),
    # up projections with short K (256) on CTA pairs, since every problem
    # averages >= 1536 rows per group: 256 x 256 tiles stored by TMA, the
    # 32-row blocks past each expert's ragged end stored per lane, and the
    # shared expert's launch (side stream) on the same kernel
    ("gemm1_pair_short_k", "ditmoe_xl", dict(T=4100, d=256, E=4, k=2, h=512, h_shared=256)),
    ("gemm2_pair_two_mma_512", "ecdit", dict(T=16 * 128, group_size=128, d=1024, E=8, h=2048, capacity=32)),
    # 160 wide (256 x 512) down-projection tiles over 74 CTA pairs: a last
    # wave of 12 tiles on a grid of many pairs
    ("ec_wide_partial_wave", "ecdit", dict(T=40 * 128, group_size=128, d=1024, E=16, h=2048, capacity=32)),
    ("all_zero_compute", "mmoe", dict(T=200, d=128, h=256, h_shared=128, zero_compute_logit_bias=60.0)),
    ("ec_full_capacity", "ecdit", dict(T=64, group_size=16, d=128, E=4, h=256, capacity=16)),
    ("ec_whole_batch", "ecdit", dict(T=2048, group_size=2048, d=128, E=8, h=256, capacity=512)),
    # capacity factors f_c = 1 and 4 (C = f_c * S / E with S = 128, E = 8)
    ("ec_capacity_factor_1", "ecdit", dict(T=512, group_size=128, d=128, E=8, h=256, capacity=16)),
    ("ec_capacity_factor_4", "ecdit", dict(T=512, group_size=128, d=128, E=8, h=256, capacity=64)),
    ("des_beta_one", "des_vote", dict(d=128, h=128, M_core=64)),
    ("odd_N_swiglu_routed", "des_vote", dict(T=37, d=128, E=16, k=4, h=128, M_core=8)),
    ("tiny_fp32_k1", "tiny_fp32", dict(k=1)),
    # fp32 token-choice layers of <= 1024 tokens without a shared expert run
    # as one launch (a CTA per token): zero-computation experts, gate
    # residual and SwiGLU; renormalised weights over 16 experts; one token.
    # Past 1024 tokens the general fp32 path (dispatch, grouped GEMMs).
    ("f32_one_launch_kinds_swiglu", "mmoe", dict(T=200, d=64, h=128, n_shared=0, dtype="f32", act="swiglu")),
    ("f32_one_launch_renorm_E16", "ditmoe_xl", dict(T=300, d=96, E=16, k=4, h=160, n_shared=0, dtype="f32", renorm=1)),
    ("f32_one_launch_one_token", "tiny_fp32", dict(T=1)),
    ("f32_general_path_T2048", "tiny_fp32", dict(T=2048)),
    # Blocks of <= 128 tokens route, dispatch and gather in one cooperative
    # kernel; 129 tokens take the separate finish / dispatch / gather kernels.
    ("small_block_T128_mmoe", "mmoe", dict(T=128, d=128, h=256, h_shared=128)),
    ("small_block_T129_mmoe", "mmoe", dict(T=129, d=128, h=256, h_shared=128)),
    ("small_block_topk_renorm", "ditmoe_xl", dict(T=77, d=128, E=16, k=4, h=256, n_shared=0, renorm=1)),
    ("small_block_des_E128", "des_vote", dict(T=100, d=128, E=128, k=8, h=128, M_core=32)),
    ("small_block_des_T128", "des_vote", dict(T=128, d=256, E=64, k=8, h=128, M_core=16)),
    ("split_router_des_T300", "des_vote", dict(T=300, d=128, E=16, k=4, h=128, M_core=8)),
    # The whole-layer kernel for small blocks without a shared expert: token
    # choice with zero-computation experts and the gate residual, the
    # 128-token boundary, and a model width whose last router slice and
    # expert widths are ragged (d = 1160, h = 264).
    ("block_topk_mmoe_kinds", "mmoe", dict(T=96, d=128, h=256, n_shared=0)),
    # mixed constant experts on a small block (the general path) and fp32
    ("small_constmix_no_shared", "mmoe_constmix", dict(T=96, d=128, h=256, n_shared=0)),
    ("constmix_fp32", "mmoe_constmix", dict(T=200, d=64, h=128, h_shared=64, dtype="f32")),
    ("block_topk_T128", "ditmoe_xl", dict(T=128, d=256, E=16, k=4, h=256, n_shared=0)),
    ("block_des_ragged_d_h", "des_vote", dict(T=40, d=1160, E=32, k=4, h=264, M_core=12)),
    # router weights over 256 KB: the router K-sliced over the CTAs; ragged last slice
    ("block_des_sliced_router", "des_vote", dict(T=32, d=4104, E=64, k=8, h=128, M_core=32)),
    # DES-Seq (core = union of local top-k_local): the whole-layer kernel,
    # a core smaller than K (one token: empty slots), the full local
    # budget (= vanilla), and the general path past 128 tokens.
    ("block_des_seq", "des_seq", dict(d=256, h=256)),
    ("block_des_seq_one_token", "des_seq", dict(T=1, d=256, h=256)),
    ("block_des_seq_full_budget", "des_seq", dict(T=16, d=256, h=256, k_local=8)),
    ("des_seq_T300_general_path", "des_seq", dict(T=300, d=128, E=16, k=4, h=128, k_local=1)),
]


@pytest.mark.parametrize("label,name,over", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases(label, name, over):
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    assert out["status"] == 0
    if cfg["T"] == 0:
        return
    hin = H.host(inp)
    _check_router(cfg, hin, out)
    sel = _check_selection(cfg, out)
    H.log_errors(f"edge/{label}", *H.check_layer_outputs(cfg, inp, hin, sel, out))
    if label == "all_zero_compute":
        assert int(out["offsets"][-1]) == 0  # no heavy rows: no GEMM tiles at all


# The library's limits and ragged widths, sampled like the full workloads:
# the largest DES block (4096 tokens), the largest expert-choice group
# (16384 tokens, one group), 128 experts under top-8 over 65536 tokens
# (half a million assignments, 512 dispatch blocks), and model / hidden
# widths that are not multiples of the 64-wide K block (K = 200 and 168:
# the last TMA box of every row is partly past the end and zero-filled).
LIMITS = [
    ("des_block_4096", "des_vote", dict(T=4096, d=256, h=128)),
    ("ec_group_16384", "ecdit", dict(T=16384, group_size=16384, d=128, E=8, h=256, capacity=2048)),
    ("topk_E128_T65536", "ditmoe_xl", dict(T=65536, d=128, E=128, k=8, h=128, n_shared=0)),
    ("ragged_K_200_168", "mmoe", dict(T=1000, d=200, h=168, h_shared=168)),
]


@pytest.mark.parametrize("label,name,over", LIMITS, ids=[c[0] for c in LIMITS])
def test_limits_and_ragged_widths_sampled(label, name, over):
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    out = H.run_layer(cfg, inp)
    assert out["status"] == 0
    hin = H.host(inp)
    _check_router(cfg, hin, out)
    sel = _check_selection(cfg, out)
    rng = np.random.default_rng(4321)
    T = cfg["T"]
    tokens = np.sort(rng.choice(T, size=min(T, 256), replace=False))
    tokens[0], tokens[-1] = 0, T - 1
    H.log_errors(f"limits/{label}", *H.check_layer_outputs(cfg, inp, hin, sel, out, tokens=tokens))


@pytest.mark.parametrize("N,kl", [(32, 2), (1, 2), (64, 1), (300, 3)])
def test_core_set_union_entry_point(N, kl):
    """moe_core_set_union against the oracle's DES-Seq on the GPU's own probabilities."""
    m = H.moe()
    cfg = gen.workload("des_seq", T=N, d=128, h=128, k_local=kl)
    inp = gen.make_inputs(cfg, "cuda")
    T, E, K = cfg["T"], cfg["E"], cfg["k"]
    logits = torch.empty(T, E, device="cuda")
    probs = torch.empty(T, E, device="cuda")
    m.router(inp["x"], inp["W_r"], logits, probs, bias=inp["logit_bias"])
    core = torch.empty(E, dtype=torch.int32, device="cuda")
    n_core = torch.empty(1, dtype=torch.int32, device="cuda")
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, device="cuda")
    m.core_set_union(probs, K, kl, core, n_core, idx, w)
    torch.cuda.synchronize()
    ref_core, ref_idx, ref_w = oracle.des_seq(probs.cpu().numpy().astype(np.float64), K, kl)
    assert int(n_core.item()) == len(ref_core)
    np.testing.assert_array_equal(core.cpu().numpy()[:len(ref_core)], ref_core)
    assert np.all(core.cpu().numpy()[len(ref_core):] == -1)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(w.cpu().numpy().astype(np.float64), ref_w)


def test_deterministic_bytes():
    cfg = gen.workload("mmoe", T=600, d=256, h=512, h_shared=256)
    inp = gen.make_inputs(cfg, "cuda")
    a = H.run_layer(cfg, inp)
    b = H.run_layer(cfg, inp)
    assert np.array_equal(a["y"].view(np.uint32), b["y"].view(np.uint32))


@pytest.mark.parametrize("T", [64, 2048], ids=["one_block", "multi_block"])
def test_bad_indices_are_flagged_not_faulted(T):
    # Host-side fault injection: corrupt expert ids in a selection; the
    # dispatch kernel's bounds checks flag them and drop those assignments
    # (T=64: the one-block dispatch; T=2048: count, scan and scatter over
    # four blocks), and the kept ones still get stable rows and their x rows.
    m = H.moe()
    cfg = gen.workload("ditmoe_xl", T=T, d=128, h=256, n_shared=0)
    c = m.make_config(cfg)
    na = m.num_assignments(c)
    g = torch.Generator(device="cpu").manual_seed(5)
    sel = torch.randint(0, cfg["E"], (na,), generator=g, dtype=torch.int32)
    sel[3] = 99
    sel[10] = -2  # (-1 marks an empty slot and is skipped without a flag)
    sel = sel.cuda()
    x = torch.randn(cfg["T"], cfg["d"], device="cuda").to(torch.bfloat16)
    ws = m.alloc_workspace(c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    offsets = torch.empty(c.n_heavy + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(na, dtype=torch.int32, device="cuda")
    row_of = torch.empty(na, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(na, cfg["d"], dtype=torch.bfloat16, device="cuda")
    m.dispatch(c, sel, x, x_perm, offsets, perm, row_of, None, None, status, ws)
    torch.cuda.synchronize()
    assert int(status.item()) & m.DEV_BAD_EXPERT
    ro = row_of.cpu().numpy()
    assert ro[3] == -1 and ro[10] == -1
    assert int(offsets[-1].item()) == na - 2
    # The kept assignments: stable rows by expert, rows gathered from x.
    keep = np.ones(na, dtype=bool)
    keep[[3, 10]] = False
    s_np = sel.cpu().numpy()
    a_tok = (np.arange(na) // cfg["k"])[keep]
    ref_off, ref_perm, ref_row, *_ = oracle.dispatch(a_tok, s_np[keep].astype(np.int64),
                                                     cfg["E_heavy"], T)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(ro[keep], ref_row)
    n_rows = int(ref_off[-1])
    np.testing.assert_array_equal(perm.cpu().numpy()[:n_rows], ref_perm)
    assert torch.equal(x_perm[:n_rows], x[perm[:n_rows].long()])
