"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI and compare it with the fp64 oracle on the same seeded inputs."""

import json
import os

import numpy as np
import torch

import oracle
from mixture_experts_layer_33_b200 import inputs as gen

# Tolerances (normwise: max |gpu - ref| / max |ref|).
ROUTER_TOL = 1e-4
Y_TOL = {"bf16": 2e-2, "f32": 1e-4}
ROWSUM_TOL = 1e-5


def moe():
    from mixture_experts_layer_33_b200 import moe as m  # loads libmoe.so
    return m


def normwise(a, ref):
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(a - ref)) / (den if den > 0 else 1.0))


def host(inp):
    return {k: gen.to_numpy_f32(v) for k, v in inp.items()}


def run_layer(cfg, inp, device="cuda", residual=True):
    """moe_forward on device inputs; returns every aux output on the host.

    ``residual=True`` adds x (the layer's residual); ``False`` passes no
    residual, so y holds the expert terms alone (routed + shared)."""
    m = moe()
    c = m.make_config(cfg)
    na = m.num_assignments(c)
    T, E = cfg["T"], cfg["E"]
    dev = device
    aux = {
        "logits": torch.empty(T, E, dtype=torch.float32, device=dev),
        "probs": torch.empty(T, E, dtype=torch.float32, device=dev),
        "sel": torch.empty(na, dtype=torch.int32, device=dev),
        "w": torch.empty(na, dtype=torch.float32, device=dev),
        "votes": torch.empty(E, dtype=torch.int64, device=dev),
        "core": torch.empty(E if cfg["routing"] == "des_seq" else max(cfg.get("M_core", 0), 1),
                            dtype=torch.int32, device=dev),
        "offsets": torch.empty(c.n_heavy + 1, dtype=torch.int32, device=dev),
    }
    ws = m.alloc_workspace(c, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y = torch.empty_like(inp["x"])
    m.forward(c, inp["x"], inp["W_r"], inp["W1"], inp["W2"], y, ws,
              residual=inp["x"] if residual else None,
              z_prev=inp["z_prev"], bias=inp["logit_bias"], Ws1=inp["Ws1"], Ws2=inp["Ws2"],
              const_vecs=inp["const_vecs"], aux=aux, dev_status=status)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in aux.items()}
    out["y"] = gen.to_numpy_f32(y)
    out["status"] = int(status.item())
    return out


def selection_of(cfg, out):
    """The GPU's selection in the oracle's format."""
    T = cfg["T"]
    if cfg["routing"] == "expert_choice":
        G = T // cfg["group_size"]
        shape = (G, cfg["E"], cfg["capacity"])
        return {"tok": out["sel"].reshape(shape), "w": out["w"].reshape(shape)}
    k = cfg["k"]
    return {"idx": out["sel"].reshape(T, k), "w": out["w"].reshape(T, k)}


def oracle_selection_from_gpu(cfg, out):
    """The oracle's selection stage fed the GPU's exact fp32 logits/affinities."""
    z = out["logits"].astype(np.float64)
    A = out["probs"].astype(np.float64)
    r = cfg["routing"]
    if r == "token_topk":
        idx = oracle.topk_token_choice(z, cfg["k"])
        w = oracle.gather_weights(A, idx)
        if cfg.get("renorm"):
            w = oracle.renormalize(w)
        return {"idx": idx, "w": w}
    if r == "expert_choice":
        tok, w = oracle.expert_choice(A, cfg["group_size"], cfg["capacity"])
        return {"tok": tok, "w": w}
    if r == "des_seq":
        core, idx, w = oracle.des_seq(A, cfg["k"], cfg["k_local"])
        return {"idx": idx, "w": w, "core": core}
    votes, core, idx, w = oracle.des_vote(A, cfg["k"], cfg["M_core"])
    return {"idx": idx, "w": w, "votes": votes, "core": core}


def oracle_layer(cfg, hin, sel, tokens=None, residual=True):
    return oracle.forward(cfg, hin["x"], hin["W1"], hin["W2"], sel, cfg["kinds"],
                          hin["const_vecs"], hin["Ws1"], hin["Ws2"],
                          residual=hin["x"] if residual else None, tokens=tokens)


def check_layer_outputs(cfg, inp, hin, sel, out, tokens=None):
    """The layer with the residual (``out``, already run) and without it.

    With x ~ N(0, 1) the residual dominates max|y|, so a normwise bound on
    y alone says little about the expert terms; the residual-free run puts
    the same bound on the routed and shared expert outputs themselves. Both
    runs must take the selection the oracle is fed (the routing does not
    depend on the residual). Returns the two normwise errors."""
    rows = slice(None) if tokens is None else tokens
    y_terms = oracle_layer(cfg, hin, sel, tokens=tokens, residual=False)
    x_rows = hin["x"][rows].astype(np.float64)
    err_res = normwise(out["y"][rows], y_terms + x_rows)
    assert err_res <= Y_TOL[cfg["dtype"]], err_res
    bare = run_layer(cfg, inp, residual=False)
    assert bare["status"] == 0
    np.testing.assert_array_equal(bare["sel"], out["sel"])
    np.testing.assert_array_equal(bare["w"], out["w"])
    err_bare = normwise(bare["y"][rows], y_terms)
    assert err_bare <= Y_TOL[cfg["dtype"]], err_bare
    return err_res, err_bare


def log_errors(case, err_res, err_bare):
    """Append a case's normwise errors (with and without the residual) to
    the JSON-lines file named by MOE_PARITY_LOG, if set."""
    path = os.environ.get("MOE_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, "err_with_residual": err_res,
                                "err_expert_terms": err_bare}) + "\n")
