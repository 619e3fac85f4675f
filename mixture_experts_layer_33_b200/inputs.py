"""Seeded synthetic inputs for the MoE layer, shared by the CUDA path's
tests and benchmark and by the oracle's tests.

This module draws random tensors of the right shapes and distributions and
nothing else: it holds none of the layer's arithmetic, and it imports
neither the CUDA binding nor the oracle.

Each tensor comes from its own ``torch.Generator`` seeded with
``seed * 1000 + tensor_id``; values are drawn in fp32 and rounded to the
workload's dtype (round-to-nearest-even for bf16). Generation on a CUDA
device and on the CPU give different (equally valid) streams, so a test
generates once and hands the same tensors to both sides.
"""

from __future__ import annotations

import copy

import torch

HEAVY, IDENTITY, ZERO, CONST = 0, 1, 2, 3

# Tensor ids of the per-tensor generator streams.
_TID = {"x": 1, "W_r": 2, "W1": 3, "W2": 4, "Ws1": 5, "Ws2": 6,
        "logit_bias": 7, "z_prev": 8, "const_vecs": 9, "const_mix": 10}

# The five workloads. Shapes and distributions follow the pages' models:
#   tiny_fp32  - small token-choice layer (fp32) for exhaustive checks;
#   ditmoe_xl  - DiT-MoE-XL (DICE page): 32 images x 256 latent tokens,
#                d=1152, 8 routed experts top-2 + 2 shared, MLP 1152-4608;
#   ecdit      - EC-DiT expert-choice layer: 64 sequences x 128 tokens,
#                d=2048, E=32, f_c=2 (C=8), MLP 2048-8192;
#   des_vote   - DES dLLM block: N=32 tokens, d=2048, M=64, K=8, beta=0.5,
#                SwiGLU 2048-1024, per-expert logit bias ~N(0,1);
#   mmoe       - MMOE MoE++ layer: 32 x 256 tokens, d=1152, 16 heavy +
#                identity + zero + constant experts, top-2, gate residual
#                0.5, 1 shared expert, MLP 1152-4608.
WORKLOADS = {
    "tiny_fp32": dict(
        routing="token_topk", dtype="f32", act="gelu", T=256, d=64, E=8, k=2,
        h=256, n_shared=0, h_shared=0, seed=0, x_std=0.02, w_std=0.02),
    "ditmoe_xl": dict(
        routing="token_topk", dtype="bf16", act="gelu", T=32 * 256, d=1152,
        E=8, k=2, h=4608, n_shared=2, h_shared=4608, seed=1, x_std=1.0,
        w_std=0.02),
    "ecdit": dict(
        routing="expert_choice", dtype="bf16", act="gelu", T=64 * 128,
        d=2048, E=32, k=0, h=8192, n_shared=0, h_shared=0, group_size=128,
        capacity_factor=2.0, capacity=8, seed=2, x_std=1.0, w_std=0.02),
    "des_vote": dict(
        routing="des_vote", dtype="bf16", act="swiglu", T=32, d=2048, E=64,
        k=8, h=1024, n_shared=0, h_shared=0, beta=0.5, M_core=32, seed=3, x_std=1.0,
        w_std=0.02, logit_bias_std=1.0),
    "mmoe": dict(
        routing="token_topk", dtype="bf16", act="gelu", T=32 * 256, d=1152,
        E=19, k=2, h=4608, n_shared=1, h_shared=4608, seed=4, x_std=1.0,
        w_std=0.02, gate_residual_scale=0.5, z_prev_std=1.0,
        kinds=[HEAVY] * 16 + [IDENTITY, ZERO, CONST]),
}

# The MMOE page reports that 44.6 % of the routing in early blocks goes to
# the zero-computation experts. This variant adds a fixed logit bias to
# those three experts so that roughly that share of the routed slots lands
# on them. The value was calibrated with the oracle's routing by
# tests/golden/calibrate_mmoe_skew.py.
MMOE_SKEW_BIAS = 0.791
WORKLOADS["mmoe_skewed"] = dict(WORKLOADS["mmoe"], zero_compute_logit_bias=MMOE_SKEW_BIAS)
# Late blocks: 23.4 % of the routing to the lightweight experts (same page,
# same calibration).
MMOE_LATE_BIAS = 0.2351
WORKLOADS["mmoe_late"] = dict(WORKLOADS["mmoe"], zero_compute_logit_bias=MMOE_LATE_BIAS)
# The constant expert as a learned-vector mixture (a0 x + a1 v, (a0, a1) =
# softmax(Wc x)), on the early-block routing so that it gets many tokens.
WORKLOADS["mmoe_constmix"] = dict(WORKLOADS["mmoe_skewed"], const_mix=1)


# The DES page's two core-set functions and the vanilla block on the same
# inputs (seed 3): DES-Seq (section 2.3) with a local budget of 2 experts
# per token, and vanilla top-8 routing with no core set (section 2.5).
WORKLOADS["des_seq"] = dict(WORKLOADS["des_vote"], routing="des_seq", k_local=2)
WORKLOADS["des_vanilla"] = dict(WORKLOADS["des_vote"], routing="token_topk")


def workload(name, **overrides):
    """The named workload's configuration, with shape overrides applied."""
    cfg = copy.deepcopy(WORKLOADS[name])
    cfg.update(overrides)
    cfg["name"] = name
    derive(cfg)
    return cfg


def derive(cfg):
    """Fill in defaults and count the heavy experts.

    The integer routing parameters are stated in the workload itself:
    ``capacity`` (EC-DiT's C = f_c*S/E: 2*128/32 = 8 for ``ecdit``) and
    ``M_core`` (DES's beta*M: 0.5*64 = 32 for ``des_vote``); a shape
    override that changes S, E or M must restate them.
    """
    cfg.setdefault("kinds", [HEAVY] * cfg["E"])
    cfg["E_heavy"] = sum(1 for k in cfg["kinds"] if k == HEAVY)
    cfg.setdefault("gate_residual_scale", 0.0)
    cfg.setdefault("renorm", 0)
    return cfg


def torch_dtype(cfg):
    return torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16


def _normal(shape, std, tid, cfg, device, dtype):
    g = torch.Generator(device=device)
    g.manual_seed(int(cfg["seed"]) * 1000 + _TID[tid])
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_inputs(cfg, device="cpu"):
    """All tensors of one layer invocation, drawn from the workload's seed.

    Layouts (row-major, contiguous):
      x          [T, d]                 dtype
      W_r        [E, d]                 dtype (row e = expert e's router weights)
      logit_bias [E] fp32 or None
      z_prev     [T, E] fp32 or None    (previous layer's gate logits)
      W1         [E_h, h, d] (GELU) or [E_h, 2h, d] (SwiGLU: gate rows, then up rows)
      W2         [E_h, d, h]
      Ws1        [n_sh*h_sh, d] or None (shared experts, concatenated hidden)
      Ws2        [d, n_sh*h_sh] or None
      const_vecs [n_const, d] or None   (constant experts' vectors, id order;
                 [n_const, 3, d] with const_mix: v, then the mixing weights Wc)
    """
    dt = torch_dtype(cfg)
    T, d, E, h = cfg["T"], cfg["d"], cfg["E"], cfg["h"]
    Eh = cfg["E_heavy"]
    ws = cfg["w_std"]
    out = {}
    out["x"] = _normal((T, d), cfg["x_std"], "x", cfg, device, dt)
    out["W_r"] = _normal((E, d), ws, "W_r", cfg, device, dt)
    bias = None
    if cfg.get("logit_bias_std"):
        bias = _normal((E,), cfg["logit_bias_std"], "logit_bias", cfg, device, torch.float32)
    if cfg.get("zero_compute_logit_bias"):
        zb = torch.tensor([cfg["zero_compute_logit_bias"] if k != HEAVY else 0.0
                           for k in cfg["kinds"]], dtype=torch.float32, device=device)
        bias = zb if bias is None else bias + zb
    out["logit_bias"] = bias
    out["z_prev"] = None
    if cfg.get("gate_residual_scale"):
        out["z_prev"] = _normal((T, E), cfg.get("z_prev_std", 1.0), "z_prev", cfg, device, torch.float32)
    rows1 = 2 * h if cfg["act"] == "swiglu" else h
    out["W1"] = _normal((Eh, rows1, d), ws, "W1", cfg, device, dt)
    out["W2"] = _normal((Eh, d, h), ws, "W2", cfg, device, dt)
    hs = cfg["n_shared"] * cfg["h_shared"]
    if hs:
        out["Ws1"] = _normal((hs, d), ws, "Ws1", cfg, device, dt)
        out["Ws2"] = _normal((d, hs), ws, "Ws2", cfg, device, dt)
    else:
        out["Ws1"] = out["Ws2"] = None
    n_const = sum(1 for k in cfg["kinds"] if k == CONST)
    out["const_vecs"] = (_normal((n_const, d), ws, "const_vecs", cfg, device, dt)
                         if n_const else None)
    if n_const and cfg.get("const_mix"):
        # [n_const, 3, d]: v, then the mixing weights Wc [2, d]
        wc = _normal((n_const, 2, d), ws, "const_mix", cfg, device, dt)
        out["const_vecs"] = torch.cat([out["const_vecs"][:, None, :], wc], dim=1).contiguous()
    return out


def to_numpy_f32(t):
    """Host fp32 copy of a tensor (exact for bf16 and fp32), or None."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float32).numpy()
