"""The expert-parallel steps on the GPU: `CudaOps` through the C ABI on a
one-rank NCCL process group (the one GPU of this test owns every expert, so
the two exchanges are copies to itself, but every kernel step of the
expert-parallel path runs: route, dispatch, regroup, grouped MLP, row
gather, shared expert, combine). The synchronous form must match the
oracle layer (and moe_forward up to bf16 rounding); DICE's interweaved
form must match the oracle's one-step-stale combine on its second step.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from mixture_experts_layer_33_b200 import inputs as gen
from mixture_experts_layer_33_b200.expert_parallel import (CudaOps, ExpertShard, InterweavedEP,
                                                           ep_forward)
from tests import parity_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=__import__("datetime").timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


def _ops(cfg, inp):
    shard = ExpertShard(cfg["E_heavy"], 1)
    ops = CudaOps(cfg, shard, 0, inp["W_r"], inp["W1"], inp["W2"], bias=inp["logit_bias"],
                  Ws1=inp["Ws1"], Ws2=inp["Ws2"], const_vecs=inp["const_vecs"])
    return shard, ops


def _gpu_selection(cfg, inp, x):
    """The router's selection of x (the same kernel CudaOps.route runs)."""
    m = H.moe()
    T, E, k = x.shape[0], cfg["E"], cfg["k"]
    logits = torch.empty(T, E, device="cuda")
    probs = torch.empty(T, E, device="cuda")
    sel = torch.empty(T * k, dtype=torch.int32, device="cuda")
    w = torch.empty(T * k, device="cuda")
    m.router(x, inp["W_r"], logits, probs, bias=inp["logit_bias"], z_prev=inp["z_prev"],
             z_prev_scale=cfg["gate_residual_scale"], k=k, idx=sel, w=w)
    torch.cuda.synchronize()
    idx = oracle.topk_token_choice(logits.cpu().numpy().astype(np.float64), k)
    np.testing.assert_array_equal(sel.cpu().numpy().reshape(T, k), idx)
    return {"idx": idx, "w": w.cpu().numpy().astype(np.float64).reshape(T, k)}


CASES = [("mmoe", dict(T=600, d=256, h=512, h_shared=256)),
         ("ditmoe_xl", dict(T=1000, d=256, h=512, h_shared=256))]


@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_cuda_expert_parallel_one_rank(group, name, over):
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    hin = H.host(inp)
    shard, ops = _ops(cfg, inp)
    x = inp["x"]
    y = ep_forward(ops, shard, x, residual=x, z_prev=inp["z_prev"], group=group)
    bare = ep_forward(ops, shard, x, residual=None, z_prev=inp["z_prev"], group=group)
    torch.cuda.synchronize()
    sel = _gpu_selection(cfg, inp, x)
    y_terms = H.oracle_layer(cfg, hin, sel, residual=False)
    tol = H.Y_TOL[cfg["dtype"]]
    assert H.normwise(gen.to_numpy_f32(y), y_terms + hin["x"]) <= tol
    assert H.normwise(gen.to_numpy_f32(bare), y_terms) <= tol
    # the one-device layer: the same arithmetic up to where bf16 rounding happens
    one = H.run_layer(cfg, inp)
    assert H.normwise(gen.to_numpy_f32(y), one["y"]) <= 1e-2


def test_cuda_interweaved_second_step_is_one_step_stale(group):
    cfg = gen.workload("mmoe", T=600, d=256, h=512, h_shared=256)
    inp = gen.make_inputs(cfg, "cuda")
    hin = H.host(inp)
    shard, ops = _ops(cfg, inp)
    g = torch.Generator(device="cuda").manual_seed(77)
    xs = [inp["x"], (inp["x"].float() + 0.5 * torch.randn(inp["x"].shape, generator=g,
                                                         device="cuda")).to(inp["x"].dtype)]
    ep = InterweavedEP(ops, shard, group)
    ys = [ep.step(x, residual=x, z_prev=inp["z_prev"]) for x in xs]
    ep.finish()
    torch.cuda.synchronize()
    n_heavy = cfg["E_heavy"]
    sels = [_gpu_selection(cfg, inp, x) for x in xs]
    xh = [gen.to_numpy_f32(x) for x in xs]

    def layer(t, keep, with_local):
        s = dict(sels[t], idx=np.where(keep(sels[t]["idx"]), sels[t]["idx"], -1))
        return oracle.forward(cfg, xh[t], hin["W1"], hin["W2"], s, cfg["kinds"],
                              hin["const_vecs"], hin["Ws1"] if with_local else None,
                              hin["Ws2"] if with_local else None,
                              residual=xh[t] if with_local else None)
    tol = H.Y_TOL[cfg["dtype"]]
    # step 0: nothing cached, the synchronous layer
    assert H.normwise(gen.to_numpy_f32(ys[0]), layer(0, lambda i: i >= 0, True)) <= tol
    # step 1: local terms of step 1 plus step 0's heavy experts
    ref1 = layer(1, lambda i: i >= n_heavy, True) + layer(0, lambda i: (i >= 0) & (i < n_heavy),
                                                         False)
    err_stale = H.normwise(gen.to_numpy_f32(ys[1]), ref1)
    assert err_stale <= tol
    # and it is not the fresh layer of step 1
    err_fresh = H.normwise(gen.to_numpy_f32(ys[1]), layer(1, lambda i: i >= 0, True))
    assert err_fresh > 3 * max(err_stale, 1e-3)
