"""Expert parallelism on CPU ranks over gloo: the exchange plan and the
two all-to-all steps of `expert_parallel.ep_forward`, with every compute
step taken by the fp64 oracle, must give each rank exactly the oracle
layer's rows for its tokens (all experts on one device). Cases: two and
three ranks, experts that do not divide evenly, a rank that owns no
expert, routing skewed onto one rank's experts, and MMOE's
zero-computation experts, gate residual and shared expert (all local to
the token's rank)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_33_b200.expert_parallel import (ExpertShard, InterweavedEP, ep_forward,
                                                           exchange_plan, merge_stale_slots)
from oracle import moe_oracle as om

H, I, Z, C = om.HEAVY, om.IDENTITY, om.ZERO, om.CONST


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """Each step of the layer by the oracle, on this rank's experts only."""

    count_device = "cpu"

    def __init__(self, cfg, shard, rank, W, kinds):
        self.cfg, self.kinds, self.W = cfg, kinds, W
        self.n_heavy = sum(1 for k in kinds if k == H)
        assert self.n_heavy == shard.n_heavy
        lo, hi = shard.bounds(rank)
        self.n_local = hi - lo
        self.W1, self.W2 = W["W1"][lo:hi], W["W2"][lo:hi]  # the shard's experts only

    def empty(self, n, d):
        return torch.empty(n, d, dtype=torch.float64)

    def route(self, x, z_prev=None):
        sel = om.route(self.cfg, x.numpy(), self.W["W_r"], self.W["bias"], z_prev)
        return torch.from_numpy(sel["idx"].reshape(-1)), torch.from_numpy(sel["w"].reshape(-1))

    def dispatch(self, sel, x):
        T, k = x.shape[0], self.cfg["k"]
        offsets, perm, row_of, _, _ = om.dispatch(np.repeat(np.arange(T), k), sel.numpy(),
                                                  self.n_heavy, T)
        return x[torch.from_numpy(perm.astype(np.int64))], offsets, row_of

    def regroup(self, x_recv, recv_expert):
        n = len(recv_expert)
        offs, perm, row_of, _, _ = om.dispatch(np.arange(n), recv_expert, self.n_local, n)
        return x_recv[torch.from_numpy(perm.astype(np.int64))], offs, row_of, recv_expert

    def experts(self, x_grp, offs):
        y = np.zeros(tuple(x_grp.shape))
        for e in range(self.n_local):
            lo, hi = offs[e], offs[e + 1]
            if hi > lo:
                y[lo:hi] = om.heavy_expert(self.cfg["act"], x_grp[lo:hi].numpy(), self.W1[e],
                                           self.W2[e], self.cfg["h"])
        return torch.from_numpy(y)

    def ungroup(self, y_grp, row_of, sel_recv, x_recv):
        return y_grp[torch.from_numpy(np.asarray(row_of, np.int64))]

    def shared(self, x):
        if self.W["Ws1"] is None:
            return None
        return om.mlp_gelu(x.numpy(), self.W["Ws1"], self.W["Ws2"])

    def check_status(self):
        pass  # no device status on the CPU ranks

    def combine(self, y_back, y_sh, sel, w, row_of, x, residual, k=None):
        T, k = x.shape[0], k or self.cfg["k"]
        sel, xs, yb = sel.numpy(), x.numpy(), y_back.numpy()
        row_of = np.asarray(row_of)
        cidx = np.cumsum([kd == C for kd in self.kinds]) - 1

        def out(a):
            e = int(sel[a])  # never -1: the oracle's combine skips empty slots
            if self.kinds[e] == H:
                return yb[row_of[a]]
            if self.kinds[e] == I:
                return xs[a // k]
            if self.kinds[e] == C:
                return self.W["cv"][cidx[e]]
            return np.zeros(xs.shape[1])

        res = None if residual is None else residual.numpy()
        return om.combine(np.arange(T), np.repeat(np.arange(T), k), sel, w.numpy(), out,
                          residual=res, shared_out=y_sh, d=xs.shape[1])


def _problem(case):
    rng = np.random.default_rng(100 + case["seed"])
    kinds = case["kinds"]
    E, Eh, d, h, T = len(kinds), sum(1 for k in kinds if k == H), 12, 16, case["T"]
    cfg = dict(routing="token_topk", E=E, k=case["k"], h=h, act=case["act"],
               gate_residual_scale=case.get("gate", 0.0), renorm=case.get("renorm", 0))
    bias = np.zeros(E)
    if case.get("skew"):
        bias[: max(1, Eh // 3)] = 3.0  # most slots to the first rank's experts
    W = dict(W_r=rng.normal(size=(E, d)), bias=bias,
             W1=rng.normal(size=(Eh, 2 * h if case["act"] == "swiglu" else h, d)) * 0.3,
             W2=rng.normal(size=(Eh, d, h)) * 0.3,
             cv=rng.normal(size=(max(1, sum(1 for k in kinds if k == C)), d)),
             Ws1=rng.normal(size=(h, d)) * 0.3 if case.get("shared") else None,
             Ws2=rng.normal(size=(d, h)) * 0.3 if case.get("shared") else None)
    x = rng.normal(size=(T, d))
    z_prev = rng.normal(size=(T, E)) if case.get("gate") else None
    return cfg, kinds, W, x, z_prev


def _reference(cfg, kinds, W, x, z_prev):
    sel = om.route(cfg, x, W["W_r"], W["bias"], z_prev)
    return om.forward(cfg, x, W["W1"], W["W2"], sel, kinds, W["cv"], W["Ws1"], W["Ws2"],
                      residual=x)


def _rank_main(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, kinds, W, x, z_prev = _problem(case)
        shard = ExpertShard(sum(1 for k in kinds if k == H), world)
        lo, hi = case["T"] * rank // world, case["T"] * (rank + 1) // world  # this rank's tokens
        xt = torch.from_numpy(x[lo:hi])
        zt = None if z_prev is None else z_prev[lo:hi]
        y = ep_forward(OracleOps(cfg, shard, rank, W, kinds), shard, xt, residual=xt, z_prev=zt)
        q.put((rank, lo, hi, np.asarray(y)))
    finally:
        dist.destroy_process_group()


CASES = [
    dict(name="two_ranks_gelu", world=2, T=40, k=2, act="gelu", kinds=[H] * 6, seed=0),
    dict(name="three_ranks_uneven_swiglu", world=3, T=31, k=3, act="swiglu", kinds=[H] * 7,
         seed=1, renorm=1),
    dict(name="rank_without_experts", world=3, T=24, k=1, act="gelu", kinds=[H] * 2, seed=2),
    dict(name="skewed_onto_rank0", world=2, T=48, k=2, act="gelu", kinds=[H] * 6, seed=3,
         skew=True),
    dict(name="mmoe_kinds_gate_shared", world=2, T=36, k=2, act="gelu",
         kinds=[H] * 5 + [I, Z, C], seed=4, gate=0.5, shared=True),
]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_expert_parallel_matches_one_device_layer(case):
    world = case["world"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, kinds, W, x, z_prev = _problem(case)
    y_ref = _reference(cfg, kinds, W, x, z_prev)
    for rank, lo, hi, y in got:
        np.testing.assert_allclose(y, y_ref[lo:hi], rtol=1e-12, atol=1e-12)


# ------------------------------------------------ interweaved (one step stale)
N_STEPS = 3


def _step_input(x0, t):
    """Diffusion-step inputs: each step moves the activations a little."""
    rng = np.random.default_rng(1000 + t)
    return x0 + 0.3 * t * rng.normal(size=x0.shape)


def _only(sel_idx, keep):
    """The selection with the slots `keep` rejects emptied (expert -1)."""
    out = dict(sel_idx)
    out["idx"] = np.where(keep(sel_idx["idx"]), sel_idx["idx"], -1)
    return out


def _interweaved_reference(cfg, kinds, W, xs, zs):
    """Step 0: the synchronous layer. Step t >= 1: residual, shared expert
    and zero-computation experts from step t's input and routing, plus the
    heavy experts' weighted outputs of step t-1 (its input and routing)."""
    n_heavy = sum(1 for k in kinds if k == H)
    outs = []
    for t, (x, z) in enumerate(zip(xs, zs)):
        sel = om.route(cfg, x, W["W_r"], W["bias"], z)
        if t == 0:
            outs.append(om.forward(cfg, x, W["W1"], W["W2"], sel, kinds, W["cv"], W["Ws1"],
                                   W["Ws2"], residual=x))
            continue
        prev = om.route(cfg, xs[t - 1], W["W_r"], W["bias"], zs[t - 1])
        stale = om.forward(cfg, xs[t - 1], W["W1"], W["W2"],
                           _only(prev, lambda i: (i >= 0) & (i < n_heavy)), kinds, W["cv"],
                           None, None, residual=None)
        fresh = om.forward(cfg, x, W["W1"], W["W2"], _only(sel, lambda i: i >= n_heavy), kinds,
                           W["cv"], W["Ws1"], W["Ws2"], residual=x)
        outs.append(fresh + stale)
    return outs


def _interweaved_rank_main(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, kinds, W, x0, z0 = _problem(case)
        shard = ExpertShard(sum(1 for k in kinds if k == H), world)
        lo, hi = case["T"] * rank // world, case["T"] * (rank + 1) // world
        ep = InterweavedEP(OracleOps(cfg, shard, rank, W, kinds), shard)
        ys = []
        for t in range(N_STEPS):
            x = _step_input(x0, t)
            xt = torch.from_numpy(x[lo:hi])
            zt = None if z0 is None else z0[lo:hi]
            ys.append(np.asarray(ep.step(xt, residual=xt, z_prev=zt)))
        ep.finish()
        q.put((rank, lo, hi, ys))
    finally:
        dist.destroy_process_group()


IW_CASES = [CASES[0], CASES[1], CASES[4]]


@pytest.mark.parametrize("case", IW_CASES, ids=[c["name"] for c in IW_CASES])
def test_interweaved_schedule_combines_one_step_stale(case):
    world = case["world"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_interweaved_rank_main, args=(r, world, port, case, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, kinds, W, x0, z0 = _problem(case)
    xs = [_step_input(x0, t) for t in range(N_STEPS)]
    zs = [z0] * N_STEPS
    refs = _interweaved_reference(cfg, kinds, W, xs, zs)
    for rank, lo, hi, ys in got:
        for t in range(N_STEPS):
            np.testing.assert_allclose(ys[t], refs[t][lo:hi], rtol=1e-12, atol=1e-12)
        # the later steps really are stale: not the synchronous layer
        sync = _reference(cfg, kinds, W, xs[1], z0)
        assert not np.allclose(ys[1], sync[lo:hi], rtol=1e-6, atol=1e-6)


def test_exchange_plan_splits_and_received_experts():
    # 2 ranks, 5 heavy experts: rank 0 owns 0..2, rank 1 owns 3..4.
    shard = ExpertShard(5, 2)
    assert [shard.bounds(r) for r in range(2)] == [(0, 3), (3, 5)]
    counts = np.array([[1, 0, 2, 3, 1],    # rows rank 0 dispatched per expert
                       [0, 4, 1, 0, 2]])   # rows rank 1 dispatched per expert
    p0, p1 = exchange_plan(counts, shard, 0), exchange_plan(counts, shard, 1)
    assert p0.send == [3, 4] and p0.recv == [3, 5]
    assert p1.send == [5, 2] and p1.recv == [4, 2]
    # received rows: source-rank major, local expert ascending within a source
    assert p0.recv_expert.tolist() == [0, 2, 2] + [1, 1, 1, 1, 2]
    assert p1.recv_expert.tolist() == [0, 0, 0, 1] + [1, 1]
    # what one rank sends to another is what that rank receives from it
    assert p0.send[1] == p1.recv[0] and p1.send[0] == p0.recv[1]


def test_shard_bounds_partition_the_experts():
    for n in range(0, 20):
        for world in range(1, 9):
            shard = ExpertShard(n, world)
            b = [shard.bounds(r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_cuda_steps_take_token_choice_only():
    # Expert-choice groups and DES blocks shard as replicas, not by expert.
    from mixture_experts_layer_33_b200.expert_parallel import CudaOps
    from mixture_experts_layer_33_b200 import inputs as gen
    for name in ("ecdit", "des_vote"):
        with pytest.raises(ValueError):
            CudaOps(gen.workload(name), ExpertShard(4, 2), 0, None, None, None, device="cpu")


def test_merge_stale_slots_keeps_previous_heavy_and_current_light_slots():
    # 3 tokens, k = 2, experts 0..3 heavy, 4..5 zero-computation; -1 empty.
    prev_sel = torch.tensor([0, 4, 5, 3, -1, 2], dtype=torch.int32)
    prev_w = torch.tensor([.1, .2, .3, .4, .5, .6])
    prev_row = np.array([7, -1, -1, 9, -1, 4], dtype=np.int32)
    sel = torch.tensor([4, 1, 2, 3, 5, 0], dtype=torch.int32)
    w = torch.tensor([.7, .8, .9, 1.0, 1.1, 1.2])
    m_sel, m_w, m_row = merge_stale_slots(prev_sel, prev_w, prev_row, sel, w, 4, 2)
    # per token: [prev slot 0, prev slot 1, current slot 0, current slot 1]
    assert m_sel.tolist() == [0, -1, 4, -1,
                              -1, 3, -1, -1,
                              -1, 2, 5, -1]
    assert m_row.tolist() == [7, -1, -1, -1,
                              -1, 9, -1, -1,
                              -1, 4, -1, -1]
    np.testing.assert_allclose(m_w.numpy(), [.1, .2, .7, .8, .3, .4, .9, 1.0, .5, .6, 1.1, 1.2])
