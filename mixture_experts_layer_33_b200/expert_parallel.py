"""Expert parallelism: the heavy experts sharded across the ranks of a
process group, tokens exchanged with two all-to-all steps.

DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
Inference, Background and motivation: under expert parallelism each device
holds a subset of the experts; a layer dispatches every token to the
devices holding its experts (all-to-all), the experts run there, and a
second all-to-all brings the outputs back to be combined. This module is
the synchronous form (fresh dispatch and combine every step), for token
choice routing: expert-choice groups and DES blocks are independent units
that shard as replicas instead.

Per rank, with experts owned in contiguous blocks (rank p owns heavy
experts [lo_p, hi_p)):

1. route its own tokens and dispatch them by global expert id; the
   dispatched rows are grouped by expert, so the rows for rank p are one
   contiguous range;
2. all-gather the per-expert row counts (small), from which every rank
   derives the send and receive splits and the local expert of each
   received row (source-rank major, expert ascending within a source);
3. all-to-all the rows; regroup the received rows by local expert with
   the same stable dispatch; run the local experts; put the outputs back
   in received order;
4. all-to-all the outputs back (splits swapped): they arrive in the order
   of step 1's dispatched rows, so the combine of step 1's routing
   applies unchanged (shared expert, residual and zero-computation experts
   are local to the token's rank).

`InterweavedEP` is DICE's interweaved schedule over the same steps (Key
designs, "Interweaved Parallelism"): the dispatch exchange completes within
the step (fresh), while the combine exchange of a step's expert outputs is
started asynchronously and consumed one step later, so the routed-expert
part of a step's output comes from the previous step (one step stale) and
only those combine results are cached. The reading taken where the page is
brief: the stale part is the sum over the previous step's heavy-expert
slots of weight times expert output, with that step's routing; everything
local to the token's rank (residual, shared expert, zero-computation
experts) uses the current step's input and routing; the first step, with
nothing cached, runs synchronously.

Every compute step is an `Ops` call: `CudaOps` runs the library's kernels
through the C ABI (one GPU per rank, NCCL); the tests drive the same
orchestration with the fp64 oracle on CPU ranks over gloo, and `CudaOps` on
one GPU as a one-rank NCCL group. The collectives are plain
`torch.distributed` calls; the fused dispatch/combine kernels over NVLink
peer memory are not built.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist


@dataclass(frozen=True)
class ExpertShard:
    """Contiguous blocks of the heavy experts over `world` ranks (the first
    n_heavy % world ranks own one more)."""

    n_heavy: int
    world: int

    def bounds(self, rank: int) -> tuple[int, int]:
        base, extra = divmod(self.n_heavy, self.world)
        lo = rank * base + min(rank, extra)
        return lo, lo + base + (1 if rank < extra else 0)


@dataclass
class ExchangePlan:
    send: list[int]          # rows to each rank
    recv: list[int]          # rows from each rank
    recv_expert: np.ndarray  # local expert id of each received row (int32)


def exchange_plan(all_counts: np.ndarray, shard: ExpertShard, rank: int) -> ExchangePlan:
    """Splits and received-row experts from every rank's per-expert counts
    (`all_counts[r, e]`: rows rank r dispatched to heavy expert e)."""
    all_counts = np.asarray(all_counts, dtype=np.int64)
    lo, hi = shard.bounds(rank)
    send = [int(all_counts[rank, slice(*shard.bounds(p))].sum()) for p in range(shard.world)]
    recv = [int(all_counts[src, lo:hi].sum()) for src in range(shard.world)]
    local = np.arange(hi - lo, dtype=np.int32)
    parts = [np.repeat(local, all_counts[src, lo:hi]) for src in range(shard.world)]
    recv_expert = np.concatenate(parts) if parts else np.zeros(0, np.int32)
    return ExchangePlan(send, recv, recv_expert.astype(np.int32))


def _all_gather_counts(counts: np.ndarray, device, group) -> np.ndarray:
    world = dist.get_world_size(group)
    t = torch.as_tensor(np.asarray(counts, dtype=np.int64), device=device)
    out = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(out, t, group=group)
    return torch.stack(out).cpu().numpy()


def _route_dispatch_compute(ops, shard: ExpertShard, x, z_prev, group):
    """Steps 1-3: route, dispatch, the dispatch exchange (completed here)
    and this rank's experts on the rows it received. Returns the routing,
    the send/receive splits and the expert outputs in received order."""
    rank = dist.get_rank(group)
    sel, w = ops.route(x, z_prev)
    x_perm, offsets, row_of = ops.dispatch(sel, x)
    offsets = np.asarray(offsets, dtype=np.int64)
    counts = np.diff(offsets)
    plan = exchange_plan(_all_gather_counts(counts, ops.count_device, group), shard, rank)
    n_send, n_recv = int(offsets[-1]), int(sum(plan.recv))
    d = x.shape[1]
    x_recv = ops.empty(n_recv, d)
    dist.all_to_all_single(x_recv, x_perm[:n_send].contiguous(), plan.recv, plan.send, group=group)
    y_recv = x_recv  # a rank that receives no row (or owns no expert) computes nothing
    if n_recv > 0:
        x_grp, offs_grp, row_of_grp, sel_recv = ops.regroup(x_recv, plan.recv_expert)
        y_grp = ops.experts(x_grp, offs_grp)
        y_recv = ops.ungroup(y_grp, row_of_grp, sel_recv, x_recv)
    return sel, w, row_of, plan, n_send, y_recv


def ep_forward(ops, shard: ExpertShard, x, residual=None, z_prev=None, group=None):
    """The layer on this rank's tokens `x` (and their previous-layer logits
    `z_prev` under MMOE's gate residual) with the heavy experts sharded over
    `group`; returns this rank's outputs. Raises if a device step flagged
    an error (bad ids, an expired bounded wait)."""
    sel, w, row_of, plan, n_send, y_recv = _route_dispatch_compute(ops, shard, x, z_prev, group)
    y_back = ops.empty(n_send, x.shape[1])
    dist.all_to_all_single(y_back, y_recv.contiguous(), plan.send, plan.recv, group=group)
    y = ops.combine(y_back, ops.shared(x), sel, w, row_of, x, residual)
    ops.check_status()
    return y


def merge_stale_slots(prev_sel, prev_w, prev_row_of, sel, w, n_heavy, k):
    """Slot lists of the interweaved combine, 2k slots per token: first the
    previous step's k slots with only their heavy experts kept (their rows
    index the previous step's returned expert outputs), then this step's k
    slots with only the zero-computation experts kept. A dropped slot is
    expert -1 with no row, which the combine skips. Index and weight
    bookkeeping only: the sums are the combine's."""
    prev_sel, sel = prev_sel.reshape(-1, k), sel.reshape(-1, k)
    heavy_prev = (prev_sel >= 0) & (prev_sel < n_heavy)
    light_now = sel >= n_heavy
    minus1 = torch.full_like(sel, -1)
    m_sel = torch.cat([torch.where(heavy_prev, prev_sel, minus1),
                       torch.where(light_now, sel, minus1)], dim=1)
    m_w = torch.cat([prev_w.reshape(-1, k), w.reshape(-1, k)], dim=1)
    prev_row = torch.as_tensor(np.asarray(prev_row_of)) if not isinstance(prev_row_of, torch.Tensor) \
        else prev_row_of
    prev_row = prev_row.to(sel.device).reshape(-1, k)
    m_row = torch.cat([torch.where(heavy_prev, prev_row.to(sel.dtype), minus1), minus1], dim=1)
    return m_sel.reshape(-1).contiguous(), m_w.reshape(-1).contiguous(), m_row.reshape(-1).contiguous()


class InterweavedEP:
    """DICE's interweaved expert-parallel schedule: fresh dispatch, combine
    one step stale (see the module docstring). Call `step` once per
    diffusion step for this layer, then `finish` before the process group
    goes away; every rank takes the same collective steps in the same
    order (one counts all-gather, one dispatch exchange and one combine
    exchange, started asynchronously, per step)."""

    def __init__(self, ops, shard: ExpertShard, group=None):
        self.ops, self.shard, self.group = ops, shard, group
        self.pending = None  # the previous step's combine exchange and routing

    def step(self, x, residual=None, z_prev=None):
        ops = self.ops
        sel, w, row_of, plan, n_send, y_recv = _route_dispatch_compute(
            ops, self.shard, x, z_prev, self.group)
        y_back = ops.empty(n_send, x.shape[1])
        y_recv = y_recv.contiguous()
        work = dist.all_to_all_single(y_back, y_recv, plan.send, plan.recv, group=self.group,
                                      async_op=True)
        prev, self.pending = self.pending, (work, y_back, y_recv, sel, w, row_of)
        y_sh = ops.shared(x)
        if prev is None:
            # nothing cached yet: this step's own combine, synchronously
            work.wait()
            y = ops.combine(y_back, y_sh, sel, w, row_of, x, residual)
        else:
            p_work, p_back, _, p_sel, p_w, p_row = prev
            p_work.wait()
            k = int(sel.numel()) // max(1, x.shape[0])
            m_sel, m_w, m_row = merge_stale_slots(p_sel, p_w, p_row, sel, w, ops.n_heavy, k)
            y = ops.combine(p_back, y_sh, m_sel, m_w, m_row, x, residual, k=2 * k)
        ops.check_status()
        return y

    def finish(self):
        """Wait for the last step's combine exchange (its result is unused)."""
        if self.pending is not None:
            self.pending[0].wait()
            self.pending = None


class CudaOps:
    """The steps on this rank's GPU through the C ABI.

    `cfg` is the layer's configuration (token choice) over all experts;
    `W1_local` / `W2_local` hold this rank's experts only (heavy experts
    [lo, hi) of `shard`), in the same layouts as the full tensors. Run on
    one GPU as a one-rank NCCL group (the exchanges are then copies to
    itself); more ranks are covered on CPU ranks with the oracle's steps.
    """

    def __init__(self, cfg, shard: ExpertShard, rank: int, W_r, W1_local, W2_local,
                 bias=None, Ws1=None, Ws2=None, const_vecs=None, device="cuda"):
        from . import moe as m
        if cfg["routing"] != "token_topk":
            raise ValueError("expert parallelism here is for token choice routing")
        self.m, self.cfg, self.device = m, cfg, device
        self.count_device = device
        self.W_r, self.bias, self.Ws1, self.Ws2, self.cv = W_r, bias, Ws1, Ws2, const_vecs
        self.W1, self.W2 = W1_local, W2_local
        lo, hi = shard.bounds(rank)
        self.n_local = hi - lo
        self.n_heavy = shard.n_heavy
        self.dtype = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def _local_cfg(self, T):
        return self.m.make_config(dict(self.cfg, T=T))

    def _group_cfg(self, n):
        # the received rows as a layer of their own: one slot per row, the
        # local experts only, no shared expert
        kinds = [0] * self.n_local
        return self.m.make_config(dict(self.cfg, T=n, E=self.n_local, k=1, kinds=kinds,
                                       n_shared=0, renorm=0))

    def empty(self, n, d):
        return torch.empty(n, d, dtype=self.dtype, device=self.device)

    def route(self, x, z_prev=None):
        T, E, k = x.shape[0], self.cfg["E"], self.cfg["k"]
        logits = torch.empty(T, E, device=self.device)
        probs = torch.empty(T, E, device=self.device)
        sel = torch.empty(T * k, dtype=torch.int32, device=self.device)
        w = torch.empty(T * k, device=self.device)
        self.m.router(x, self.W_r, logits, probs, bias=self.bias, z_prev=z_prev,
                      z_prev_scale=self.cfg.get("gate_residual_scale", 0.0), k=k,
                      renorm=self.cfg.get("renorm", 0), idx=sel, w=w)
        return sel, w

    def dispatch(self, sel, x):
        c = self._local_cfg(x.shape[0])
        na = self.m.num_assignments(c)
        self._ws = self.m.alloc_workspace(c, self.device)
        x_perm = torch.empty(na, x.shape[1], dtype=x.dtype, device=self.device)
        offsets = torch.empty(c.n_heavy + 1, dtype=torch.int32, device=self.device)
        perm = torch.empty(na, dtype=torch.int32, device=self.device)
        row_of = torch.empty(na, dtype=torch.int32, device=self.device)
        self.m.dispatch(c, sel, x, x_perm, offsets, perm, row_of, None, None, self.status, self._ws)
        return x_perm, offsets.cpu().numpy(), row_of

    def regroup(self, x_recv, recv_expert):
        n = x_recv.shape[0]
        c = self._group_cfg(n)
        sel_recv = torch.as_tensor(recv_expert, device=self.device)
        self._gws = self.m.alloc_workspace(c, self.device)
        x_grp = torch.empty_like(x_recv)
        offs = torch.empty(self.n_local + 1, dtype=torch.int32, device=self.device)
        perm = torch.empty(n, dtype=torch.int32, device=self.device)
        row_of = torch.empty(n, dtype=torch.int32, device=self.device)
        self.m.dispatch(c, sel_recv, x_recv, x_grp, offs, perm, row_of, None, None, self.status,
                        self._gws)
        return x_grp, offs, row_of, sel_recv

    def experts(self, x_grp, offs):
        c = self._group_cfg(x_grp.shape[0])
        y_grp = torch.empty_like(x_grp)
        self.m.grouped_mlp(c, x_grp, offs, self.W1, self.W2, None, None, None, y_grp, None,
                           self.status, self._gws)
        return y_grp

    def ungroup(self, y_grp, row_of, sel_recv, x_recv):
        # y_recv[i] = 1 * y_grp[row_of[i]]: the combine with one unit-weight
        # slot per row and no residual is an exact row gather
        n = y_grp.shape[0]
        c = self._group_cfg(n)
        ones = torch.ones(n, device=self.device)
        y_recv = torch.empty_like(y_grp)
        self.m.combine(c, y_grp, None, sel_recv, ones, row_of, None, None, x_recv, None, None,
                       y_recv, self.status)
        return y_recv

    def shared(self, x):
        if not self.cfg.get("n_shared"):
            return None
        # the shared expert(s) alone: a layer of one zero-computation expert
        # (no heavy experts, so no routed problem) and the shared problem
        c = self.m.make_config(dict(self.cfg, T=x.shape[0], E=1, k=1, kinds=[self.m.ZERO],
                                    renorm=0))
        ws = self.m.alloc_workspace(c, self.device)
        y_sh = torch.empty_like(x)
        self.m.grouped_mlp(c, None, None, None, None, x, self.Ws1, self.Ws2, None, y_sh,
                           self.status, ws)
        return y_sh

    def combine(self, y_back, y_sh, sel, w, row_of, x, residual, k=None):
        c = self.m.make_config(dict(self.cfg, T=x.shape[0], k=k or self.cfg["k"]))
        y = torch.empty_like(x)
        self.m.combine(c, y_back, y_sh, sel, w, row_of, None, None, x, self.cv, residual, y,
                       self.status)
        return y

    def check_status(self):
        """Raise if any step flagged an error in the device status word."""
        st = int(self.status.item())
        if st != 0:
            raise RuntimeError(f"expert-parallel layer: device status {st:#x}")
