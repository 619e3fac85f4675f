"""moe_forward's side stream for the shared expert, through the C ABI.

For a bf16 layer with a shared expert and routed rows, moe_forward runs the
shared expert's up projection on a library-owned side stream, forked from
the caller's stream after the routing and joined before the down
projections (the oracle parity tests check the values). These tests check
the ordering: a CUDA graph captured around moe_forward (the capture takes
the side stream in through the fork event) replays to the bytes of an
eager call, and two callers on two streams with their own workspaces,
enqueueing at the same time from two host threads, each get the bytes a
lone call gives. A join missing or out of order would let the down
projection read a half-written hidden buffer; every comparison is exact,
since the same kernels run on the same inputs and only their overlap
differs.
"""

import threading

import pytest
import torch

from mixture_experts_layer_33_b200 import inputs as gen

pytestmark = pytest.mark.gpu

# Small layers that take the grouped-GEMM path with a shared expert
# (more than 128 tokens, bf16): DiT-MoE-style top-2 with two shared
# experts, and MMOE-style with zero-computation experts and one shared.
CASES = [
    ("ditmoe_shared", "ditmoe_xl", dict(T=600, d=256, h=512, h_shared=256)),
    ("mmoe_shared", "mmoe", dict(T=520, d=256, h=512, h_shared=512)),
]


def _moe():
    from mixture_experts_layer_33_b200 import moe
    return moe


def _forward(m, c, inp, y, ws, status, stream=None):
    m.forward(c, inp["x"], inp["W_r"], inp["W1"], inp["W2"], y, ws, residual=inp["x"],
              z_prev=inp["z_prev"], bias=inp["logit_bias"], Ws1=inp["Ws1"], Ws2=inp["Ws2"],
              const_vecs=inp["const_vecs"], dev_status=status, stream=stream)


@pytest.mark.parametrize("label,name,over", CASES, ids=[c[0] for c in CASES])
def test_graph_replay_matches_eager(label, name, over):
    m = _moe()
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    c = m.make_config(cfg)
    ws = m.alloc_workspace(c, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    y_eager = torch.empty_like(inp["x"])
    _forward(m, c, inp, y_eager, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    # Captured once, replayed twice, into another output buffer.
    y_graph = torch.full_like(inp["x"], 7.0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _forward(m, c, inp, y_graph, ws, status, stream=side)  # warm-up off the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _forward(m, c, inp, y_graph, ws, status)
    for _ in range(2):
        y_graph.fill_(7.0)
        g.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y_graph, y_eager)
    del g


def test_concurrent_callers_on_two_streams():
    m = _moe()
    cfgs = [gen.workload(n, **o) for _, n, o in CASES]
    inps = [gen.make_inputs(cfg, "cuda") for cfg in cfgs]
    cs = [m.make_config(cfg) for cfg in cfgs]
    wss = [m.alloc_workspace(c, "cuda") for c in cs]
    sts = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in cfgs]

    ref = []
    for c, inp, ws, st in zip(cs, inps, wss, sts):
        y = torch.empty_like(inp["x"])
        _forward(m, c, inp, y, ws, st)
        ref.append(y)
    torch.cuda.synchronize()

    streams = [torch.cuda.Stream() for _ in cfgs]
    outs = [[torch.empty_like(inp["x"]) for _ in range(4)] for inp in inps]
    errors = []
    start = threading.Barrier(len(cfgs))

    def run(i):
        try:
            torch.cuda.set_device(0)
            start.wait()
            for y in outs[i]:
                _forward(m, cs[i], inps[i], y, wss[i], sts[i], stream=streams[i])
        except Exception as exc:  # noqa: BLE001
            errors.append(exc)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(len(cfgs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    assert not errors, errors
    for i in range(len(cfgs)):
        assert int(sts[i].item()) == 0
        for y in outs[i]:
            assert torch.equal(y, ref[i])
