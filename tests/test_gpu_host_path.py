"""moe_forward_host against moe_forward on the same inputs.

The host entry point cuts a large batch into token chunks (whole groups
for expert choice, never a DES block) and overlaps each chunk's copies
with the layer on its neighbours. Routing is per token (token choice) or
per group (expert choice) and every later step is per row or per token, so
the chunked layer must return the bytes the one-shot device call returns.
The device call itself is checked against the oracle in test_gpu_parity.
"""

import numpy as np
import pytest
import torch

from mixture_experts_layer_33_b200 import inputs as gen
from tests import parity_helpers as H

pytestmark = pytest.mark.gpu

CASES = [
    # token choice, two chunks (2304 + 2176 tokens), shared experts
    ("ditmoe_xl", dict(T=4480), False),
    # expert choice: two chunks of 16 whole 128-token groups
    ("ecdit", dict(T=4096, h=2048), False),
    # gate-residual z_prev and a residual other than x, three chunks (1:2:1)
    ("mmoe", dict(T=8320), True),
    # a DES block is routed as one unit: one chunk
    ("des_vote", {}, False),
    # below two minimum chunks: one chunk
    ("ditmoe_xl", dict(T=3000, d=256, h=512, h_shared=256), True),
    # a small fp32 layer: one chunk, the one-launch fp32 path
    ("tiny_fp32", {}, True),
]


def _device_y(m, c, inp, residual):
    ws = m.alloc_workspace(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.empty_like(inp["x"])
    m.forward(c, inp["x"], inp["W_r"], inp["W1"], inp["W2"], y, ws, residual=residual,
              z_prev=inp["z_prev"], bias=inp["logit_bias"], Ws1=inp["Ws1"], Ws2=inp["Ws2"],
              const_vecs=inp["const_vecs"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return y.cpu()


@pytest.mark.parametrize("name,over,own_residual", CASES,
                         ids=[f"{c[0]}_T{gen.workload(c[0], **c[1])['T']}" for c in CASES])
def test_host_path_matches_device_path(name, over, own_residual):
    m = H.moe()
    cfg = gen.workload(name, **over)
    inp = gen.make_inputs(cfg, "cuda")
    c = m.make_config(cfg)
    residual = inp["x"]
    if own_residual:
        g = torch.Generator(device="cuda").manual_seed(77)
        residual = torch.randn(inp["x"].shape, generator=g, device="cuda").to(inp["x"].dtype)
    y_dev = _device_y(m, c, inp, residual)

    x_h = inp["x"].cpu().pin_memory()
    r_h = residual.cpu().pin_memory() if own_residual else x_h
    zp_h = inp["z_prev"].cpu().pin_memory() if inp["z_prev"] is not None else None
    ws = m.alloc_workspace(c)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    # Two calls back to back with no host synchronisation between them: the
    # second must wait for the first's copies out before it overwrites the
    # staging buffers, and the shared side-stream events are reused.
    for _ in range(2):
        y_h = torch.full_like(x_h, float("nan")).pin_memory()
        m.forward_host(c, x_h, inp["W_r"], inp["W1"], inp["W2"], y_h, ws, residual_host=r_h,
                       z_prev_host=zp_h, bias=inp["logit_bias"], Ws1=inp["Ws1"],
                       Ws2=inp["Ws2"], const_vecs=inp["const_vecs"], dev_status=st)
        outs.append(y_h)
    torch.cuda.current_stream().synchronize()
    assert int(st.item()) == 0
    for y_h in outs:
        a = gen.to_numpy_f32(y_h)
        b = gen.to_numpy_f32(y_dev)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), \
            f"max |diff| {np.nanmax(np.abs(a - b))}"


def test_host_path_on_a_side_stream():
    m = H.moe()
    cfg = gen.workload("ditmoe_xl", T=4224, d=256, h=512, h_shared=256)
    inp = gen.make_inputs(cfg, "cuda")
    c = m.make_config(cfg)
    y_dev = _device_y(m, c, inp, inp["x"])
    x_h = inp["x"].cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    ws = m.alloc_workspace(c)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        m.forward_host(c, x_h, inp["W_r"], inp["W1"], inp["W2"], y_h, ws, residual_host=x_h,
                       bias=inp["logit_bias"], Ws1=inp["Ws1"], Ws2=inp["Ws2"], stream=s)
    s.synchronize()
    assert torch.equal(y_h, y_dev)
