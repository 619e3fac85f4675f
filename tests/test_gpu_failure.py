"""Failure detection on the GPU without a GPU fault: a bounded device wait
is made to run out on purpose, and the library reports it.

Blocks of at most 128 bf16 tokens with a shared expert finish their routing
in one cooperative kernel whose CTAs meet at grid barriers: software
barriers on a global counter, each wait bounded. The test hook
moe_test_set_barrier_wait shortens the bound to 100 us and makes the
barriers wait for one arrival more than the grid has, so every CTA's wait
expires. Nothing else changes: no trap, no bad address, no endless loop.
The call must come back with MOE_DEV_TIMEOUT in the status word and an
in-bounds, empty routing (every slot -1, no rows), so the rest of the
layer gives y = x + shared(x); the next call, with the defaults restored,
must match the oracle as usual.
"""

import numpy as np
import pytest

import oracle
from mixture_experts_layer_33_b200 import inputs as gen
from tests import parity_helpers as H

pytestmark = pytest.mark.gpu

# T = 128 with a shared expert: the split router, then the cooperative
# small-block routing kernel (token choice over 16 heavy experts and the
# three zero-computation experts).
CFG = dict(T=128, d=128, h=256, h_shared=128)


def test_expired_grid_barrier_reports_timeout_then_recovers():
    m = H.moe()
    cfg = gen.workload("mmoe", **CFG)
    inp = gen.make_inputs(cfg, "cuda")
    hin = H.host(inp)
    try:
        m.set_barrier_wait_for_tests(limit_ns=100_000, extra_arrivals=1)
        bad = H.run_layer(cfg, inp)
    finally:
        m.set_barrier_wait_for_tests(0, 0)
    assert bad["status"] & m.DEV_TIMEOUT
    assert np.all(bad["sel"] == -1)
    assert np.all(bad["w"] == 0)
    assert np.all(bad["offsets"] == 0)
    # no routed term at all: the residual plus the shared expert
    empty = {"idx": np.full((cfg["T"], cfg["k"]), -1), "w": np.zeros((cfg["T"], cfg["k"]))}
    y_ref = H.oracle_layer(cfg, hin, empty)
    assert H.normwise(bad["y"], y_ref) <= H.Y_TOL[cfg["dtype"]]

    good = H.run_layer(cfg, inp)
    assert good["status"] == 0
    z = good["logits"].astype(np.float64)
    idx = oracle.topk_token_choice(z, cfg["k"])
    np.testing.assert_array_equal(good["sel"].reshape(cfg["T"], cfg["k"]), idx)
    sel = {"idx": idx, "w": oracle.gather_weights(good["probs"].astype(np.float64), idx)}
    assert H.normwise(good["y"], H.oracle_layer(cfg, hin, sel)) <= H.Y_TOL[cfg["dtype"]]
