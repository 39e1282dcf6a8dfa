"""Parity of the CUDA path with the fp64 CPU oracle on small shapes.

Every call goes through the C ABI (via the ctypes binding). Shapes span
several router chunks (64 tokens), several 128-row expert tiles, ragged
tails, every BLOCK_M, H with and without a 256-column L2 tile, bias and no
bias, k = 1 and k = E. Routing must match bit-exactly, y within the
tolerances in parity_util.
"""
import ctypes

import numpy as np
import pytest
import torch

from synth.moe_inputs import custom_shape, make_inputs
from tests.parity_util import assert_routing_equal, assert_y_close, oracle_forward

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _plan(shape, block_m=0, T_max=None):
    from moe_megakernel_b200 import MoEPlan
    return MoEPlan(T_max or shape.T, shape.H, shape.I, shape.E, shape.k, block_m=block_m)


def _poison(plan):
    """Fill the workspace with 0xFF (NaN / -1) so reads of unwritten memory show up."""
    plan.workspace.fill_(0xFF)
    rc = plan.lib.moe_plan_bind_workspace(plan._plan, ctypes.c_void_p(plan.workspace.data_ptr()),
                                          plan.workspace_bytes)
    assert rc == 0


def _run_and_compare(shape, block_m=0, poison=True):
    inp = make_inputs(shape, device=DEV)
    plan = _plan(shape, block_m)
    if poison:
        _poison(plan)
    y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    ref = oracle_forward(inp, block_m=plan.block_m)
    assert_routing_equal(plan.routing(shape.T), ref)
    assert torch.isfinite(y).all()
    fro, mx = assert_y_close(y, ref["y"])
    return plan, inp, y, ref, (fro, mx)


SMALL = [
    # T,   H,   I,   E,  k, block_m, zipf
    (64, 128, 256, 8, 2, 0, False),      # the tiny workload shape (BLOCK_M 16)
    (300, 256, 384, 16, 4, 0, False),    # ragged T, H % 256 != 0, BLOCK_M 128
    (300, 256, 384, 16, 4, 16, False),
    (300, 256, 384, 16, 4, 32, False),
    (300, 256, 384, 16, 4, 64, False),
    (129, 384, 256, 32, 8, 0, True),     # Zipf-biased gate, 8 experts per token
    (1, 128, 128, 8, 1, 0, False),       # one token, k = 1
    (77, 128, 256, 8, 8, 0, False),      # k = E: every expert selected
    (200, 256, 256, 256, 8, 0, False),   # 256 experts, ~6 tokens each
    (500, 512, 256, 128, 8, 0, True),    # skewed routing, hot experts span many blocks
    (1000, 256, 512, 8, 2, 0, False),    # 2000 routed rows: many m-blocks per expert
]


@pytest.mark.parametrize("T,H,I,E,k,bm,zipf", SMALL)
def test_forward_matches_oracle(T, H, I, E, k, bm, zipf):
    shape = custom_shape(T, H, I, E, k, zipf)
    _, _, _, _, (fro, mx) = _run_and_compare(shape, bm)
    print(f"T={T} H={H} I={I} E={E} k={k} bm={bm}: rel_fro={fro:.2e} max_abs={mx:.2e}")


def test_uniform_routing_is_mean_of_experts():
    """Wg = 0, k = E: weights exactly 1/E, y = mean of all expert FFNs."""
    from synth.moe_inputs import make_expert_weights, _normal_bf16, _gen
    shape = custom_shape(96, 256, 256, 8, 8)
    x = _normal_bf16((96, 256), 1.0, _gen(torch.device(DEV), 0, 1), DEV)
    Wg = torch.zeros((256, 8), dtype=torch.bfloat16, device=DEV)
    W1, W3, W2 = make_expert_weights(shape, DEV)
    inp = dict(x=x, Wg=Wg, bias=None, W1=W1, W3=W3, W2=W2, k=8)
    plan = _plan(shape)
    y = plan.forward(x, Wg, None, W1, W3, W2)
    plan.check()
    r = plan.routing(96)
    assert torch.all(r["topk_w"] == 0.125)
    ref = oracle_forward(inp, block_m=plan.block_m)
    assert_routing_equal(r, ref)
    assert_y_close(y, ref["y"])


def test_plan_reuse_smaller_T_and_repeat():
    shape = custom_shape(256, 256, 256, 16, 4)
    plan = _plan(shape, T_max=512)
    inp = make_inputs(shape, device=DEV)
    y1 = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    r1 = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in plan.routing(256).items()}
    y2 = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    r2 = plan.routing(256)
    for key in ("topk_idx", "expert_count", "expert_offset", "slot_token", "slot_topk"):
        assert torch.equal(r1[key], r2[key]), key
    # fp32 atomics may reorder additions: y agrees to rounding
    assert (y1.float() - y2.float()).abs().max().item() <= 1e-2
    ref = oracle_forward(inp, block_m=plan.block_m)
    assert_y_close(y2, ref["y"])


def test_empty_batch_is_a_no_op():
    shape = custom_shape(64, 128, 256, 8, 2)
    plan = _plan(shape)
    inp = make_inputs(shape, device=DEV)
    y = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    plan.forward(inp["x"][:0], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"], y=y)
    plan.check()


def test_T_above_plan_limit_rejected():
    from moe_megakernel_b200 import MoEError
    shape = custom_shape(64, 128, 256, 8, 2)
    plan = _plan(shape, T_max=32)
    inp = make_inputs(shape, device=DEV)
    with pytest.raises(MoEError):
        plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])


def test_route_only_matches_oracle():
    shape = custom_shape(700, 384, 256, 64, 6, True)
    plan = _plan(shape)
    inp = make_inputs(shape, device=DEV)
    plan.route(inp["x"], inp["Wg"], inp["bias"])
    plan.check()
    from tests.parity_util import oracle_route
    assert_routing_equal(plan.routing(700), oracle_route(inp, plan.block_m))


def test_route_only_tcgen05_router_back_to_back():
    """Routing-only calls on the tcgen05 router (at least one 64-token tile per
    SM, E a multiple of 64), three in a row without a host sync, then the
    result against the oracle."""
    shape = custom_shape(10000, 256, 128, 64, 4)
    plan = _plan(shape)
    inp = make_inputs(shape, device=DEV)
    for _ in range(3):
        plan.route(inp["x"], inp["Wg"], inp["bias"])
    plan.check()
    from tests.parity_util import oracle_route
    assert_routing_equal(plan.routing(shape.T), oracle_route(inp, plan.block_m))


def test_host_io_entry_matches_device_entry():
    shape = custom_shape(128, 256, 256, 8, 2)
    plan = _plan(shape)
    inp = make_inputs(shape, device=DEV)
    y_dev = plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty((128, 256), dtype=torch.bfloat16).pin_memory()
    plan.forward_host(x_host, inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"], y_host)
    plan.check()
    assert (y_host.float() - y_dev.cpu().float()).abs().max().item() <= 1e-2


def test_bounded_wait_reports_timeout_and_context_survives():
    """A withheld L1 completion makes the dependent L2 tasks give up after the
    timeout; the error is reported by moe_check and the next run is clean."""
    from moe_megakernel_b200 import MoEError
    shape = custom_shape(256, 128, 256, 8, 2)
    plan = _plan(shape)
    inp = make_inputs(shape, device=DEV)
    plan.set_debug(withhold_block=0, timeout_ns=20_000_000)
    plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    with pytest.raises(MoEError) as ei:
        plan.check()
    assert ei.value.status == 6
    plan.set_debug(-1, 0)
    y = plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    ref = oracle_forward(inp, block_m=plan.block_m)
    assert_y_close(y, ref["y"])


def test_profiling_counts_forwards():
    shape = custom_shape(128, 128, 256, 8, 2)
    plan = _plan(shape)
    inp = make_inputs(shape, device=DEV)
    plan.set_profiling(True)
    for _ in range(3):
        plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    ms, n = plan.profile_read()
    assert n == 3 and all(v >= 0 for v in ms.values()) and ms["expert_gemm"] > 0


def test_h_ring_wraps_many_times():
    """I = 14336 makes the task groups 3-6 blocks, so the h ring is 18 blocks
    for ~70 expert blocks: every slot is reused several times."""
    from tests.parity_util import sample_tokens
    shape = custom_shape(4096, 128, 14336, 32, 2)
    inp = make_inputs(shape, device=DEV)
    plan = _plan(shape)
    _poison(plan)
    y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    rows = sample_tokens(shape.T, 256)
    ref = oracle_forward(inp, tokens=rows, block_m=plan.block_m)
    assert_routing_equal(plan.routing(shape.T), ref)
    assert int(ref["num_padded"]) // plan.block_m > 3 * 18
    assert_y_close(y[torch.from_numpy(rows).to(y.device)], ref["y"])
