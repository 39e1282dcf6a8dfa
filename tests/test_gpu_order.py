"""The expert GEMM's two task orders give the same layer.

The persistent kernel hands out its L1 (x W1, x W3 + SwiGLU) and L2 (h W2 +
combine) tasks from one queue ("MegaMoE 在 MoE 系统谱系中的位置", section 2.7).
Staggered: L1 of group 0, L1 of group 1, L2 of group 0, L1 of group 2, ...;
interleaved: after a lag, the L1 tasks of group m mixed evenly with the L2
tasks of group m-1. Both must match the oracle on shapes with several block
groups (so that the ring of h rows wraps and the L2-after-L1 and ring waits
are exercised in both orders), on both kernels.
"""
import pytest
import torch

from synth.moe_inputs import custom_shape, make_inputs
from tests.parity_util import assert_routing_equal, assert_y_close, oracle_forward

pytestmark = pytest.mark.gpu

ORDER_SHAPES = [
    # T,    H,   I,   E,  k, zipf   (expected blocks of 128: T*k/128 + padding)
    (8192, 256, 256, 16, 8, False),   # 512+ blocks: 3+ groups on both kernels, N1 = 2, N2 = 1
    (6000, 512, 768, 64, 8, True),    # Zipf-skewed: one hot expert spans several groups
    (4096, 384, 1280, 8, 2, False),   # H % 256 != 0, N1 = 10
]


@pytest.mark.parametrize("pairs", [True, False], ids=["pairs", "single"])
@pytest.mark.parametrize("T,H,I,E,k,zipf", ORDER_SHAPES)
def test_task_orders_match_oracle(T, H, I, E, k, zipf, pairs):
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device="cuda")
    ref = oracle_forward(inp, block_m=128)
    ys = []
    for order in (0, 1):
        plan = MoEPlan(T, H, I, E, k, block_m=128)
        plan.set_cta_pairs(pairs)
        plan.set_task_order(order)
        assert plan.task_order == order
        y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
        plan.check()
        assert_routing_equal(plan.routing(T), ref)
        fro, mx = assert_y_close(y, ref["y"], f"y (order {order})")
        print(f"{'pairs' if pairs else 'single'} order={order} T={T} H={H} I={I} E={E} k={k}: "
              f"rel_fro={fro:.2e} max_abs={mx:.2e}")
        ys.append(y.float())
    # the two orders add the same products in a different order into fp32: equal up to rounding
    assert (ys[0] - ys[1]).abs().max().item() <= 2e-2


def test_task_order_setter_rejects_unknown_modes():
    from moe_megakernel_b200 import MoEError, MoEPlan
    plan = MoEPlan(256, 256, 256, 8, 2)
    with pytest.raises(MoEError):
        plan.set_task_order(2)
    plan.set_task_order(-1)
    assert plan.task_order == 0                  # automatic: staggered
    plan.set_task_order(1)
    assert plan.task_order == 1
