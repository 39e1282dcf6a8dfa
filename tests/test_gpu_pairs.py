"""Parity of both expert-GEMM kernels with the oracle, each forced on.

The plan runs 128-row blocks on CTA pairs (tcgen05 cta_group::2: two
consecutive blocks of an expert per task, each CTA of a cluster holding its
own block's rows and half of the weight tile) and smaller blocks on the
single-CTA kernel. Here every shape runs on both, and the full workloads on
the kernel the plan would not pick. Shapes include experts with an odd block
count (the second CTA of the last pair has no block), BLOCK_M below 128,
H % 256 != 0 and a ring that wraps.
"""
import numpy as np
import pytest
import torch

from synth.moe_inputs import WORKLOADS, custom_shape, make_inputs
from tests.parity_util import assert_routing_equal, assert_y_close, full_oracle, oracle_forward, sample_tokens

pytestmark = pytest.mark.gpu

DEV = "cuda"

PAIR_SHAPES = [
    # T,   H,   I,   E,  k, block_m, zipf
    (64, 128, 256, 8, 2, 0, False),
    (300, 256, 384, 16, 4, 0, False),      # H % 256 != 0 (L2 tile 128 columns)
    (300, 256, 384, 16, 4, 16, False),
    (129, 384, 256, 32, 8, 0, True),
    (1000, 256, 512, 8, 2, 0, False),      # several pairs per expert, odd block counts
    (500, 512, 256, 128, 8, 0, True),
    (4096, 128, 14336, 32, 2, 0, False),   # N1 = 112: small groups, the h ring wraps
]


def _plan(shape, block_m=0, pairs=True):
    from moe_megakernel_b200 import MoEPlan
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, block_m=block_m)
    plan.set_cta_pairs(pairs)
    return plan


@pytest.mark.parametrize("pairs", [True, False], ids=["pairs", "single"])
@pytest.mark.parametrize("T,H,I,E,k,bm,zipf", PAIR_SHAPES)
def test_pairs_forward_matches_oracle(T, H, I, E, k, bm, zipf, pairs):
    """Both expert-GEMM kernels on every shape, whichever the plan would pick."""
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device=DEV)
    plan = _plan(shape, bm, pairs)
    plan.workspace.fill_(0xFF)   # poison: unwritten reads show up as NaN
    plan.lib.moe_plan_bind_workspace(plan._plan, plan.workspace.data_ptr(), plan.workspace_bytes)
    y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    ref = oracle_forward(inp, block_m=plan.block_m)   # every token row
    assert_routing_equal(plan.routing(T), ref)
    fro, mx = assert_y_close(y, ref["y"])
    print(f"{'pairs' if pairs else 'single'} T={T} H={H} I={I} E={E} k={k}: rel_fro={fro:.2e} max_abs={mx:.2e}")


def test_pairs_and_single_agree_and_repeat():
    shape = custom_shape(1000, 256, 512, 8, 2)
    inp = make_inputs(shape, device=DEV)
    plan = _plan(shape)
    y_pair = plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"]).float()
    plan.check()
    y_pair2 = plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"]).float()
    plan.check()
    plan.set_cta_pairs(False)
    y_single = plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"]).float()
    plan.check()
    assert (y_pair - y_single).abs().max().item() <= 1e-2
    assert (y_pair - y_pair2).abs().max().item() <= 1e-2


def test_pairs_bounded_wait_reports_timeout():
    from moe_megakernel_b200 import MoEError
    shape = custom_shape(256, 128, 256, 8, 2)
    inp = make_inputs(shape, device=DEV)
    plan = _plan(shape)
    plan.set_debug(withhold_block=0, timeout_ns=20_000_000)   # pair 0's L1 completion never published
    plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    with pytest.raises(MoEError) as ei:
        plan.check()
    assert ei.value.status == 6
    plan.set_debug(-1, 0)
    y = plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    assert_y_close(y, oracle_forward(inp, block_m=plan.block_m)["y"])


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mixtral", "fine_grained_prefill", "decode", "skewed"])
def test_pairs_workload_matches_oracle(name):
    """The full workloads on the kernel the plan does NOT pick by default."""
    shape = WORKLOADS[name]
    inp = make_inputs(shape, device=DEV)
    plan = _plan(shape)
    plan.set_cta_pairs(plan.block_m != 128)
    y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    ref = full_oracle(name, inp, plan.block_m)   # every token row
    assert_routing_equal(plan.routing(shape.T), ref)
    fro, mx = assert_y_close(y, ref["y"])
    print(f"{'pairs' if plan.block_m != 128 else 'single'} {name}: all {shape.T} rows rel_fro={fro:.2e} "
          f"max_abs={mx:.2e}")


HALF_SHAPES = [
    # T,    H,   I,   E,  k, zipf   odd block counts; with Zipf many cold experts of one block
    (1000, 256, 512, 8, 2, False),
    (3000, 512, 768, 64, 8, True),
    (700, 384, 256, 32, 4, True),     # H % 256 != 0: L2 tile of 128 columns, 64 per warp in half tasks
    (2600, 128, 1024, 16, 2, False),
]


@pytest.mark.parametrize("T,H,I,E,k,zipf", HALF_SHAPES)
def test_half_tail_tasks_match_oracle(T, H, I, E, k, zipf):
    """An expert's lone last block as M = 128 pair MMAs (64 rows per CTA) against full pairs and the oracle."""
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device=DEV)
    ref = oracle_forward(inp, block_m=128)
    nb = (ref["count"] + 127) // 128
    assert (nb % 2 == 1).any(), "the shape must have experts with an odd block count"
    ys = []
    for half in (True, False):
        plan = _plan(shape, 128, True)
        plan.set_half_tails(half)
        assert plan.half_tails == half
        plan.workspace.fill_(0xFF)   # poison: rows the half tasks miss would show up as NaN
        plan.lib.moe_plan_bind_workspace(plan._plan, plan.workspace.data_ptr(), plan.workspace_bytes)
        y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
        plan.check()
        assert_routing_equal(plan.routing(T), ref)
        fro, mx = assert_y_close(y, ref["y"], f"y (half tails {half})")
        print(f"half={half} T={T} H={H} I={I} E={E} k={k}: odd-block experts {int((nb % 2 == 1).sum())} "
              f"rel_fro={fro:.2e} max_abs={mx:.2e}")
        ys.append(y.float())
    assert (ys[0] - ys[1]).abs().max().item() <= 2e-2


WIDE_SHAPES = [
    # T,    H,   I,   E,  k, zipf   (I % 256 == 0: wide first-GEMM tasks apply)
    (1000, 256, 512, 8, 2, False),
    (3000, 512, 768, 64, 8, True),
    (4096, 128, 2048, 16, 2, False),   # H % 256 != 0 (L2 tile of 128 columns)
    (2600, 384, 256, 16, 2, False),    # one wide task per pair (I = 256)
]


@pytest.mark.parametrize("T,H,I,E,k,zipf", WIDE_SHAPES)
def test_wide_l1_tasks_match_oracle(T, H, I, E, k, zipf):
    """256-column first-GEMM tasks (two N = 256 MMAs on one gathered x tile), with and without
    half tail tasks, against 128-column tasks and the oracle."""
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device=DEV)
    ref = oracle_forward(inp, block_m=128)
    ys = {}
    for wide in (True, False):
        for half in (True, False):
            plan = _plan(shape, 128, True)
            plan.set_wide_l1(wide)
            plan.set_half_tails(half)
            assert plan.wide_l1 == wide
            plan.workspace.fill_(0xFF)
            plan.lib.moe_plan_bind_workspace(plan._plan, plan.workspace.data_ptr(), plan.workspace_bytes)
            y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
            plan.check()
            assert_routing_equal(plan.routing(T), ref)
            fro, mx = assert_y_close(y, ref["y"], f"y (wide {wide}, half {half})")
            print(f"wide={wide} half={half} T={T} H={H} I={I} E={E} k={k}: rel_fro={fro:.2e} max_abs={mx:.2e}")
            ys[(wide, half)] = y.float()
    base = ys[(False, False)]
    for key, y in ys.items():
        assert (y - base).abs().max().item() <= 2e-2, key
