"""Shared experts on the GPU against the oracle.

A plan made with n_shared > 0 runs every token through each shared expert
(weight 1) as more blocks of the same persistent expert GEMM ("MegaMoE 在 MoE
系统谱系中的位置", section 2.7: shared experts are phases of the routed
experts' task queue). Checked on both expert-GEMM kernels: routing unchanged
and bit-exact, the shared slot records, y against the oracle.
"""
import numpy as np
import pytest
import torch

from synth.moe_inputs import WORKLOADS, custom_shape, make_inputs
import oracle.moe_oracle as O
from tests.parity_util import (assert_routing_equal, assert_y_close, expert_loader, full_oracle, oracle_forward,
                                sample_tokens, to_f64)

pytestmark = pytest.mark.gpu

DEV = "cuda"

SHAPES = [
    # T,   H,   I,   E,  k, S, block_m, zipf
    (64, 128, 256, 8, 2, 1, 0, False),
    (300, 256, 384, 16, 4, 2, 0, False),     # H % 256 != 0, two shared experts
    (129, 384, 256, 32, 8, 1, 0, True),      # ragged T, bias
    (1000, 256, 512, 8, 2, 1, 0, False),     # several blocks per shared expert, odd counts
    (40, 256, 256, 64, 8, 3, 0, False),      # BLOCK_M 16 (decode-like), three shared experts
]


def _plan(shape, S, block_m=0, pairs=None):
    from moe_megakernel_b200 import MoEPlan
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, block_m=block_m, n_shared=S)
    if pairs is not None:
        plan.set_cta_pairs(pairs)
    return plan


def _fwd(plan, inp, **kw):
    return plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        Ws1=inp["Ws1"], Ws3=inp["Ws3"], Ws2=inp["Ws2"], **kw)


@pytest.mark.parametrize("pairs", [True, False], ids=["pairs", "single"])
@pytest.mark.parametrize("T,H,I,E,k,S,bm,zipf", SHAPES)
def test_shared_forward_matches_oracle(T, H, I, E, k, S, bm, zipf, pairs):
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device=DEV, n_shared=S)
    plan = _plan(shape, S, bm, pairs)
    plan.workspace.fill_(0xFF)   # poison: unwritten reads show up as NaN
    plan.lib.moe_plan_bind_workspace(plan._plan, plan.workspace.data_ptr(), plan.workspace_bytes)
    y = _fwd(plan, inp)
    plan.check()
    ref = oracle_forward(inp, block_m=plan.block_m)
    r = plan.routing(T)
    assert_routing_equal(r, ref)
    # shared slots: every token once per shared expert, in order, record (t, -2), padded with (-1, -1)
    P, BM = int(ref["num_padded"]), plan.block_m
    per = (T + BM - 1) // BM * BM
    tok = r["slot_token"][P:P + S * per].cpu().numpy().reshape(S, per)
    topk = r["slot_topk"][P:P + S * per].cpu().numpy().reshape(S, per)
    want = np.where(np.arange(per) < T, np.arange(per), -1)
    for s in range(S):
        np.testing.assert_array_equal(tok[s], want)
        np.testing.assert_array_equal(topk[s], np.where(np.arange(per) < T, -2, -1))
    fro, mx = assert_y_close(y, ref["y"])
    print(f"shared S={S} {'pairs' if pairs else 'single'} T={T} H={H} I={I} E={E} k={k}: "
          f"rel_fro={fro:.2e} max_abs={mx:.2e}")


def test_shared_plan_rejects_plain_forward_and_missing_weights():
    shape = custom_shape(64, 128, 256, 8, 2)
    inp = make_inputs(shape, device=DEV, n_shared=1)
    plan = _plan(shape, 1)
    y = torch.empty_like(inp["x"])
    rc = plan.lib.moe_forward(plan._plan, inp["x"].data_ptr(), inp["Wg"].data_ptr(), None, inp["W1"].data_ptr(),
                              inp["W3"].data_ptr(), inp["W2"].data_ptr(), 64, y.data_ptr(), None)
    assert rc == 1   # MOE_ERR_INVALID_ARG: the plan has a shared expert
    rc = plan.lib.moe_forward_shared(plan._plan, inp["x"].data_ptr(), inp["Wg"].data_ptr(), None,
                                     inp["W1"].data_ptr(), inp["W3"].data_ptr(), inp["W2"].data_ptr(),
                                     None, None, None, 64, y.data_ptr(), None)
    assert rc == 1   # shared weights missing
    with pytest.raises(TypeError):
        plan.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])   # the binding checks too
    plan.check()


def test_zero_shared_plan_matches_plain_plan():
    shape = custom_shape(300, 256, 384, 16, 4)
    inp = make_inputs(shape, device=DEV)
    from moe_megakernel_b200 import MoEPlan
    a = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k)
    b = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, n_shared=0)
    ya = a.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    yb = b.forward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    a.check()
    b.check()
    assert torch.equal(ya, yb) or (ya.float() - yb.float()).abs().max().item() <= 1e-2


def test_shared_host_entry_matches_device_entry():
    shape = custom_shape(300, 256, 384, 16, 4)
    inp = make_inputs(shape, device=DEV, n_shared=2)
    plan = _plan(shape, 2)
    y = _fwd(plan, inp).float()
    plan.check()
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty((shape.T, shape.H), dtype=torch.bfloat16).pin_memory()
    plan.forward_host(x_host, inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"], y_host,
                      Ws1=inp["Ws1"], Ws3=inp["Ws3"], Ws2=inp["Ws2"])
    plan.check()
    assert (y_host.float() - y.cpu()).abs().max().item() <= 1e-2


@pytest.mark.slow
@pytest.mark.parametrize("name", ["fine_grained_prefill", "decode"])
def test_shared_workload_matches_oracle(name):
    """DeepSeek-shaped layers (256 routed experts, top-8) with one shared expert."""
    shape = WORKLOADS[name]
    inp = make_inputs(shape, device=DEV, n_shared=1)
    plan = _plan(shape, 1)
    y = _fwd(plan, inp)
    plan.check()
    # every token row: the routed layer (shared with the other full-size tests) plus the
    # oracle's sum of the shared experts' FFNs, as the oracle's layer adds them
    ref = full_oracle(name, inp, plan.block_m)
    assert_routing_equal(plan.routing(shape.T), ref)
    y_ref = ref["y"] + O.shared_ffn_sum(to_f64(inp["x"]), expert_loader(inp["Ws1"], inp["Ws3"], inp["Ws2"]), 1)
    fro, mx = assert_y_close(y, y_ref)
    print(f"shared {name}: all {shape.T} rows rel_fro={fro:.2e} max_abs={mx:.2e}")
