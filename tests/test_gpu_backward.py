"""The backward kernels against the fp64 backward oracle.

moe_backward recomputes the routing, runs dgrad (g, u and dy W2^T on the
tensor cores, the SwiGLU and softmax derivatives in the epilogues, dx added
through the slot records), the gate backward, and the weight gradients as
reductions over each expert's slots. Every gradient is compared with the
oracle's (oracle/moe_oracle_backward.py, itself pinned against finite
differences and fp64 autograd) on the same seeded inputs.

Tolerance, per gradient tensor G: relative Frobenius error <= 1e-2 and
max |G_gpu - G_ref| <= 5e-2 * max |G_ref|. Derivation: every product on the
GPU has bf16 operands (exact) accumulated in fp32; the intermediates dg, du
and w * activation are stored as bf16 (relative rounding <= 2^-9 = 2e-3 per
element), as are dx and the weight gradients (another 2^-9); sums over K
terms of such independently rounded values carry a relative error of a few
1e-3, so 1e-2 leaves margin while a wrong term (a dropped factor, a sign, a
transposed operand) moves the result by O(1).
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
import oracle.moe_oracle_backward as B
from synth.moe_inputs import custom_shape, make_dy, make_inputs
from tests.parity_util import assert_routing_equal, oracle_route, to_f64

pytestmark = pytest.mark.gpu

REL_FRO = 1e-2
MAX_REL = 5e-2

BWD_SHAPES = [
    # T,    H,   I,   E,  k, block_m, zipf, bias
    (64, 128, 256, 8, 2, 0, False, False),      # tiny layer: BLOCK_M 16, H % 256 != 0
    (300, 256, 384, 16, 4, 0, False, True),     # BLOCK_M 128, ragged T
    (129, 384, 256, 32, 8, 0, True, True),      # BLOCK_M 32: weight-gradient K blocks cross experts
    (40, 256, 256, 64, 8, 0, False, False),     # BLOCK_M 16, idle experts (zero gradients)
    (1000, 256, 512, 8, 2, 0, False, False),    # several blocks per expert
    (500, 512, 256, 128, 8, 0, True, True),     # E = 128, Zipf-skewed
    (700, 256, 256, 16, 4, 64, False, False),   # BLOCK_M 64 forced
]


def _compare(name, got: torch.Tensor, ref: np.ndarray):
    g = got.to(torch.float64).cpu().numpy()
    d = g - ref
    fro = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)
    mx = float(np.abs(d).max()) if d.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    assert fro <= REL_FRO and mx <= MAX_REL * max(scale, 1e-30), \
        f"{name}: rel Frobenius {fro:.3e}, max abs {mx:.3e} (max |ref| {scale:.3e})"
    return fro


@pytest.mark.parametrize("T,H,I,E,k,bm,zipf,with_bias", BWD_SHAPES)
def test_backward_matches_oracle(T, H, I, E, k, bm, zipf, with_bias):
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device="cuda")
    bias = inp["bias"]
    if with_bias and bias is None:
        bias = (torch.arange(E, dtype=torch.float32, device="cuda") % 3 - 1.0) * 0.25
    dy = make_dy(shape, device="cuda")
    plan = MoEPlan(T, H, I, E, k, block_m=bm, backward=True)
    plan.workspace.fill_(0xFF)   # poison: anything read before it is written shows up as NaN
    plan.lib.moe_plan_bind_workspace(plan._plan, plan.workspace.data_ptr(), plan.workspace_bytes)
    g = plan.backward(inp["x"], inp["Wg"], bias, inp["W1"], inp["W3"], inp["W2"], dy)
    plan.check()
    r = oracle_route(dict(inp, bias=bias), plan.block_m)
    assert_routing_equal(plan.routing(T), r)
    ref = B.moe_backward(to_f64(inp["x"]), to_f64(inp["Wg"]), None if bias is None else to_f64(bias),
                         O.stacked_expert_weights(to_f64(inp["W1"]), to_f64(inp["W3"]), to_f64(inp["W2"])), k,
                         to_f64(dy))
    errs = {n: _compare(n, g[n], ref[n]) for n in ("dx", "dWg", "dW1", "dW3", "dW2")}
    if bias is not None:
        errs["dbias"] = _compare("dbias", g["dbias"], ref["dbias"])
    idle = np.nonzero(r["count"] == 0)[0]
    for e in idle:   # experts no token chose: exactly zero weight gradients
        assert g["dW1"][e].abs().max().item() == 0 and g["dW2"][e].abs().max().item() == 0
    print(f"backward T={T} H={H} I={I} E={E} k={k} bm={plan.block_m} idle={len(idle)} "
          + " ".join(f"{n}={v:.2e}" for n, v in errs.items()))


def test_backward_needs_backward_regions():
    from moe_megakernel_b200 import MoEError, MoEPlan
    shape = custom_shape(64, 128, 256, 8, 2)
    inp = make_inputs(shape, device="cuda")
    plan = MoEPlan(64, 128, 256, 8, 2)
    plan.has_backward = True   # the binding's own check bypassed: the library must refuse
    with pytest.raises(MoEError):
        plan.backward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"], make_dy(shape, device="cuda"))


def test_backward_twice_gives_the_same_gradients():
    """Outputs are overwritten, not accumulated into; the workspace carries no state between calls."""
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(300, 256, 384, 16, 4)
    inp = make_inputs(shape, device="cuda")
    dy = make_dy(shape, device="cuda")
    plan = MoEPlan(300, 256, 384, 16, 4, backward=True)
    a = plan.backward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"], dy)
    a = {n: v.clone() for n, v in a.items() if v is not None}
    b = plan.backward(inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"], dy)
    plan.check()
    for n in a:
        d = (a[n].float() - b[n].float()).abs().max().item()
        assert d <= 2e-2 * max(a[n].float().abs().max().item(), 1e-30), n


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny", "mixtral", "decode", "skewed", "fine_grained_prefill"])
def test_backward_workload_matches_oracle(name):
    """moe_backward at the five workloads' full sizes, every gradient compared in full: dx on every
    row, dWg and dbias, and each expert's dW1 / dW3 / dW2 (the oracle hands them over one expert
    at a time; the tolerances apply to each whole gradient tensor)."""
    from threadpoolctl import threadpool_limits

    from moe_megakernel_b200 import MoEPlan
    from synth.moe_inputs import WORKLOADS
    from tests.parity_util import expert_loader, oracle_workers
    shape = WORKLOADS[name]
    inp = make_inputs(shape, device="cuda")
    dy = make_dy(shape, device="cuda")
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, backward=True)
    g = plan.backward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], dy)
    plan.check()
    acc = {n: [0.0, 0.0, 0.0, 0.0] for n in ("dW1", "dW3", "dW2")}   # |d|^2, |ref|^2, max|d|, max|ref|
    idle = []

    def on_expert(e, dW1e, dW3e, dW2e):
        if dW1e is None:
            idle.append(e)
            return
        for n, ref in (("dW1", dW1e), ("dW3", dW3e), ("dW2", dW2e)):
            got = g[n][e].to(torch.float64).cpu().numpy()
            d = got - ref
            a = acc[n]
            a[0] += float(np.sum(d * d))
            a[1] += float(np.sum(ref * ref))
            a[2] = max(a[2], float(np.abs(d).max()))
            a[3] = max(a[3], float(np.abs(ref).max()))

    with threadpool_limits(limits=1):
        ref = B.moe_backward(to_f64(inp["x"]), to_f64(inp["Wg"]), None if inp["bias"] is None else to_f64(inp["bias"]),
                             expert_loader(inp["W1"], inp["W3"], inp["W2"]), shape.k, to_f64(dy),
                             workers=oracle_workers(), on_expert=on_expert)
    errs = {n: _compare(n, g[n], ref[n]) for n in ("dx", "dWg")}
    if inp["bias"] is not None:
        errs["dbias"] = _compare("dbias", g["dbias"], ref["dbias"])
    for n, (d2, r2, mx, rmax) in acc.items():
        fro = (d2 / max(r2, 1e-300)) ** 0.5
        assert fro <= REL_FRO and mx <= MAX_REL * max(rmax, 1e-30), f"{n}: rel Frobenius {fro:.3e}, max abs {mx:.3e}"
        errs[n] = fro
    for e in idle:
        assert g["dW1"][e].abs().max().item() == 0 and g["dW2"][e].abs().max().item() == 0
    print(f"backward {name}: idle experts {len(idle)} " + " ".join(f"{n}={v:.2e}" for n, v in errs.items()))
