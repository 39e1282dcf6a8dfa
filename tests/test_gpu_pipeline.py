"""The pipelined host-buffer entry against the device entry.

Several calls in a row (more than the two staging buffers, so each buffer is
reused after its previous copy-out) with different inputs and their own host
outputs, bf16 and FP8; every y equals the device entry's y for the same input
(up to the order of the fp32 combine reductions).
"""
import pytest
import torch

from synth.moe_inputs import custom_shape, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "fp8"])
def test_pipelined_host_entry_matches_device_entry(fp8):
    from moe_megakernel_b200 import MoEPlan, quantize_weights_fp8
    shape = custom_shape(300, 256, 384, 16, 4)
    inp = make_inputs(shape, device=DEV)
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, fp8=fp8)
    fw = []
    if fp8:
        for w in ("W1", "W3", "W2"):
            fw += list(quantize_weights_fp8(inp[w]))
    xs = [(inp["x"].float() * s).to(torch.bfloat16) for s in (1.0, 2.0, 0.5, 1.5, 3.0)]
    ref = []
    for x in xs:
        if fp8:
            ref.append(plan.forward_fp8(x, inp["Wg"], inp["bias"], *fw).float().cpu())
        else:
            ref.append(plan.forward(x, inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"]).float().cpu())
    plan.check()
    x_host = [x.cpu().pin_memory() for x in xs]
    y_host = [torch.empty_like(x_host[0]).pin_memory() for _ in xs]
    for xh, yh in zip(x_host, y_host):
        if fp8:
            plan.forward_host_pipelined_fp8(xh, inp["Wg"], inp["bias"], *fw, yh)
        else:
            plan.forward_host_pipelined(xh, inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], yh)
    plan.host_pipeline_join()
    plan.check()
    for i, (yh, r) in enumerate(zip(y_host, ref)):
        err = (yh.float() - r).abs().max().item()
        assert err <= 1e-2 * max(1.0, r.abs().max().item()), f"call {i}: max abs difference {err:.3e}"
