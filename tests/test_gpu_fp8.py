"""FP8 E4M3 expert GEMMs on the GPU against the oracle.

"MegaMoE 在 MoE 系统谱系中的位置", section 一 (the expert GEMMs take 8-bit
operands with scale factors beside them) and section 2.1 (activation amax and
quantization between the GEMMs): x and the activation are quantized per
token, W1 / W3 / W2 per (expert, column), with power-of-two scales, and both
GEMMs run on tcgen05 kind::f8f6f4. Codes and scales are compared bit-exactly
with the oracle's (both sides convert the same fp32 / fp64-exact quotient with
round to nearest even), y with the layer tolerances on the oracle's FP8 layer.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from synth.moe_inputs import WORKLOADS, custom_shape, make_inputs
from tests.parity_util import assert_routing_equal, assert_y_close, full_oracle, oracle_forward, sample_tokens, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each E4M3 byte: sign, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent 0 is subnormal (m/8 * 2**-6); 0x7f / 0xff are NaN."""
    b = codes.astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 15
    m = b & 7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * np.ldexp(1.0, e - 7))
    v = np.where((b & 0x7F) == 0x7F, np.nan, v)
    return s * v


def _x_cases(T=261, H=512, seed=3):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, H), generator=g)
    x *= torch.exp2(torch.randint(-24, 24, (T, 1), generator=g).float())   # scales across 48 binades
    x[0] = 0.0                          # amax 0: scale 1, codes 0
    x[1, :] = 0.001
    x[1, 7] = 448.0 * 8                 # amax exactly 448 * 2**3: scale 8, code 448
    x[2, :] = 1.0 + 1.0 / 16           # halfway between E4M3 1.0 and 1.125 after scaling by 1
    x[2, 0] = 300.0
    x[3, :] = -2.0 ** -10               # E4M3 subnormal range after scaling
    x[3, 1] = 1.0
    return x.to(torch.bfloat16)


def test_quantize_x_codes_and_scales_match_oracle():
    from moe_megakernel_b200 import quantize_x_fp8
    x = _x_cases()
    xq, sx = quantize_x_fp8(x.to(DEV))
    torch.cuda.synchronize()
    codes_ref, sc_ref = O.quantize_fp8(to_f64(x), axis=1)
    np.testing.assert_array_equal(sx.cpu().numpy().astype(np.float64), sc_ref[:, 0])
    np.testing.assert_array_equal(e4m3_decode(xq.cpu().numpy()), codes_ref)
    assert sx[0].item() == 1.0 and sx[1].item() == 8.0
    assert (xq[0] == 0).all()


def test_quantize_weights_codes_and_scales_match_oracle():
    from moe_megakernel_b200 import quantize_weights_fp8
    E, H, I = 3, 320, 192
    g = torch.Generator().manual_seed(5)
    W = torch.randn((E, H, I), generator=g) * 0.02
    W *= torch.exp2(torch.randint(-6, 6, (E, 1, I), generator=g).float())   # per-column magnitudes
    W[1, :, 5] = 0.0                                                        # an all-zero column
    W = W.to(torch.bfloat16)
    Wq, sc = quantize_weights_fp8(W.to(DEV))
    torch.cuda.synchronize()
    assert Wq.shape == (E, I, H) and sc.shape == (E, I)
    Wq, sc = Wq.cpu().numpy(), sc.cpu().numpy().astype(np.float64)
    for e in range(E):
        codes_ref, s_ref = O.quantize_fp8(to_f64(W[e]), axis=0)   # [H, I], [1, I]
        np.testing.assert_array_equal(sc[e], s_ref[0])
        np.testing.assert_array_equal(e4m3_decode(Wq[e]).T, codes_ref)
    assert sc[1, 5] == 1.0


SHAPES = [
    # T,   H,   I,   E,  k, block_m, zipf
    (64, 128, 256, 8, 2, 0, False),
    (300, 256, 384, 16, 4, 0, False),    # H % 256 != 0
    (129, 384, 256, 32, 8, 0, True),     # ragged T, bias
    (1000, 256, 512, 8, 2, 0, False),    # several full blocks per expert
    (40, 256, 256, 64, 8, 0, False),     # BLOCK_M 16 (decode-like)
    (500, 512, 256, 16, 2, 32, False),   # forced BLOCK_M 32
    (500, 512, 256, 16, 2, 64, False),   # forced BLOCK_M 64
]


def _fp8_weights(inp):
    from moe_megakernel_b200 import quantize_weights_fp8
    W1q, s1 = quantize_weights_fp8(inp["W1"])
    W3q, s3 = quantize_weights_fp8(inp["W3"])
    W2q, s2 = quantize_weights_fp8(inp["W2"])
    return W1q, s1, W3q, s3, W2q, s2


@pytest.mark.parametrize("pairs", [True, False], ids=["pairs", "single"])
@pytest.mark.parametrize("T,H,I,E,k,bm,zipf", SHAPES)
def test_fp8_forward_matches_oracle(T, H, I, E, k, bm, zipf, pairs):
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device=DEV)
    plan = MoEPlan(T, H, I, E, k, block_m=bm, fp8=True)
    plan.set_cta_pairs(pairs)
    plan.workspace.fill_(0xFF)   # poison: unwritten reads show up as NaN
    plan.lib.moe_plan_bind_workspace(plan._plan, plan.workspace.data_ptr(), plan.workspace_bytes)
    fw = _fp8_weights(inp)
    y = plan.forward_fp8(inp["x"], inp["Wg"], inp["bias"], *fw)
    plan.check()
    ref = oracle_forward(inp, block_m=plan.block_m, fp8=True)
    assert_routing_equal(plan.routing(T), ref)
    fro, mx = assert_y_close(y, ref["y"], "y (fp8)")
    # the FP8 layer differs from the bf16 one by the quantization, well above the kernel's own error
    # (the W2 codes are [E, H, I]: W2 transposed per expert)
    assert fw[4].shape == (E, H, I) and fw[5].shape == (E, H)
    ref16 = oracle_forward(inp, block_m=plan.block_m)
    q_err = np.linalg.norm(ref["y"] - ref16["y"]) / np.linalg.norm(ref16["y"])
    print(f"fp8 {'pairs' if pairs else 'single'} T={T} H={H} I={I} E={E} k={k} BM={plan.block_m}: "
          f"rel_fro={fro:.2e} max_abs={mx:.2e} (fp8 vs bf16 layer {q_err:.2e})")


def test_fp8_forward_rejects_shared_plan_and_bad_pointers():
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(64, 128, 256, 8, 2)
    inp = make_inputs(shape, device=DEV)
    fw = _fp8_weights(inp)
    y = torch.empty_like(inp["x"])
    W1q, s1, W3q, s3, W2q, s2 = fw
    shared = MoEPlan(64, 128, 256, 8, 2, n_shared=1)
    rc = shared.lib.moe_forward_fp8(shared._plan, inp["x"].data_ptr(), inp["Wg"].data_ptr(), None,
                                    W1q.data_ptr(), s1.data_ptr(), W3q.data_ptr(), s3.data_ptr(),
                                    W2q.data_ptr(), s2.data_ptr(), 64, y.data_ptr(), None)
    assert rc == 1   # MOE_ERR_INVALID_ARG: the FP8 layer has no shared experts
    assert shared.lib.moe_plan_set_fp8(shared._plan, 1) == 2   # MOE_ERR_UNSUPPORTED_SHAPE: shared experts
    plain = MoEPlan(64, 128, 256, 8, 2)   # no FP8 workspace regions
    rc = plain.lib.moe_forward_fp8(plain._plan, inp["x"].data_ptr(), inp["Wg"].data_ptr(), None,
                                   W1q.data_ptr(), s1.data_ptr(), W3q.data_ptr(), s3.data_ptr(),
                                   W2q.data_ptr(), s2.data_ptr(), 64, y.data_ptr(), None)
    assert rc == 1
    plan = MoEPlan(64, 128, 256, 8, 2, fp8=True)
    assert plan.workspace_bytes > plain.workspace_bytes
    for missing in ("s1", "s2"):
        rc = plan.lib.moe_forward_fp8(plan._plan, inp["x"].data_ptr(), inp["Wg"].data_ptr(), None,
                                      W1q.data_ptr(), None if missing == "s1" else s1.data_ptr(), W3q.data_ptr(),
                                      s3.data_ptr(), W2q.data_ptr(), None if missing == "s2" else s2.data_ptr(),
                                      64, y.data_ptr(), None)
        assert rc == 1   # missing column scales
    with pytest.raises(ValueError):
        plan.forward_fp8(inp["x"], inp["Wg"], None, W1q, s1, W3q, s3, inp["W2"], s2)   # bf16 W2: wrong layout
    shared.check()
    plain.check()
    plan.check()


def test_fp8_back_to_back_calls_do_not_leak_state():
    """x1, then a different x2 (larger activations), then x1 again on one plan: the third call
    matches the first (the per-row activation amax and scales are rebuilt every call)."""
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(300, 256, 384, 16, 4)
    inp = make_inputs(shape, device=DEV)
    fw = _fp8_weights(inp)
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, fp8=True)
    x2 = (inp["x"].float() * 8.0).to(torch.bfloat16)
    y1 = plan.forward_fp8(inp["x"], inp["Wg"], None, *fw).float().clone()
    plan.forward_fp8(x2, inp["Wg"], None, *fw)
    y3 = plan.forward_fp8(inp["x"], inp["Wg"], None, *fw).float()
    plan.check()
    # equal up to the order of the fp32 combine reductions
    assert (y1 - y3).abs().max().item() <= 1e-2 * max(1.0, y1.abs().max().item())


def test_fp8_host_entry_matches_device_entry():
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(300, 256, 384, 16, 4)
    inp = make_inputs(shape, device=DEV)
    fw = _fp8_weights(inp)
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, fp8=True)
    y = plan.forward_fp8(inp["x"], inp["Wg"], None, *fw).float()
    plan.check()
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty((shape.T, shape.H), dtype=torch.bfloat16).pin_memory()
    plan.forward_host_fp8(x_host, inp["Wg"], None, *fw, y_host)
    plan.check()
    assert (y_host.float() - y.cpu()).abs().max().item() <= 1e-2


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mixtral", "fine_grained_prefill", "decode"])
def test_fp8_workload_matches_oracle(name):
    """Full-size layers with FP8 expert GEMMs, y on every token row."""
    from moe_megakernel_b200 import MoEPlan
    shape = WORKLOADS[name]
    inp = make_inputs(shape, device=DEV)
    fw = _fp8_weights(inp)
    plan = MoEPlan(shape.T, shape.H, shape.I, shape.E, shape.k, fp8=True)
    y = plan.forward_fp8(inp["x"], inp["Wg"], inp["bias"], *fw)
    plan.check()
    ref = full_oracle(name, inp, plan.block_m, fp8=True)
    assert_routing_equal(plan.routing(shape.T), ref)
    fro, mx = assert_y_close(y, ref["y"], "y (fp8)")
    print(f"fp8 {name}: all {shape.T} rows rel_fro={fro:.2e} max_abs={mx:.2e}")
