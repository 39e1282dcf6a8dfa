"""The seeded synthetic inputs (synth/moe_inputs.py) keep the recipe they state (CPU).

The generator draws x ~ N(0,1), Wg/W1/W3 ~ N(0,1/H), W2 ~ N(0,1/I) in fp32 and
rounds to bf16, each tensor from its own seeded stream; it redraws tokens whose
k-th and (k+1)-th gate logits are closer than GAP_MIN, so routing cannot flip
under fp32 rounding; the skewed workload adds b_e = 1.5 ln(1 / (e+1)^1.2).
"""
import math

import pytest
import torch

from synth.moe_inputs import (GAP_MIN, WORKLOADS, custom_shape, make_dy, make_expert_weights, make_inputs,
                              make_router_inputs, zipf_bias)


def test_same_seed_same_tensors_other_seed_other_tokens():
    a = make_inputs("tiny")
    b = make_inputs("tiny")
    for key in ("x", "Wg", "W1", "W3", "W2"):
        assert torch.equal(a[key], b[key]), key
    c = make_inputs("tiny", x_seed=1)
    assert not torch.equal(a["x"], c["x"])          # other tokens
    for key in ("Wg", "W1", "W3", "W2"):              # the same weights
        assert torch.equal(a[key], c[key]), key


@pytest.mark.parametrize("T,H,E,k,zipf", [(512, 128, 16, 4, False), (256, 256, 64, 8, True), (300, 128, 8, 2, False)])
def test_every_token_clears_the_routing_gap(T, H, E, k, zipf):
    shape = custom_shape(T, H, 128, E, k, zipf)
    x, Wg, bias, redrawn = make_router_inputs(shape)
    l = x.double() @ Wg.double()
    if bias is not None:
        l = l + bias.double()
    top = torch.topk(l, k + 1, dim=1).values
    gap = top[:, k - 1] - top[:, k]
    assert (gap >= GAP_MIN).all()
    assert redrawn >= 0


def test_zipf_bias_formula():
    b = zipf_bias(128)
    for e in (0, 1, 9, 127):
        assert abs(float(b[e]) - 1.5 * math.log(1.0 / (e + 1) ** 1.2)) < 1e-6
    assert float(b[0]) == 0.0 and (b[1:] < b[:-1]).all()   # decreasing with rank
    x, Wg, bias, _ = make_router_inputs(custom_shape(64, 128, 128, 32, 4, True))
    assert torch.equal(bias, zipf_bias(32))
    assert make_router_inputs(custom_shape(64, 128, 128, 32, 4, False))[2] is None


def test_values_are_bf16_with_the_stated_variances():
    shape = custom_shape(2048, 512, 384, 4, 2)
    x, Wg, _, _ = make_router_inputs(shape)
    W1, W3, W2 = make_expert_weights(shape)
    for t in (x, Wg, W1, W3, W2):
        assert t.dtype == torch.bfloat16
    # sample variances within a few standard errors of the stated ones
    for t, var in ((x, 1.0), (Wg, 1.0 / 512), (W1, 1.0 / 512), (W3, 1.0 / 512), (W2, 1.0 / 384)):
        v = float(t.double().var())
        assert abs(v / var - 1.0) < 0.05, (v, var)
    assert abs(float(x.double().mean())) < 0.01


def test_upstream_gradient_has_its_own_stream():
    shape = WORKLOADS["tiny"]
    dy = make_dy(shape)
    assert dy.shape == (shape.T, shape.H) and dy.dtype == torch.bfloat16
    assert torch.equal(dy, make_dy(shape))
    assert not torch.equal(dy, make_inputs(shape)["x"])
