"""Pins of the fp64 CPU oracle against things other than itself.

Each pin checks the oracle against a hand-derived fixture, a closed form, an
invariant of the method, or an independent library routine (torch on CPU),
so that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them. The mutation tests at the end plant such
mistakes in the oracle and check that a pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bf16_vals(rng, shape, std=1.0):
    """Random values that are exactly representable in bf16, as fp64."""
    v = torch.from_numpy(rng.standard_normal(shape) * std).to(torch.float32)
    return v.to(torch.bfloat16).double().numpy()


def _tiny_layer(rng, T=12, H=16, I=32, E=4):
    x = _bf16_vals(rng, (T, H))
    Wg = _bf16_vals(rng, (H, E), 1 / math.sqrt(H))
    W1 = _bf16_vals(rng, (E, H, I), 1 / math.sqrt(H))
    W3 = _bf16_vals(rng, (E, H, I), 1 / math.sqrt(H))
    W2 = _bf16_vals(rng, (E, I, H), 1 / math.sqrt(I))
    return x, Wg, W1, W3, W2


def _torch_ffn(xr, W1e, W3e, W2e):
    """Textbook SwiGLU FFN with torch fp64 ops; the activation rounded by the
    oracle's bf16 rounding (itself pinned against torch's conversion below)."""
    xt = torch.from_numpy(xr)
    g = xt @ torch.from_numpy(W1e)
    u = xt @ torch.from_numpy(W3e)
    a = torch.nn.functional.silu(g) * u
    a = torch.from_numpy(O.bf16_round(a.numpy()))
    return (a @ torch.from_numpy(W2e)).numpy()


# ----------------------------------------------------------------- rounding

def test_bf16_round_golden():
    fx = json.load(open(os.path.join(GOLDEN, "bf16_rounding.json")))
    for inp, exp in fx["cases"]:
        got = O.bf16_round(np.array([eval(inp)], dtype=np.float64))[0]
        want = float(eval(exp, {"inf": math.inf}))
        assert got == want, (inp, got, want)


def test_bf16_round_matches_torch_on_fp32_values():
    # torch converts fp32 -> bf16 with round-to-nearest-even; on values that
    # are exactly fp32 there is a single rounding, so the two must agree.
    rng = _rng(1)
    v32 = (rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 20, 200_000))).astype(np.float32)
    # add exact halfway points between neighbouring bf16 values
    base = torch.from_numpy(v32[:1000]).to(torch.bfloat16).float().numpy()
    half = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    v32 = np.concatenate([v32, half])
    want = torch.from_numpy(v32).to(torch.bfloat16).double().numpy()
    got = O.bf16_round(v32.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_silu_matches_torch():
    g = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(O.silu(g), torch.nn.functional.silu(torch.from_numpy(g)).numpy(),
                               rtol=1e-15, atol=1e-300)
    assert O.silu(np.array([0.0]))[0] == 0.0


# ----------------------------------------------------------------- gate

def test_routing_golden():
    fx = json.load(open(os.path.join(GOLDEN, "routing_small.json")))
    l = np.array(fx["logits"], dtype=np.float64)
    x = np.eye(l.shape[0])
    idx, w, logits = O.route(x, l, None, fx["k"])
    np.testing.assert_array_equal(idx, np.array(fx["topk_idx"]))
    exp = np.array([[eval(s, {"exp": math.exp}) for s in row] for row in fx["topk_w_closed_form"]])
    np.testing.assert_allclose(w, exp, rtol=0, atol=1e-15)
    d = O.dispatch(idx, l.shape[1], fx["block_m"])
    np.testing.assert_array_equal(d["count"], fx["count"])
    np.testing.assert_array_equal(d["offset"], fx["offset"])
    np.testing.assert_array_equal(d["slot_token"], fx["slot_token"])
    np.testing.assert_array_equal(d["slot_topk"], fx["slot_topk"])


def test_gate_logits_match_torch_matmul_and_bias_sign():
    rng = _rng(2)
    x, Wg = rng.standard_normal((7, 5)), rng.standard_normal((5, 3))
    b = np.array([0.5, -1.0, 2.0])
    want = (torch.from_numpy(x) @ torch.from_numpy(Wg)).numpy() + b
    np.testing.assert_allclose(O.gate_logits(x, Wg, b), want, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (256, 8), (5, 5), (3, 1)])
def test_top_k_matches_torch_topk(E, k):
    rng = _rng(E * 10 + k)
    l = rng.standard_normal((300, E))
    idx = O.top_k_select(l, k)
    ref = torch.topk(torch.from_numpy(l), k, dim=1).indices.sort(dim=1).values.numpy()
    np.testing.assert_array_equal(idx, ref)
    assert np.all(np.diff(idx, axis=1) > 0)


def test_weights_are_full_softmax_renormalised():
    # softmax over all E, keep the k selected, divide by their sum: same w
    rng = _rng(3)
    l = rng.standard_normal((50, 16)) * 3
    idx = O.top_k_select(l, 4)
    w = O.renormalised_softmax(l, idx)
    full = torch.softmax(torch.from_numpy(l), dim=1).numpy()
    sel = np.take_along_axis(full, idx, axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-13)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # larger logit, larger weight
    ls = np.take_along_axis(l, idx, axis=1)
    for t in range(50):
        assert np.all(np.argsort(ls[t], kind="stable") == np.argsort(w[t], kind="stable"))


# ----------------------------------------------------------------- dispatch

def test_block_m_rule_table():
    # the candidate steps: <=16 -> 16, <=32 -> 32, <=64 -> 64, else 128
    assert O.block_m_rule(64, 2, 8) == 16          # 16 per expert
    assert O.block_m_rule(4096, 2, 8) == 128       # 1024 per expert
    assert O.block_m_rule(16384, 8, 256) == 128    # 512 per expert
    assert O.block_m_rule(32, 8, 256) == 16        # 1 per expert
    assert O.block_m_rule(16384, 8, 128) == 128
    assert O.block_m_rule(68, 2, 8) == 32          # 17 per expert
    assert O.block_m_rule(128, 2, 8) == 32         # 32 per expert
    assert O.block_m_rule(129, 2, 8) == 64
    assert O.block_m_rule(257, 2, 8) == 128


def test_pool_capacity_matches_pages_formula_one_rank():
    # pool = ranks * max_tokens * min(topk, experts_per_rank) + experts_per_rank * (BLOCK_M - 1);
    # one rank, all experts local: T*k + E*(BLOCK_M-1) (the pages' 191 is BLOCK_M 192 - 1)
    assert O.pool_capacity(100, 8, 256, 192) == 100 * min(8, 256) + 256 * 191
    assert O.pool_capacity(16384, 8, 256, 128) == 163584


@pytest.mark.parametrize("T,E,k,bm", [(64, 8, 2, 16), (300, 16, 4, 32), (37, 5, 5, 8), (200, 64, 8, 128)])
def test_dispatch_invariants_and_stable_sort(T, E, k, bm):
    rng = _rng(T + E)
    l = rng.standard_normal((T, E)) + np.linspace(0, 2, E)[None, :]
    idx = O.top_k_select(l, k)
    d = O.dispatch(idx, E, bm)
    c, p, off = d["count"], d["padded"], d["offset"]
    assert c.sum() == T * k
    assert np.all(p % bm == 0)
    assert np.all((c <= p) & (p <= c + bm - 1))
    assert np.all((p == 0) == (c == 0))
    assert d["num_padded"] <= O.pool_capacity(T, k, E, bm)
    st, sk = d["slot_token"], d["slot_topk"]
    real = st >= 0
    assert real.sum() == T * k
    pairs = set(zip(st[real].tolist(), sk[real].tolist()))
    assert pairs == {(t, j) for t in range(T) for j in range(k)}
    # independent formulation: stable sort of the flattened pairs by expert id
    flat_e = idx.reshape(-1)
    order = np.argsort(flat_e, kind="stable")
    ref_t, ref_j = order // k, order % k
    np.testing.assert_array_equal(st[real], ref_t)
    np.testing.assert_array_equal(sk[real], ref_j)
    for e in range(E):
        seg_t = st[off[e]:off[e + 1]]
        seg_j = sk[off[e]:off[e + 1]]
        assert np.all(seg_t[:c[e]] >= 0) and np.all(seg_t[c[e]:] == -1) and np.all(seg_j[c[e]:] == -1)
        assert np.all(np.diff(seg_t[:c[e]]) > 0)
        assert np.all(idx[seg_t[:c[e]], seg_j[:c[e]]] == e)


# ----------------------------------------------------------------- FFN + combine

def test_brute_force_dense_masked():
    """y from the oracle == dense all-experts compute, masked by routing."""
    rng = _rng(4)
    x, Wg, W1, W3, W2 = _tiny_layer(rng)
    T, E, k = x.shape[0], Wg.shape[1], 2
    r = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), k)
    idx, w = r["topk_idx"], r["topk_w"]
    dense = np.stack([_torch_ffn(x, W1[e], W3[e], W2[e]) for e in range(E)])  # [E,T,H]
    gate = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            gate[t, idx[t, j]] = w[t, j]
    y_ref = np.einsum("te,eth->th", gate, dense)
    np.testing.assert_allclose(r["y"], y_ref, rtol=1e-12, atol=1e-14)


def test_k_equals_E_uniform_weights_is_mean_of_experts():
    rng = _rng(5)
    x, _, W1, W3, W2 = _tiny_layer(rng)
    E = W1.shape[0]
    Wg = np.zeros((x.shape[1], E))
    r = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), E)
    assert np.all(r["topk_w"] == 1.0 / E)
    mean = np.mean([_torch_ffn(x, W1[e], W3[e], W2[e]) for e in range(E)], axis=0)
    np.testing.assert_allclose(r["y"], mean, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("mode", ["k1", "bias"])
def test_single_expert_is_dense_ffn(mode):
    rng = _rng(6)
    x, Wg, W1, W3, W2 = _tiny_layer(rng)
    E = Wg.shape[1]
    if mode == "k1":
        r = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), 1)
        assert np.all(r["topk_w"] == 1.0)
        ref = np.stack([_torch_ffn(x[t:t + 1], W1[e], W3[e], W2[e])[0]
                        for t, e in enumerate(r["topk_idx"][:, 0])])
    else:
        b = np.zeros(E)
        b[0] = 100.0
        r = O.moe_forward(x, Wg, b, O.stacked_expert_weights(W1, W3, W2), 1)
        assert np.all(r["topk_idx"][:, 0] == 0)
        ref = _torch_ffn(x, W1[0], W3[0], W2[0])
    np.testing.assert_allclose(r["y"], ref, rtol=1e-12, atol=1e-14)


def test_metamorphic_token_permutation_expert_relabel_and_w2_scale():
    rng = _rng(7)
    x, Wg, W1, W3, W2 = _tiny_layer(rng, T=20, E=6)
    k = 2
    base = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), k)
    # token permutation permutes y
    perm = rng.permutation(x.shape[0])
    r = O.moe_forward(x[perm], Wg, None, O.stacked_expert_weights(W1, W3, W2), k)
    np.testing.assert_allclose(r["y"], base["y"][perm], rtol=1e-13, atol=1e-15)
    # consistent expert relabelling leaves y unchanged
    q = rng.permutation(Wg.shape[1])
    r = O.moe_forward(x, Wg[:, q], None, O.stacked_expert_weights(W1[q], W3[q], W2[q]), k)
    np.testing.assert_allclose(r["y"], base["y"], rtol=1e-13, atol=1e-15)
    # scaling W2 by 2 scales y by exactly 2
    r = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, 2 * W2), k)
    np.testing.assert_array_equal(r["y"], 2 * base["y"])


def test_token_subset_matches_full():
    rng = _rng(8)
    x, Wg, W1, W3, W2 = _tiny_layer(rng, T=30)
    full = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), 2)
    sub = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), 2, tokens=[3, 17, 29, 0])
    np.testing.assert_allclose(sub["y"], full["y"][[3, 17, 29, 0]], rtol=1e-14, atol=1e-16)


# ----------------------------------------------------------------- shared experts

def test_shared_experts_add_dense_ffns():
    """With the routed experts' W2 = 0 the routed combine is exactly 0, so y is
    the sum of the shared experts' textbook dense FFNs (weight 1 each)."""
    rng = _rng(11)
    x, Wg, W1, W3, W2 = _tiny_layer(rng)
    S = 2
    Ws1 = _bf16_vals(rng, (S, x.shape[1], W1.shape[2]), 0.25)
    Ws3 = _bf16_vals(rng, (S, x.shape[1], W1.shape[2]), 0.25)
    Ws2 = _bf16_vals(rng, (S, W1.shape[2], x.shape[1]), 0.2)
    r = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, 0 * W2), 2,
                      shared_weights=O.stacked_expert_weights(Ws1, Ws3, Ws2), n_shared=S)
    ref = sum(_torch_ffn(x, Ws1[s], Ws3[s], Ws2[s]) for s in range(S))
    np.testing.assert_allclose(r["y"], ref, rtol=1e-12, atol=1e-14)
    # routing and dispatch do not see the shared experts
    r0 = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), 2)
    for key in ("topk_idx", "offset", "slot_token", "slot_topk"):
        np.testing.assert_array_equal(r[key], r0[key])


def test_shared_expert_equal_to_routed_doubles_y():
    """Every token routed to expert 0 with weight 1 (bias +100, k = 1) and one
    shared expert with expert 0's weights: y = 2 * FFN_0(x)."""
    rng = _rng(12)
    x, Wg, W1, W3, W2 = _tiny_layer(rng)
    b = np.zeros(Wg.shape[1])
    b[0] = 100.0
    r = O.moe_forward(x, Wg, b, O.stacked_expert_weights(W1, W3, W2), 1,
                      shared_weights=O.stacked_expert_weights(W1[:1], W3[:1], W2[:1]), n_shared=1)
    np.testing.assert_allclose(r["y"], 2 * _torch_ffn(x, W1[0], W3[0], W2[0]), rtol=1e-12, atol=1e-14)


def test_two_shared_experts_equal_one_of_double_width():
    """Shared experts add up: S experts of width I equal one of width S*I
    (W1/W3 concatenated along I, W2 along I), since the activation is rounded
    element by element."""
    rng = _rng(13)
    x, Wg, W1, W3, W2 = _tiny_layer(rng)
    H, I = x.shape[1], W1.shape[2]
    Ws1 = _bf16_vals(rng, (2, H, I), 0.25)
    Ws3 = _bf16_vals(rng, (2, H, I), 0.25)
    Ws2 = _bf16_vals(rng, (2, I, H), 0.2)
    two = O.shared_ffn_sum(x, O.stacked_expert_weights(Ws1, Ws3, Ws2), 2)
    wide = O.expert_ffn(x, np.concatenate([Ws1[0], Ws1[1]], 1), np.concatenate([Ws3[0], Ws3[1]], 1),
                        np.concatenate([Ws2[0], Ws2[1]], 0))
    np.testing.assert_allclose(two, wide, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------- FP8 expert GEMMs

def test_e4m3_round_golden_and_matches_torch():
    """E4M3 rounding: hand-derived values (ties to even on the 1/8 mantissa
    grid, the 2**-9 subnormal grid, saturation at 448) and torch's float8
    conversion on 20000 random in-range values."""
    golden = {1.0: 1.0, 1.0625: 1.0, 1.1875: 1.25, 3.5: 3.5, 2.0 ** -9: 2.0 ** -9,
              1.5 * 2.0 ** -9: 2.0 ** -8, 2.0 ** -10: 0.0, 447.0: 448.0, 460.0: 448.0, -0.3: -0.3125}
    for v, want in golden.items():
        assert O.e4m3_round(v) == want, (v, O.e4m3_round(v), want)
    rng = _rng(21)
    v = np.clip(rng.standard_normal(20000) * np.exp(rng.uniform(-12, 6, 20000)), -448, 448)
    t = torch.from_numpy(v).to(torch.float32)
    np.testing.assert_array_equal(O.e4m3_round(t.double().numpy()), t.to(torch.float8_e4m3fn).double().numpy())


def test_pow2_scale_is_the_smallest_power_of_two():
    rng = _rng(22)
    amax = np.concatenate([np.exp(rng.uniform(-20, 20, 5000)), [448.0, 896.0, 224.0, 1.0]])
    p = O.pow2_scale(amax)
    k = np.log2(p)
    assert np.all(k == np.round(k))                       # powers of two
    assert np.all(amax / p <= 448.0) and np.all(amax / (p / 2) > 448.0)
    assert O.pow2_scale(0.0) == 1.0 and O.pow2_scale(448.0) == 1.0 and O.pow2_scale(449.0) == 2.0


def test_fp8_forward_matches_textbook_dequantized_ffn():
    """fp8=True equals the bf16 layer's combine with x, W1, W3, W2 and the
    bf16 activation replaced by their dequantized FP8 values (quantized here
    with torch's float8 cast and scales from torch log2/ceil; x and the
    activation per row, the weights per column)."""
    rng = _rng(23)
    x, Wg, W1, W3, W2 = _tiny_layer(rng, T=20, H=32, I=48, E=4)
    k = 2

    def tq(a, dim):
        amax = torch.from_numpy(np.abs(a)).amax(dim=dim, keepdim=True)
        sc = torch.where(amax > 0, torch.exp2(torch.ceil(torch.log2(amax / 448.0))), torch.ones_like(amax))
        q = (torch.from_numpy(a) / sc).to(torch.float32).to(torch.float8_e4m3fn).double()
        return (q * sc).numpy()

    xd = tq(x, 1)
    W1d = np.stack([tq(W1[e], 0) for e in range(W1.shape[0])])
    W3d = np.stack([tq(W3[e], 0) for e in range(W3.shape[0])])
    W2d = np.stack([tq(W2[e], 0) for e in range(W2.shape[0])])
    r = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), k, fp8=True)
    idx, w = r["topk_idx"], r["topk_w"]
    y = np.zeros_like(x)
    for t in range(x.shape[0]):
        for j in range(k):
            e = idx[t, j]
            xt = torch.from_numpy(xd[t:t + 1])
            g, u = xt @ torch.from_numpy(W1d[e]), xt @ torch.from_numpy(W3d[e])
            a = (torch.nn.functional.silu(g) * u).to(torch.bfloat16).double().numpy()
            y[t] += w[t, j] * (torch.from_numpy(tq(a, 1)) @ torch.from_numpy(W2d[e])).numpy()[0]
    np.testing.assert_allclose(r["y"], y, rtol=1e-12, atol=1e-14)
    # and it stays near the bf16 layer (FP8 has 3 mantissa bits)
    b = O.moe_forward(x, Wg, None, O.stacked_expert_weights(W1, W3, W2), k)
    assert np.linalg.norm(r["y"] - b["y"]) / np.linalg.norm(b["y"]) < 0.1


# ----------------------------------------------------------------- planted mistakes

_MUTANTS = {
    "no_activation_rounding": ("expert_ffn", lambda xr, W1e, W3e, W2e, round_activation=True:
                               (O.silu(xr @ W1e) * (xr @ W3e)) @ W2e),
    "swapped_gate_and_up": ("expert_ffn", lambda xr, W1e, W3e, W2e, round_activation=True:
                            O.bf16_round(O.silu(xr @ W3e) * (xr @ W1e)) @ W2e),
    "silu_sign": ("silu", lambda g: g / (1.0 + np.exp(g))),
    "no_renormalisation": ("renormalised_softmax", lambda l, idx:
                           np.take_along_axis(np.exp(l) / np.exp(l).sum(1, keepdims=True), idx, 1)),
    "descending_order": ("top_k_select", lambda l, k: np.argsort(-l, axis=1, kind="stable")[:, :k]),
    "round_half_away": ("bf16_round", lambda a: np.ldexp(np.floor(np.ldexp(np.frexp(np.asarray(a, float))[0], 8) + 0.5),
                                                          np.frexp(np.asarray(a, float))[1] - 8)),
    "shared_averaged": ("shared_ffn_sum", lambda xr, sw, S: sum(O.expert_ffn(xr, *sw(s)) for s in range(S)) / S),
    "shared_first_only": ("shared_ffn_sum", lambda xr, sw, S: O.expert_ffn(xr, *sw(0))),
    "e4m3_truncation": ("e4m3_round", lambda a: np.clip(np.ldexp(np.trunc(np.ldexp(np.asarray(a, float),
                        -(np.maximum(np.frexp(np.asarray(a, float))[1] - 1, -6) - 3))),
                        np.maximum(np.frexp(np.asarray(a, float))[1] - 1, -6) - 3), -448, 448)),
    "fp8_scale_dropped": ("expert_ffn_fp8", lambda xq, sx, W1q, s1, W3q, s3, W2q, s2:
                          (O.quantize_fp8(O.bf16_round(O.silu((xq @ W1q) * s1) * ((xq @ W3q) * s3)), 1)[0] @ W2q)
                          * O.quantize_fp8(O.bf16_round(O.silu((xq @ W1q) * s1) * ((xq @ W3q) * s3)), 1)[1] * s2),
    "fp8_activation_not_quantized": ("expert_ffn_fp8", lambda xq, sx, W1q, s1, W3q, s3, W2q, s2:
                                     (O.bf16_round(O.silu((xq @ W1q) * sx * s1) * ((xq @ W3q) * sx * s3)) @ W2q) * s2),
    "fp8_second_scale_dropped": ("expert_ffn_fp8", lambda xq, sx, W1q, s1, W3q, s3, W2q, s2:
                                 (O.quantize_fp8(O.bf16_round(O.silu((xq @ W1q) * sx * s1) * ((xq @ W3q) * sx * s3)),
                                                 1)[0] @ W2q) * s2),
    "pow2_scale_floor": ("pow2_scale", lambda amax: np.where(np.asarray(amax) > 0, np.ldexp(1.0, np.frexp(
                         np.asarray(amax, float) / 448.0)[1] - 1), 1.0)),
}


def _pins_pass():
    tests = [test_bf16_round_golden, test_bf16_round_matches_torch_on_fp32_values, test_silu_matches_torch,
             test_routing_golden, test_weights_are_full_softmax_renormalised, test_brute_force_dense_masked,
             test_k_equals_E_uniform_weights_is_mean_of_experts,
             lambda: test_top_k_matches_torch_topk(8, 2),
             lambda: test_single_expert_is_dense_ffn("bias"),
             test_shared_experts_add_dense_ffns, test_shared_expert_equal_to_routed_doubles_y,
             test_e4m3_round_golden_and_matches_torch, test_pow2_scale_is_the_smallest_power_of_two,
             test_fp8_forward_matches_textbook_dequantized_ffn]
    for t in tests:
        try:
            t()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("name", sorted(_MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = _MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    assert not _pins_pass(), f"mutant {name} slipped past every pin"


def test_moe_forward_threaded_experts_give_the_same_y():
    """The worker threads only compute the experts' outputs; y is added in expert order."""
    rng = _rng(7)
    T, H, I, E, k = 97, 128, 256, 16, 4
    x, Wg = _bf16_vals(rng, (T, H)), _bf16_vals(rng, (H, E), H ** -0.5)
    W1, W3 = _bf16_vals(rng, (E, H, I), H ** -0.5), _bf16_vals(rng, (E, H, I), H ** -0.5)
    W2 = _bf16_vals(rng, (E, I, H), I ** -0.5)
    load = O.stacked_expert_weights(W1, W3, W2)
    a = O.moe_forward(x, Wg, None, load, k)
    b = O.moe_forward(x, Wg, None, load, k, workers=4)
    assert np.array_equal(a["y"], b["y"])
