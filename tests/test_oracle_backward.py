"""The backward oracle pinned against things other than itself (CPU).

* central finite differences of L = sum(dy * y) through the forward oracle
  (activation unrounded: the smooth function the backward differentiates);
* torch autograd in fp64 through an independent dense formulation of the
  layer (every expert on every token, masked by the routing);
* invariants: linearity in dy, zero weight gradients for an expert no token
  chooses, and the straight-through reading (dW1, dW3 do not depend on the
  rounding of the activation);
* planted mistakes, each caught by one of the above.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
import oracle.moe_oracle_backward as B


def _layer(seed, T=6, H=8, I=16, E=4):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    Wg = rng.standard_normal((H, E)) / np.sqrt(H)
    bias = rng.standard_normal(E) * 0.3
    W1 = rng.standard_normal((E, H, I)) / np.sqrt(H)
    W3 = rng.standard_normal((E, H, I)) / np.sqrt(H)
    W2 = rng.standard_normal((E, I, H)) / np.sqrt(I)
    dy = rng.standard_normal((T, H))
    return x, Wg, bias, W1, W3, W2, dy


def _loss(x, Wg, bias, W1, W3, W2, dy, k):
    r = O.moe_forward(x, Wg, bias, O.stacked_expert_weights(W1, W3, W2), k, round_activation=False)
    return float(np.sum(dy * r["y"])), r["topk_idx"]


def _grads(x, Wg, bias, W1, W3, W2, dy, k, round_activation=False):
    return B.moe_backward(x, Wg, bias, O.stacked_expert_weights(W1, W3, W2), k, dy, round_activation)


def test_backward_matches_finite_differences():
    k = 2
    params = list(_layer(11))
    dy = params.pop()
    g = _grads(*params, dy, k)
    names = ["x", "Wg", "bias", "W1", "W3", "W2"]
    want = {"x": g["dx"], "Wg": g["dWg"], "bias": g["dbias"], "W1": g["dW1"], "W3": g["dW3"], "W2": g["dW2"]}
    rng = np.random.default_rng(12)
    _, idx0 = _loss(*params, dy, k)
    h = 1e-6
    for pi, name in enumerate(names):
        p = params[pi]
        for _ in range(6):
            pos = tuple(rng.integers(0, n) for n in p.shape)
            plus = [q.copy() for q in params]
            minus = [q.copy() for q in params]
            plus[pi][pos] += h
            minus[pi][pos] -= h
            lp, ip = _loss(*plus, dy, k)
            lm, im = _loss(*minus, dy, k)
            assert np.array_equal(ip, idx0) and np.array_equal(im, idx0), "routing changed under the step"
            fd = (lp - lm) / (2 * h)
            an = want[name][pos]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, pos, fd, an)


def _torch_dense_layer(x, Wg, bias, W1, W3, W2, k):
    """Every expert on every token, then the k selected outputs weighted by the softmax of their logits."""
    logits = x @ Wg + bias
    sel = torch.topk(logits.detach(), k, dim=1).indices
    w = torch.softmax(torch.gather(logits, 1, sel), dim=1)                    # [T, k]
    g = torch.einsum("th,ehi->eti", x, W1)
    u = torch.einsum("th,ehi->eti", x, W3)
    o = torch.einsum("eti,eih->eth", torch.nn.functional.silu(g) * u, W2)    # [E, T, H]
    T = x.shape[0]
    picked = o[sel.T, torch.arange(T)[None, :]]                               # [k, T, H]
    return torch.einsum("tk,kth->th", w, picked)


@pytest.mark.parametrize("seed,k", [(21, 1), (22, 2), (23, 3), (24, 4)])
def test_backward_matches_torch_autograd(seed, k):
    params = list(_layer(seed, T=9, H=8, I=12, E=5))
    dy = params.pop()
    g = _grads(*params, dy, k)
    tp = [torch.tensor(p, dtype=torch.float64, requires_grad=True) for p in params]
    y = _torch_dense_layer(*tp, k)
    y.backward(torch.tensor(dy))
    for t, key in zip(tp, ["dx", "dWg", "dbias", "dW1", "dW3", "dW2"]):
        np.testing.assert_allclose(g[key], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=key)


def test_backward_is_linear_in_dy():
    params = list(_layer(31))
    dy1 = params.pop()
    dy2 = np.random.default_rng(32).standard_normal(dy1.shape)
    a, b, c = (_grads(*params, d, 2) for d in (dy1, dy2, 2.0 * dy1 - 3.0 * dy2))
    for key in ["dx", "dWg", "dbias", "dW1", "dW3", "dW2"]:
        np.testing.assert_allclose(c[key], 2.0 * a[key] - 3.0 * b[key], rtol=1e-9, atol=1e-12, err_msg=key)


def test_unchosen_expert_has_zero_gradients():
    x, Wg, bias, W1, W3, W2, dy = _layer(41)
    bias[-1] = -1e3                      # no token picks the last expert
    g = _grads(x, Wg, bias, W1, W3, W2, dy, 2)
    assert not np.any(g["topk_idx"] == Wg.shape[1] - 1)
    for key in ["dW1", "dW3", "dW2"]:
        assert np.all(g[key][-1] == 0.0)
    assert g["dbias"][-1] == 0.0 and np.all(g["dWg"][:, -1] == 0.0)


def test_straight_through_rounding():
    """The rounding of the activation only changes what depends on the rounded value (dW2 and,
    through o, the gate gradients); dW1 and dW3 come from da = w dy W2^T and are identical."""
    params = list(_layer(51))
    dy = params.pop()
    a = _grads(*params, dy, 2, round_activation=True)
    b = _grads(*params, dy, 2, round_activation=False)
    np.testing.assert_array_equal(a["dW1"], b["dW1"])
    np.testing.assert_array_equal(a["dW3"], b["dW3"])
    assert not np.array_equal(a["dW2"], b["dW2"])
    # and dW2 moves by about the bf16 rounding of the activation (2**-9 relative)
    assert np.linalg.norm(a["dW2"] - b["dW2"]) <= 1e-2 * np.linalg.norm(b["dW2"])


_MUTANTS = {
    "silu_grad_is_silu": ("silu_grad", lambda g: O.silu(g)),
    "silu_grad_missing_g_term": ("silu_grad", lambda g: 1.0 / (1.0 + np.exp(-g))),
    "softmax_grad_without_mean": ("selected_softmax_grad", lambda w, dw: w * dw),
    "softmax_grad_sign": ("selected_softmax_grad", lambda w, dw: -w * (dw - np.sum(w * dw, axis=1, keepdims=True))),
}


def _pins_pass():
    tests = [test_backward_matches_finite_differences, lambda: test_backward_matches_torch_autograd(22, 2)]
    for t in tests:
        try:
            t()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("name", sorted(_MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    fn, repl = _MUTANTS[name]
    monkeypatch.setattr(B, fn, repl)
    assert not _pins_pass(), f"mutant {name} was not caught"


def test_threaded_experts_and_per_expert_callback_give_the_same_gradients():
    """The full-size parity tests run the backward oracle with experts on host threads and take
    each expert's weight gradients through a callback; both give the plain run's values."""
    x, Wg, bias, W1, W3, W2, dy = _layer(51, T=20, E=6)
    bias[-1] = -1e3                      # one expert no token picks: the callback gets None for it
    plain = _grads(x, Wg, bias, W1, W3, W2, dy, 2, round_activation=True)
    got = {}

    def on_expert(e, dW1e, dW3e, dW2e):
        got[e] = (dW1e, dW3e, dW2e)

    t = B.moe_backward(x, Wg, bias, O.stacked_expert_weights(W1, W3, W2), 2, dy, True, workers=3,
                       on_expert=on_expert)
    assert t["dW1"] is None and sorted(got) == list(range(6))
    assert got[5] == (None, None, None)
    for e in range(5):
        for i, key in enumerate(("dW1", "dW3", "dW2")):
            np.testing.assert_allclose(got[e][i], plain[key][e], rtol=1e-12, atol=1e-14, err_msg=f"{key}[{e}]")
    for key in ("dx", "dWg", "dbias", "dw"):
        np.testing.assert_allclose(t[key], plain[key], rtol=1e-12, atol=1e-14, err_msg=key)
