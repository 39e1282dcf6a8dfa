"""Comparison helpers shared by the GPU parity tests.

Tolerances (written here once, used by every parity test):
* routing (topk_idx, expert_count, expert_offset, slot_token, slot_topk,
  num_padded): bit-exact.
* topk_w: |gpu - oracle| <= TOPK_W_ATOL. The GPU forms the logits with fp32
  accumulation of H exact bf16 x bf16 products; with O(1) partial sums the
  accumulated error is about sqrt(H) * 2**-24 ~ 1e-5 for H <= 8192 and the
  renormalised softmax moves by at most half the logit error, so 1e-4 leaves
  an order of magnitude of margin while still catching a wrong weight formula
  (those are off by > 1e-2).
* y: relative Frobenius error <= 1e-2 and max |gpu - oracle| <= 5e-2 on the
  compared rows.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle.moe_oracle as O

TOPK_W_ATOL = 1e-4
Y_REL_FRO = 1e-2
Y_MAX_ABS = 5e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).cpu().numpy()


def expert_loader(W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor):
    """Oracle expert weights, one expert at a time (exact bf16 -> fp64 widening)."""
    def load(e):
        return to_f64(W1[e]), to_f64(W3[e]), to_f64(W2[e])
    return load


def oracle_forward(inp: dict, tokens=None, block_m=None, fp8: bool = False):
    x = to_f64(inp["x"])
    Wg = to_f64(inp["Wg"])
    bias = None if inp["bias"] is None else to_f64(inp["bias"])
    S = inp.get("n_shared", 0)
    shared = expert_loader(inp["Ws1"], inp["Ws3"], inp["Ws2"]) if S else None
    return O.moe_forward(x, Wg, bias, expert_loader(inp["W1"], inp["W3"], inp["W2"]), inp["k"],
                         block_m=block_m, tokens=tokens, shared_weights=shared, n_shared=S, fp8=fp8)


def oracle_route(inp: dict, block_m: int):
    x = to_f64(inp["x"])
    Wg = to_f64(inp["Wg"])
    bias = None if inp["bias"] is None else to_f64(inp["bias"])
    idx, w, _ = O.route(x, Wg, bias, inp["k"])
    d = O.dispatch(idx, Wg.shape[1], block_m)
    return dict(topk_idx=idx, topk_w=w, **d)


def assert_routing_equal(gpu: dict, ref: dict):
    T, k = ref["topk_idx"].shape
    np.testing.assert_array_equal(gpu["topk_idx"].cpu().numpy(), ref["topk_idx"], err_msg="topk_idx")
    np.testing.assert_array_equal(gpu["expert_count"].cpu().numpy(), ref["count"], err_msg="expert_count")
    np.testing.assert_array_equal(gpu["expert_offset"].cpu().numpy(), ref["offset"], err_msg="expert_offset")
    P = int(ref["num_padded"])
    assert int(gpu["num_padded"].item()) == P, "num_padded"
    np.testing.assert_array_equal(gpu["slot_token"][:P].cpu().numpy(), ref["slot_token"], err_msg="slot_token")
    np.testing.assert_array_equal(gpu["slot_topk"][:P].cpu().numpy(), ref["slot_topk"], err_msg="slot_topk")
    w = gpu["topk_w"].to(torch.float64).cpu().numpy()
    err = np.abs(w - ref["topk_w"]).max() if T else 0.0
    assert err <= TOPK_W_ATOL, f"topk_w max abs error {err:.3e} > {TOPK_W_ATOL}"
    if T:
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-6)


def y_errors(y_gpu: np.ndarray, y_ref: np.ndarray):
    d = y_gpu - y_ref
    fro = np.linalg.norm(d) / max(np.linalg.norm(y_ref), 1e-300)
    return float(fro), float(np.abs(d).max()) if d.size else 0.0


def assert_y_close(y_gpu: torch.Tensor, y_ref: np.ndarray, what="y"):
    fro, mx = y_errors(to_f64(y_gpu), y_ref)
    assert fro <= Y_REL_FRO and mx <= Y_MAX_ABS, f"{what}: rel Frobenius {fro:.3e}, max abs {mx:.3e}"
    return fro, mx


def sample_tokens(T: int, n: int, seed: int = 1):
    if n >= T:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, n - 2, replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(s))
