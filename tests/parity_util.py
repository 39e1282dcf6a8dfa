"""Comparison helpers shared by the GPU parity tests.

Tolerances (written here once, used by every parity test):
* routing (topk_idx, expert_count, expert_offset, slot_token, slot_topk,
  num_padded): bit-exact.
* topk_w: |gpu - oracle| <= TOPK_W_ATOL = 1e-5. The GPU forms each logit by
  fp32 accumulation of H exact bf16 x bf16 products (tensor-core steps of 16
  products, or H/64 chunks of the warp MMA), so it carries about H/16 roundings
  of partial sums of size |l| <= ~10 (logits ~ N(0,1), plus the skewed
  workload's bias down to -8.7), each at most 2**-24 |partial|: a random-walk
  sum of sqrt(H/16) * 2**-24 * 10 ~ 1.3e-5 at H = 7168, ~3e-6 for the |l| ~ 2
  of the selected experts. The renormalised softmax weight moves by
  w_j (dl_j - sum_i w_i dl_i), at most half of the largest logit error, and
  the fp32 exp / division add a few 2**-24. So 1e-5 holds with margin for the
  selected logits and still catches any wrong weight formula (those are off by
  > 1e-2). The measured maximum is printed by the workload tests.
* y: relative Frobenius error <= 1e-2 and max |gpu - oracle| <= 5e-2 on the
  compared rows.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle.moe_oracle as O

TOPK_W_ATOL = 1e-5
Y_REL_FRO = 1e-2
Y_MAX_ABS = 5e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).cpu().numpy()


def expert_loader(W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor):
    """Oracle expert weights, one expert at a time (exact bf16 -> fp64 widening)."""
    def load(e):
        return to_f64(W1[e]), to_f64(W3[e]), to_f64(W2[e])
    return load


def oracle_workers() -> int:
    """Threads for the oracle's per-expert loop in full-size tests."""
    return max(1, min(16, os.cpu_count() or 1))


def oracle_forward(inp: dict, tokens=None, block_m=None, fp8: bool = False, workers: int = 1):
    x = to_f64(inp["x"])
    Wg = to_f64(inp["Wg"])
    bias = None if inp["bias"] is None else to_f64(inp["bias"])
    S = inp.get("n_shared", 0)
    shared = expert_loader(inp["Ws1"], inp["Ws3"], inp["Ws2"]) if S else None
    load = expert_loader(inp["W1"], inp["W3"], inp["W2"])
    if workers > 1:
        # one BLAS thread per expert worker (the workers are the parallelism)
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            return O.moe_forward(x, Wg, bias, load, inp["k"], block_m=block_m, tokens=tokens,
                                 shared_weights=shared, n_shared=S, fp8=fp8, workers=workers)
    return O.moe_forward(x, Wg, bias, load, inp["k"], block_m=block_m, tokens=tokens,
                         shared_weights=shared, n_shared=S, fp8=fp8)


_FULL = {}


def _fingerprint(inp: dict):
    """A few sums of the inputs, so that a cached oracle result is only reused for the same tensors."""
    fp = [float(inp["x"].float().sum()), float(inp["Wg"].float().sum()), float(inp["W1"][0, 0].float().sum()),
          float(inp["W2"][-1, -1].float().sum())]
    return tuple(fp) + (None if inp["bias"] is None else float(inp["bias"].sum()),)


def full_oracle(name: str, inp: dict, block_m: int, fp8: bool = False) -> dict:
    """The oracle's layer over ALL tokens of a full-size workload (routed experts only),
    computed once per test session and shared by every test that compares that workload."""
    key = (name, fp8, block_m, _fingerprint(inp))
    if key not in _FULL:
        routed = dict(inp, n_shared=0)
        _FULL[key] = oracle_forward(routed, block_m=block_m, fp8=fp8, workers=oracle_workers())
    return _FULL[key]


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
    err = float(np.abs(w - ref["topk_w"]).max()) if T else 0.0
    assert err <= TOPK_W_ATOL, f"topk_w max abs error {err:.3e} > {TOPK_W_ATOL}"
    if T:
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-6)
    return err


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
