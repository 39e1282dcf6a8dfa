"""CPU oracle for the MoE-layer backward: plain, slow, fp64.

TEST INFRASTRUCTURE ONLY, like moe_oracle (only the tests may import it).

What it computes: the gradients of the forward layer of moe_oracle,
y[t] = sum_j w[t,j] * FFN_{e_j}(x[t]), FFN_e(x) = a W2[e], a = silu(x W1[e]) *
(x W3[e]), w = softmax over the k selected gate logits, for an upstream dy [T,H]:
dx, dWg, dbias, dW1, dW3, dW2. The pages name a backward MoE megakernel without
defining it ("MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
Replication", abstract: forward and backward megakernels, the backward reducing
the experts' weight gradients); "MegaMoE 在 MoE 系统谱系中的位置", section 五
(Mega MoE itself has no backward; the training path stays dispatch -> grouped
GEMM -> SwiGLU -> GEMM -> combine). Readings taken here:

* the gradient of the layer as written, by the chain rule; the top-k selection
  is piecewise constant (no gradient through which experts are chosen);
* the bf16 rounding of the activation is passed straight through (its
  derivative taken as 1): da is the gradient of the unrounded activation,
  while dW2 uses the rounded activation that the forward multiplied;
* no shared experts and no FP8 (the bf16 layer).

Steps, per expert e and the rows (t, j) routed to it, with do = w[t,j] dy[t]:
  dW2[e] += a^T do;  da = do W2[e]^T;
  dg = da * u * silu'(g);  du = da * silu(g);  silu'(g) = s (1 + g (1 - s)), s = sigmoid(g);
  dW1[e] += x^T dg;  dW3[e] += x^T du;  dx[t] += dg W1[e]^T + du W3[e]^T;
  dw[t,j] = dy[t] . o[t,j];
and for the gate, w = softmax(l_sel): dl[t,j] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]),
  dWg[:, e_j] += x[t] dl[t,j];  dbias[e_j] += dl[t,j];  dx[t] += Wg[:, e_j] dl[t,j].
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np

from oracle.moe_oracle import bf16_round, route, silu


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d silu(g) / dg = s (1 + g (1 - s)) with s = sigmoid(g)."""
    s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def selected_softmax_grad(w: np.ndarray, dw: np.ndarray) -> np.ndarray:
    """Gradient of the selected logits [T,k] of w = softmax(l_sel) for the upstream dw [T,k]."""
    return w * (dw - np.sum(w * dw, axis=1, keepdims=True))


def expert_ffn_backward(xr: np.ndarray, W1e: np.ndarray, W3e: np.ndarray, W2e: np.ndarray, do: np.ndarray,
                        round_activation: bool = True):
    """For rows xr [n,H] and the upstream do [n,H] of o = a W2e: (o, dxr, dW1e, dW3e, dW2e)."""
    g = xr @ W1e
    u = xr @ W3e
    a = silu(g) * u
    a_used = bf16_round(a) if round_activation else a
    o = a_used @ W2e
    dW2e = a_used.T @ do
    da = do @ W2e.T                     # straight through the rounding
    dg = da * u * silu_grad(g)
    du = da * silu(g)
    return o, dg @ W1e.T + du @ W3e.T, xr.T @ dg, xr.T @ du, dW2e


def moe_backward(x, Wg, bias, expert_weights: Callable[[int], tuple], k: int, dy,
                 round_activation: bool = True, workers: int = 1,
                 on_expert: Optional[Callable[..., None]] = None) -> dict:
    """Gradients of the layer for the upstream dy [T,H] (see the module notes).

    x [T,H], Wg [H,E], bias [E] or None, expert_weights(e) -> (W1[e] [H,I], W3[e] [H,I], W2[e] [I,H]).
    Returns dx [T,H], dWg [H,E], dbias [E] (zeros when bias is None), dW1/dW3 [E,H,I],
    dW2 [E,I,H], and the routing (topk_idx, topk_w) and dw [T,k] for inspection.

    workers > 1 runs the experts' backward in that many threads; their contributions are
    still added in ascending expert order. With on_expert, each expert's weight gradients are
    handed to on_expert(e, dW1e, dW3e, dW2e) (None for an expert no token chose) instead of
    being kept (dW1, dW3, dW2 are then returned as None).
    """
    x = np.asarray(x, np.float64)
    Wg = np.asarray(Wg, np.float64)
    dy = np.asarray(dy, np.float64)
    T, H = x.shape
    E = Wg.shape[1]
    idx, w, _ = route(x, Wg, bias, k)
    dx = np.zeros_like(x)
    dw = np.zeros((T, k))
    dW1 = dW3 = dW2 = None

    def expert_part(e):
        t, j = np.nonzero(idx == e)
        if t.size == 0:
            return e, t, j, None
        W1e, W3e, W2e = expert_weights(e)
        do = w[t, j][:, None] * dy[t]
        return e, t, j, (W1e.shape[1],) + expert_ffn_backward(x[t], W1e, W3e, W2e, do, round_activation)

    if workers > 1:
        from concurrent.futures import ThreadPoolExecutor
        pool = ThreadPoolExecutor(max_workers=workers)
        parts = pool.map(expert_part, range(E))
    else:
        pool = None
        parts = map(expert_part, range(E))
    for e, t, j, res in parts:
        if res is None:
            if on_expert is not None:
                on_expert(e, None, None, None)
            continue
        I, o, dxr, dW1e, dW3e, dW2e = res
        if on_expert is not None:
            on_expert(e, dW1e, dW3e, dW2e)
        else:
            if dW1 is None:
                dW1 = np.zeros((E, H, I))
                dW3 = np.zeros((E, H, I))
                dW2 = np.zeros((E, I, H))
            dW1[e], dW3[e], dW2[e] = dW1e, dW3e, dW2e
        dx[t] += dxr                      # a token chooses an expert at most once: rows t are distinct
        dw[t, j] = np.sum(dy[t] * o, axis=1)
    if pool is not None:
        pool.shutdown()
    dl = selected_softmax_grad(w, dw)
    # the gate gradients with the selected logits' gradients as a dense [T, E] matrix (zero where
    # an expert was not chosen): dWg = x^T dl, dbias = column sums of dl, dx += dl Wg^T
    dl_dense = np.zeros((T, E))
    np.put_along_axis(dl_dense, idx, dl, axis=1)
    dWg = x.T @ dl_dense
    dbias = dl_dense.sum(axis=0)
    dx += dl_dense @ Wg.T
    return dict(dx=dx, dWg=dWg, dbias=dbias, dW1=dW1, dW3=dW3, dW2=dW2, topk_idx=idx, topk_w=w, dw=dw)
