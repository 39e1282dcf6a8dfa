"""CPU oracle for the MoE-layer forward: plain, slow, fp64.

TEST INFRASTRUCTURE ONLY. Only the tests, the package's ``smoke()`` check and
the CPU-baseline leg of the benchmark may import this module. The CUDA library
never imports it and shares no code, table or constant generator with it.

What it computes is the plain dropless top-k mixture-of-experts layer, the
operation that the pages fuse into one kernel:

* "FlashMoE Kernel", opening paragraph: the layer is gate -> dispatch ->
  expert FFN -> combine, in that order.
* "FlashMoE Kernel", section "架构" (unified task abstraction t=(M,*,phi)): the
  two FFN matmuls and the combine's Hadamard weighting are the tasks.
* "FlashMoE Kernel", section "通信" (in-place padding): tokens are padded to the
  tile only for local compute.
* "MegaMoE 在 MoE 系统谱系中的位置", section 2.4 (TokenSrcMetadata): each pool
  slot records the (token, top-k position) it came from; the combine writes
  through that record.
* "MegaMoE 在 MoE 系统谱系中的位置", sections 2.5/2.6: BLOCK_M is chosen from
  the expected tokens per expert T*k/E, and the pool is dropless with at most
  BLOCK_M-1 padding rows per expert.

Readings where the pages are silent (each is also listed in the design notes):

* Gate: softmax over all E logits, keep the k largest, renormalise over the k
  kept. This equals a softmax over the k selected logits, which is what is
  computed here.
* Ties in the top-k go to the lower expert id. Within a token the k selected
  experts are listed in ascending expert id.
* W1 is the gated branch (SiLU applied), W3 the linear branch, W2 the down
  projection: a = silu(x W1) * (x W3), o = a W2.
* The SwiGLU activation a is rounded to bf16 (round to nearest, ties to even)
  before the down projection, because the GPU path stores it as bf16.
* The gate bias, when present, is added to the logits before both the
  selection and the softmax.
* BLOCK_M rule for one GPU: with n = T*k/E expected tokens per expert,
  BLOCK_M = 16 if n <= 16, 32 if n <= 32, 64 if n <= 64, else 128.
* Padding slots of the per-expert blocks hold the record (-1, -1).
* Shared experts ("MegaMoE 在 MoE 系统谱系中的位置", section 2.7: the shared
  experts' two GEMM phases run in the same task queue as the routed ones):
  each of the S shared experts is the same SwiGLU FFN (same H and I, same
  bf16 rounding of the activation) applied to every token with weight 1 and
  added to the routed combine: y[t] += sum_s FFN_shared_s(x[t]). Routing and
  dispatch do not see them.

* FP8 expert GEMMs (optional; "MegaMoE 在 MoE 系统谱系中的位置", section 一:
  the Mega MoE kernel runs its GEMMs on 8-bit operands with scale factors
  loaded beside them, and section 2.1: the activation is quantized from its
  amax between the two GEMMs). Reading taken here: every operand of both
  expert GEMMs as OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3
  mantissa bits, largest finite 448, round to nearest even, saturating), with
  power-of-two scales, the smallest power of two p with amax / p <= 448 (1
  for an all-zero row or column): one per token over H for x; one per
  (expert, column i) over H for W1 and W3; one per token over I for the
  activation a = bf16(silu(g) * u) (rounded to bf16 first, as in the bf16
  layer); one per (expert, output column) over I for W2.
  g = sx[t] * s1[e,i] * sum_h xq[t,h] W1q[e,h,i], the same for u;
  o[t,c] = sa[t] * s2[e,c] * sum_i aq[t,i] W2q[e,i,c].

Everything is fp64 on inputs given as fp64 arrays holding bf16 values.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import numpy as np

# --------------------------------------------------------------------------
# Rounding


def bf16_round(a) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), as fp64.

    bf16 keeps 8 significant bits (1 implicit + 7 stored) and fp32's exponent
    range. Written from that definition: split a = m * 2**e with m in
    [0.5, 1), round m * 2**8 to the nearest integer (numpy's rint rounds half
    to even), scale back. Values below the smallest normal bf16 (2**-126) are
    rounded on the fixed subnormal grid 2**-133. Overflow rounds to +-inf.
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.empty_like(a)
    finite = np.isfinite(a)
    m, e = np.frexp(a[finite])
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    tiny = np.abs(a[finite]) < 2.0 ** -126
    if np.any(tiny):
        r[tiny] = np.rint(a[finite][tiny] * 2.0 ** 133) * 2.0 ** -133
    # largest finite bf16 is (2 - 2**-7) * 2**127
    big = np.abs(r) > (2.0 - 2.0 ** -7) * 2.0 ** 127
    r[big] = np.copysign(np.inf, r[big])
    out[finite] = r
    out[~finite] = a[~finite]
    return out


E4M3_MAX = 448.0


def e4m3_round(a) -> np.ndarray:
    """Round fp64 values to the nearest FP8 E4M3 value (ties to even), as fp64,
    saturating at +-448.

    Written from the format: normal values (1 + m/8) * 2**e for e in -6..8, so
    for |a| in [2**e, 2**(e+1)) the grid step is 2**(e-3); below 2**-6 the
    subnormal step is 2**-9.
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                      # a = m * 2**e, |m| in [0.5, 1)
    step_exp = np.maximum(e - 1, -6) - 3    # exponent of the grid step
    r = np.ldexp(np.rint(np.ldexp(a, -step_exp)), step_exp)
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def pow2_scale(amax) -> np.ndarray:
    """Smallest power of two p with amax / p <= 448 (1 where amax == 0)."""
    amax = np.asarray(amax, dtype=np.float64)
    q = amax / E4M3_MAX
    m, e = np.frexp(q)                      # q = m * 2**e, m in [0.5, 1)
    k = np.where(m == 0.5, e - 1, e)        # 2**k >= q, and 2**(k-1) < q
    return np.where(amax > 0, np.ldexp(1.0, k), 1.0)


def quantize_fp8(a: np.ndarray, axis: int):
    """(codes, scales): scales = pow2_scale(max |a| along `axis`), codes = e4m3_round(a / scales)."""
    sc = pow2_scale(np.max(np.abs(a), axis=axis, keepdims=True))
    return e4m3_round(a / sc), sc


# --------------------------------------------------------------------------
# Gate


def gate_logits(x: np.ndarray, Wg: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """l[t,e] = sum_h x[t,h] Wg[h,e] (+ b[e]), fp64. x [T,H], Wg [H,E]."""
    l = np.asarray(x, np.float64) @ np.asarray(Wg, np.float64)
    if bias is not None:
        l = l + np.asarray(bias, np.float64)[None, :]
    return l


def top_k_select(l: np.ndarray, k: int) -> np.ndarray:
    """For each token the k largest logits, ties to the lower expert id.

    Returns expert ids [T,k] listed in ascending expert id.
    """
    T, E = l.shape
    idx = np.empty((T, k), dtype=np.int64)
    experts = np.arange(E)
    for t in range(T):
        # lexsort sorts by the last key first: descending logit, then ascending id
        order = np.lexsort((experts, -l[t]))
        idx[t] = np.sort(order[:k])
    return idx


def renormalised_softmax(l: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """w[t,j] = exp(l[t,idx_j] - m) / sum_i exp(l[t,idx_i] - m), m = max over the k kept."""
    sel = np.take_along_axis(l, idx, axis=1)
    m = sel.max(axis=1, keepdims=True)
    p = np.exp(sel - m)
    return p / p.sum(axis=1, keepdims=True)


def route(x, Wg, bias, k: int):
    """Gate step: (topk_idx [T,k] int64 ascending, topk_w [T,k] fp64, logits [T,E])."""
    l = gate_logits(x, Wg, bias)
    idx = top_k_select(l, k)
    w = renormalised_softmax(l, idx)
    return idx, w, l


# --------------------------------------------------------------------------
# Dispatch


def block_m_rule(T: int, k: int, E: int) -> int:
    """BLOCK_M from the expected tokens per expert n = T*k/E (one GPU).

    The pages' candidate table steps BLOCK_M up with n; on one GPU with a
    128-row MMA tile the candidates kept are 16, 32, 64 and 128.
    """
    n = T * k / E
    if n <= 16:
        return 16
    if n <= 32:
        return 32
    if n <= 64:
        return 64
    return 128


def dispatch(idx: np.ndarray, E: int, block_m: int) -> dict:
    """Histogram, padded exclusive scan and stable slot permutation.

    count[e]   = number of (t, j) with idx[t,j] == e
    padded[e]  = ceil(count[e] / block_m) * block_m
    offset[e]  = sum of padded[e'] over e' < e  (offset has E+1 entries)
    Slot offset[e] + r holds the r-th token, in ascending token order, routed
    to e, with its top-k position j; the remaining slots of the expert's
    blocks hold (-1, -1).
    """
    T, k = idx.shape
    count = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            count[idx[t, j]] += 1
    padded = (count + block_m - 1) // block_m * block_m
    offset = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offset[e + 1] = offset[e] + padded[e]
    P = int(offset[E])
    slot_token = np.full(P, -1, dtype=np.int64)
    slot_topk = np.full(P, -1, dtype=np.int64)
    fill = offset[:E].copy()
    for t in range(T):              # ascending t makes the permutation stable
        for j in range(k):
            e = idx[t, j]
            slot_token[fill[e]] = t
            slot_topk[fill[e]] = j
            fill[e] += 1
    return dict(count=count, padded=padded, offset=offset, num_padded=P,
                slot_token=slot_token, slot_topk=slot_topk, block_m=block_m)


def pool_capacity(T: int, k: int, E: int, block_m: int) -> int:
    """Worst-case number of slots: every routed pair plus BLOCK_M-1 padding per expert."""
    return T * k + E * (block_m - 1)


# --------------------------------------------------------------------------
# Expert FFN and combine


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def expert_ffn(xr: np.ndarray, W1e: np.ndarray, W3e: np.ndarray, W2e: np.ndarray,
               round_activation: bool = True) -> np.ndarray:
    """o = bf16(silu(xr W1e) * (xr W3e)) W2e for rows xr [n,H]; W1e,W3e [H,I]; W2e [I,H].
    round_activation=False leaves the activation unrounded (the smooth function whose
    derivative the backward computes)."""
    g = xr @ W1e
    u = xr @ W3e
    a = silu(g) * u
    if round_activation:
        a = bf16_round(a)
    return a @ W2e


def expert_ffn_fp8(xq: np.ndarray, sx: np.ndarray, W1q: np.ndarray, s1: np.ndarray, W3q: np.ndarray,
                   s3: np.ndarray, W2q: np.ndarray, s2: np.ndarray) -> np.ndarray:
    """The expert FFN on FP8 operands: xq [n,H] codes with scales sx [n,1];
    W1q, W3q [H,I] codes with column scales s1, s3 [1,I]; W2q [I,H] codes with
    column scales s2 [1,H]. The bf16-rounded activation is quantized per row."""
    g = (xq @ W1q) * sx * s1
    u = (xq @ W3q) * sx * s3
    a = bf16_round(silu(g) * u)
    aq, sa = quantize_fp8(a, axis=1)
    return (aq @ W2q) * sa * s2


def stacked_expert_weights(W1, W3, W2) -> Callable[[int], tuple]:
    """Expert loader over stacked arrays W1,W3 [E,H,I], W2 [E,I,H] (any float dtype)."""
    def load(e):
        return (np.asarray(W1[e], np.float64), np.asarray(W3[e], np.float64),
                np.asarray(W2[e], np.float64))
    return load


def moe_forward(x, Wg, bias, expert_weights: Callable[[int], tuple], k: int,
                block_m: Optional[int] = None, tokens: Optional[Sequence[int]] = None,
                shared_weights: Optional[Callable[[int], tuple]] = None, n_shared: int = 0,
                fp8: bool = False, round_activation: bool = True, workers: int = 1) -> dict:
    """The whole layer: gate, dispatch, expert FFN, gate-weighted combine.

    x [T,H] fp64; Wg [H,E] fp64; bias [E] or None; ``expert_weights(e)``
    returns (W1[e], W3[e], W2[e]) as fp64. If ``tokens`` is given, y is
    computed only for those token rows (routing and dispatch always cover all
    T tokens). y[t] = sum_j w[t,j] * FFN_{idx[t,j]}(x[t])
                      + sum_{s < n_shared} FFN_shared_s(x[t]),
    with ``shared_weights(s)`` returning the shared expert's (W1, W3, W2).
    fp8=True runs both expert GEMMs on FP8 E4M3 operands (see the module notes):
    x and the activation per token, W1/W3/W2 per (expert, column); no shared experts.

    workers > 1 computes the experts' FFN outputs in that many threads (the
    matrix and rounding routines release the interpreter lock); they are still
    added into y one expert at a time in ascending expert order, so y is the
    same for any number of workers.
    """
    x = np.asarray(x, np.float64)
    T, H = x.shape
    E = np.asarray(Wg).shape[1]
    idx, w, logits = route(x, Wg, bias, k)
    bm = block_m_rule(T, k, E) if block_m is None else block_m
    disp = dispatch(idx, E, bm)
    rows = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    y = np.zeros((len(rows), H), dtype=np.float64)
    if fp8:
        if n_shared:
            raise ValueError("the FP8 layer is defined without shared experts")
        xq, sx = quantize_fp8(x, axis=1)

    def expert_part(e):
        # (row position in `rows`, top-k position) of every selected pair routed to e,
        # and the expert's FFN output for those rows
        hit = np.nonzero(idx[rows] == e)
        if hit[0].size == 0:
            return hit, None
        W1e, W3e, W2e = expert_weights(e)
        if fp8:
            W1q, s1 = quantize_fp8(W1e, axis=0)
            W3q, s3 = quantize_fp8(W3e, axis=0)
            W2q, s2 = quantize_fp8(W2e, axis=0)
            o = expert_ffn_fp8(xq[rows[hit[0]]], sx[rows[hit[0]]], W1q, s1, W3q, s3, W2q, s2)
        else:
            o = expert_ffn(x[rows[hit[0]]], W1e, W3e, W2e, round_activation)
        return hit, o

    if workers > 1:
        from concurrent.futures import ThreadPoolExecutor
        pool = ThreadPoolExecutor(max_workers=workers)
        parts = pool.map(expert_part, range(E))
    else:
        pool = None
        parts = map(expert_part, range(E))
    for hit, o in parts:
        if o is None:
            continue
        wt = w[rows[hit[0]], hit[1]]
        # a token selects an expert at most once, so the rows hit[0] are distinct
        y[hit[0]] += wt[:, None] * o
    if pool is not None:
        pool.shutdown()
    if n_shared:
        y += shared_ffn_sum(x[rows], shared_weights, n_shared)
    return dict(topk_idx=idx, topk_w=w, logits=logits, y=y, tokens=rows, **disp)


def shared_ffn_sum(xr: np.ndarray, shared_weights: Callable[[int], tuple], n_shared: int) -> np.ndarray:
    """sum over the n_shared shared experts of FFN_shared_s(xr), each with weight 1."""
    out = np.zeros((xr.shape[0], xr.shape[1]), dtype=np.float64)
    for sh in range(n_shared):
        W1s, W3s, W2s = shared_weights(sh)
        out += expert_ffn(xr, W1s, W3s, W2s)
    return out
