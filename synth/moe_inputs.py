"""Seeded synthetic inputs for the MoE-layer forward.

This module only draws inputs. It holds none of the layer's arithmetic: no
top-k, no softmax, no dispatch, no expert FFN, no combine. The one place it
looks at the inputs is the routing-gap screen: it computes fp64 gate logits
``x @ Wg + b`` solely to redraw tokens whose k-th and (k+1)-th largest logit
lie closer than ``GAP_MIN``, so that the set of selected experts cannot flip
under fp32 rounding. The layer itself is computed elsewhere, by the CUDA
library and, separately, by the CPU oracle; both consume the same tensors
produced here.

Workloads (one per named configuration):

* ``tiny``       T=64,    H=128,  I=256,   E=8,   k=2
* ``mixtral``    T=4096,  H=4096, I=14336, E=8,   k=2
* ``fine_grained_prefill``  T=16384, H=7168, I=2048, E=256, k=8
* ``decode``     T=32,    H=7168, I=2048,  E=256, k=8
* ``skewed``     T=16384, H=2048, I=768,   E=128, k=8, Zipf-like gate bias

Distributions: x ~ N(0,1); Wg, W1, W3 ~ N(0, 1/H); W2 ~ N(0, 1/I) (the
second argument is the variance). Every value is drawn in fp32 and rounded
to bf16 (round to nearest even, torch's conversion). The skewed workload adds
``b_e = 1.5 * ln(1 / (e+1)**1.2)`` (natural log, rank_e = e+1) to the gate
logits.

Every tensor has its own generator stream, seeded from (seed, stream id), so
a tensor does not change when another one's shape changes. Weights are drawn
one expert at a time so host memory stays bounded.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

GAP_MIN = 1e-2          # minimum gap between the k-th and (k+1)-th gate logit
MAX_REDRAWS = 64        # redraw rounds before giving up

_STREAM_X, _STREAM_WG, _STREAM_W1, _STREAM_W3, _STREAM_W2 = 1, 2, 3, 4, 5
_STREAM_WS1, _STREAM_WS3, _STREAM_WS2 = 6, 7, 8   # shared experts
_STREAM_DY = 9          # upstream gradient of the backward
_STREAM_REDRAW = 100    # + attempt number


@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    zipf_bias: bool = False

    @property
    def routed(self) -> int:
        return self.T * self.k


WORKLOADS = {
    "tiny": MoEShape("tiny", 64, 128, 256, 8, 2),
    "mixtral": MoEShape("mixtral", 4096, 4096, 14336, 8, 2),
    "fine_grained_prefill": MoEShape("fine_grained_prefill", 16384, 7168, 2048, 256, 8),
    "decode": MoEShape("decode", 32, 7168, 2048, 256, 8),
    "skewed": MoEShape("skewed", 16384, 2048, 768, 128, 8, zipf_bias=True),
}


def _gen(device: torch.device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        v.mul_(std)
    return v.to(torch.bfloat16)


def zipf_bias(E: int) -> torch.Tensor:
    """b_e = 1.5 * ln(1 / rank_e**1.2) with rank_e = e + 1, as fp32."""
    r = torch.arange(1, E + 1, dtype=torch.float64)
    return (1.5 * torch.log(1.0 / r.pow(1.2))).to(torch.float32)


def _ambiguous_tokens(x, Wg, bias, k: int) -> torch.Tensor:
    """Indices of tokens whose k-th/(k+1)-th largest gate logit differ by < GAP_MIN.

    The logits are formed in fp64 from the bf16 values, only to screen inputs.
    """
    E = Wg.shape[1]
    if k >= E:
        return torch.empty(0, dtype=torch.long, device=x.device)
    l = x.double() @ Wg.double()
    if bias is not None:
        l = l + bias.double().to(l.device)
    top = torch.topk(l, k + 1, dim=1, largest=True, sorted=True).values
    gap = top[:, k - 1] - top[:, k]
    return torch.nonzero(gap < GAP_MIN).flatten()


def make_router_inputs(shape: MoEShape, device="cpu", seed: int = 0,
                       T: Optional[int] = None, wg_zero: bool = False, x_seed: Optional[int] = None):
    """x [T,H] bf16, Wg [H,E] bf16, bias [E] fp32 or None, with the gap screen applied.
    ``x_seed`` (default ``seed``) seeds the tokens and their redraws only, so that replicas
    with the same weights can draw different tokens."""
    device = torch.device(device)
    T = shape.T if T is None else T
    H, E, k = shape.H, shape.E, shape.k
    xs = seed if x_seed is None else x_seed
    x = _normal_bf16((T, H), 1.0, _gen(device, xs, _STREAM_X), device)
    if wg_zero:
        Wg = torch.zeros((H, E), dtype=torch.bfloat16, device=device)
    else:
        Wg = _normal_bf16((H, E), 1.0 / math.sqrt(H), _gen(device, seed, _STREAM_WG), device)
    bias = zipf_bias(E).to(device) if shape.zipf_bias else None
    redrawn = 0
    if not wg_zero:
        for attempt in range(MAX_REDRAWS + 1):
            bad = _ambiguous_tokens(x, Wg, bias, k)
            if bad.numel() == 0:
                break
            if attempt == MAX_REDRAWS:
                raise RuntimeError(f"{shape.name}: {bad.numel()} tokens still ambiguous "
                                   f"after {MAX_REDRAWS} redraws")
            g = _gen(device, xs, _STREAM_REDRAW + attempt)
            x[bad] = _normal_bf16((bad.numel(), H), 1.0, g, device)
            if attempt == 0:
                redrawn = bad.numel()
    return x, Wg, bias, redrawn


def make_expert_weights(shape: MoEShape, device="cpu", seed: int = 0):
    """W1, W3 [E,H,I] and W2 [E,I,H], bf16, drawn one expert at a time."""
    device = torch.device(device)
    E, H, I = shape.E, shape.H, shape.I
    W1 = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
    W3 = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
    W2 = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    g1 = _gen(device, seed, _STREAM_W1)
    g3 = _gen(device, seed, _STREAM_W3)
    g2 = _gen(device, seed, _STREAM_W2)
    s_h, s_i = 1.0 / math.sqrt(H), 1.0 / math.sqrt(I)
    for e in range(E):
        W1[e] = _normal_bf16((H, I), s_h, g1, device)
        W3[e] = _normal_bf16((H, I), s_h, g3, device)
        W2[e] = _normal_bf16((I, H), s_i, g2, device)
    return W1, W3, W2


def make_shared_weights(shape: MoEShape, n_shared: int, device="cpu", seed: int = 0):
    """Shared experts Ws1, Ws3 [S,H,I] and Ws2 [S,I,H], bf16, same init as the routed experts
    (their own generator streams)."""
    device = torch.device(device)
    H, I = shape.H, shape.I
    Ws1 = torch.empty((n_shared, H, I), dtype=torch.bfloat16, device=device)
    Ws3 = torch.empty((n_shared, H, I), dtype=torch.bfloat16, device=device)
    Ws2 = torch.empty((n_shared, I, H), dtype=torch.bfloat16, device=device)
    g1 = _gen(device, seed, _STREAM_WS1)
    g3 = _gen(device, seed, _STREAM_WS3)
    g2 = _gen(device, seed, _STREAM_WS2)
    s_h, s_i = 1.0 / math.sqrt(H), 1.0 / math.sqrt(I)
    for e in range(n_shared):
        Ws1[e] = _normal_bf16((H, I), s_h, g1, device)
        Ws3[e] = _normal_bf16((H, I), s_h, g3, device)
        Ws2[e] = _normal_bf16((I, H), s_i, g2, device)
    return Ws1, Ws3, Ws2


def make_inputs(shape, device="cpu", seed: int = 0, T: Optional[int] = None, n_shared: int = 0,
                x_seed: Optional[int] = None):
    """All inputs of one workload as a dict of tensors on ``device`` (plus
    ``n_shared`` shared experts Ws1/Ws3/Ws2 when asked for). ``x_seed`` (default
    ``seed``) draws the tokens from another seed with the same weights."""
    if isinstance(shape, str):
        shape = WORKLOADS[shape]
    x, Wg, bias, redrawn = make_router_inputs(shape, device, seed, T, x_seed=x_seed)
    W1, W3, W2 = make_expert_weights(shape, device, seed)
    out = dict(shape=shape, x=x, Wg=Wg, bias=bias, W1=W1, W3=W3, W2=W2,
               k=shape.k, redrawn=redrawn, n_shared=n_shared)
    if n_shared:
        out["Ws1"], out["Ws3"], out["Ws2"] = make_shared_weights(shape, n_shared, device, seed)
    return out


def custom_shape(T, H, I, E, k, zipf=False, name="custom") -> MoEShape:
    return MoEShape(name, T, H, I, E, k, zipf)


def make_dy(shape: MoEShape, device="cpu", seed: int = 0, T: Optional[int] = None) -> torch.Tensor:
    """Upstream gradient dy [T,H] ~ N(0,1), bf16, for the backward."""
    device = torch.device(device)
    T = shape.T if T is None else T
    return _normal_bf16((T, shape.H), 1.0, _gen(device, seed, _STREAM_DY), device)
