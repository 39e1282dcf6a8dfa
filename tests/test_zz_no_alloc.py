"""The allocation-free routing entry point, moe_route_static, through the C ABI.

Some callers cannot allocate device memory: an inference engine's
enqueue-style callback that forbids allocation, a process whose device memory
a framework pool has already reserved, or a latency-critical loop that cannot
take cudaMalloc's implicit synchronisation. moe_route_static serves them with
a fixed scratch array inside the library. These tests check that it routes
exactly like the plan-and-workspace path (moe_route), on two calls in a row,
and that sizes beyond its fixed scratch are refused up front.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one.
"""
import ctypes

import pytest
import torch

from synth.moe_inputs import custom_shape, make_router_inputs
from tests.parity_util import TOPK_W_ATOL

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


@pytest.mark.parametrize("T,H,E,k,zipf", [(1000, 256, 64, 6, True), (300, 384, 8, 2, False)])
def test_route_static_matches_planned_route_twice(T, H, E, k, zipf):
    from moe_megakernel_b200 import MoEPlan, load_library
    lib = load_library()
    shape = custom_shape(T, H, 128, E, k, zipf)
    x, Wg, bias, _ = make_router_inputs(shape, device="cuda")
    plan = MoEPlan(T, H, 128, E, k)
    plan.route(x, Wg, bias)
    plan.check()
    ref = {key: (v.clone() if torch.is_tensor(v) else v) for key, v in plan.routing(T).items()}
    pool = plan.pool_capacity
    P = int(ref["num_padded"].item())

    dev = x.device
    out = dict(topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
               topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
               expert_count=torch.empty(E, dtype=torch.int32, device=dev),
               expert_offset=torch.empty(E + 1, dtype=torch.int32, device=dev),
               slot_token=torch.empty(pool, dtype=torch.int32, device=dev),
               slot_topk=torch.empty(pool, dtype=torch.int32, device=dev),
               num_padded=torch.empty(1, dtype=torch.int32, device=dev),
               error_word=torch.empty(1, dtype=torch.int32, device=dev))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        for v in out.values():
            v.fill_(-7)   # stale values must not survive a call
        rc = lib.moe_route_static(_p(x), _p(Wg), _p(bias), T, H, E, k, 0,
                                  _p(out["topk_idx"]), _p(out["topk_w"]), _p(out["expert_count"]),
                                  _p(out["expert_offset"]), _p(out["slot_token"]), _p(out["slot_topk"]), pool,
                                  _p(out["num_padded"]), _p(out["error_word"]), stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        assert out["error_word"].item() == 0, f"call {call}"
        assert out["num_padded"].item() == P, f"call {call}"
        for key in ("topk_idx", "expert_count", "expert_offset"):
            assert torch.equal(out[key], ref[key]), f"call {call}: {key}"
        assert torch.equal(out["slot_token"][:P], ref["slot_token"][:P]), f"call {call}: slot_token"
        assert torch.equal(out["slot_topk"][:P], ref["slot_topk"][:P]), f"call {call}: slot_topk"
        err = (out["topk_w"] - ref["topk_w"]).abs().max().item()
        assert err <= TOPK_W_ATOL, f"call {call}: topk_w differs by {err}"


def test_route_static_refuses_sizes_beyond_its_scratch():
    from moe_megakernel_b200 import load_library
    lib = load_library()
    # T*k alone exceeds the fixed scratch; nothing is enqueued, no pointer is touched
    rc = lib.moe_route_static(None, None, None, 1 << 17, 256, 64, 8, 0, None, None, None, None, None, None,
                              0, None, None, None)
    assert rc == 9
    assert lib.moe_status_string(rc).startswith(b"sizes exceed")
