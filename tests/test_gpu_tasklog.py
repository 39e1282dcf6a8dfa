"""The expert GEMM's task log: one record per task of the launch, consistent with the task
queue's rules ("MegaMoE 在 MoE 系统谱系中的位置", section 2.7: one queue holds both GEMMs'
tasks; a second-GEMM task runs after every first-GEMM task of its rows).

Checked on both kernels: every task number of the launch appears exactly once and every
(unit, phase, column tile) exactly once; each record's stamps are ordered; a CTA's MMA
issue intervals do not overlap; and no second-GEMM task of a unit issues its first MMA
before the last first-GEMM MMA of that unit was issued.
"""
import pytest
import torch

from synth.moe_inputs import custom_shape, make_inputs
from tests.parity_util import assert_y_close, oracle_forward

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pairs", [True, False], ids=["pairs", "single"])
@pytest.mark.parametrize("T,H,I,E,k,zipf", [(8192, 256, 256, 16, 8, False), (3000, 512, 768, 64, 8, True)])
def test_task_log_records_every_task_once(T, H, I, E, k, zipf, pairs):
    from moe_megakernel_b200 import MoEPlan
    shape = custom_shape(T, H, I, E, k, zipf)
    inp = make_inputs(shape, device="cuda")
    plan = MoEPlan(T, H, I, E, k, block_m=128, task_log=True)
    plan.set_cta_pairs(pairs)
    y = plan.forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    plan.check()
    assert_y_close(y, oracle_forward(inp, block_m=128)["y"])
    log = plan.task_log()
    n = log["task"].numel()
    assert n > 0
    assert torch.equal(torch.sort(log["task"]).values, torch.arange(n)), "task numbers 0 .. n-1, once each"
    key = (log["unit"] * 2 + log["phase"]) * 65536 + log["n"]
    assert torch.unique(key).numel() == n, "each (unit, phase, tile) once"
    # the number of tasks: every unit's first-GEMM tiles and second-GEMM tiles
    n1 = int(log["n"][log["phase"] == 0].max()) + 1
    n2 = int(log["n"][log["phase"] == 1].max()) + 1
    units = int(log["unit"].max()) + 1
    assert n == units * (n1 + n2)
    assert (log["t_first_mma"] <= log["t_last_mma"]).all() and (log["t_last_mma"] <= log["t_done"]).all()
    for cta in torch.unique(log["cta"]).tolist():   # one MMA warp per CTA: intervals in sequence
        m = log["cta"] == cta
        order = torch.argsort(log["t_first_mma"][m])
        a, b = log["t_first_mma"][m][order], log["t_last_mma"][m][order]
        assert (a[1:] >= b[:-1]).all(), f"CTA {cta}: overlapping MMA intervals"
    last_l1 = torch.zeros(units, dtype=torch.int64)
    l1 = log["phase"] == 0
    last_l1.scatter_reduce_(0, log["unit"][l1], log["t_last_mma"][l1], reduce="amax")
    l2 = log["phase"] == 1
    assert (log["t_first_mma"][l2] >= last_l1[log["unit"][l2]]).all(), "a second-GEMM task ran before its rows"
    span = int(log["t_done"].max() - log["t_first_mma"].min())
    busy = torch.zeros(int(log["cta"].max()) + 1, dtype=torch.int64)
    busy.scatter_add_(0, log["cta"], log["t_last_mma"] - log["t_first_mma"])
    print(f"{'pairs' if pairs else 'single'} T={T}: {n} tasks over {int((busy > 0).sum())} CTAs, "
          f"span {span / 1e3:.1f} us, MMA-issue occupancy mean {float(busy[busy > 0].float().mean()) / span:.2f}")


def test_task_log_needs_the_option():
    from moe_megakernel_b200 import MoEError, MoEPlan
    plan = MoEPlan(64, 128, 256, 8, 2)
    with pytest.raises(MoEError):
        plan.task_log()
