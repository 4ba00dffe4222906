"""Failure detection on the GPU without a GPU fault: every device wait of the attention kernel
is bounded.  With the diagnostics fault on, each CTA's MMA warp withholds one "S ready"
signal; the waiting softmax warps run past a short limit, the CTA stops cleanly (bounded
drains, TMEM released) and the host reads ULTRAGEN_ERR_TIMEOUT.  The context stays usable:
the next normal call gives exactly the output of a fresh plan."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


@pytest.mark.parametrize("qk", ["bf16", "e4m3"])
def test_withheld_signal_times_out_and_context_survives(ug, qk):
    import torch
    wl = ug.WORKLOADS["1k"]
    q, k, v = (t.cuda() for t in ug.make_qkv(wl))
    plan = ug.plan_for(wl)
    plan.set_qk_format(qk)
    lay = ug.Layer(plan, wl.batch)
    ug.permute_rope(q, k, v, lay.qp, lay.kp, lay.vp, plan)
    assert plan.sync_status() == 0

    plan.set_diagnostics(fault=1, wait_limit_s=0.05)
    ug.hla_forward(lay.qp, lay.kp, lay.vp, lay.op, plan)
    assert plan.sync_status() == 5          # ULTRAGEN_ERR_TIMEOUT
    assert plan.sync_status() == 0          # the error word was cleared

    plan.set_diagnostics(fault=0, wait_limit_s=2.0)
    ug.hla_forward(lay.qp, lay.kp, lay.vp, lay.op, plan)
    assert plan.sync_status() == 0
    fresh = ug.plan_for(wl)
    fresh.set_qk_format(qk)
    lay2 = ug.Layer(fresh, wl.batch)
    ug.permute_rope(q, k, v, lay2.qp, lay2.kp, lay2.vp, fresh)
    ug.hla_forward(lay2.qp, lay2.kp, lay2.vp, lay2.op, fresh)
    assert fresh.sync_status() == 0
    torch.cuda.synchronize()
    assert torch.equal(lay.op.view(torch.int16), lay2.op.view(torch.int16))


def test_launch_clock_record(ug):
    """The launch clock record counts the attention launches and gives the SM clock they ran
    at (cycles of the first CTA over its nanoseconds), then clears."""
    import torch
    wl = ug.WORKLOADS["1k"]
    q, k, v = (t.cuda() for t in ug.make_qkv(wl))
    plan = ug.plan_for(wl)
    lay = ug.Layer(plan, wl.batch)
    ug.permute_rope(q, k, v, lay.qp, lay.kp, lay.vp, plan)
    plan.set_clock_record(True)
    for _ in range(3):
        ug.hla_forward(lay.qp, lay.kp, lay.vp, lay.op, plan)
    assert plan.sync_status() == 0
    rec = plan.read_clock()
    assert rec["launches"] == 3
    assert 300.0 < rec["sm_mhz"] < 2500.0, rec
    assert plan.read_clock()["launches"] == 0
    plan.set_clock_record(False)
    ug.hla_forward(lay.qp, lay.kp, lay.vp, lay.op, plan)
    assert plan.sync_status() == 0
    assert plan.read_clock()["launches"] == 0
    torch.cuda.synchronize()
