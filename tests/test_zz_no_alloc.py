"""ultragen_hla_forward_noalloc against the ordinary ultragen_hla_forward, through the C ABI.

Some callers cannot allocate device memory when they call the library: a framework's caching
allocator may own the whole device, a real-time loop must not meet cudaMalloc's implicit
synchronisation, or the process runs under a fixed memory budget.  The no-allocation entry
point serves them with one fixed scratch array shared by all calls.  It runs the same kernels
as the ordinary entry point, so the two must agree bit for bit.  These checks run two calls in
a row (the second one finds the first call's partials still in the array), and check that a
plan changed after its upload is refused instead of being uploaded again.  The file name makes
pytest collect it last.
"""
import dataclasses

import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


def run_both(ug, plan, lay, call_noalloc=True):
    """hla_forward and hla_forward_noalloc on the same permuted inputs; both outputs start as
    NaN so that a row either call leaves unwritten shows up."""
    import torch
    ref = torch.full_like(lay.qp, float("nan"))
    got = torch.full_like(lay.qp, float("nan"))
    ug.hla_forward(lay.qp, lay.kp, lay.vp, ref, plan)
    if call_noalloc:
        ug.hla_forward_noalloc(lay.qp, lay.kp, lay.vp, got, plan)
    assert plan.sync_status() == 0
    torch.cuda.synchronize()
    return ref, got


def bit_equal(a, b) -> bool:
    import torch
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_noalloc_matches_hla_forward_bitwise_on_two_calls_in_a_row(ug):
    base = ug.WORKLOADS["1k"]
    for call in range(2):
        wl = dataclasses.replace(base, cfg=base.cfg + 100 * (call + 1), batch=2)
        plan = ug.plan_for(wl)
        plan.set_split(11)                     # text groups split: their partials use the scratch
        need = plan.info["workspace_bytes_per_head"] * wl.heads * wl.batch
        assert plan.info["n_split_items"] > 0 and 0 < need <= (64 << 20)
        q, k, v = (t.cuda() for t in ug.make_qkv(wl))
        lay = ug.Layer(plan, wl.batch)
        ug.permute_rope(q, k, v, lay.qp, lay.kp, lay.vp, plan)   # puts the plan on the GPU
        ref, got = run_both(ug, plan, lay)
        assert bit_equal(ref, got), f"no-alloc call {call + 1} differs from hla_forward"


def test_noalloc_refuses_a_plan_changed_after_upload(ug):
    import torch
    wl = ug.WORKLOADS["1k"]
    plan = ug.plan_for(wl)
    plan.set_split(11)
    q, k, v = (t.cuda() for t in ug.make_qkv(wl))
    lay = ug.Layer(plan, wl.batch)
    ug.permute_rope(q, k, v, lay.qp, lay.kp, lay.vp, plan)
    torch.cuda.synchronize()
    plan.set_split(0)                          # no split now: the device tables are out of date
    L = ug.lib()
    out = torch.empty_like(lay.qp)
    st = L.ultragen_hla_forward_noalloc(lay.qp.data_ptr(), lay.kp.data_ptr(), lay.vp.data_ptr(),
                                        out.data_ptr(), plan.handle, wl.batch, None)
    assert st == 6                             # ULTRAGEN_ERR_PLAN_MISMATCH: nothing uploaded
    # a device call that may allocate puts the changed plan on the GPU; then it is served
    ug.permute_rope(q, k, v, lay.qp, lay.kp, lay.vp, plan)
    ref, got = run_both(ug, plan, lay)
    assert bit_equal(ref, got)


def test_noalloc_refuses_what_it_cannot_serve(ug):
    import torch
    L = ug.lib()
    buf = torch.empty(1024, dtype=torch.bfloat16, device="cuda")
    a = buf.data_ptr()
    # split partials beyond the fixed scratch: 8K layer, 24 heads, text groups split
    big = ug.plan_for(ug.WORKLOADS["8k"])
    big.set_split(41)
    need = big.info["workspace_bytes_per_head"] * 24
    assert need > (64 << 20)
    assert L.ultragen_hla_forward_noalloc(a, a, a, a, big.handle, 1, None) == 2
    # a plan whose tables are not on the device yet: the call uploads nothing and refuses
    cold = ug.plan_for(ug.WORKLOADS["tiny"])
    assert L.ultragen_hla_forward_noalloc(a, a, a, a, cold.handle, 1, None) == 6
    assert L.ultragen_hla_forward_noalloc(None, a, a, a, cold.handle, 1, None) == 1
