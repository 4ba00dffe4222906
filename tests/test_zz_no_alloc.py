"""ultragen_hla_forward_noalloc against the ordinary ultragen_hla_forward, through the C ABI.

Some callers cannot allocate device memory when they call the library: a framework's caching
allocator may own the whole device, a real-time loop must not meet cudaMalloc's implicit
synchronisation, or the process runs under a fixed memory budget.  The no-allocation entry
point serves them with one fixed scratch array shared by all calls.  These checks run two
calls in a row (the second one finds the first call's partials still in the array) and
compare each with the ordinary entry point on the same inputs, within the attention
tolerance the other tests use.  The file name makes pytest collect it last.
"""
import dataclasses

import numpy as np
import pytest

from helpers import check_attention, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


def run_both(ug, wl, plan):
    import torch
    q, k, v = (t.cuda() for t in ug.make_qkv(wl))
    lay = ug.Layer(plan, wl.batch)
    ug.permute_rope(q, k, v, lay.qp, lay.kp, lay.vp, plan)      # also puts the plan on the GPU
    ref = torch.full_like(lay.qp, float("nan"))
    got = torch.full_like(lay.qp, float("nan"))
    ug.hla_forward(lay.qp, lay.kp, lay.vp, ref, plan)
    ug.hla_forward_noalloc(lay.qp, lay.kp, lay.vp, got, plan)
    assert plan.sync_status() == 0
    torch.cuda.synchronize()
    assert not torch.isnan(got).any()
    return to_np64(ref), to_np64(got)


def test_noalloc_matches_hla_forward_on_two_calls_in_a_row(ug):
    base = ug.WORKLOADS["1k"]
    for call in range(2):
        wl = dataclasses.replace(base, cfg=base.cfg + 100 * (call + 1), batch=2)
        plan = ug.plan_for(wl)                 # default split: text groups write partials
        need = plan.info["workspace_bytes_per_head"] * wl.heads * wl.batch
        assert plan.info["n_split_items"] > 0 and 0 < need <= (64 << 20)
        ref, got = run_both(ug, wl, plan)
        check_attention(got.ravel(), ref.ravel(), f"no-alloc call {call + 1}")


def test_noalloc_refuses_what_it_cannot_serve(ug):
    import torch
    L = ug.lib()
    buf = torch.empty(1024, dtype=torch.bfloat16, device="cuda")
    a = buf.data_ptr()
    # split partials beyond the fixed scratch: 8K layer, 24 heads, default split
    big = ug.plan_for(ug.WORKLOADS["8k"])
    need = big.info["workspace_bytes_per_head"] * 24
    assert need > (64 << 20)
    assert L.ultragen_hla_forward_noalloc(a, a, a, a, big.handle, 1, None) == 2
    # a plan whose tables are not on the device yet: the call uploads nothing and refuses
    cold = ug.plan_for(ug.WORKLOADS["tiny"])
    assert L.ultragen_hla_forward_noalloc(a, a, a, a, cold.handle, 1, None) == 6
    assert L.ultragen_hla_forward_noalloc(None, a, a, a, cold.handle, 1, None) == 1
