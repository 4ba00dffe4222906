"""The host-buffer runner gives the same bits as the device path (same kernels per head)."""
import dataclasses

import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


@pytest.mark.parametrize("name,hpc,split", [("1k", 5, None), ("1k", 24, None), ("ragged", 7, None),
                                            ("tiny", 1, 2), ("1k", 3, 0)])
def test_host_runner_matches_device_path(ug, name, hpc, split):
    import torch
    wl = ug.WORKLOADS[name]
    plan = ug.plan_for(wl)
    if split is not None:
        plan.set_split(split)
    q, k, v = (x.to(torch.bfloat16) for x in ug.make_qkv(wl))
    shape = (wl.batch, plan.info["N_raster"], wl.heads, wl.D)
    # device path: permute_rope + hla_forward_raster on the same bf16 inputs
    lay = ug.Layer(plan, wl.batch)
    o_dev = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    lay(q.cuda(), k.cuda(), v.cuda(), o_dev)
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    # host path
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.full(shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    run = ug.HostRunner(plan, wl.batch, hpc)
    run(qh, kh, vh, oh)
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    assert run.last_launch_count() >= 2 * ((wl.heads + hpc - 1) // hpc) * wl.batch
    assert torch.equal(oh.view(torch.int16), o_dev.cpu().view(torch.int16))
    # a second call on the same runner (staging reuse) gives the same bits
    oh2 = torch.full(shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    run(qh, kh, vh, oh2)
    torch.cuda.synchronize()
    assert torch.equal(oh2.view(torch.int16), oh.view(torch.int16))
    run.close()


def test_host_runner_pageable_memory(ug):
    """Pageable host buffers work too (the copies then do not overlap)."""
    import torch
    wl = dataclasses.replace(ug.WORKLOADS["1k"], heads=4)
    plan = ug.plan_for(wl)
    q, k, v = ug.make_qkv(wl)
    shape = (wl.batch, plan.info["N_raster"], wl.heads, wl.D)
    lay = ug.Layer(plan, wl.batch)
    o_dev = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    lay(q.cuda(), k.cuda(), v.cuda(), o_dev)
    oh = torch.empty(shape, dtype=torch.bfloat16)
    run = ug.HostRunner(plan, wl.batch, 3)
    run(q, k, v, oh)
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    assert torch.equal(oh.view(torch.int16), o_dev.cpu().view(torch.int16))


def test_host_runner_at_the_benchmarked_4k_configuration(ug):
    """The end-to-end figure's own call: the 4K layer in bf16 with the plan's automatic choice
    (compact halo blocks at 4K) and 2-head units, bit for bit the device path's output."""
    import torch
    wl = ug.WORKLOADS["4k"]
    plan = ug.plan_for(wl)
    assert plan.info["halo_copy"] > 0          # the automatic choice takes halo blocks here
    q, k, v = ug.make_qkv(wl)
    shape = (wl.batch, plan.info["N_raster"], wl.heads, wl.D)
    lay = ug.Layer(plan, wl.batch)
    o_dev = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    lay(q.cuda(), k.cuda(), v.cuda(), o_dev)
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.full(shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    run = ug.HostRunner(plan, wl.batch, 2)
    run(qh, kh, vh, oh)
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    assert torch.equal(oh.view(torch.int16), o_dev.cpu().view(torch.int16))
    run.close()
