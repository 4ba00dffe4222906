"""The layer's launches can be captured in a CUDA graph and replayed (same bits as eager)."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


@pytest.mark.parametrize("name,split,qk", [("1k", None, "bf16"), ("1k", 5, "bf16"),
                                           ("ragged", None, "bf16"), ("1k", 5, "e4m3")])
def test_layer_replays_from_a_cuda_graph(ug, name, split, qk):
    import torch
    wl = ug.WORKLOADS[name]
    plan = ug.plan_for(wl)
    if split is not None:
        plan.set_split(split)
    plan.set_qk_format(qk)
    q, k, v = (x.cuda() for x in ug.make_qkv(wl))
    shape = (wl.batch, plan.info["N_raster"], wl.heads, wl.D)
    lay = ug.Layer(plan, wl.batch)
    o_eager = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        lay(q, k, v, o_eager)          # first call: uploads the plan's tables (not capturable)
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    o_graph = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        lay(q, k, v, o_graph)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert plan.sync_status() == 0
    assert torch.equal(o_graph.view(torch.int16), o_eager.view(torch.int16))
    del g
