"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Bars: permutation and V gather bit-exact; Q/K after RoPE within 1 bf16 ulp of the oracle's
fp64 RoPE rounded to nearest-even, plus the fp32 rotation error bound (see FP32_ROT);
attention output within max-abs 2e-2 and mean-rel 5e-3
of the oracle on every real row (pad rows exactly 0).
"""
import dataclasses

import numpy as np
import pytest

from helpers import check_attention, geometry, oracle_rows, sample_rows, to_np64
from oracle import hla_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


def _wl(name, **kw):
    from diffusion_transformer_ultra_b200 import WORKLOADS
    return dataclasses.replace(WORKLOADS[name], **kw) if kw else WORKLOADS[name]


def run_layer(ug, wl, split=None, poison=True, lr_radius=-1, halo=None, lr_order=None):
    import torch
    plan = ug.plan_for(wl)
    if lr_radius != -1:
        plan.set_lr_scope(lr_radius)
    if lr_order is not None:
        plan.set_lr_order(lr_order)
    if halo is not None:
        plan.set_halo(halo)
    if split is not None:
        plan.set_split(split)
    q, k, v = ug.make_qkv(wl)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lay = ug.Layer(plan, wl.batch)
    if poison:
        for t in (lay.qp, lay.kp, lay.vp, lay.op):
            t.fill_(float("nan"))
    o = torch.full((wl.batch, plan.info["N_raster"], wl.heads, wl.D), float("nan"),
                   dtype=torch.bfloat16, device="cuda")
    lay(qd, kd, vd, o, fused=False)
    assert plan.sync_status() == 0
    torch.cuda.synchronize()
    return plan, (q, k, v), lay, o


# ------------------------------------------------------------------ permute / RoPE
CUSTOM = {
    "odd": dict(name="odd", cfg=11, H=37, W=29, l=12, b=5, rho=3, T=70, heads=3, D=128, batch=2),
    "small_l": dict(name="small_l", cfg=12, H=20, W=18, l=4, b=3, rho=5, T=9, heads=2, D=64,
                    batch=1, axes=(16, 24, 24), dtype="f32", sinusoid=False),
    "no_lr_text": dict(name="no_lr_text", cfg=13, H=40, W=24, l=8, b=8, rho=0, T=0, heads=2, D=128, batch=1),
    # ablation shapes of the pages: 512-px windows (l = 32) and rho = 2
    "win32_rho2": dict(name="win32_rho2", cfg=15, H=96, W=96, l=32, b=8, rho=2, T=64, heads=2, D=128, batch=1),
    "text_only_pad": dict(name="text_only_pad", cfg=14, H=16, W=16, l=16, b=0, rho=2, T=200, heads=2, D=64,
                          batch=1, axes=(8, 28, 28)),
    # degenerate cases: one HR token (and one LR token); a window larger than the image; rho
    # larger than the image; a 3-row strip whose text segment ends one past a tile boundary
    "single": dict(name="single", cfg=16, H=1, W=1, l=1, b=0, rho=1, T=0, heads=2, D=128, batch=1),
    "win_exceeds": dict(name="win_exceeds", cfg=17, H=5, W=7, l=16, b=3, rho=8, T=3, heads=2, D=64,
                        batch=2, axes=(16, 24, 24)),
    "rho_exceeds": dict(name="rho_exceeds", cfg=18, H=4, W=4, l=2, b=2, rho=8, T=1, heads=1, D=128, batch=1),
    "thin": dict(name="thin", cfg=19, H=3, W=130, l=4, b=1, rho=2, T=129, heads=2, D=128, batch=1),
    # halo tiles the attention gathers itself (whole windows, b * b a multiple of 8); border
    # windows take zero boxes for their pieces outside the image
    "l16_b8": dict(name="l16_b8", cfg=20, H=48, W=64, l=16, b=8, rho=4, T=20, heads=2, D=128, batch=2),
    "l32_b4": dict(name="l32_b4", cfg=21, H=64, W=96, l=32, b=4, rho=4, T=33, heads=2, D=64, batch=1,
                   axes=(16, 24, 24)),
    "l8_b4": dict(name="l8_b4", cfg=22, H=24, W=40, l=8, b=4, rho=2, T=5, heads=3, D=128, batch=1),
}


def custom(name):
    from diffusion_transformer_ultra_b200 import WORKLOADS
    return dataclasses.replace(WORKLOADS["1k"], **CUSTOM[name])


def expected_qkv_perm(wl, q, k, v, b, h, halo=False):
    """Oracle RoPE'd, permuted Q, K (rounded to bf16), V -- K and V in the K/V layout, with the
    halo blocks when the plan has them -- and the per-element pair magnitude |x_2k| + |x_2k+1|
    of the unrotated inputs in the same layouts."""
    g = dataclasses.replace(geometry(wl), halo_copy=halo)
    pos = O.positions(g)
    qh, kh, vh = (to_np64(x[b:b + 1, :, h:h + 1, :]) for x in (q, k, v))
    qp = O.permute(O.rope(qh, pos, wl.axes), g)[0, 0]
    kp = O.permute_kv(O.rope(kh, pos, wl.axes), g)[0, 0]
    vp = O.permute_kv(vh, g)[0, 0]

    def pair_mag(x, perm):
        xp = np.abs(perm(x, g)[0, 0])
        s = xp[:, 0::2] + xp[:, 1::2]
        return np.repeat(s, 2, axis=1)

    return (O.round_bf16(qp), O.round_bf16(kp), O.round_bf16(vp), pair_mag(qh, O.permute),
            pair_mag(kh, O.permute_kv))


# RoPE is evaluated in fp32 from fp32 cos/sin tables, then rounded to bf16 (nearest even).
# Against the fp64 rotation rounded to bf16, an element may differ by one bf16 ulp (the
# rounding of a value that moved across a tie) plus the fp32 evaluation error, which is
# bounded by 2^-22 * (|x_2k| + |x_2k+1|): table rounding of cos and sin (2^-24 each, relative)
# and at most two product/sum roundings.  The second term only matters where the rotation
# cancels to a value far below the pair's magnitude.
FP32_ROT = 2.0 ** -22


def ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (np.maximum(e, -126) - 7), 2.0 ** -133)


@pytest.mark.parametrize("name,halo", [("tiny", None), ("1k", None), ("ragged", None), ("odd", None),
                                       ("small_l", None), ("text_only_pad", None), ("single", None),
                                       ("win_exceeds", None), ("thin", None), ("1k", 1), ("odd", 1),
                                       ("thin", 1), ("1k", 2), ("l16_b8", 2), ("l32_b4", 2),
                                       ("l8_b4", 2)])
def test_permute_rope_parity(ug, name, halo):
    wl = _wl(name) if name in ("tiny", "1k", "ragged") else custom(name)
    plan, (q, k, v), lay, _ = run_layer(ug, wl, halo=halo)
    heads = range(wl.heads) if wl.heads <= 3 else (0, wl.heads // 2, wl.heads - 1)
    for b in range(wl.batch):
        for h in heads:
            # copied halo blocks (mode 1) are part of the K/V buffers; gathered ones (mode 2)
            # are not
            eq, ek, ev, mq, mk = expected_qkv_perm(wl, q, k, v, b, h, plan.info["halo_copy"] == 1)
            gq, gk, gv = (to_np64(t[b, h]) for t in (lay.qp, lay.kp, lay.vp))
            np.testing.assert_array_equal(gv, ev, err_msg="V gather must be bit-exact")
            for got, exp, mag, nm in ((gq, eq, mq, "Q"), (gk, ek, mk, "K")):
                tol = ulp_bf16(np.maximum(np.abs(got), np.abs(exp))) + FP32_ROT * mag
                bad = np.abs(got - exp) > tol
                assert not bad.any(), f"{nm} outside 1 ulp + fp32 bound at {np.argwhere(bad)[:5]}"
                # almost every element is within one plain ulp
                assert (np.abs(got - exp) > ulp_bf16(exp)).mean() < 1e-5
    # text tokens and axis-0 dims are copies
    g = geometry(wl)
    if g.T:
        src = q[0, :g.T].to("cuda").to(lay.qp.dtype)
        assert (lay.qp[0, :, :g.T].permute(1, 0, 2) == src).all()


@pytest.mark.parametrize("name", ["1k", "ragged"])
def test_unpermute_inverts_permute_bitwise(ug, name):
    import torch
    wl = _wl(name)
    plan, (q, k, v), lay, _ = run_layer(ug, wl)
    vd = v.cuda()
    vq = lay.vp[:, :, :plan.info["N_tot"]].contiguous()   # the window segment (Q layout)
    back = torch.empty_like(vd)
    ug.unpermute(vq, back, plan)
    back32 = torch.empty(vd.shape, dtype=torch.float32, device="cuda")
    ug.unpermute(vq, back32, plan)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), vd.view(torch.int16))
    assert torch.equal(back32, vd.float())


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("name,split,halo", [
    ("tiny", None, None), ("tiny", 0, None), ("tiny", 2, None), ("1k", None, None), ("1k", 0, None),
    ("1k", 5, None), ("odd", None, None), ("odd", 3, None), ("small_l", None, None),
    ("no_lr_text", None, None), ("win32_rho2", None, None), ("text_only_pad", 1, None),
    ("single", None, None), ("win_exceeds", None, None), ("rho_exceeds", None, None),
    ("thin", None, None), ("thin", 1, None),
    # compact halo blocks forced on (R18): the same attention
    ("tiny", None, 1), ("1k", None, 1), ("1k", 5, 1), ("odd", 3, 1), ("small_l", None, 1),
    ("win32_rho2", None, 1), ("win_exceeds", None, 1), ("thin", 1, 1),
    # and forced off where the automatic choice takes them
    ("win32_rho2", None, 0),
    # halo tiles gathered by the attention from the window segment (the automatic choice for
    # l = 16, b = 4), with split groups and border windows; copied and no blocks beside
    ("1k", 5, 2), ("l16_b8", None, 2), ("l16_b8", 3, 2), ("l32_b4", None, 2), ("l8_b4", None, 2),
    ("l16_b8", None, 1), ("1k", None, 0)])
def test_attention_full_parity(ug, name, split, halo):
    wl = _wl(name) if name in ("tiny", "1k") else custom(name)
    plan, (q, k, v), lay, o = run_layer(ug, wl, split=split, halo=halo)
    g = geometry(wl)
    perm = O.perm_map(g)
    rows = np.arange(g.N_tot)
    real = perm >= 0
    heads = range(wl.heads) if wl.heads <= 3 else (0, 7, wl.heads - 1)
    for b in range(wl.batch):
        ref = oracle_rows(q, k, v, wl, b, heads, rows)
        got = np.stack([to_np64(lay.op[b, h]) for h in heads])
        assert np.all(got[:, ~real] == 0), "pad rows must be 0"
        check_attention(got[:, real], ref[:, real], f"{name} split={split} b={b}")
    # the raster output is the unpermuted window-first output, bit for bit
    import torch
    assert not torch.isnan(o).any()
    for b in range(wl.batch):
        slot = O.slot_of_tokens(g)
        assert torch.equal(o[b].permute(1, 0, 2).view(torch.int16),
                           lay.op[b][:, torch.as_tensor(slot, device="cuda")].view(torch.int16))


# rows sampled per layer: the fp64 oracle is dense, so the 8K and 16K samples are smaller
SAMPLE = {"4k": {}, "ragged": {}, "8k": dict(n_text=128, n_lr=128),
          "16k": dict(n_text=64, n_lr=64, windows="corners")}


@pytest.mark.parametrize("name,heads", [("4k", (0, 12, 23)), ("ragged", (0, 12, 23)),
                                        ("8k", (23,)), ("16k", (1,))])
def test_attention_full_size_sampled(ug, name, heads):
    """Full-size layers in the configuration the benchmark runs, checked on sampled rows; the
    16K layer (the largest considered, 1024 x 1024 HR tokens) runs with 2 heads."""
    import torch
    wl = _wl(name, heads=2) if name == "16k" else _wl(name)
    plan, (q, k, v), lay, o = run_layer(ug, wl)
    assert not torch.isnan(lay.op).any()
    rows = sample_rows(wl, **SAMPLE[name])
    g = geometry(wl)
    real = O.perm_map(g)[rows] >= 0
    for b in range(wl.batch):
        ref = oracle_rows(q, k, v, wl, b, heads, rows)
        got = np.stack([to_np64(lay.op[b, h, torch.as_tensor(rows, device="cuda")]) for h in heads])
        assert np.all(got[:, ~real] == 0)
        check_attention(got[:, real], ref[:, real], f"{name} b={b}")


@pytest.mark.parametrize("name,heads,windows", [("4k", (0, 12, 23), "corners"),
                                                 ("8k", (0, 11, 23), "corners")])
def test_benchmarked_raster_call_at_full_size(ug, name, heads, windows):
    """The call bench.py times, in its own configuration: permute_rope + hla_forward_raster on
    the default plan (all LR tokens, compact halo blocks chosen automatically), checked on the
    raster output against the oracle for sampled rows of three heads, the corner (edge)
    windows and the centre window among them."""
    import torch
    wl = _wl(name)
    plan = ug.plan_for(wl)
    assert plan.info["halo_copy"] > 0
    q, k, v = ug.make_qkv(wl)
    lay = ug.Layer(plan, wl.batch)
    o = torch.full((wl.batch, plan.info["N_raster"], wl.heads, wl.D), float("nan"),
                   dtype=torch.bfloat16, device="cuda")
    ug.permute_rope(q.cuda(), k.cuda(), v.cuda(), lay.qp, lay.kp, lay.vp, plan)
    ug.hla_forward_raster(lay.qp, lay.kp, lay.vp, o, plan)
    assert plan.sync_status() == 0
    torch.cuda.synchronize()
    assert not torch.isnan(o).any()
    g = geometry(wl)
    rows = sample_rows(wl, n_text=128, n_lr=128, windows=windows)
    tok = O.perm_map(g)[rows]
    real = tok >= 0
    rows, tok = rows[real], tok[real]
    got_all = o[0][torch.as_tensor(tok, device="cuda")]            # [rows, heads, D]
    ref = oracle_rows(q, k, v, wl, 0, heads, rows)
    got = np.stack([to_np64(got_all[:, h]) for h in heads])
    check_attention(got, ref, f"{name} raster, heads {heads}")


@pytest.mark.parametrize("name,r,heads,order", [("1k", 4, (0, 11, 23), None), ("tiny", 0, (0,), None),
                                                ("4k", 4, (9,), None), ("8k", 0, (2,), None),
                                                ("1k", 4, (0, 23), 1), ("tiny", 0, (0,), 1),
                                                ("odd", 3, (0, 2), 1), ("4k", 4, (9,), 0)])
def test_attention_lr_region_parity(ug, name, r, heads, order):
    """The LR-region reading (HR queries see only the anchors of their window, grown by r), with
    the LR segment in the order the plan picks (4K, 8K: 8 x 16 blocks, R20) or the one forced."""
    import torch
    wl = _wl(name) if name in ("tiny", "1k", "4k", "8k") else custom(name)
    plan, (q, k, v), lay, o = run_layer(ug, wl, lr_radius=r, lr_order=order)
    assert plan.info["lr_radius"] == r
    lrb = bool(plan.info["lr_block"])
    if order is not None:
        assert lrb == bool(order)
    elif name in ("4k", "8k"):
        assert lrb                              # the automatic choice takes the blocks there
    assert not torch.isnan(lay.op).any()
    g = geometry(wl, r, lrb)
    rows = np.arange(g.N_tot) if name in ("1k", "tiny", "odd") else sample_rows(wl, n_text=128, n_lr=128)
    rows = rows[rows < g.N_tot]
    real = O.perm_map(g)[rows] >= 0
    ref = np.concatenate([oracle_rows(q, k, v, wl, b, heads, rows, lr_radius=r, lr_block=lrb)
                          for b in range(wl.batch)])
    got = np.concatenate([np.stack([to_np64(lay.op[b, h, torch.as_tensor(rows, device="cuda")])
                                    for h in heads]) for b in range(wl.batch)])
    assert np.all(got[:, ~real] == 0)
    check_attention(got[:, real], ref[:, real], f"{name} lr_radius={r} lr_block={lrb}")


@pytest.mark.parametrize("name,split,r", [("1k", None, -1), ("1k", 5, -1), ("ragged", None, -1),
                                          ("odd", 3, -1), ("tiny", 2, -1), ("4k", None, 4),
                                          ("text_only_pad", 1, -1)])
def test_fused_raster_equals_forward_then_unpermute(ug, name, split, r):
    """The unpermute folded into the attention epilogue gives the same bits as the two passes."""
    import torch
    wl = _wl(name) if name in ("tiny", "1k", "ragged", "4k") else custom(name)
    plan, (q, k, v), lay, o_two = run_layer(ug, wl, split=split, lr_radius=r)
    o_one = torch.full_like(o_two, float("nan"))
    if o_one.dtype != torch.bfloat16:
        o_one = torch.full(o_two.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ug.hla_forward_raster(lay.qp, lay.kp, lay.vp, o_one, plan)
    assert plan.sync_status() == 0
    torch.cuda.synchronize()
    assert torch.equal(o_one.view(torch.int16), o_two.to(torch.bfloat16).view(torch.int16))


def test_deterministic(ug):
    import torch
    wl = _wl("1k")
    _, _, lay1, o1 = run_layer(ug, wl)
    _, _, lay2, o2 = run_layer(ug, wl)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
