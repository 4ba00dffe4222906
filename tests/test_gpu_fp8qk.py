"""GPU parity of the 8-bit Q K^T format (Q and K stored as scaled e4m3 after RoPE) against the
oracle's reading of it, through the C ABI.

Stored bytes: each permuted Q / K byte is the e4m3 rounding of the RoPE'd value times 2^-exp.
The kernel evaluates RoPE in fp32 (error at most 2^-22 (|x_2k| + |x_2k+1|), see the bf16
permute test) and the oracle in fp64, so a value that lies within that error of a rounding
midpoint may round the other way: there the kernel's value must be the rounding of some point
inside the error interval; everywhere else the values are equal.  V is bit-exact.

Attention: the kernel against the oracle's forward with the same quantization (the logits of
the stored values times 2^(q_exp + k_exp)), to the tolerance of the bf16 path (max-abs 2e-2,
mean-rel 5e-3).  The distance to the unquantized oracle is larger (e4m3 keeps 3 mantissa
bits); a test checks that the kernel is much closer to the quantized reading than to it.
"""
import dataclasses

import numpy as np
import pytest

from helpers import check_attention, geometry, oracle_rows, sample_rows, to_np64
from oracle import hla_oracle as O
from test_gpu_parity import CUSTOM, FP32_ROT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


def _wl(name, **kw):
    from diffusion_transformer_ultra_b200 import WORKLOADS
    if name in CUSTOM:
        return dataclasses.replace(WORKLOADS["1k"], **CUSTOM[name])
    return dataclasses.replace(WORKLOADS[name], **kw) if kw else WORKLOADS[name]


def run_fp8(ug, wl, split=None, halo=None, q_exp=0, k_exp=0, qs=0, ks=0, fused=False):
    """The layer with e4m3 Q/K on inputs whose Q, K are scaled by 2^qs, 2^ks (exact in bf16)."""
    import torch
    plan = ug.plan_for(wl)
    if halo is not None:
        plan.set_halo(halo)
    if split is not None:
        plan.set_split(split)
    plan.set_qk_format("e4m3", q_exp, k_exp)
    q, k, v = ug.make_qkv(wl)
    q, k = q * 2.0 ** qs, k * 2.0 ** ks
    lay = ug.Layer(plan, wl.batch)
    assert lay.qp.dtype == torch.float8_e4m3fn and lay.kp.dtype == torch.float8_e4m3fn
    lay.qp.view(torch.uint8).fill_(0x7F)          # NaN bytes: every slot must be written
    lay.kp.view(torch.uint8).fill_(0x7F)
    lay.vp.fill_(float("nan"))
    lay.op.fill_(float("nan"))
    o = torch.full((wl.batch, plan.info["N_raster"], wl.heads, wl.D), float("nan"),
                   dtype=torch.bfloat16, device="cuda")
    lay(q.cuda(), k.cuda(), v.cuda(), o, fused=fused)
    assert plan.sync_status() == 0
    torch.cuda.synchronize()
    return plan, (q, k, v), lay, o


def check_stored(got, x, mag, exp, what):
    """got: the kernel's stored values (decoded, times 2^exp); x: oracle fp64 RoPE values;
    mag: |x_2k| + |x_2k+1| of the unrotated inputs, in the same layout."""
    exact = O.quantize_e4m3(x, exp)
    diff = got != exact
    if diff.any():
        d = FP32_ROT * mag[diff]
        lo = O.quantize_e4m3(x[diff] - d, exp)
        hi = O.quantize_e4m3(x[diff] + d, exp)
        ok = (got[diff] == lo) | (got[diff] == hi)
        assert ok.all(), f"{what}: {np.count_nonzero(~ok)} bytes are not a rounding of the RoPE value"
    assert diff.mean() < 1e-4, f"{what}: {diff.mean():.2e} of the bytes sit on the other side of a tie"


def expected_fp8_inputs(wl, q, k, v, b, h, halo):
    g = dataclasses.replace(geometry(wl), halo_copy=halo)
    pos = O.positions(g)
    qh, kh, vh = (to_np64(x[b:b + 1, :, h:h + 1, :]) for x in (q, k, v))

    def mag(x, perm):
        xp = np.abs(perm(x, g)[0, 0])
        return np.repeat(xp[:, 0::2] + xp[:, 1::2], 2, axis=1)

    return (O.permute(O.rope(qh, pos, wl.axes), g)[0, 0], mag(qh, O.permute),
            O.permute_kv(O.rope(kh, pos, wl.axes), g)[0, 0], mag(kh, O.permute_kv),
            O.round_bf16(O.permute_kv(vh, g)[0, 0]))


@pytest.mark.parametrize("name,halo,q_exp,k_exp", [("1k", None, 0, 0), ("1k", 1, -2, 3), ("1k", 2, 1, 0),
                                                   ("odd", 1, 1, 0), ("thin", None, 0, -1),
                                                   ("win32_rho2", None, 0, 0)])
def test_permute_stores_e4m3_codes(ug, name, halo, q_exp, k_exp):
    import torch
    wl = _wl(name)
    plan, (q, k, v), lay, _ = run_fp8(ug, wl, halo=halo, q_exp=q_exp, k_exp=k_exp)
    heads = range(wl.heads) if wl.heads <= 3 else (0, wl.heads // 2, wl.heads - 1)
    for b in range(wl.batch):
        for h in heads:
            xq, mq, xk, mk, ev = expected_fp8_inputs(wl, q, k, v, b, h, plan.info["halo_copy"] == 1)
            gq = lay.qp[b, h].to(torch.float64).cpu().numpy() * 2.0 ** q_exp
            gk = lay.kp[b, h].to(torch.float64).cpu().numpy() * 2.0 ** k_exp
            check_stored(gq, xq, mq, q_exp, f"{name} Q b={b} h={h}")
            check_stored(gk, xk, mk, k_exp, f"{name} K b={b} h={h}")
            np.testing.assert_array_equal(to_np64(lay.vp[b, h]), ev, err_msg="V must be bit-exact")


@pytest.mark.parametrize("name,split,halo,q_exp,k_exp", [
    ("1k", None, None, 0, 0), ("1k", 0, None, 0, 0), ("1k", 5, None, 0, 0), ("1k", None, 1, 0, 0),
    ("1k", 5, 1, 1, -1), ("odd", 3, 1, 1, 1), ("odd", None, 0, 0, 0), ("no_lr_text", None, None, 0, 0),
    ("win32_rho2", None, None, 0, 0), ("single", None, None, 0, 0), ("rho_exceeds", None, None, 0, 0),
    ("thin", 1, 1, 0, 0)])
def test_attention_fp8_parity(ug, name, split, halo, q_exp, k_exp):
    import torch
    wl = _wl(name)
    plan, (q, k, v), lay, o = run_fp8(ug, wl, split=split, halo=halo, q_exp=q_exp, k_exp=k_exp)
    g = geometry(wl)
    real = O.perm_map(g) >= 0
    rows = np.arange(g.N_tot)
    heads = range(wl.heads) if wl.heads <= 3 else (0, 7, wl.heads - 1)
    for b in range(wl.batch):
        ref = oracle_rows(q, k, v, wl, b, heads, rows, qk_format="e4m3", q_exp=q_exp, k_exp=k_exp)
        got = np.stack([to_np64(lay.op[b, h]) for h in heads])
        assert np.all(got[:, ~real] == 0), "pad rows must be 0"
        check_attention(got[:, real], ref[:, real], f"{name} e4m3 split={split} b={b}")
    # the unpermuted output, and the fused raster epilogue, equal the window-first output
    slot = torch.as_tensor(O.slot_of_tokens(g), device="cuda")
    o2 = torch.full_like(o, float("nan"))
    ug.hla_forward_raster(lay.qp, lay.kp, lay.vp, o2, plan)
    torch.cuda.synchronize()
    for b in range(wl.batch):
        want = lay.op[b][:, slot].view(torch.int16)
        assert torch.equal(o[b].permute(1, 0, 2).view(torch.int16), want)
        assert torch.equal(o2[b].permute(1, 0, 2).view(torch.int16), want)


def test_quantized_path_is_closer_to_its_reading_than_to_exact_attention(ug):
    wl = _wl("1k")
    plan, (q, k, v), lay, _ = run_fp8(ug, wl)
    g = geometry(wl)
    real = O.perm_map(g) >= 0
    rows = np.arange(g.N_tot)
    heads = (0, 11, 23)
    got = np.stack([to_np64(lay.op[0, h]) for h in heads])[:, real]
    ref8 = oracle_rows(q, k, v, wl, 0, heads, rows, qk_format="e4m3")[:, real]
    ref = oracle_rows(q, k, v, wl, 0, heads, rows)[:, real]
    rel8 = np.abs(got - ref8).sum() / np.abs(ref8).sum()
    rel = np.abs(got - ref).sum() / np.abs(ref).sum()
    assert rel8 < 0.3 * rel, (rel8, rel)


def test_moving_powers_of_two_between_inputs_and_exponents_is_bitwise_neutral(ug):
    """Q x 4 with q_exp = 2 and K / 4 with k_exp = -2 store the same bytes and scale the
    logits by 2^0: the output is bit-identical to the unscaled run."""
    import torch
    wl = _wl("odd")
    _, _, lay0, o0 = run_fp8(ug, wl, halo=1)
    _, _, lay1, o1 = run_fp8(ug, wl, halo=1, q_exp=2, k_exp=-2, qs=2, ks=-2)
    assert torch.equal(lay0.qp.view(torch.uint8), lay1.qp.view(torch.uint8))
    assert torch.equal(lay0.kp.view(torch.uint8), lay1.kp.view(torch.uint8))
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))


@pytest.mark.parametrize("name,heads", [("4k", (0, 12, 23)), ("8k", (23,))])
def test_attention_fp8_full_size_sampled(ug, name, heads):
    """The full-size layers in the benchmark's configuration (automatic halo blocks)."""
    wl = _wl(name)
    plan, (q, k, v), lay, o = run_fp8(ug, wl, fused=True)
    kw = {} if name == "4k" else dict(n_text=128, n_lr=128)
    rows = sample_rows(wl, **kw)
    g = geometry(wl)
    slots = O.slot_of_tokens(g)
    perm = O.perm_map(g)
    real = perm[rows] >= 0
    ref = oracle_rows(q, k, v, wl, 0, heads, rows, qk_format="e4m3")
    tok = perm[rows[real]]
    got = np.stack([to_np64(o[0, :, h][tok]) for h in heads])
    check_attention(got, ref[:, real], f"{name} e4m3 sampled")
    assert (slots[tok] == rows[real]).all()


def test_host_runner_and_noalloc_follow_the_format(ug):
    import torch
    wl = _wl("1k", batch=2)
    plan, (q, k, v), lay, o = run_fp8(ug, wl, split=5, halo=1, q_exp=1, k_exp=0, fused=True)
    r = ug.HostRunner(plan, wl.batch, heads_per_chunk=5)
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.full(o.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    r(qh, kh, vh, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh.view(torch.int16), o.cpu().view(torch.int16))
    # the no-allocation call's fixed scratch holds this layer's partials with chunks of 12
    plan.set_split(12)
    assert wl.batch * wl.heads * plan.info["workspace_bytes_per_head"] <= 64 << 20
    op2 = torch.full_like(lay.op, float("nan"))
    ug.hla_forward(lay.qp, lay.kp, lay.vp, lay.op, plan)     # uploads the rebuilt tables
    ug.hla_forward_noalloc(lay.qp, lay.kp, lay.vp, op2, plan)
    torch.cuda.synchronize()
    assert torch.equal(op2.view(torch.int16), lay.op.view(torch.int16))
    r.close()
