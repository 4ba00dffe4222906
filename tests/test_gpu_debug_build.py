"""The debug build (ULTRAGEN_DEBUG) on the GPU: its kernels check every plan index and tile
coordinate against the table or tensor it indexes before using it.  On valid plans every
check passes: the debug library returns status 0 and the same output bits as the release
library, on layers that exercise the split merge, compact halo blocks, the raster epilogue,
ragged edge windows, head_dim 64 and the e4m3 Q/K format.  Each library runs in its own
process (ULTRAGEN_LIB_PATH selects it)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import dataclasses, hashlib, json, sys
sys.path.insert(0, ROOT)
import torch
import diffusion_transformer_ultra_b200 as ug
cases = [("1k", dict(), 5, None, "bf16"), ("ragged", dict(), None, None, "bf16"),
         ("1k", dict(name="odd", cfg=11, H=37, W=29, l=12, b=5, rho=3, T=70, heads=3, batch=2), 3, 1, "bf16"),
         ("1k", dict(name="small_l", cfg=12, H=20, W=18, l=4, b=3, rho=5, T=9, heads=2, D=64,
                     axes=(16, 24, 24), dtype="f32", sinusoid=False), None, None, "bf16"),
         ("1k", dict(heads=4), None, 1, "e4m3")]
out = []
for base, kw, split, halo, qk in cases:
    wl = dataclasses.replace(ug.WORKLOADS[base], **kw)
    plan = ug.plan_for(wl)
    if split is not None:
        plan.set_split(split)
    if halo is not None:
        plan.set_halo(halo)
    if qk != "bf16":
        plan.set_qk_format(qk)
    q, k, v = (t.cuda() for t in ug.make_qkv(wl))
    lay = ug.Layer(plan, wl.batch)
    o = torch.empty((wl.batch, plan.info["N_raster"], wl.heads, wl.D), dtype=torch.bfloat16, device="cuda")
    lay(q, k, v, o)                         # permute_rope + hla_forward_raster (+ merge)
    st = plan.sync_status()
    torch.cuda.synchronize()
    out.append([st, hashlib.sha256(o.view(torch.int16).cpu().numpy().tobytes()).hexdigest()])
print("RESULT " + json.dumps(out))
"""


def run_with(lib_path):
    env = dict(os.environ, ULTRAGEN_LIB_PATH=lib_path)
    r = subprocess.run([sys.executable, "-c", SCRIPT.replace("ROOT", repr(ROOT))], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


def test_debug_build_passes_its_checks_and_matches_release(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    release = build.build()
    debug = build.build(debug=True)
    rel = run_with(release)
    dbg = run_with(debug)
    assert all(st == 0 for st, _ in rel)
    assert all(st == 0 for st, _ in dbg), dbg
    assert [h for _, h in dbg] == [h for _, h in rel]
