"""UltraGen hierarchical local attention (HLA) hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libultragen.so`` (hand-written CUDA behind a C ABI, see
``include/ultragen.h``); this package holds its ctypes binding, the in-tree build script and
the seeded synthetic-input generator.
"""
from ._ffi import (BF16, F32, QK_BF16, QK_E4M3, HostRunner, Layer, Plan, UltragenError,  # noqa: F401
                   hla_forward,
                   hla_forward_noalloc, hla_forward_raster, lib, permute_rope,
                   unpermute, warm_start)
from .inputs import (WARM_WORKLOADS, WORKLOADS, WarmWorkload, Workload,  # noqa: F401
                     make_qkv, make_warm)


def plan_for(wl: "Workload") -> "Plan":
    """Plan for one of the named workloads (geometry, heads, head_dim and RoPE axes)."""
    p = Plan(wl.H, wl.W, wl.l, wl.b, wl.rho, wl.T, wl.heads, wl.D)
    p.set_rope(wl.axes)
    return p
