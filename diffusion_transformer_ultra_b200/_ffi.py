"""ctypes binding of libultragen.so: argument marshalling only.

Every step of the hot path runs in the library's CUDA kernels; this module checks shapes,
dtypes and devices of torch tensors and passes raw pointers.  There is no fallback: if the
library is missing the import of any entry point raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# the in-tree library; ULTRAGEN_LIB_PATH selects another build of it (e.g. the debug build,
# libultragen_debug.so)
LIB_PATH = os.environ.get("ULTRAGEN_LIB_PATH") or os.path.join(_HERE, "libultragen.so")

OK = 0
STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
    4: "out of memory", 5: "device wait timed out", 6: "plan does not match the call",
    7: "no sm_100 device", 8: "index outside its table (debug build check)",
}
BF16, F32 = 0, 1
QK_BF16, QK_E4M3 = 0, 1          # storage of the permuted Q and K (Plan.set_qk_format)

# exported names of include/ultragen.h
SYMBOLS = (
    "ultragen_status_string", "ultragen_plan", "ultragen_plan_set_rope", "ultragen_plan_set_split",
    "ultragen_plan_info", "ultragen_plan_export", "ultragen_plan_export_rowmasks",
    "ultragen_plan_destroy", "ultragen_permute_rope", "ultragen_hla_forward",
    "ultragen_unpermute", "ultragen_sync_status", "ultragen_last_launch_count",
    "ultragen_hla_forward_noalloc", "ultragen_plan_set_diagnostics", "ultragen_plan_set_lr_scope",
    "ultragen_hla_forward_raster", "ultragen_warm_start", "ultragen_host_runner_create",
    "ultragen_host_runner_forward", "ultragen_host_runner_last_launch_count",
    "ultragen_host_runner_destroy", "ultragen_plan_set_halo", "ultragen_plan_export_kv",
    "ultragen_plan_set_qk_format", "ultragen_plan_set_lr_order",
    "ultragen_plan_set_clock_record", "ultragen_plan_read_clock",
    "ultragen_plan_export_halo_ops", "ultragen_plan_export_items",
)


class PlanInfo(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("l", ctypes.c_int32), ("b", ctypes.c_int32),
        ("rho", ctypes.c_int32), ("text_len", ctypes.c_int32), ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("nWh", ctypes.c_int32), ("nWw", ctypes.c_int32),
        ("h", ctypes.c_int32), ("w", ctypes.c_int32), ("N_raster", ctypes.c_int64),
        ("N_tot", ctypes.c_int64), ("off_hr", ctypes.c_int64), ("off_lr", ctypes.c_int64),
        ("n_qtiles", ctypes.c_int32), ("n_items", ctypes.c_int32), ("n_entries", ctypes.c_int64),
        ("n_partial", ctypes.c_int64), ("useful_pairs", ctypes.c_int64),
        ("rope_axes", ctypes.c_int32 * 3), ("rope_theta", ctypes.c_double),
        ("split_chunk", ctypes.c_int32), ("n_split_groups", ctypes.c_int32),
        ("n_split_items", ctypes.c_int32), ("workspace_bytes_per_head", ctypes.c_int64),
        ("lr_radius", ctypes.c_int32), ("halo_copy", ctypes.c_int32),
        ("halo_slots_per_window", ctypes.c_int32), ("N_kv", ctypes.c_int64),
        ("off_halo", ctypes.c_int64), ("qk_format", ctypes.c_int32), ("q_exp", ctypes.c_int32),
        ("k_exp", ctypes.c_int32), ("lr_block", ctypes.c_int32), ("kv_rows", ctypes.c_int64),
        ("n_halo_ops", ctypes.c_int32), ("n_long_items", ctypes.c_int32),
    ]

    def as_dict(self):
        d = {f: getattr(self, f) for f, _ in self._fields_}
        d["rope_axes"] = tuple(self.rope_axes)
        return d


class UltragenError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what} failed: {STATUS.get(status, status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m diffusion_transformer_ultra_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, cint = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int
    L.ultragen_status_string.restype = ctypes.c_char_p
    L.ultragen_status_string.argtypes = [cint]
    L.ultragen_plan.argtypes = [cint] * 8 + [ctypes.POINTER(vp)]
    L.ultragen_plan_set_rope.argtypes = [vp, cint, cint, cint, ctypes.c_double]
    L.ultragen_plan_set_split.argtypes = [vp, cint]
    L.ultragen_plan_set_lr_scope.argtypes = [vp, cint]
    L.ultragen_plan_set_halo.argtypes = [vp, cint]
    L.ultragen_plan_export_kv.argtypes = [vp, vp]
    L.ultragen_plan_export_halo_ops.argtypes = [vp, vp]
    L.ultragen_plan_export_items.argtypes = [vp, vp]
    L.ultragen_plan_set_qk_format.argtypes = [vp, cint, cint, cint]
    L.ultragen_plan_set_lr_order.argtypes = [vp, cint]
    L.ultragen_plan_set_clock_record.argtypes = [vp, cint]
    L.ultragen_plan_read_clock.argtypes = [vp, vp]
    L.ultragen_plan_info.argtypes = [vp, ctypes.POINTER(PlanInfo)]
    L.ultragen_plan_export.argtypes = [vp, vp, vp, vp]
    L.ultragen_plan_export_rowmasks.argtypes = [vp, cint, vp]
    L.ultragen_plan_destroy.argtypes = [vp]
    L.ultragen_permute_rope.argtypes = [vp, vp, vp, cint, vp, vp, vp, cint, vp, vp]
    L.ultragen_hla_forward.argtypes = [vp, vp, vp, vp, vp, cint, vp]
    L.ultragen_hla_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, cint, vp]
    L.ultragen_hla_forward_raster.argtypes = [vp, vp, vp, vp, vp, cint, vp]
    L.ultragen_unpermute.argtypes = [vp, vp, cint, cint, vp, vp]
    L.ultragen_sync_status.argtypes = [vp, vp]
    L.ultragen_last_launch_count.argtypes = [vp]
    L.ultragen_plan_set_diagnostics.argtypes = [vp, cint, ctypes.c_double]
    L.ultragen_warm_start.argtypes = [vp, vp, vp] + [cint] * 6 + [ctypes.c_float] * 2 + \
        [ctypes.c_uint64] * 2 + [vp]
    L.ultragen_host_runner_create.argtypes = [vp, cint, cint, ctypes.POINTER(vp)]
    L.ultragen_host_runner_forward.argtypes = [vp, vp, vp, vp, vp, vp]
    L.ultragen_host_runner_last_launch_count.argtypes = [vp]
    L.ultragen_host_runner_destroy.argtypes = [vp]
    for name in SYMBOLS:
        if name != "ultragen_status_string":
            getattr(L, name).restype = cint
    _lib = L
    return L


def _check(what: str, st: int):
    if st != OK:
        raise UltragenError(what, st)


class Plan:
    """Owner of one ultragen_plan_t."""

    def __init__(self, H, W, l, b, rho, text_len, heads, head_dim):
        self._h = ctypes.c_void_p()
        _check("ultragen_plan", lib().ultragen_plan(H, W, l, b, rho, text_len, heads, head_dim,
                                                    ctypes.byref(self._h)))
        self._refresh()

    def _refresh(self):
        info = PlanInfo()
        _check("ultragen_plan_info", lib().ultragen_plan_info(self._h, ctypes.byref(info)))
        self.info = info.as_dict()

    @property
    def handle(self):
        return self._h

    def set_rope(self, axes, theta=1.0e4):
        _check("ultragen_plan_set_rope", lib().ultragen_plan_set_rope(self._h, *axes, float(theta)))
        self._refresh()

    def set_split(self, chunk: int):
        _check("ultragen_plan_set_split", lib().ultragen_plan_set_split(self._h, int(chunk)))
        self._refresh()

    def set_lr_scope(self, radius: int):
        _check("ultragen_plan_set_lr_scope", lib().ultragen_plan_set_lr_scope(self._h, int(radius)))
        self._refresh()

    def set_lr_order(self, mode: int):
        """LR segment order: 1 blocks of 8 x 16 LR tokens, 0 raster, -1 automatic (the
        default; blocks only with an LR-region scope, when they give fewer tile entries)."""
        _check("ultragen_plan_set_lr_order", lib().ultragen_plan_set_lr_order(self._h, int(mode)))
        self._refresh()

    def set_halo(self, mode: int):
        """Compact halo blocks in the K/V layout: 1 on, 0 off, -1 automatic (the default)."""
        _check("ultragen_plan_set_halo", lib().ultragen_plan_set_halo(self._h, int(mode)))
        self._refresh()

    def set_qk_format(self, fmt, q_exp: int = 0, k_exp: int = 0):
        """Storage of the permuted Q and K: "bf16" (the default) or "e4m3" -- Q and K as e4m3
        bytes of x * 2^-q_exp and x * 2^-k_exp, multiplied by 8-bit tensor-core products."""
        code = {"bf16": QK_BF16, "e4m3": QK_E4M3}.get(fmt, fmt)
        _check("ultragen_plan_set_qk_format",
               lib().ultragen_plan_set_qk_format(self._h, int(code), int(q_exp), int(k_exp)))
        self._refresh()

    def qk_dtypes(self):
        """Tensor dtypes accepted for the permuted Q and K under the plan's Q/K format."""
        import torch
        if self.info["qk_format"] == QK_E4M3:
            return (torch.float8_e4m3fn, torch.uint8)
        return (torch.bfloat16,)

    def export_kv(self):
        kv = np.empty(self.info["N_kv"], np.int32)
        _check("ultragen_plan_export_kv", lib().ultragen_plan_export_kv(self._h, kv.ctypes.data))
        return kv

    def export_items(self):
        """The work items of one (batch, head): [n_items, 8] int32 (qt0, qt1, e0, e1, split
        slot, row classes, first window, 0)."""
        items = np.zeros((max(1, self.info["n_items"]), 8), np.int32)
        _check("ultragen_plan_export_items", lib().ultragen_plan_export_items(self._h, items.ctypes.data))
        return items[:self.info["n_items"]]

    def export_halo_ops(self):
        ops = np.zeros(max(1, self.info["n_halo_ops"]), np.int32)
        _check("ultragen_plan_export_halo_ops",
               lib().ultragen_plan_export_halo_ops(self._h, ops.ctypes.data))
        return ops[:self.info["n_halo_ops"]]

    def export(self):
        i = self.info
        perm = np.empty(i["N_tot"], np.int32)
        row_ptr = np.empty(i["n_qtiles"] + 1, np.int32)
        entries = np.empty(max(1, i["n_entries"]), np.int32)
        _check("ultragen_plan_export", lib().ultragen_plan_export(
            self._h, perm.ctypes.data, row_ptr.ctypes.data, entries.ctypes.data))
        return perm, row_ptr, entries[:i["n_entries"]]

    def rowmasks(self, qtile: int, n_entries: int):
        out = np.empty((max(1, n_entries), 128, 4), np.uint32)
        _check("ultragen_plan_export_rowmasks",
               lib().ultragen_plan_export_rowmasks(self._h, int(qtile), out.ctypes.data))
        return out[:n_entries]

    def set_diagnostics(self, fault: int = 0, wait_limit_s: float = 2.0):
        _check("ultragen_plan_set_diagnostics",
               lib().ultragen_plan_set_diagnostics(self._h, int(fault), float(wait_limit_s)))

    def set_clock_record(self, on: bool = True):
        _check("ultragen_plan_set_clock_record",
               lib().ultragen_plan_set_clock_record(self._h, 1 if on else 0))

    def read_clock(self) -> dict:
        """The attention launches' clock record since the last read: launches, SM cycles and
        nanoseconds of the first CTA summed, and their ratio in MHz (then cleared)."""
        out = (ctypes.c_uint64 * 3)()
        _check("ultragen_plan_read_clock", lib().ultragen_plan_read_clock(self._h, out))
        n, cyc, ns = int(out[0]), int(out[1]), int(out[2])
        return {"launches": n, "cycles": cyc, "ns": ns,
                "sm_mhz": (1e3 * cyc / ns) if ns else None}

    def sync_status(self, stream=None) -> int:
        return lib().ultragen_sync_status(self._h, _stream_ptr(stream))

    def last_launch_count(self) -> int:
        return lib().ultragen_last_launch_count(self._h)

    def close(self):
        if self._h:
            lib().ultragen_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, shape, dtypes, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def permute_rope(q, k, v, qp, kp, vp, plan: Plan, stream=None):
    """Raster Q/K/V [B, N_raster, H, D] -> window-first [B, H, N_tot, D] bf16 with RoPE on Q, K."""
    import torch
    i = plan.info
    B = q.shape[0]
    raster = (B, i["N_raster"], i["heads"], i["head_dim"])
    q_shape = (B, i["heads"], i["N_tot"], i["head_dim"])
    kv_shape = (B, i["heads"], i["kv_rows"], i["head_dim"])
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, raster, (torch.bfloat16, torch.float32), n)
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share a dtype")
    _need(qp, q_shape, plan.qk_dtypes(), "qp")
    _need(kp, kv_shape, plan.qk_dtypes(), "kp")
    _need(vp, kv_shape, (torch.bfloat16,), "vp")
    dt = BF16 if q.dtype == torch.bfloat16 else F32
    _check("ultragen_permute_rope", lib().ultragen_permute_rope(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dt, qp.data_ptr(), kp.data_ptr(), vp.data_ptr(),
        B, plan.handle, _stream_ptr(stream)))


def hla_forward(qp, kp, vp, op, plan: Plan, stream=None):
    """Block-sparse masked attention over the window-first layout."""
    import torch
    i = plan.info
    B = qp.shape[0]
    shape = (B, i["heads"], i["N_tot"], i["head_dim"])
    kv_shape = (B, i["heads"], i["kv_rows"], i["head_dim"])
    _need(qp, shape, plan.qk_dtypes(), "qp")
    _need(op, shape, (torch.bfloat16,), "op")
    _need(kp, kv_shape, plan.qk_dtypes(), "kp")
    _need(vp, kv_shape, (torch.bfloat16,), "vp")
    _check("ultragen_hla_forward", lib().ultragen_hla_forward(
        qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(), plan.handle, B,
        _stream_ptr(stream)))


def hla_forward_raster(qp, kp, vp, o, plan: Plan, stream=None):
    """hla_forward writing O straight to the raster layout [B, N_raster, H, D] (bf16)."""
    import torch
    i = plan.info
    B = qp.shape[0]
    _need(qp, (B, i["heads"], i["N_tot"], i["head_dim"]), plan.qk_dtypes(), "qp")
    _need(kp, (B, i["heads"], i["kv_rows"], i["head_dim"]), plan.qk_dtypes(), "kp")
    _need(vp, (B, i["heads"], i["kv_rows"], i["head_dim"]), (torch.bfloat16,), "vp")
    _need(o, (B, i["N_raster"], i["heads"], i["head_dim"]), (torch.bfloat16,), "o")
    _check("ultragen_hla_forward_raster", lib().ultragen_hla_forward_raster(
        qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), o.data_ptr(), plan.handle, B,
        _stream_ptr(stream)))


def hla_forward_noalloc(qp, kp, vp, op, plan: Plan, stream=None):
    """hla_forward without any device allocation: split partials go to the library's fixed
    scratch array.  The plan's tables must already be on the device (any earlier device call
    with this plan uploads them)."""
    import torch
    i = plan.info
    B = qp.shape[0]
    shape = (B, i["heads"], i["N_tot"], i["head_dim"])
    kv_shape = (B, i["heads"], i["kv_rows"], i["head_dim"])
    _need(qp, shape, plan.qk_dtypes(), "qp")
    _need(op, shape, (torch.bfloat16,), "op")
    _need(kp, kv_shape, plan.qk_dtypes(), "kp")
    _need(vp, kv_shape, (torch.bfloat16,), "vp")
    _check("ultragen_hla_forward_noalloc", lib().ultragen_hla_forward_noalloc(
        qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(), plan.handle, B,
        _stream_ptr(stream)))


def unpermute(op, o, plan: Plan, stream=None):
    """Window-first [B, H, N_tot, D] bf16 -> raster [B, N_raster, H, D] (bf16 or fp32)."""
    import torch
    i = plan.info
    B = op.shape[0]
    _need(op, (B, i["heads"], i["N_tot"], i["head_dim"]), (torch.bfloat16,), "op")
    _need(o, (B, i["N_raster"], i["heads"], i["head_dim"]), (torch.bfloat16, torch.float32), "o")
    dt = BF16 if o.dtype == torch.bfloat16 else F32
    _check("ultragen_unpermute", lib().ultragen_unpermute(
        op.data_ptr(), o.data_ptr(), dt, B, plan.handle, _stream_ptr(stream)))


def warm_start(x_lr, x_hr, alpha: float, sharpen: float = 1.0, noise=None, seed: int = 0,
               offset: int = 0, stream=None):
    """Warm-start latent x_hr [B, C, H, W] = alpha * X_T + (1 - alpha) * sharpen(upsample(x_lr))
    (fp32).  X_T is `noise` [B, C, H, W], or the Philox/Box-Muller stream (seed, offset) drawn
    in the kernel when noise is None."""
    import torch
    if x_lr.dim() != 4 or x_hr.dim() != 4:
        raise ValueError("x_lr and x_hr must be [B, C, h, w] and [B, C, H, W]")
    B, C, h, w = x_lr.shape
    H, W = x_hr.shape[2:]
    _need(x_lr, (B, C, h, w), (torch.float32,), "x_lr")
    _need(x_hr, (B, C, H, W), (torch.float32,), "x_hr")
    if noise is not None:
        _need(noise, (B, C, H, W), (torch.float32,), "noise")
    _check("ultragen_warm_start", lib().ultragen_warm_start(
        x_lr.data_ptr(), None if noise is None else noise.data_ptr(), x_hr.data_ptr(), B, C, h, w,
        H, W, float(alpha), float(sharpen), int(seed), int(offset), _stream_ptr(stream)))
    return x_hr


class HostRunner:
    """The whole layer for Q/K/V and O in host memory, PCIe copies overlapped with the kernels
    (units of heads_per_chunk heads; see ultragen_host_runner_create)."""

    def __init__(self, plan: Plan, batch: int, heads_per_chunk: int = 2):
        self.plan = plan
        self.batch = batch
        self._h = ctypes.c_void_p()
        _check("ultragen_host_runner_create", lib().ultragen_host_runner_create(
            plan.handle, int(batch), int(heads_per_chunk), ctypes.byref(self._h)))

    def __call__(self, q, k, v, o, stream=None):
        """q, k, v, o: CPU bf16 [batch, N_raster, heads, D] (page-locked for overlap)."""
        import torch
        i = self.plan.info
        shape = (self.batch, i["N_raster"], i["heads"], i["head_dim"])
        for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
            if not isinstance(t, torch.Tensor) or t.is_cuda:
                raise ValueError(f"{n} must be a host tensor")
            if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or not t.is_contiguous():
                raise ValueError(f"{n} must be contiguous bf16 {shape}")
        _check("ultragen_host_runner_forward", lib().ultragen_host_runner_forward(
            self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _stream_ptr(stream)))
        return o

    def last_launch_count(self) -> int:
        return lib().ultragen_host_runner_last_launch_count(self._h)

    def close(self):
        if self._h:
            lib().ultragen_host_runner_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Layer:
    """The whole path for one shape: permute_rope -> hla_forward -> unpermute, with the
    permuted buffers kept resident between calls."""

    def __init__(self, plan: Plan, batch: int, device="cuda"):
        import torch
        i = plan.info
        self.plan = plan
        shape = (batch, i["heads"], i["N_tot"], i["head_dim"])
        kv_shape = (batch, i["heads"], i["kv_rows"], i["head_dim"])
        qk = plan.qk_dtypes()[0]
        self.qp = torch.empty(shape, dtype=qk, device=device)
        self.op = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.kp = torch.empty(kv_shape, dtype=qk, device=device)
        self.vp = torch.empty(kv_shape, dtype=torch.bfloat16, device=device)

    def __call__(self, q, k, v, o, stream=None, fused=None):
        """o: raster [B, N_raster, H, D].  With a bf16 o the unpermute runs inside the
        attention epilogue (fused=None or True); fused=False, or an fp32 o, keeps the three
        separate passes (the permuted output stays in self.op)."""
        import torch
        permute_rope(q, k, v, self.qp, self.kp, self.vp, self.plan, stream)
        if fused is None:
            fused = o.dtype == torch.bfloat16
        if fused:
            hla_forward_raster(self.qp, self.kp, self.vp, o, self.plan, stream)
        else:
            hla_forward(self.qp, self.kp, self.vp, self.op, self.plan, stream)
            unpermute(self.op, o, self.plan, stream)
        return o
