"""Shared test helpers: the tolerance check and oracle runs on sampled rows/heads."""
import numpy as np

from oracle import hla_oracle as O

MAX_ABS = 2e-2      # attention output from bf16 inputs: max |gpu - oracle| over real rows
MEAN_REL = 5e-3     # sum |gpu - oracle| / sum |oracle| over the same elements


def to_np64(t):
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


def geometry(wl, lr_radius=-1, lr_block=False):
    return O.Geometry(wl.H, wl.W, wl.l, wl.b, wl.rho, wl.T, lr_radius, lr_block=lr_block)


def check_attention(got, ref, what=""):
    d = np.abs(got - ref)
    max_abs = float(d.max()) if d.size else 0.0
    mean_rel = float(d.sum() / max(np.abs(ref).sum(), 1e-30))
    assert max_abs <= MAX_ABS and mean_rel <= MEAN_REL, (
        f"{what}: max_abs {max_abs:.3e} (<= {MAX_ABS}), mean_rel {mean_rel:.3e} (<= {MEAN_REL})")
    return max_abs, mean_rel


def oracle_rows(q, k, v, wl, b, heads, rows, lr_radius=-1, lr_block=False, **fwd):
    """Oracle output [len(heads), len(rows), D] for batch b, the given heads and permuted rows
    (``fwd``: further options of the oracle's forward, e.g. the Q/K format)."""
    g = geometry(wl, lr_radius, lr_block)
    out = []
    for h in heads:
        qh = to_np64(q[b:b + 1, :, h:h + 1, :])
        kh = to_np64(k[b:b + 1, :, h:h + 1, :])
        vh = to_np64(v[b:b + 1, :, h:h + 1, :])
        o, _ = O.forward(qh, kh, vh, g, wl.axes, rows=rows, **fwd)
        out.append(o[0, 0])
    return np.stack(out)


def sample_rows(wl, n_text=512, n_lr=512, windows="all12"):
    """Permuted rows checked at full size: all text rows (up to n_text, evenly spaced beyond),
    every row of 12 windows (the 4 corners, the 4 edge middles, 4 interior windows at the
    quarter points; at a ragged right edge the corner and edge windows are the partial ones;
    windows="corners" keeps the corners and the centre), and n_lr evenly spaced LR rows."""
    g = geometry(wl)
    rows = list(np.linspace(0, max(0, g.T - 1), min(n_text, g.T)).astype(int)) if g.T else []
    l2 = g.l * g.l
    R, C = g.nWh - 1, g.nWw - 1
    cells = {(0, 0), (0, C), (R, 0), (R, C)}                     # corners
    if windows == "all12":
        cells |= {(0, C // 2), (R, C // 2), (R // 2, 0), (R // 2, C),   # edge middles
                  (R // 4, C // 4), (R // 4, 3 * C // 4), (3 * R // 4, C // 4), (3 * R // 4, 3 * C // 4)}
    else:
        cells |= {(R // 2, C // 2)}
    for (wr, wc) in sorted(cells):
        w = wr * g.nWw + wc
        rows += list(range(g.off_hr + w * l2, g.off_hr + (w + 1) * l2))
    if g.N_lr:
        rows += list(np.linspace(g.off_lr, g.off_lr + g.N_lr - 1, min(n_lr, g.N_lr)).astype(int))
    return np.array(sorted(set(int(r) for r in rows)), np.int64)
