"""Oracle for UltraGen's hierarchical local attention (HLA). TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct fp64 NumPy restatement of what the hot path computes.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline leg and its
reference arm) may import or run this module.  It shares no code, table or helper with the
CUDA library, and it imports nothing from the product package.

Sources (page title, then the section on the page):
  [UG-note]  "UltraGen: Efficient Ultra-High-Resolution Image Generation with Hierarchical
             Local Attention" -- papernotes.org note (ECCV 2026), section 方法详解 / 关键设计 1-3
             and the MMA equation under 关键设计 3.
  [UG-gist]  same title -- gist.science English summary of arXiv 2510.16325, section
             "2. Methodology", parts A (window-first permutation) and B (low-resolution
             global guidance, "Attention Masking").

What each function follows:
  * geometry / window partition ............ [UG-note] 关键设计 1; [UG-gist] 2.A
  * window-first permutation ............... [UG-note] 关键设计 1 (window-first token order)
  * LR position scaling (m,n)->(rho m,rho n) [UG-note] 关键设计 2, the scaling equation
  * sequence order [C_T; X; X_lr] .......... [UG-note] 关键设计 3
  * visibility (mask M) .................... [UG-note] 关键设计 2 (last paragraph);
                                             [UG-gist] 2.B "Attention Masking"
  * masked softmax attention ............... [UG-note] 关键设计 3, the MMA equation
  * 2D RoPE on Q/K ......................... implied by [UG-note] 关键设计 1 and 3 ("RoPE"),
                                             convention fixed by the readings below

Tables returned by the cached geometry helpers (raster_tokens, slot_of_tokens, perm_map,
slot_info) are shared between calls: callers must not modify them.

Readings taken where the pages are silent or garbled:
  R1  l counts latent tokens (l=16 <-> 256x256 pixels at a 16x VAE).
  R2  Halo: the query's own window box grown by b tokens on every side, clipped to the
      image; every query of a window sees the same set.  0 <= b <= l.
  R3  HR queries see ALL low-resolution tokens (lr_radius = -1, the default).  The variant
      lr_radius = r >= 0 follows the other reading of the pages (the "corresponding" LR
      anchors, [UG-note] 关键设计 2 and the German summary's "entsprechenden skalierten
      Regionen"): an HR query of window (wr, wc) sees LR token (m, n) iff its scaled position
      (rho m, rho n) lies in the window's l x l box grown by r tokens on every side.
  R4  LR queries see LR and text.  R5 text queries see text and HR, not LR.
  R6  The "* M" inside the softmax is read as an additive -inf on masked pairs; the
      scale is 1/sqrt(head_dim).
  R7  RoPE: interleaved pairs (2k, 2k+1); dims split into axes (a0, a1, a2) laid out
      consecutively; pair k of an axis of width d rotates by pos * theta**(-2k/d);
      theta = 1e4; axis 0 position is always 0; text tokens sit at (0, 0, 0).
  R8  Sequence layout [text | pad | HR window-first | pad | LR | pad], every segment
      starting on a multiple of 128; partial edge windows keep l*l slots: their tokens first,
      in raster order of the window's part inside the image, then pad slots.
  R9  H counts rows (axis 1 <- row i), W counts columns (axis 2 <- column j).
  R13 Windows in row-major order; raster order inside a window (of its part inside the
      image, for a partial edge window: rows of min(l, W - wc*l) tokens).
  R15 Pad slots are not tokens: never visible as keys; pad query rows output 0; tile lists
      are derived from the mask rows of real tokens only.
  R18 Optional compact halo blocks (halo_copy): the K/V layout appends, per window w, a block
      of G slots holding w's halo tokens -- the HR tokens of its grown box outside the window.
      The block is eight pieces, in this order: the top and bottom strips (b rows x l
      columns, in the window's columns), the left and right strips (l rows x b columns, in the
      window's rows), and the top-left, top-right, bottom-left and bottom-right corners (b x b);
      each piece is in raster order of its rectangle, starts on a multiple of 8 slots, and a
      piece of at most 128 slots does not cross a multiple of 128 (a longer one starts on
      one).  A piece position outside the image is a pad slot, so every window's block has the
      same shape; G is its length padded to 128.  (A strip of a window is then a box of the
      window-first layout, which a tile copy can fetch.)  An HR query of window w takes the
      other windows' tokens of its box from w's block instead of their window segments; halo
      blocks are visible to nothing else.  Every query sees the same tokens as without them,
      so the attention output is the same function.
  R20 Optional block order of the LR segment (lr_block; a layout choice for the LR-region
      reading of R3): LR token (m, n) takes slot off_lr + ((m // 8) * nbw + n // 16) * 128 +
      (m % 8) * 16 + n % 16, nbw = ceil(w / 16), so every 128-slot tile holds one 8 x 16 block
      of the LR grid (partial blocks at the bottom and right edges keep their pad slots).  The
      window-grown LR region of an HR window then falls into a few dense tiles instead of one
      row per tile.  Every query sees the same tokens, so the attention is the same function.
  R19 Optional 8-bit Q K^T (qk_format = "e4m3"; the pages only place the permuted layout next
      to SageAttention's tiling, [UG-note] 关键设计 1): after RoPE, every element x of Q (of K)
      is stored as the e4m3 value nearest to x * 2^-q_exp (x * 2^-k_exp), ties to even, values
      beyond the largest finite e4m3 magnitude 448 clamped to +-448; the logits are formed from
      those stored values times 2^(q_exp + k_exp).  The exponents are per tensor and chosen by
      the caller (default 0); a power of two makes the scaling itself exact.  V, the softmax
      and P V keep their precision.  e4m3 is the OCP 8-bit float with 4 exponent bits
      (bias 7) and 3 mantissa bits, subnormals, no infinities, one NaN pattern per sign.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` (brute force
on tiny grids, closed forms, textbook special cases, invariants).  The pages print no
numeric worked example for this method, so no value is pinned to a printed number except
the closed forms the pages state (the 256x window reduction at 4K, rho = H/h).
"""
from __future__ import annotations

import functools
import math
from dataclasses import dataclass

import numpy as np

TEXT, HR, LR, PAD = 0, 1, 2, -1
TILE = 128
LR_BH, LR_BW = 8, 16      # LR block of one tile in the block order (R20)


def pad128(n: int) -> int:
    return TILE * ((n + TILE - 1) // TILE)


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


@dataclass(frozen=True)
class Geometry:
    """Token geometry of one joint sequence [C_T; X; X_lr] ([UG-note] 关键设计 1-3)."""

    H: int          # HR latent rows
    W: int          # HR latent columns
    l: int          # window side in latent tokens (R1)
    b: int          # halo width in tokens (R2)
    rho: int        # LR down-scale factor, rho = H / h ([UG-note] 关键设计 2); 0 = no LR
    T: int          # text tokens
    lr_radius: int = -1   # -1: HR sees all LR (R3); r >= 0: only the window's region grown by r
    halo_copy: bool = False   # K/V carry a compact halo block per window (R18)
    lr_block: bool = False    # LR segment in 8 x 16 blocks of the LR grid (R20)

    @property
    def nWh(self) -> int:
        return cdiv(self.H, self.l)

    @property
    def nWw(self) -> int:
        return cdiv(self.W, self.l)

    @property
    def h(self) -> int:
        return cdiv(self.H, self.rho) if self.rho > 0 else 0

    @property
    def w(self) -> int:
        return cdiv(self.W, self.rho) if self.rho > 0 else 0

    @property
    def N_hr(self) -> int:
        return self.H * self.W

    @property
    def N_lr(self) -> int:
        return self.h * self.w

    @property
    def N_hrp(self) -> int:
        return self.nWh * self.nWw * self.l * self.l

    @property
    def off_hr(self) -> int:
        return pad128(self.T)

    @property
    def off_lr(self) -> int:
        return self.off_hr + pad128(self.N_hrp)

    @property
    def N_lrp(self) -> int:
        """Slots of the LR segment: padded to 128, or whole 8 x 16 blocks (R20)."""
        if self.lr_block:
            return cdiv(self.h, LR_BH) * cdiv(self.w, LR_BW) * TILE
        return pad128(self.N_lr)

    @property
    def N_tot(self) -> int:
        return self.off_lr + self.N_lrp

    @property
    def N_raster(self) -> int:
        return self.T + self.N_hr + self.N_lr

    @property
    def n_windows(self) -> int:
        return self.nWh * self.nWw

    @property
    def G(self) -> int:
        """Slots of one window's halo block in the K/V layout (R18): the packed pieces, padded
        to a multiple of 128; 0 without halo blocks."""
        if not self.halo_copy:
            return 0
        kind, r, c, off = halo_pieces(self)[-1]
        return pad128(off + r * c)

    @property
    def off_halo(self) -> int:
        return self.N_tot

    @property
    def N_kv(self) -> int:
        """K/V slots: the permuted layout plus one halo block per window (R18)."""
        return self.N_tot + self.n_windows * self.G


# --------------------------------------------------------------------------------------
# Tokens, raster order and the window-first permutation
# --------------------------------------------------------------------------------------

@functools.lru_cache(maxsize=8)
def raster_tokens(g: Geometry):
    """Every token of [C_T; X; X_lr] in raster order: (segment, a, b) per token.

    text t -> (TEXT, t, 0); HR (i, j) -> (HR, i, j); LR (m, n) -> (LR, m, n).
    """
    seg = np.empty(g.N_raster, np.int64)
    ca = np.empty(g.N_raster, np.int64)
    cb = np.empty(g.N_raster, np.int64)
    r = 0
    seg[r:r + g.T] = TEXT
    ca[r:r + g.T] = np.arange(g.T)
    cb[r:r + g.T] = 0
    r += g.T
    ii, jj = np.meshgrid(np.arange(g.H), np.arange(g.W), indexing="ij")
    seg[r:r + g.N_hr] = HR
    ca[r:r + g.N_hr] = ii.ravel()
    cb[r:r + g.N_hr] = jj.ravel()
    r += g.N_hr
    mm, nn = np.meshgrid(np.arange(g.h), np.arange(g.w), indexing="ij")
    seg[r:r + g.N_lr] = LR
    ca[r:r + g.N_lr] = mm.ravel()
    cb[r:r + g.N_lr] = nn.ravel()
    return seg, ca, cb


@functools.lru_cache(maxsize=8)
def slot_of_tokens(g: Geometry) -> np.ndarray:
    """Permuted slot of every raster token (window-first order, [UG-note] 关键设计 1; R8, R13).

    HR token (i, j) lies in window (i // l, j // l); windows are numbered row-major and
    tokens inside a window are numbered in raster order of the window's part inside the
    image, whose rows hold min(l, W - wc * l) tokens (R8, R13).
    """
    seg, ca, cb = raster_tokens(g)
    slot = np.empty(g.N_raster, np.int64)
    t = seg == TEXT
    slot[t] = ca[t]
    hr = seg == HR
    i, j = ca[hr], cb[hr]
    window = (i // g.l) * g.nWw + (j // g.l)
    cols = np.minimum(g.l, g.W - (j // g.l) * g.l)       # the window's columns in the image
    slot[hr] = g.off_hr + window * g.l * g.l + (i % g.l) * cols + (j % g.l)
    lr = seg == LR
    m, n = ca[lr], cb[lr]
    if g.lr_block:
        nbw = cdiv(g.w, LR_BW)
        slot[lr] = (g.off_lr + ((m // LR_BH) * nbw + n // LR_BW) * TILE
                    + (m % LR_BH) * LR_BW + n % LR_BW)
    else:
        slot[lr] = g.off_lr + m * g.w + n
    return slot


@functools.lru_cache(maxsize=8)
def perm_map(g: Geometry) -> np.ndarray:
    """pi: permuted slot -> raster index, -1 for pad slots."""
    perm = np.full(g.N_tot, -1, np.int64)
    perm[slot_of_tokens(g)] = np.arange(g.N_raster)
    return perm


@functools.lru_cache(maxsize=8)
def slot_info(g: Geometry):
    """Per permuted slot: segment (PAD for pad slots) and the token's two coordinates."""
    seg_r, ca_r, cb_r = raster_tokens(g)
    perm = perm_map(g)
    real = perm >= 0
    seg = np.full(g.N_tot, PAD, np.int64)
    ca = np.zeros(g.N_tot, np.int64)
    cb = np.zeros(g.N_tot, np.int64)
    seg[real] = seg_r[perm[real]]
    ca[real] = ca_r[perm[real]]
    cb[real] = cb_r[perm[real]]
    return seg, ca, cb


def permute(x: np.ndarray, g: Geometry) -> np.ndarray:
    """Raster [B, N_raster, Hh, D] -> window-first [B, Hh, N_tot, D]; pad slots are zero."""
    B, N, Hh, D = x.shape
    assert N == g.N_raster
    perm = perm_map(g)
    out = np.zeros((B, Hh, g.N_tot, D), x.dtype)
    real = perm >= 0
    out[:, :, real, :] = np.transpose(x, (0, 2, 1, 3))[:, :, perm[real], :]
    return out


def unpermute(xp: np.ndarray, g: Geometry) -> np.ndarray:
    """Window-first [B, Hh, N_tot, D] -> raster [B, N_raster, Hh, D]; pad slots dropped."""
    B, Hh, N, D = xp.shape
    assert N == g.N_tot
    slot = slot_of_tokens(g)
    return np.transpose(xp[:, :, slot, :], (0, 2, 1, 3)).copy()


# --------------------------------------------------------------------------------------
# Compact halo blocks of K/V (R18)
# --------------------------------------------------------------------------------------

HALO = 3   # segment of a K/V slot in a window's halo block


@functools.lru_cache(maxsize=4096)
def halo_tokens(g: Geometry, w: int) -> tuple:
    """Raster indices of window w's halo: the HR tokens of its box grown by b (clipped to the
    image, R2) that lie outside the window itself, in raster order of the grown box (R18)."""
    wr, wc = divmod(w, g.nWw)
    r0, r1 = max(0, wr * g.l - g.b), min(g.H, (wr + 1) * g.l + g.b)
    c0, c1 = max(0, wc * g.l - g.b), min(g.W, (wc + 1) * g.l + g.b)
    out = []
    for i in range(r0, r1):
        for j in range(c0, c1):
            if i // g.l == wr and j // g.l == wc:
                continue
            out.append(g.T + i * g.W + j)
    return tuple(out)


# the eight pieces of a halo block, in block order: (row offset, column offset) of each
# piece's rectangle from the window's top-left token, in units where "-b" is b before the
# window and "l" is right after it; and its shape in (b or l) units
HALO_PIECES = ("top", "bottom", "left", "right", "top_left", "top_right", "bottom_left",
               "bottom_right")


def halo_piece_rect(g: Geometry, kind: str, wr: int, wc: int):
    """Rows [i0, i0 + nr) x cols [j0, j0 + nc) of image coordinates covered by one piece of
    window (wr, wc)'s halo (R18); coordinates may fall outside the image."""
    top, left = wr * g.l, wc * g.l
    rows = {"top": (top - g.b, g.b), "bottom": (top + g.l, g.b), "left": (top, g.l),
            "right": (top, g.l), "top_left": (top - g.b, g.b), "top_right": (top - g.b, g.b),
            "bottom_left": (top + g.l, g.b), "bottom_right": (top + g.l, g.b)}[kind]
    cols = {"top": (left, g.l), "bottom": (left, g.l), "left": (left - g.b, g.b),
            "right": (left + g.l, g.b), "top_left": (left - g.b, g.b),
            "top_right": (left + g.l, g.b), "bottom_left": (left - g.b, g.b),
            "bottom_right": (left + g.l, g.b)}[kind]
    return rows[0], cols[0], rows[1], cols[1]


@functools.lru_cache(maxsize=64)
def halo_pieces(g: Geometry):
    """(kind, rows, cols, slot offset) of the eight pieces of a halo block (R18): each at the
    next multiple of 8; a piece of at most 128 slots that would cross a multiple of 128 moves
    to it, and a longer piece starts on one."""
    out, off = [], 0
    for kind in HALO_PIECES:
        _, _, nr, nc = halo_piece_rect(g, kind, 0, 0)
        n = nr * nc
        off = -(-off // 8) * 8
        if n > 128 or (off % 128) + n > 128:
            off = pad128(off) if off % 128 else off
        out.append((kind, nr, nc, off))
        off += n
    return tuple(out)


@functools.lru_cache(maxsize=4096)
def halo_layout(g: Geometry, w: int) -> tuple:
    """Window w's halo block (R18): G entries, the raster index of the token in each slot or
    -1 for a pad slot."""
    wr, wc = divmod(w, g.nWw)
    out = [-1] * g.G
    for kind, nr, nc, off in halo_pieces(g):
        i0, j0, _, _ = halo_piece_rect(g, kind, wr, wc)
        for a in range(nr):
            for c in range(nc):
                i, j = i0 + a, j0 + c
                if 0 <= i < g.H and 0 <= j < g.W:
                    out[off + a * nc + c] = g.T + i * g.W + j
    return tuple(out)


@functools.lru_cache(maxsize=8)
def kv_perm_map(g: Geometry) -> np.ndarray:
    """K/V slot -> raster index (-1 pad): the permuted layout, then window w's halo block at
    off_halo + w * G in the piece order of halo_layout (R18)."""
    kv = np.full(g.N_kv, -1, np.int64)
    kv[:g.N_tot] = perm_map(g)
    if g.halo_copy:
        for w in range(g.n_windows):
            kv[g.off_halo + w * g.G:g.off_halo + (w + 1) * g.G] = halo_layout(g, w)
    return kv


@functools.lru_cache(maxsize=8)
def kv_slot_info(g: Geometry):
    """Per K/V slot: segment (HALO for halo-block slots, PAD for pad), the token's coordinates,
    and the owning window (HR window-segment and halo-block slots; -1 otherwise)."""
    seg_r, ca_r, cb_r = raster_tokens(g)
    kv = kv_perm_map(g)
    real = kv >= 0
    seg = np.full(g.N_kv, PAD, np.int64)
    ca = np.zeros(g.N_kv, np.int64)
    cb = np.zeros(g.N_kv, np.int64)
    seg[real] = seg_r[kv[real]]
    ca[real] = ca_r[kv[real]]
    cb[real] = cb_r[kv[real]]
    owner = np.full(g.N_kv, -1, np.int64)
    s = np.arange(g.N_kv)
    win_seg = (s >= g.off_hr) & (s < g.off_hr + g.N_hrp)
    owner[win_seg] = (s[win_seg] - g.off_hr) // (g.l * g.l)
    if g.halo_copy:
        halo = s >= g.off_halo
        owner[halo] = (s[halo] - g.off_halo) // g.G
        seg[halo & real] = HALO
    return seg, ca, cb, owner


def permute_kv(x: np.ndarray, g: Geometry) -> np.ndarray:
    """Raster [B, N_raster, Hh, D] -> K/V layout [B, Hh, N_kv, D]; pad slots are zero."""
    B, N, Hh, D = x.shape
    assert N == g.N_raster
    kv = kv_perm_map(g)
    out = np.zeros((B, Hh, g.N_kv, D), x.dtype)
    real = kv >= 0
    out[:, :, real, :] = np.transpose(x, (0, 2, 1, 3))[:, :, kv[real], :]
    return out


# --------------------------------------------------------------------------------------
# Positions and 2D RoPE
# --------------------------------------------------------------------------------------

def positions(g: Geometry) -> np.ndarray:
    """(p0, p1, p2) per raster token: text (0,0,0); HR (0,i,j); LR (0, rho*m, rho*n).

    The LR scaling is the equation of [UG-note] 关键设计 2; the rest is R7/R9.
    """
    seg, ca, cb = raster_tokens(g)
    pos = np.zeros((g.N_raster, 3), np.int64)
    hr = seg == HR
    pos[hr, 1] = ca[hr]
    pos[hr, 2] = cb[hr]
    lr = seg == LR
    pos[lr, 1] = g.rho * ca[lr]
    pos[lr, 2] = g.rho * cb[lr]
    return pos


def rope(x: np.ndarray, pos: np.ndarray, axes, theta: float = 1.0e4) -> np.ndarray:
    """Axial RoPE in fp64 on x [B, N, Hh, D] with per-token positions pos [N, 3] (R7).

    For axis a of width d_a starting at dim o_a, pair k = (o_a + 2k, o_a + 2k + 1) rotates
    by phi = pos_a * theta**(-2k / d_a):  (x0, x1) -> (x0 cos phi - x1 sin phi,
    x0 sin phi + x1 cos phi).
    """
    x = np.asarray(x, np.float64)
    assert sum(axes) == x.shape[-1] and all(d % 2 == 0 for d in axes)
    out = x.copy()
    o = 0
    for a, d in enumerate(axes):
        k = np.arange(d // 2, dtype=np.float64)
        omega = theta ** (-2.0 * k / d)
        phi = pos[:, a].astype(np.float64)[:, None] * omega[None, :]      # [N, d/2]
        c = np.cos(phi)[None, :, None, :]
        s = np.sin(phi)[None, :, None, :]
        x0 = x[..., o + 0:o + d:2]
        x1 = x[..., o + 1:o + d:2]
        out[..., o + 0:o + d:2] = x0 * c - x1 * s
        out[..., o + 1:o + d:2] = x0 * s + x1 * c
        o += d
    return out


# --------------------------------------------------------------------------------------
# The mask M
# --------------------------------------------------------------------------------------

def window_box(g: Geometry, i: np.ndarray, j: np.ndarray):
    """Halo box of the window holding HR token (i, j): [r0, r1) x [c0, c1) (R2)."""
    wr, wc = i // g.l, j // g.l
    r0 = np.maximum(0, wr * g.l - g.b)
    r1 = np.minimum(g.H, (wr + 1) * g.l + g.b)
    c0 = np.maximum(0, wc * g.l - g.b)
    c1 = np.minimum(g.W, (wc + 1) * g.l + g.b)
    return r0, r1, c0, c1


def visible_rows(g: Geometry, q_slots: np.ndarray) -> np.ndarray:
    """Explicit boolean mask rows M[q, :] over all N_kv key slots (R2-R5, R15, R18).

    text q -> text and HR keys;  HR q -> text, LR, and HR keys in its window's halo box;
    LR q -> LR and text keys;  pad q -> nothing.  Pad keys are never visible.
    With halo blocks (R18) an HR query takes its own window's keys from the window segment and
    every other key of its halo box from its window's halo block; halo-block keys are visible
    to nothing else, so every query sees the same tokens as without them.
    """
    seg, ca, cb = slot_info(g)
    kseg_a, ki_a, kj_a, kown_a = kv_slot_info(g)
    q_slots = np.asarray(q_slots, np.int64)
    qs = seg[q_slots]
    kseg = kseg_a[None, :]
    vis = np.zeros((len(q_slots), g.N_kv), bool)

    t = qs == TEXT
    vis[t] = ((kseg == TEXT) | (kseg == HR))[0]

    lr = qs == LR
    vis[lr] = ((kseg == LR) | (kseg == TEXT))[0]

    hr = np.nonzero(qs == HR)[0]
    if len(hr):
        qi, qj = ca[q_slots[hr]], cb[q_slots[hr]]
        ki, kj = ki_a[None, :], kj_a[None, :]
        if g.halo_copy:
            qw = (q_slots[hr] - g.off_hr) // (g.l * g.l)
            in_box = ((kseg == HR) | (kseg == HALO)) & (kown_a[None, :] == qw[:, None])
        else:
            r0, r1, c0, c1 = window_box(g, qi, qj)
            in_box = ((kseg == HR) & (ki >= r0[:, None]) & (ki < r1[:, None])
                      & (kj >= c0[:, None]) & (kj < c1[:, None]))
        if g.lr_radius < 0:
            lr_vis = kseg == LR
        else:
            # LR anchors whose scaled position lies in the window grown by lr_radius
            rr0 = (qi // g.l) * g.l - g.lr_radius
            rr1 = (qi // g.l + 1) * g.l + g.lr_radius
            cc0 = (qj // g.l) * g.l - g.lr_radius
            cc1 = (qj // g.l + 1) * g.l + g.lr_radius
            pm, pn = g.rho * ki, g.rho * kj
            lr_vis = ((kseg == LR) & (pm >= rr0[:, None]) & (pm < rr1[:, None])
                      & (pn >= cc0[:, None]) & (pn < cc1[:, None]))
        vis[hr] = in_box | (kseg == TEXT) | lr_vis
    return vis


# --------------------------------------------------------------------------------------
# Masked softmax attention ([UG-note] 关键设计 3, MMA equation; R6)
# --------------------------------------------------------------------------------------

def attention_rows(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, g: Geometry,
                   rows: np.ndarray, heads=None, chunk: int = 256) -> np.ndarray:
    """Dense fp64 masked softmax attention for selected permuted query rows.

    qp: [B, Hh, N_tot, D], kp, vp: [B, Hh, N_kv, D] (already RoPE'd and permuted; N_kv = N_tot
    without halo blocks).  Returns [B, Hh', len(rows), D]
    with heads' = ``heads`` (all by default).  Pad rows give 0.
    """
    B, Hh, N, D = qp.shape
    heads = range(Hh) if heads is None else heads
    rows = np.asarray(rows, np.int64)
    out = np.zeros((B, len(list(heads)), len(rows), D), np.float64)
    scale = 1.0 / math.sqrt(D)
    for c0 in range(0, len(rows), chunk):
        rr = rows[c0:c0 + chunk]
        vis = visible_rows(g, rr)
        any_vis = vis.any(axis=1)
        for bi in range(B):
            for hi, h in enumerate(heads):
                K = np.asarray(kp[bi, h], np.float64)
                V = np.asarray(vp[bi, h], np.float64)
                q = np.asarray(qp[bi, h, rr], np.float64)
                s = (q @ K.T) * scale
                s = np.where(vis, s, -np.inf)
                m = np.max(np.where(any_vis[:, None], s, 0.0), axis=1, keepdims=True)
                p = np.exp(s - m)
                p[~any_vis] = 0.0
                den = p.sum(axis=1, keepdims=True)
                den[~any_vis] = 1.0
                p = p / den
                ok = np.abs(p[any_vis].sum(axis=1) - 1.0) < 1e-12
                assert ok.all(), "softmax rows must sum to 1"
                out[bi, hi, c0:c0 + len(rr)] = p @ V
    return out


def forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, g: Geometry, axes,
            theta: float = 1.0e4, rows=None, heads=None, qk_format: str = "bf16",
            q_exp: int = 0, k_exp: int = 0):
    """Whole path on raster inputs [B, N_raster, Hh, D]: RoPE -> permute -> attention.

    qk_format "e4m3" stores the RoPE'd Q and K as scaled e4m3 values first (R19); "bf16"
    keeps them exact.  Returns (O_rows [B, Hh', n, D] for the permuted ``rows`` (all slots by
    default), rows).  Unpermute the full result with ``unpermute``.
    """
    pos = positions(g)
    qr = rope(q, pos, axes, theta)
    kr = rope(k, pos, axes, theta)
    if qk_format == "e4m3":
        qr, kr = quantize_e4m3(qr, q_exp), quantize_e4m3(kr, k_exp)
    elif qk_format != "bf16":
        raise ValueError(f"unknown qk_format {qk_format!r}")
    qp, kp, vp = permute(qr, g), permute_kv(kr, g), permute_kv(np.asarray(v, np.float64), g)
    rows = np.arange(g.N_tot) if rows is None else np.asarray(rows, np.int64)
    return attention_rows(qp, kp, vp, g, rows, heads=heads), rows


# --------------------------------------------------------------------------------------
# Tile lists derived from the explicit mask (R15)
# --------------------------------------------------------------------------------------

def qtile_entries(g: Geometry, t: int):
    """Entries of query tile t: ascending key tiles with any visible (real row, col) cell;
    bit 31 marks a partial tile (some real-row cell not visible).  Also returns the
    per-entry row masks [n_entries, 128, 4] uint32 (bit c%32 of word c//32 = column c
    visible for that row; rows of pad slots are 0)."""
    perm = perm_map(g)
    slots = np.arange(t * TILE, (t + 1) * TILE)
    real = perm[slots] >= 0
    nk = g.N_kv // TILE
    vis = np.zeros((TILE, g.N_kv), bool)
    if real.any():
        vis[real] = visible_rows(g, slots[real])
    blocks = vis.reshape(TILE, nk, TILE)
    anyv = blocks[real].any(axis=(0, 2)) if real.any() else np.zeros(nk, bool)
    allv = blocks[real].all(axis=(0, 2)) if real.any() else np.zeros(nk, bool)
    ks = np.nonzero(anyv)[0]
    entries = (ks.astype(np.uint64) | ((~allv[ks]).astype(np.uint64) << np.uint64(31)))
    bits = blocks[:, ks, :].transpose(1, 0, 2).reshape(len(ks), TILE, 4, 32)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    words = (bits.astype(np.uint64) * weights).sum(axis=-1).astype(np.uint32)
    return entries.astype(np.uint32), words


def tile_lists(g: Geometry, qtiles=None):
    """CSR over query tiles: (row_ptr, entries) as uint32, for the given q-tiles (all)."""
    qtiles = range(g.N_tot // TILE) if qtiles is None else qtiles
    row_ptr = [0]
    ents = []
    for t in qtiles:
        e, _ = qtile_entries(g, t)
        ents.append(e)
        row_ptr.append(row_ptr[-1] + len(e))
    entries = np.concatenate(ents) if ents else np.zeros(0, np.uint32)
    return np.asarray(row_ptr, np.int64), entries


def visible_pair_count(g: Geometry, chunk: int = 1024) -> int:
    """Number of visible (query, key) pairs of one head, from the explicit mask."""
    total = 0
    for c0 in range(0, g.N_tot, chunk):
        total += int(visible_rows(g, np.arange(c0, min(g.N_tot, c0 + chunk))).sum())
    return total


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even); returns fp64.

    Works on the fp64 bit pattern so there is no double rounding through fp32.
    Finite inputs only.
    """
    x = np.asarray(x, np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    xv = x[nz]
    e = np.floor(np.log2(np.abs(xv)))
    # guard against log2 rounding at exact powers of two
    e = np.where(np.abs(xv) < 2.0 ** e, e - 1, e)
    e = np.where(np.abs(xv) >= 2.0 ** (e + 1), e + 1, e)
    e = np.maximum(e, -126.0)                 # below 2**-126 the ulp stays 2**-133
    ulp = 2.0 ** (e - 7)
    out[nz] = np.round(xv / ulp) * ulp        # np.round: ties to even
    return out


# --------------------------------------------------------------------------------------
# 8-bit Q K^T (R19)
# --------------------------------------------------------------------------------------

E4M3_MAX = 448.0             # largest finite e4m3 magnitude: 2^8 * (1 + 6/8)
E4M3_MIN_NORMAL_EXP = -6     # 1 - bias 7; below 2^-6 the spacing stays 2^-9 (subnormals)


def round_e4m3(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value (ties to even), clamped to +-448; returns fp64 (R19).

    A finite x with 2^e <= |x| < 2^(e+1) has spacing 2^(e-3) between its e4m3 neighbours
    (3 mantissa bits); below the smallest normal 2^-6 the spacing stays 2^-9.  Rounding x
    to a multiple of that spacing, ties to even, is exact in fp64.  Finite inputs only.
    """
    x = np.asarray(x, np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    xv = x[nz]
    e = np.floor(np.log2(np.abs(xv)))
    e = np.where(np.abs(xv) < 2.0 ** e, e - 1, e)          # log2 rounding at powers of two
    e = np.where(np.abs(xv) >= 2.0 ** (e + 1), e + 1, e)
    e = np.maximum(e, float(E4M3_MIN_NORMAL_EXP))
    ulp = 2.0 ** (e - 3)
    out[nz] = np.clip(np.round(xv / ulp) * ulp, -E4M3_MAX, E4M3_MAX)   # np.round: ties to even
    return out


def quantize_e4m3(x: np.ndarray, exp: int) -> np.ndarray:
    """The value an e4m3-stored tensor with scale 2^exp represents: round(x 2^-exp) 2^exp."""
    return round_e4m3(np.asarray(x, np.float64) * 2.0 ** -exp) * 2.0 ** exp


def e4m3_codes(x: np.ndarray, exp: int) -> np.ndarray:
    """The stored bytes of round_e4m3(x 2^-exp) (R19): sign bit 7, exponent bits 6..3
    (bias 7, field 0 for zero and subnormals), mantissa bits 2..0."""
    y = round_e4m3(np.asarray(x, np.float64) * 2.0 ** -exp)
    sign = (y < 0) | ((y == 0) & np.signbit(y))
    a = np.abs(y)
    code = np.zeros(y.shape, np.int64)
    nz = a > 0
    av = a[nz]
    e = np.floor(np.log2(av))
    e = np.where(av < 2.0 ** e, e - 1, e)
    e = np.where(av >= 2.0 ** (e + 1), e + 1, e)
    sub = e < E4M3_MIN_NORMAL_EXP
    field = np.where(sub, 0, e + 7).astype(np.int64)
    mant = np.where(sub, av / 2.0 ** -9, (av / 2.0 ** e - 1.0) * 8.0)
    code[nz] = (field << 3) | np.rint(mant).astype(np.int64)
    return (code | (sign.astype(np.int64) << 7)).astype(np.uint8)
