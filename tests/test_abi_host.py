"""C-ABI checks that need no GPU: the library loads, exports every symbol of
include/ultragen.h, rejects bad arguments, and its host plan (permutation, tile lists,
per-row masks, pair counts) is bit-exact against the oracle's explicit mask."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import hla_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session")
def ffi():
    from diffusion_transformer_ultra_b200 import build
    build.build()
    from diffusion_transformer_ultra_b200 import _ffi
    return _ffi


def header_functions():
    src = open(os.path.join(ROOT, "include", "ultragen.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(ultragen_\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported(ffi):
    names = header_functions()
    assert len(names) >= 13
    lib = ctypes.CDLL(ffi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ffi.SYMBOLS)


def test_status_strings(ffi):
    L = ffi.lib()
    for code in range(9):
        assert L.ultragen_status_string(code).decode() != "unknown status"
    assert L.ultragen_status_string(99).decode() == "unknown status"


def test_clock_record_arguments(ffi):
    import ctypes as C
    L = ffi.lib()
    buf = (C.c_uint64 * 3)(7, 7, 7)
    assert L.ultragen_plan_set_clock_record(None, 1) == 1
    assert L.ultragen_plan_read_clock(None, buf) == 1
    p = ffi.Plan(32, 32, 8, 2, 4, 16, 1, 64)
    assert L.ultragen_plan_set_clock_record(p.handle, 2) == 1
    assert L.ultragen_plan_read_clock(p.handle, None) == 1
    p.set_clock_record(True)
    # no tables on a device yet: an empty record
    assert p.read_clock() == {"launches": 0, "cycles": 0, "ns": 0, "sm_mhz": None}


def test_debug_build_compiles_and_exports_every_symbol(ffi):
    """The ULTRAGEN_DEBUG build (index checks in the kernels) builds in-tree and exports the
    same C ABI; nothing here calls into a GPU."""
    from diffusion_transformer_ultra_b200 import build
    path = build.build(debug=True)
    assert path.endswith("libultragen_debug.so") and os.path.exists(path)
    lib = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(lib, n), n


@pytest.mark.parametrize("args,status", [
    ((0, 8, 4, 1, 2, 3, 1, 64), 1),     # H < 1
    ((8, 8, 4, 5, 2, 3, 1, 64), 2),     # b > l
    ((8, 8, 4, 1, -1, 3, 1, 64), 1),    # rho < 0
    ((8, 8, 4, 1, 2, 3, 1, 96), 2),     # head_dim not 64/128
    ((8, 8, 0, 0, 2, 3, 1, 64), 1),     # l < 1
    ((8, 8, 4, 1, 2, -3, 1, 64), 1),    # text_len < 0
])
def test_plan_rejects_bad_arguments(ffi, args, status):
    h = ctypes.c_void_p()
    assert ffi.lib().ultragen_plan(*args, ctypes.byref(h)) == status
    assert not h.value


def test_set_rope_validation(ffi):
    p = ffi.Plan(8, 8, 4, 1, 2, 3, 1, 64)
    L = ffi.lib()
    assert L.ultragen_plan_set_rope(p.handle, 16, 24, 22, 1e4) == 1   # sum != D
    assert L.ultragen_plan_set_rope(p.handle, 15, 25, 24, 1e4) == 1   # odd
    assert L.ultragen_plan_set_rope(p.handle, 16, 24, 24, -1.0) == 1
    assert L.ultragen_plan_set_rope(p.handle, 0, 32, 32, 5e3) == 0
    p._refresh()
    assert p.info["rope_axes"] == (0, 32, 32) and p.info["rope_theta"] == 5e3


def test_device_calls_without_device_fail_cleanly(ffi):
    """On a host with no GPU the device entry points return an error status, never crash."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = ffi.Plan(8, 8, 4, 1, 2, 3, 1, 64)
    L = ffi.lib()
    buf = ctypes.create_string_buffer(1 << 16)
    a = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16
    st = L.ultragen_hla_forward(a, a, a, a, p.handle, 1, None)
    assert st in (3, 7)
    assert L.ultragen_hla_forward(None, a, a, a, p.handle, 1, None) == 1
    assert L.ultragen_permute_rope(a, a, a, 5, a, a, a, 1, p.handle, None) == 1
    assert L.ultragen_warm_start(a, None, a, 1, 1, 4, 4, 16, 16, 0.5, 1.0, 0, 0, None) in (3, 7)
    r = ctypes.c_void_p()
    assert L.ultragen_host_runner_create(p.handle, 1, 4, ctypes.byref(r)) in (3, 7)
    assert not r.value


def test_host_runner_argument_checks(ffi):
    """Argument errors of the host runner come back before any device work."""
    L = ffi.lib()
    p = ffi.Plan(8, 8, 4, 1, 2, 3, 2, 64)
    r = ctypes.c_void_p()
    assert L.ultragen_host_runner_create(None, 1, 1, ctypes.byref(r)) == 1
    assert L.ultragen_host_runner_create(p.handle, 0, 1, ctypes.byref(r)) == 1
    assert L.ultragen_host_runner_create(p.handle, 1, 0, ctypes.byref(r)) == 1
    assert L.ultragen_host_runner_create(p.handle, 1, 1, None) == 1
    buf = ctypes.create_string_buffer(64)
    a = ctypes.addressof(buf)
    assert L.ultragen_host_runner_forward(None, a, a, a, a, None) == 1
    assert L.ultragen_host_runner_destroy(None) == 1
    assert L.ultragen_host_runner_last_launch_count(None) == -1


def test_warm_start_argument_checks(ffi):
    """Argument errors come back before any device work (safe with or without a GPU)."""
    L = ffi.lib()
    buf = ctypes.create_string_buffer(1 << 12)
    a = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16
    ok = (a, None, a, 1, 4, 8, 8, 32, 32, 0.5, 1.0, 7, 0, None)

    def call(**kw):
        args = list(ok)
        for i, name in enumerate(("lr", "noise", "out", "B", "C", "h", "w", "H", "W", "alpha",
                                  "sharpen", "seed", "offset", "stream")):
            if name in kw:
                args[i] = kw[name]
        return L.ultragen_warm_start(*args)

    assert call(lr=None) == 1
    assert call(out=None) == 1
    assert call(B=0) == 1 and call(C=-1) == 1 and call(h=0) == 1 and call(W=0) == 1
    assert call(sharpen=-0.5) == 1
    assert call(alpha=float("nan")) == 1 and call(sharpen=float("inf")) == 1
    assert call(lr=a + 2) == 1 and call(noise=a + 1) == 1
    assert call(B=300, C=300) == 2


GEOMS = {
    "tiny": (32, 32, 8, 2, 4, 16),
    "1k": (64, 64, 16, 4, 4, 512),
    "ragged": (256, 135, 16, 16, 4, 256),
    "odd": (37, 29, 12, 5, 3, 70),
    "small_l": (20, 18, 4, 3, 5, 9),
    "no_lr_text": (40, 24, 8, 8, 0, 0),
    # window-size / rho ablation shapes of the pages (ws 512 px -> l = 32; rho = 2)
    "win32_rho2": (96, 96, 32, 8, 2, 64),
    # degenerate cases: one token; a window larger than the image; rho larger than the image
    # (one LR token); a 3-row strip with a text segment one past a tile boundary
    "single": (1, 1, 1, 0, 1, 0),
    "win_exceeds": (5, 7, 16, 3, 8, 3),
    "rho_exceeds": (4, 4, 2, 2, 8, 1),
    "thin": (3, 130, 4, 1, 2, 129),
}


def sample_qtiles(g, n_hr=40, seed=0):
    nq = g.N_tot // 128
    text = list(range(0, g.off_hr // 128))
    lr = list(range(g.off_lr // 128, nq))
    hr = list(range(g.off_hr // 128, g.off_lr // 128))
    rng = np.random.default_rng(seed)
    pick = sorted(set(hr[:4] + hr[-4:] + list(rng.choice(hr, size=min(n_hr, len(hr)), replace=False))))
    return sorted(set(text + lr[:3] + lr[-3:] + pick))


def compare_plan(ffi, geom, qtiles=None, halo=None):
    p = ffi.Plan(*geom, 2, 64)
    if halo is not None:
        p.set_halo(halo)
    info = p.info
    g = O.Geometry(*geom, halo_copy=bool(info["halo_copy"]))
    assert info["N_tot"] == g.N_tot and info["N_raster"] == g.N_raster
    assert info["off_hr"] == g.off_hr and info["off_lr"] == g.off_lr
    assert info["N_kv"] == g.N_kv and info["halo_slots_per_window"] == g.G
    perm, row_ptr, entries = p.export()
    np.testing.assert_array_equal(perm, O.perm_map(g))
    np.testing.assert_array_equal(p.export_kv(), O.kv_perm_map(g))
    qtiles = range(g.N_tot // 128) if qtiles is None else qtiles
    for t in qtiles:
        e_ref, m_ref = O.qtile_entries(g, t)
        e_got = entries[row_ptr[t]:row_ptr[t + 1]].view(np.uint32)
        np.testing.assert_array_equal(e_got, e_ref, err_msg=f"q-tile {t}")
        np.testing.assert_array_equal(p.rowmasks(t, len(e_ref)), m_ref, err_msg=f"q-tile {t} masks")
    return g, p


@pytest.mark.parametrize("halo", [None, 0, 1])
@pytest.mark.parametrize("name", ["tiny", "1k", "odd", "small_l", "no_lr_text", "win32_rho2",
                                  "single", "win_exceeds", "rho_exceeds", "thin"])
def test_plan_bit_exact_full(ffi, name, halo):
    g, p = compare_plan(ffi, GEOMS[name], halo=halo)
    assert p.info["useful_pairs"] == O.visible_pair_count(g)


# shapes whose halo tiles the attention can gather (whole windows, b * b a multiple of 8,
# pieces within one tile); their border windows take zero boxes for the pieces outside
GATHER_GEOMS = {
    "1k": GEOMS["1k"],
    "l16_b8": (48, 64, 16, 8, 4, 20),
    "l32_b4": (64, 96, 32, 4, 4, 33),
    "l8_b4": (24, 40, 8, 4, 2, 5),
}


@pytest.mark.parametrize("name", sorted(GATHER_GEOMS))
def test_plan_bit_exact_gathered_halo(ffi, name):
    g, p = compare_plan(ffi, GATHER_GEOMS[name], halo=2)
    assert p.info["halo_copy"] == 2 and p.info["kv_rows"] == p.info["N_tot"]


@pytest.mark.parametrize("name", sorted(GATHER_GEOMS))
def test_gathered_halo_tiles_assemble_the_oracle_blocks(ffi, name):
    """Replays the attention's halo-tile copies on the host: every box is read from the window
    segment the way the tiled copy reads it (raster order of the box; zeros for a zero box or
    a window outside the image) and must rebuild each halo-block tile of the oracle's K/V slot
    map token for token, every row written exactly once, every box on an 8-row boundary."""
    geom = GATHER_GEOMS[name]
    p = ffi.Plan(*geom, 2, 64)
    p.set_halo(2)
    g = O.Geometry(*geom, halo_copy=True)
    kv, perm, ops = O.kv_perm_map(g), O.perm_map(g), p.export_halo_ops()
    l, b, G = g.l, g.b, g.G
    gt = G // 128
    shapes = [(b, l), (l, b), (b, b)]                      # (rows, columns) of a box
    assert len(ops) == p.info["n_halo_ops"] and ops[0] == gt + 1 and ops[gt] == len(ops)
    for w in range(g.nWh * g.nWw):
        wr, wc = divmod(w, g.nWw)
        for t in range(gt):
            got = np.full(128, -2, np.int64)
            for o in range(ops[t], ops[t + 1]):
                c = int(ops[o])
                row, shape, zero = c & 127, (c >> 7) & 3, (c >> 9) & 1
                sr, sc = wr + ((c >> 10) & 3) - 1, wc + ((c >> 12) & 3) - 1
                i0, j0 = (c >> 14) & 255, (c >> 22) & 255
                nr, nc = shapes[shape]
                assert row % 8 == 0 and row + nr * nc <= 128
                assert i0 + nr <= l and j0 + nc <= l
                outside = zero or not (0 <= sr < g.nWh and 0 <= sc < g.nWw)
                for a in range(nr):
                    for cc in range(nc):
                        assert got[row + a * nc + cc] == -2, "row written twice"
                        src = g.off_hr + (sr * g.nWw + sc) * l * l + (i0 + a) * l + j0 + cc
                        got[row + a * nc + cc] = -1 if outside else perm[src]
            assert (got != -2).all(), "row left unwritten"
            s0 = g.off_halo + w * G + t * 128
            np.testing.assert_array_equal(got, kv[s0:s0 + 128], err_msg=f"window {w} tile {t}")


def test_qk_format_argument_checks(ffi):
    """The Q/K storage format: validated on the host, kept across plan rebuilds, and the
    bf16 format carries no exponents."""
    L = ffi.lib()
    p = ffi.Plan(64, 64, 16, 4, 4, 512, 2, 128)
    assert p.info["qk_format"] == ffi.QK_BF16 and p.info["q_exp"] == p.info["k_exp"] == 0
    assert L.ultragen_plan_set_qk_format(None, 1, 0, 0) == 1
    assert L.ultragen_plan_set_qk_format(p.handle, 2, 0, 0) == 1
    assert L.ultragen_plan_set_qk_format(p.handle, -1, 0, 0) == 1
    assert L.ultragen_plan_set_qk_format(p.handle, 1, 33, 0) == 1
    assert L.ultragen_plan_set_qk_format(p.handle, 1, 0, -33) == 1
    p.set_qk_format("e4m3", -32, 32)
    assert (p.info["qk_format"], p.info["q_exp"], p.info["k_exp"]) == (ffi.QK_E4M3, -32, 32)
    p.set_halo(0)
    entries = p.info["n_entries"]
    p.set_halo(1)
    p.set_split(3)
    assert p.info["n_entries"] < entries                # the halo blocks rebuilt the lists
    assert (p.info["qk_format"], p.info["q_exp"], p.info["k_exp"]) == (ffi.QK_E4M3, -32, 32)
    p.set_qk_format("bf16", 5, 5)
    assert (p.info["qk_format"], p.info["q_exp"], p.info["k_exp"]) == (ffi.QK_BF16, 0, 0)
    # e4m3 products read 128-byte rows: head_dim 64 is not supported
    q = ffi.Plan(64, 64, 16, 4, 4, 512, 2, 64)
    assert L.ultragen_plan_set_qk_format(q.handle, 1, 0, 0) == 2
    q.set_qk_format("bf16")


def test_halo_mode_argument_checks_and_auto_choice(ffi):
    p = ffi.Plan(64, 64, 16, 4, 4, 512, 2, 64)
    assert ffi.lib().ultragen_plan_set_halo(p.handle, 3) == 1
    assert ffi.lib().ultragen_plan_set_halo(p.handle, -2) == 1
    useful = p.info["useful_pairs"]
    for mode in (0, 1, 2, -1):
        p.set_halo(mode)
        assert p.info["useful_pairs"] == useful            # the same attention either way
    p.set_halo(1)
    assert p.info["halo_copy"] == 1 and p.info["N_kv"] > p.info["N_tot"]
    assert p.info["kv_rows"] == p.info["N_kv"]            # the permute copies the blocks
    entries = p.info["n_entries"]
    p.set_halo(2)
    assert p.info["halo_copy"] == 2 and p.info["N_kv"] > p.info["N_tot"]
    assert p.info["kv_rows"] == p.info["N_tot"]           # the attention gathers them
    assert p.info["n_entries"] == entries                 # over the same tile lists
    p.set_halo(0)
    assert p.info["halo_copy"] == 0 and p.info["N_kv"] == p.info["N_tot"] == p.info["kv_rows"]
    # l = 16, b = 4 can be gathered, so the automatic choice gathers
    p.set_halo(-1)
    assert p.info["halo_copy"] == 2
    # b = 3: a corner of 9 tokens cannot land on a 1 KB boundary; copied blocks still work
    s = ffi.Plan(64, 64, 16, 3, 4, 512, 2, 64)
    assert ffi.lib().ultragen_plan_set_halo(s.handle, 2) == 2
    s.set_halo(1)
    assert s.info["halo_copy"] == 1
    # partial edge windows (W = 72) pack their tokens at the front: no gather; copied blocks
    # still work
    e = ffi.Plan(64, 72, 16, 4, 4, 512, 2, 64)
    assert e.info["halo_copy"] != 2
    assert ffi.lib().ultragen_plan_set_halo(e.handle, 2) == 2
    e.set_halo(1)
    assert e.info["halo_copy"] == 1
    # b = l: every neighbour tile is fully visible, so the automatic choice keeps them
    q = ffi.Plan(256, 135, 16, 16, 4, 256, 2, 64)
    assert q.info["halo_copy"] == 0
    # b = 0: no halo at all
    r = ffi.Plan(64, 64, 16, 0, 4, 16, 2, 64)
    assert r.info["halo_copy"] == 0


@pytest.mark.parametrize("name", ["ragged"])
def test_plan_bit_exact_sampled(ffi, name):
    compare_plan(ffi, GEOMS[name], sample_qtiles(O.Geometry(*GEOMS[name])))


def test_plan_4k_8k_sampled_and_pair_counts(ffi):
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from test_oracle_pins import closed_form_pairs
    for side in (256, 512):
        geom = (side, side, 16, 4, 4, 512)
        g = O.Geometry(*geom)
        _, p = compare_plan(ffi, geom, sample_qtiles(g, n_hr=12))
        assert p.info["useful_pairs"] == sum(closed_form_pairs(*geom).values())
    # the totals quoted for these layers: 390,873,088 (4K) and 4,988,354,560 (8K) pairs per head
    assert sum(closed_form_pairs(256, 256, 16, 4, 4, 512).values()) == 390_873_088
    assert sum(closed_form_pairs(512, 512, 16, 4, 4, 512).values()) == 4_988_354_560


def check_schedule(p):
    """The work items cover every query tile's key list exactly once: a paired item covers two
    adjacent query tiles with identical lists and the same masks on every real row, a split
    group's items partition its
    list in order with distinct partial slots, and the long groups come first, longest first,
    then the split items, then the rest."""
    info = p.info
    perm, row_ptr, entries = p.export()
    items = p.export_items()
    assert len(items) == info["n_items"] and (items[:, 7] == 0).all()
    ranges = {}
    second = set()
    for qt0, qt1, e0, e1, ws, _, _, _ in items.tolist():
        assert row_ptr[qt0] <= e0 <= e1 <= row_ptr[qt0 + 1]
        ranges.setdefault(qt0, []).append((e0, e1, ws))
        if qt1 >= 0:
            assert qt1 == qt0 + 1
            n = row_ptr[qt0 + 1] - row_ptr[qt0]
            assert row_ptr[qt1 + 1] - row_ptr[qt1] == n
            np.testing.assert_array_equal(entries[row_ptr[qt0]:row_ptr[qt0 + 1]],
                                          entries[row_ptr[qt1]:row_ptr[qt1 + 1]])
            # the same masks on every real row of both tiles (pad rows export as 0)
            m0, m1 = p.rowmasks(qt0, n), p.rowmasks(qt1, n)
            r0 = perm[qt0 * 128:(qt0 + 1) * 128] >= 0
            r1 = perm[qt1 * 128:(qt1 + 1) * 128] >= 0
            ref = m0[:, np.argmax(r0)]
            assert (m0[:, r0] == ref[:, None]).all() and (m1[:, r1] == ref[:, None]).all()
            second.add(qt1)
    # every query tile is the first tile of exactly one group or the second tile of a pair
    assert set(ranges) | second == set(range(info["n_qtiles"]))
    assert not set(ranges) & second
    slots = []
    for qt0, rs in ranges.items():
        rs.sort()
        assert rs[0][0] == row_ptr[qt0] and rs[-1][1] == row_ptr[qt0 + 1]
        assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
        if len(rs) > 1:
            assert all(ws >= 0 for _, _, ws in rs)
            slots += [ws for _, _, ws in rs]
        else:
            assert rs[0][2] == -1
    assert sorted(slots) == list(range(info["n_split_items"]))
    # order: long groups (longest first), split items, the rest
    n = items[:, 3] - items[:, 2]
    nl = info["n_long_items"]
    assert (items[:nl, 4] == -1).all() and (np.diff(n[:nl]) <= 0).all()
    rest = items[nl:]
    split_end = int((rest[:, 4] >= 0).sum())
    assert (rest[:split_end, 4] >= 0).all() and (rest[split_end:, 4] == -1).all()
    if nl and split_end < len(rest):
        assert n[:nl].min() > n[nl + split_end:].max()


@pytest.mark.parametrize("name", ["tiny", "1k", "odd", "small_l", "no_lr_text", "win32_rho2",
                                  "single", "win_exceeds", "thin"])
@pytest.mark.parametrize("split", [None, 0, 3])
def test_schedule_covers_every_query_tile_once(ffi, name, split):
    p = ffi.Plan(*GEOMS[name], 2, 64)
    if split is not None:
        p.set_split(split)
    check_schedule(p)


@pytest.mark.parametrize("heads", [1, 24])
def test_schedule_at_4k(ffi, heads):
    """4K with one head splits its text groups; with 24 it splits nothing and hands the two text
    groups out first."""
    p = ffi.Plan(256, 256, 16, 4, 4, 512, heads, 128)
    check_schedule(p)
    assert (p.info["n_split_items"] > 0) == (heads == 1)


def test_split_policy(ffi):
    # 24 heads: the longest group (a text pair over all 548 key tiles) is below one SM's share
    # of the layer (24 heads x the key-tile steps of a head / 148), so nothing is split and the
    # two text groups of a head are its long items, handed out first
    p24 = ffi.Plan(256, 256, 16, 4, 4, 512, 24, 128)
    assert p24.info["split_chunk"] == 0 and p24.info["n_split_groups"] == 0
    assert p24.info["n_long_items"] == 2
    # one head: the text groups outlast that share and are split
    p = ffi.Plan(256, 256, 16, 4, 4, 512, 1, 128)
    i = p.info
    # automatic chunk: the longest HR / LR query-tile list, applied to the text groups only
    _, row_ptr, _ = p.export()
    longest = int(np.diff(row_ptr)[i["off_hr"] // 128:].max())
    assert i["split_chunk"] == max(longest, 8) and i["n_split_groups"] == 2
    assert i["n_long_items"] == 0
    p.set_split(0)
    assert p.info["n_split_groups"] == 0 and p.info["workspace_bytes_per_head"] == 0
    p.set_split(7)
    assert p.info["split_chunk"] == 7 and p.info["n_split_groups"] > 2
    assert p.info["workspace_bytes_per_head"] == p.info["n_split_items"] * 2 * 128 * 129 * 4


def test_diagnostics_validation(ffi):
    p = ffi.Plan(8, 8, 4, 1, 2, 3, 1, 64)
    L = ffi.lib()
    assert L.ultragen_plan_set_diagnostics(p.handle, 2, 1.0) == 1
    assert L.ultragen_plan_set_diagnostics(p.handle, 0, 0.0) == 1
    assert L.ultragen_plan_set_diagnostics(p.handle, 0, 61.0) == 1
    assert L.ultragen_plan_set_diagnostics(p.handle, 1, 0.05) == 0
    assert L.ultragen_plan_set_diagnostics(p.handle, 0, 2.0) == 0


def compare_region_plan(ffi, geom, r, qtiles=None, order=None):
    p = ffi.Plan(*geom, 2, 64)
    p.set_lr_scope(r)
    if order is not None:
        p.set_lr_order(order)
    assert p.info["lr_radius"] == r
    g = O.Geometry(*geom, lr_radius=r, halo_copy=bool(p.info["halo_copy"]),
                   lr_block=bool(p.info["lr_block"]))
    if callable(qtiles):
        qtiles = qtiles(g)
    perm, row_ptr, entries = p.export()
    np.testing.assert_array_equal(perm, O.perm_map(g))
    np.testing.assert_array_equal(p.export_kv(), O.kv_perm_map(g))
    for t in (range(g.N_tot // 128) if qtiles is None else qtiles):
        e_ref, m_ref = O.qtile_entries(g, t)
        np.testing.assert_array_equal(entries[row_ptr[t]:row_ptr[t + 1]].view(np.uint32), e_ref,
                                      err_msg=f"q-tile {t}")
        np.testing.assert_array_equal(p.rowmasks(t, len(e_ref)), m_ref, err_msg=f"q-tile {t} masks")
    return g, p


@pytest.mark.parametrize("order", [None, 0, 1])
@pytest.mark.parametrize("name,r", [("tiny", 0), ("1k", 4), ("odd", 3), ("small_l", 1)])
def test_region_plan_bit_exact(ffi, name, r, order):
    g, p = compare_region_plan(ffi, GEOMS[name], r, order=order)
    if order is not None:
        assert p.info["lr_block"] == order
    assert p.info["useful_pairs"] == O.visible_pair_count(g)


def test_lr_order_argument_checks_and_auto_choice(ffi):
    p = ffi.Plan(256, 256, 16, 4, 4, 512, 2, 64)
    L = ffi.lib()
    assert L.ultragen_plan_set_lr_order(p.handle, 2) == 1
    assert L.ultragen_plan_set_lr_order(p.handle, -2) == 1
    p.set_lr_order(1)
    assert p.info["lr_block"] == 0                  # all LR visible: the order stays raster
    p.set_lr_scope(4)
    auto = p.info["n_entries"]
    assert p.info["lr_block"] == 1                  # the 4K region: blocks give fewer entries
    p.set_lr_order(0)
    assert p.info["lr_block"] == 0 and p.info["n_entries"] > auto
    p.set_lr_order(-1)
    assert p.info["lr_block"] == 1 and p.info["n_entries"] == auto
    q = ffi.Plan(256, 135, 16, 16, 4, 256, 2, 64)   # ragged: raster packs the region better
    q.set_lr_scope(4)
    assert q.info["lr_block"] == 0


def test_region_plan_large_sampled(ffi):
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from test_oracle_pins import closed_form_pairs
    for geom, r in (((256, 256, 16, 4, 4, 512), 4), ((512, 512, 16, 4, 4, 512), 0),
                    ((256, 135, 16, 16, 4, 256), 16)):
        _, p = compare_region_plan(ffi, geom, r, lambda g: sample_qtiles(g, n_hr=10))
        assert p.info["useful_pairs"] == sum(closed_form_pairs(*geom, lr_radius=r).values())
    p = ffi.Plan(64, 64, 16, 4, 4, 512, 2, 64)
    assert ffi.lib().ultragen_plan_set_lr_scope(p.handle, -2) == 1


def test_plan_at_16k_maximum_size(ffi):
    """The largest layer considered (a 16K image: 1024 x 1024 HR tokens, 256 x 256 LR): the plan
    builds, stays inside the int32 limits of the launch arithmetic for 24 heads, and its visible
    pair count equals the closed form."""
    import importlib.util
    import os
    spec = importlib.util.spec_from_file_location(
        "pins", os.path.join(os.path.dirname(__file__), "test_oracle_pins.py"))
    pins = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(pins)
    geom = (1024, 1024, 16, 4, 4, 512)
    p = ffi.Plan(*geom, 24, 128)
    i = p.info
    assert sum(pins.closed_form_pairs(*geom).values()) == i["useful_pairs"]
    assert 24 * i["N_tot"] < 2 ** 31 and 24 * i["N_raster"] < 2 ** 31
    assert 24 * i["n_items"] < 2 ** 31
    g = O.Geometry(*geom)
    assert (i["N_tot"], i["N_raster"], i["off_hr"], i["off_lr"]) == (g.N_tot, g.N_raster, g.off_hr, g.off_lr)


def test_plan_matches_oracle_on_random_geometries(ffi):
    """60 seeded random small geometries (any H, W, l, b <= l, rho including 0, text length,
    LR scope, halo mode): layout, K/V slot map, tile lists, partial flags and row masks are
    bit-exact against the oracle's explicit mask."""
    rng = np.random.default_rng(2026)
    for case in range(60):
        H, W = (int(x) for x in rng.integers(1, 49, 2))
        l = int(rng.integers(1, 21))
        b = int(rng.integers(0, l + 1))
        rho = int(rng.integers(0, 7))
        T = int(rng.choice([0, 1, 3, 127, 128, 129, 300]))
        r = int(rng.choice([-1, -1, 0, 2, 5])) if rho else -1
        halo = [None, 0, 1][case % 3]
        order = [None, 1, 0, None][case % 4]
        p = ffi.Plan(H, W, l, b, rho, T, 2, 64)
        if r >= 0:
            p.set_lr_scope(r)
        if order is not None:
            p.set_lr_order(order)
        if halo is not None:
            p.set_halo(halo)
        info = p.info
        g = O.Geometry(H, W, l, b, rho, T, r, halo_copy=bool(info["halo_copy"]),
                       lr_block=bool(info["lr_block"]))
        what = f"case {case}: H={H} W={W} l={l} b={b} rho={rho} T={T} r={r} halo={halo} order={order}"
        assert (info["N_tot"], info["N_kv"], info["off_lr"]) == (g.N_tot, g.N_kv, g.off_lr), what
        perm, row_ptr, entries = p.export()
        np.testing.assert_array_equal(perm, O.perm_map(g), err_msg=what)
        np.testing.assert_array_equal(p.export_kv(), O.kv_perm_map(g), err_msg=what)
        for t in range(g.N_tot // 128):
            e_ref, m_ref = O.qtile_entries(g, t)
            e_got = entries[row_ptr[t]:row_ptr[t + 1]].view(np.uint32)
            np.testing.assert_array_equal(e_got, e_ref, err_msg=f"{what}, q-tile {t}")
            np.testing.assert_array_equal(p.rowmasks(t, len(e_ref)), m_ref,
                                          err_msg=f"{what}, q-tile {t} masks")
        assert info["useful_pairs"] == O.visible_pair_count(g), what
