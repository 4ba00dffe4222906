// Internal plan representation shared by the host plan builder and the device entry points.
#pragma once

#include <array>
#include <cstdint>
#include <vector>

#include "ultragen.h"

namespace ug {

constexpr int kTile = 128;          // query and key tile edge (rows / columns)
constexpr int kPlanSMs = 148;       // streaming multiprocessors the split policy plans for

// One piece of a window's halo block (R18): rows [di, di + nr) x cols [dj, dj + nc) relative
// to the window's top-left token, stored in raster order from slot `off` of the block.
struct HaloPiece {
  int di, dj, nr, nc;
  int64_t off;
};

// The eight pieces in block order -- top, bottom (b x l), left, right (l x b), top-left,
// top-right, bottom-left, bottom-right (b x b) -- each from the next multiple of 8 slots; a
// piece of at most 128 slots does not cross a multiple of 128 (a longer one starts on one).
inline std::array<HaloPiece, 8> halo_pieces(int l, int b) {
  const int sh[8][4] = {{-b, 0, b, l}, {l, 0, b, l}, {0, -b, l, b}, {0, l, l, b},
                        {-b, -b, b, b}, {-b, l, b, b}, {l, -b, b, b}, {l, l, b, b}};
  std::array<HaloPiece, 8> out{};
  int64_t off = 0;
  for (int k = 0; k < 8; ++k) {
    const int64_t n = (int64_t)sh[k][2] * sh[k][3];
    off = (off + 7) / 8 * 8;
    if ((n <= kTile && off / kTile != (off + n - 1) / kTile) || (n > kTile && off % kTile))
      off = (off / kTile + 1) * kTile;
    out[k] = HaloPiece{sh[k][0], sh[k][1], sh[k][2], sh[k][3], off};
    off += n;
  }
  return out;
}

// Slots of a halo block: its pieces, padded to a multiple of 128.
inline int64_t halo_block_slots(int l, int b) {
  const HaloPiece q = halo_pieces(l, b)[7];
  return (q.off + (int64_t)q.nr * q.nc + kTile - 1) / kTile * kTile;
}

// Whether the attention can assemble the halo tiles itself from the window-first K/V (halo
// mode 2): every piece fits one tile and starts, ends and leaves gaps on multiples of b * b
// rows (8 at least), so that each piece is one TMA box landing on a 1 KB boundary of the
// 128-byte-swizzled slot and the gaps can be zero-filled with b x b boxes; box sides up to 256.
inline bool halo_gather_supported(int l, int b, int qk_format) {
  (void)qk_format;
  if (b < 1 || b >= l || l > 256 || (int64_t)b * b % 8 != 0) return false;
  const std::array<HaloPiece, 8> pc = halo_pieces(l, b);
  const int64_t unit = (int64_t)b * b;
  for (const HaloPiece& q : pc) {
    const int64_t n = (int64_t)q.nr * q.nc;
    if (n > kTile || q.off % unit || n % unit) return false;
  }
  return true;
}

// Copy lists of gathered halo tiles (halo mode 2).  The first G/128 + 1 words bound each tile's
// copies (CSR, indices into the same array); a copy is one word: its first row in the tile
// (bits 0-6), box shape (7-8: 0 b x l, 1 l x b, 2 b x b), zero fill (9), source window offset
// plus one in rows (10-11) and columns (12-13), and the box's first local row (14-21) and
// column (22-29) in that window.  Together a tile's copies cover its 128 rows exactly: the
// gaps between pieces and after the last are zero-filled boxes.
inline std::vector<int32_t> halo_gather_ops(int l, int b) {
  const std::array<HaloPiece, 8> pc = halo_pieces(l, b);
  const int64_t G = halo_block_slots(l, b);
  const int gt = (int)(G / kTile);
  const auto word = [](int row, int shape, int zero, int dwr, int dwc, int i0, int j0) {
    return (int32_t)((uint32_t)row | (uint32_t)shape << 7 | (uint32_t)zero << 9 |
                     (uint32_t)(dwr + 1) << 10 | (uint32_t)(dwc + 1) << 12 |
                     (uint32_t)i0 << 14 | (uint32_t)j0 << 22);
  };
  std::vector<std::vector<int32_t>> tiles(gt);
  // zero boxes over rows [r0, r1) of tile t: b x l boxes while they fit, then b x b
  const auto fill = [&](int t, int r0, int r1) {
    while (r0 < r1) {
      const int shape = r1 - r0 >= b * l ? 0 : 2;
      tiles[t].push_back(word(r0, shape, 1, 0, 0, 0, 0));
      r0 += shape == 0 ? b * l : b * b;
    }
  };
  std::vector<int> cursor(gt, 0);
  for (int k = 0; k < 8; ++k) {
    const HaloPiece& q = pc[k];
    const int t = (int)(q.off / kTile), r = (int)(q.off % kTile);
    fill(t, cursor[t], r);
    const int dwr = q.di < 0 ? -1 : (q.di >= l ? 1 : 0);
    const int dwc = q.dj < 0 ? -1 : (q.dj >= l ? 1 : 0);
    tiles[t].push_back(word(r, k < 2 ? 0 : (k < 4 ? 1 : 2), 0, dwr, dwc, q.di - dwr * l,
                            q.dj - dwc * l));
    cursor[t] = r + q.nr * q.nc;
  }
  for (int t = 0; t < gt; ++t) fill(t, cursor[t], kTile);
  std::vector<int32_t> out(gt + 1);
  for (int t = 0; t < gt; ++t) {
    out[t] = (int32_t)out.size();
    out.insert(out.end(), tiles[t].begin(), tiles[t].end());
  }
  out[gt] = (int32_t)out.size();
  return out;
}
constexpr int kItemInts = 8;        // int32 fields per work item

// SEG_HALO: a K/V slot of a window's compact halo block
enum Seg : int8_t { SEG_PAD = -1, SEG_TEXT = 0, SEG_HR = 1, SEG_LR = 2, SEG_HALO = 3 };

// One unit of kernel work for one (batch, head): one or two query tiles that share the same
// key-tile list and masks, over a contiguous range of that list.
//   [0] qtile0   [1] qtile1 (-1: single tile)   [2] entry begin   [3] entry end
//   [4] workspace slot (-1: write the output directly)   [5] row classes C of qtile0
//   [6] first window of qtile0 (HR tiles) or -1   [7] unused
struct Item {
  int32_t v[kItemInts];
};

// A query group whose key list is split: partials of its nsplit items are merged.
struct CombineGroup {
  int32_t qtile0, qtile1, ws_first, nsplit;
};

struct DeviceTables {
  int device = -1;
  bool valid = false;
  int32_t* items = nullptr;
  int32_t* entries = nullptr;
  int32_t* mask_off = nullptr;
  uint32_t* mask_pool = nullptr;
  int32_t* perm = nullptr;         // K/V slot -> raster over N_kv (its first N_tot: Q slots)
  int32_t* inv_perm = nullptr;
  uint32_t* slot_pos = nullptr;    // (pos_row << 16) | pos_col per K/V slot; 0 for text/pad
  int32_t* halo_ptr = nullptr;     // halo-block copies of each window-segment slot (CSR)
  int32_t* halo_dst = nullptr;
  int32_t* halo_pad = nullptr;     // pad slots of the halo blocks
  int32_t* halo_ops = nullptr;     // gathered halo tiles: per-tile copy lists (halo_gather_ops)
  int32_t* item_order = nullptr;   // items by decreasing key-tile count
  float* rope = nullptr;           // [max(H,W)][head_dim/2][2] (cos, sin)
  int32_t* combine = nullptr;      // CombineGroup[]
  int* error = nullptr;            // device error word
  unsigned long long* clock = nullptr;   // launch clock record: launches, cycles, ns; 2 scratch
  int* sched = nullptr;            // the attention's work counter (2 words, zero between launches)
  float* ws = nullptr;             // split partials
  size_t ws_bytes = 0;
};

}  // namespace ug

struct ultragen_plan {
  // arguments
  int H, W, l, b, rho, T, heads, D;
  // geometry
  int nWh, nWw, h, w;
  int64_t N_hr, N_lr, N_hrp, off_hr, off_lr, N_tot, N_raster;
  int n_qtiles;
  // rope
  int axes[3];
  double theta;
  // split policy (-1 auto, 0 off, >0 chunk) and the chunk in effect
  int split_req = -1;
  int split_chunk = 0;
  // HR -> LR scope: -1 all LR tokens; r >= 0 the anchors within r of the query's window
  int lr_radius = -1;
  // compact halo blocks in the K/V layout: requested (-1 auto, 0 off, 1 on) and in effect;
  // G K/V slots per window, N_kv = N_tot + nWh * nWw * G
  int halo_req = -1;
  int halo_copy = 0;
  // LR segment order: requested (-1 auto, 0 raster, 1 blocks of 8 x 16 LR tokens) and in effect
  // (blocks only with the LR-region scope)
  int lr_order_req = -1;
  int lr_block = 0;
  int64_t G = 0, N_kv = 0, off_halo = 0;
  // rows per (batch, head) of the K/V buffers: N_kv, or N_tot when the attention gathers the
  // halo tiles itself (halo_copy == 2)
  int64_t kv_rows = 0;
  // format of the permuted Q and K: ULTRAGEN_QK_BF16, or ULTRAGEN_QK_E4M3 with the stored
  // values x * 2^-q_exp (Q) and x * 2^-k_exp (K)
  int qk_format = 0;
  int q_exp = 0, k_exp = 0;
  // diagnostics: device wait limit and injected fault (ultragen_plan_set_diagnostics)
  unsigned long long wait_limit_ns = 2000ull * 1000 * 1000;
  int fault = 0;
  // launch clock record (ultragen_plan_set_clock_record)
  int clock_record = 0;

  // host tables
  std::vector<int32_t> perm;       // K/V slot -> raster (-1 pad), N_kv long; Q slots are its
                                   // first N_tot entries
  std::vector<int32_t> inv_perm;   // raster -> slot (the window segment copy)
  std::vector<int8_t> seg;         // per K/V slot
  std::vector<int32_t> ci, cj;     // per K/V slot coordinates (HR: i,j; LR: m,n; text: t,0)
  std::vector<int32_t> owner;      // per K/V slot: window of an HR or halo slot, else -1
  std::vector<uint32_t> slot_pos;  // per K/V slot packed RoPE positions
  std::vector<int32_t> halo_ops;   // gathered halo tiles (halo_copy == 2): halo_gather_ops(l, b)
  std::vector<int32_t> halo_ptr;   // halo blocks: CSR over window-segment slots (N_hrp + 1) of
  std::vector<int32_t> halo_dst;   //   the halo-block slots that copy the slot's token
  std::vector<int32_t> halo_pad;   // halo-block slots that hold no token (written as zeros)
  std::vector<int32_t> item_order; // item indices by decreasing key-tile count (stable)
  std::vector<int32_t> row_ptr;    // CSR over query tiles
  std::vector<int32_t> entries;    // key tile | partial << 31
  std::vector<int32_t> mask_off;   // per entry: offset into mask_pool, -1 when full
  std::vector<uint32_t> mask_pool; // per partial entry: C classes x 4 words
  std::vector<int32_t> qt_classes; // per query tile: C
  std::vector<int32_t> qt_wfirst;  // per query tile: first window (HR) or -1
  std::vector<int32_t> qt_real;    // per query tile: real rows
  int64_t useful_pairs = 0;
  int64_t n_partial = 0;

  // schedule
  std::vector<ug::Item> items;               // per (batch, head)
  std::vector<ug::CombineGroup> combine;     // split groups
  int n_split_items = 0;
  int n_long_items = 0;            // items[0, n_long_items): long groups, longest first

  // device
  ug::DeviceTables dev;
  bool dirty = true;
  int last_launches = 0;
};

namespace ug {
// Builds every host table of `p` from its arguments (plan.cpp).
int build_tables(ultragen_plan_t* p);
// Rebuilds the schedule (pairing, splitting) from the tile lists (plan.cpp).
void build_schedule(ultragen_plan_t* p);
// Fills the RoPE table on the host: [max(H,W)][D/2][2] (cos, sin) floats (plan.cpp).
std::vector<float> rope_table(const ultragen_plan_t* p);

// Device-side launch helpers shared by the entry points (api.cu).  They take the number of
// (batch, head) units and the raster head count explicitly, so a caller can run a slice of the
// heads; the plan's tables must already be on the current device.
int ensure_device_tables(ultragen_plan_t* p);
size_t split_workspace_bytes(const ultragen_plan_t* p, int64_t units);
int launch_permute(const ultragen_plan_t* p, const void* q, const void* k, const void* v,
                   int in_dtype, void* qp, void* kp, void* vp, int batch, int heads,
                   ultragen_stream_t s);
int launch_attention(const ultragen_plan_t* p, const void* qp, const void* kp, const void* vp,
                     void* op, int units, int heads, int raster, float* ws, ultragen_stream_t s,
                     int* launches);
}  // namespace ug
