// Internal plan representation shared by the host plan builder and the device entry points.
#pragma once

#include <cstdint>
#include <vector>

#include "ultragen.h"

namespace ug {

constexpr int kTile = 128;          // query and key tile edge (rows / columns)
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
  int32_t* item_order = nullptr;   // items by decreasing key-tile count
  float* rope = nullptr;           // [max(H,W)][head_dim/2][2] (cos, sin)
  int32_t* combine = nullptr;      // CombineGroup[]
  int* error = nullptr;            // device error word
  unsigned long long* clock = nullptr;   // launch clock record: launches, cycles, ns; 2 scratch
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
