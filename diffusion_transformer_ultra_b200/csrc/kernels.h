// Argument blocks and launchers of the device kernels (host side includes this).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ug {

// Division of 0 <= n < 2^31 by a fixed divisor d >= 1 as a multiply-high and a shift (the
// round-up method of Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (mulhi(n, m) + n) >> s.  The sum stays below 2^32 because n < 2^31.
struct FastDiv {
  uint32_t d, m, s;
  FastDiv() : d(1), m(0), s(0) {}
  explicit FastDiv(uint32_t div) : d(div), m(0), s(0) {
    while ((1ull << s) < div) ++s;
    m = (uint32_t)((((1ull << 32) * ((1ull << s) - div)) / div) + 1);
  }
#ifdef __CUDACC__
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
#endif
};

struct PermuteArgs {
  const void* in[3];               // q, k, v raster [B, N_raster, heads, D]
  void* out[3];                    // qp [B, heads, N_tot, D]; kp, vp [B, heads, N_kv, D]:
                                   // bf16, or e4m3 bytes for qp and kp when qk8 is set
  int qk8;                         // 1: Q and K stored as e4m3 of x * qk_inv[0 / 1]
  float qk_inv[2];                 // 2^-q_exp, 2^-k_exp
  const int32_t* perm;             // K/V slot -> raster, -1 pad (first N_tot: the Q slots)
  const uint32_t* slot_pos;        // (row_pos << 16) | col_pos per K/V slot
  const float* rope;               // [max(H,W)][D/2][2] (cos, sin)
  int64_t rows_total;              // B * heads * (N_tot + number of halo pad slots)
  int N_tot, N_kv, N_raster, heads;
  FastDiv div_heads, div_rows;     // by heads, by N_tot + number of halo pad slots
  const int32_t* halo_pad;         // halo-block pad slots (rows past N_tot of each (b, h))
  // halo blocks (null when the plan has none): the halo-block copies of window-segment slot
  // off_hr + k are halo_dst[halo_ptr[k] .. halo_ptr[k+1]); the kernel writes them from the same
  // read, and writes only the pad slots of the halo region itself
  const int32_t* halo_ptr;
  const int32_t* halo_dst;
  int off_hr, N_hrp;
  int pair_a0, pair_a01;           // pairs [0,a0) axis 0, [a0,a01) axis 1, rest axis 2
  // index checks of debug builds (ULTRAGEN_DEBUG): the device error word and table sizes
  int* err = nullptr;
  int rope_rows = 0;               // rows of the cos/sin table
  int n_halo_dst = 0;              // halo-copy targets
};

struct UnpermuteArgs {
  const __nv_bfloat16* in;         // [B, heads, N_tot, D]
  void* out;                       // [B, N_raster, heads, D]
  const int32_t* inv_perm;         // raster -> slot
  int64_t rows_total;              // B * N_raster * heads
  int N_tot, N_raster, heads;
  FastDiv div_heads, div_nraster;
};

struct CombineArgs {
  const float* ws;                 // split partials
  __nv_bfloat16* out;              // [B*heads, N_tot, D]
  const int32_t* groups;           // 4 ints per split group: qt0, qt1, ws_first, nsplit
  const int32_t* perm;
  int n_groups, n_ws_head, N_tot, BH;
  int raster = 0;                  // 1: out is raster [B, N_raster, heads, D] (pad rows skipped)
  int N_raster = 0, heads = 1;
};

struct FwdParams {
  const int32_t* items;            // 8 ints per item (per batch-head)
  const int32_t* entries;          // key tile | partial << 31
  const int32_t* mask_off;         // per entry, -1 full
  const uint32_t* mask_pool;       // per partial entry: classes x 4 words
  const int32_t* perm;             // slot -> raster, -1 pad
  __nv_bfloat16* out;              // [B*heads, N_tot, D]
  float* ws;                       // split partials [B*heads][n_ws_head][2][128][D+1]
  int* err;                        // device error word
  int n_items_head;
  int n_long = 0;                  // the first n_long items of each head are long groups
  // work order: 0 head-major -- the long items of every (batch, head) first (item i < n_long *
  // units is item i / units of (batch, head) i % units), then the rest head by head (item
  // n_long * units + i is item n_long + i % (n_items_head - n_long) of (batch, head)
  // i / (n_items_head - n_long)); 1 item-major over item_order, longest first (item i is item
  // item_order[i / units] of (batch, head) i % units), used when a layer has few items per CTA
  int item_major = 0;
  int units = 1;                   // batch * heads of the launch
  const int32_t* item_order = nullptr;
  int total_items;
  int N_tot;                       // Q / O rows per (batch, head)
  int N_kv;                        // K / V rows per (batch, head) in the buffers
  int n_ktiles = 0;                // key tiles the entries may name (the halo blocks' included)
  // gathered halo tiles (halo mode 2; null otherwise): key tiles from halo_tile0 on are the
  // halo blocks' tiles, halo_gtiles per window, assembled from the window segment with the
  // copies of halo_ops (CSR per tile of a block, then one packed word per copy)
  const int32_t* halo_ops = nullptr;
  int halo_tile0 = 0, halo_gtiles = 1, nWh = 1, nWw = 1, n_halo_ops = 0;
  int off_hr;
  int l2;                          // l * l
  int n_ws_head;
  float scale_log2;                // log2(e) / sqrt(D)
  unsigned long long timeout_ns;   // limit of every device-side wait
  int fault = 0;                   // 1: withhold one "S ready" signal (tests the timeout path)
  int raster = 0;                  // 1: out is raster [B, N_raster, heads, D] (pad rows skipped)
  int N_raster = 0, heads = 1;
  int n_entries = 0;               // table sizes for the index checks of debug builds
  int n_mask_words = 0;
  // work counter (2 words, zero between launches; null: round-robin items): word 0 hands out
  // item indices, word 1 counts the CTAs that are done taking them
  int* sched = nullptr;
  // launch clock record: CTA 0 adds 1, its cycles and its nanoseconds to words 0-2, keeping
  // its start in words 3-4 (null: not recorded)
  unsigned long long* clock = nullptr;
};

// Device error codes shared by the kernels and the host (ultragen_sync_status): the bounded
// waits write DEV_TIMEOUT_* (ptx.cuh); the index checks of debug builds write DEV_BOUNDS.
constexpr int DEV_BOUNDS = 0x105;

struct WarmArgs {
  const float* lr;                 // [planes, h, w] low-resolution latent
  const float* noise;              // [planes, H, W] X_T, or null: drawn in the kernel
  float* out;                      // [planes, H, W]
  int planes, h, w, H, W;          // planes = batch * channels
  float sy, sx;                    // h / H, w / W in fp32
  float alpha, amount;             // blend weight of the noise, unsharp-mask amount
  unsigned long long seed, offset; // Philox key and the high counter words
  int vec;                         // 1: W % 4 == 0 and 16-byte aligned noise / out
};

cudaError_t launch_permute_rope(const PermuteArgs& a, int in_dtype, int D, int grid_x,
                                cudaStream_t st);
cudaError_t launch_unpermute(const UnpermuteArgs& a, int out_dtype, int D, int grid_x,
                             cudaStream_t st);
cudaError_t launch_combine(const CombineArgs& a, int D, cudaStream_t st);
// 2D bf16 tensor map [rows, D] with [128 x 64] boxes and the 128-byte swizzle (api.cu).
int make_tmap(CUtensorMap* m, const void* base, uint64_t rows, int D);
// 2D byte tensor map [rows, D] with [128 x 128] boxes and the 128-byte swizzle (api.cu).
int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, int D);
// Streaming multiprocessors of the current device (api.cu).
int sm_count();
cudaError_t launch_warm_start(const WarmArgs& a, cudaStream_t st);
// Launches the block-sparse attention kernel; tensor maps are built by the caller.
// qk8 = 1: tmQ and tmK are byte maps of e4m3 Q and K (D = 128 only).
// Window views of K (0-2) and V (3-5) with the b x l, l x b and b x b piece boxes of the
// gathered halo tiles (unused without them).
struct HaloMaps {
  CUtensorMap m[6];
};
cudaError_t launch_hla_fwd(const void* tmQ, const void* tmK, const void* tmV,
                           const HaloMaps* halo, const FwdParams& p, int D, int qk8, int grid,
                           cudaStream_t st);

}  // namespace ug
