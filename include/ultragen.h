/*
 * ultragen.h -- C ABI of the B200 (sm_100a) hot path of UltraGen's hierarchical local
 * attention (HLA): window-first permuted, block-masked multi-head attention of one MMDiT
 * layer over the joint sequence [C_T; X; X_lr].
 *
 * Sources (page title, then section):
 *   [UG-note] "UltraGen: Efficient Ultra-High-Resolution Image Generation with Hierarchical
 *             Local Attention", papernotes.org note (ECCV 2026), 方法详解 / 关键设计 1-3.
 *   [UG-gist] same title, gist.science summary of arXiv 2510.16325, "2. Methodology" A-B.
 *
 * Conventions shared by every call
 *   - Every function returns an int status (ULTRAGEN_OK or an ULTRAGEN_ERR_* code); no C++
 *     exception crosses this boundary.  Argument errors are reported before any work.
 *   - Device pointers are CUDA global-memory pointers of the current device, contiguous,
 *     16-byte aligned.  The caller owns every tensor; the plan owns its own tables.
 *   - "stream" is a cudaStream_t (0 = legacy default stream).  Device calls are
 *     asynchronous on that stream; errors raised by a kernel while it runs (a wait that
 *     timed out) are read back by ultragen_sync_status().
 *   - A plan is not thread-safe: do not use one plan from two host threads or on two
 *     streams at once (its device tables, split workspace and work counter are shared by its
 *     calls).  The first device call on a plan uploads its tables with a synchronous copy;
 *     make that call before any stream capture.
 *   - A plan's device tables live on one device at a time: a device call on another current
 *     device frees them and uploads them there.  A process that drives several GPUs at once
 *     keeps one plan per device.
 *
 * Sequence layout (the "permuted" layout; where the pages leave it open, the plainest reading):
 *   slots [0, T) text | pad to a multiple of 128 | HR tokens window-first (windows row-major,
 *   l*l slots each, raster order inside; a partial edge window holds its tokens first, in
 *   raster order of its part inside the image, then pad slots) | pad to 128 |
 *   LR tokens raster, or in 8 x 16 blocks of the LR grid (ultragen_plan_set_lr_order) |
 *   pad to 128.   N_tot = number of slots, a multiple of 128.
 *   K/V slots: the same N_tot slots, then, when the plan uses compact halo blocks
 *   (ultragen_plan_set_halo), one block of G slots per window holding that window's halo
 *   tokens; N_kv = N_tot + nWh * nWw * G (N_kv = N_tot without blocks).  The K/V buffers hold
 *   kv_rows rows per (batch, head): N_kv when the permute copies the blocks, N_tot when the
 *   attention gathers them (ultragen_plan_info).  Q and O use N_tot.
 *   Raster layout: tokens ordered text, HR raster (row i, column j), LR raster.
 */
#ifndef ULTRAGEN_H
#define ULTRAGEN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                       /* cudaStream_t is struct CUstream_st* */
typedef struct CUstream_st* ultragen_stream_t;

enum ultragen_status {
  ULTRAGEN_OK = 0,
  ULTRAGEN_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size         */
  ULTRAGEN_ERR_UNSUPPORTED = 2,   /* head_dim not 64/128, b > l, sizes past int32 limits */
  ULTRAGEN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed                   */
  ULTRAGEN_ERR_OOM = 4,           /* device allocation failed                            */
  ULTRAGEN_ERR_TIMEOUT = 5,       /* a device-side wait ran past its limit               */
  ULTRAGEN_ERR_PLAN_MISMATCH = 6, /* plan built for another shape / device               */
  ULTRAGEN_ERR_NO_DEVICE = 7,     /* no sm_100 device is current                         */
  ULTRAGEN_ERR_BOUNDS = 8         /* a debug build (ULTRAGEN_DEBUG) found a plan index or
                                     tile coordinate outside its table or tensor             */
};

enum ultragen_dtype { ULTRAGEN_BF16 = 0, ULTRAGEN_F32 = 1 };

/* Storage of the permuted Q and K (ultragen_plan_set_qk_format). */
enum ultragen_qk_format { ULTRAGEN_QK_BF16 = 0, ULTRAGEN_QK_E4M3 = 1 };
#define ULTRAGEN_QK_EXP_MAX 32   /* |q_exp|, |k_exp| <= this */

typedef struct ultragen_plan ultragen_plan_t;   /* opaque, owned by the library */

typedef struct {
  int32_t H, W, l, b, rho, text_len, heads, head_dim;
  int32_t nWh, nWw;           /* windows per column / per row: ceil(H/l), ceil(W/l)   */
  int32_t h, w;               /* LR grid: ceil(H/rho), ceil(W/rho); 0 when rho = 0      */
  int64_t N_raster;           /* text_len + H*W + h*w                                   */
  int64_t N_tot;              /* slots in the permuted layout                           */
  int64_t off_hr, off_lr;     /* first slot of the HR and LR segments                   */
  int32_t n_qtiles;           /* N_tot / 128                                            */
  int32_t n_items;            /* work items per (batch, head) after pairing/splitting   */
  int64_t n_entries;          /* tile-list entries (all query tiles)                    */
  int64_t n_partial;          /* entries that need per-element masking                  */
  int64_t useful_pairs;       /* visible (query, key) pairs of one head                 */
  int32_t rope_axes[3];       /* RoPE dims per axis (text/time, row, column)            */
  double rope_theta;
  int32_t split_chunk;        /* key tiles per split of a long query group (0 = none)   */
  int32_t n_split_groups;     /* query groups whose key list is split                   */
  int32_t n_split_items;      /* items that write split partials (per head)             */
  int64_t workspace_bytes_per_head; /* split partial storage per (batch, head)          */
  int32_t lr_radius;          /* HR -> LR scope (ultragen_plan_set_lr_scope)            */
  int32_t halo_copy;          /* halo blocks (ultragen_plan_set_halo): 0 none, 1 copied by
                                 the permute, 2 gathered by the attention              */
  int32_t halo_slots_per_window; /* G: slots of one window's halo block (0 without)      */
  int64_t N_kv;               /* K/V slots the tile lists address: N_tot + nWh * nWw * G */
  int64_t off_halo;           /* first halo-block slot (= N_tot)                         */
  int32_t qk_format;          /* ULTRAGEN_QK_BF16 or ULTRAGEN_QK_E4M3                    */
  int32_t q_exp, k_exp;       /* e4m3 scale exponents (0 for bf16)                       */
  int32_t lr_block;           /* 1: LR segment in 8 x 16 blocks (ultragen_plan_set_lr_order) */
  int64_t kv_rows;            /* rows per (batch, head) of the K/V buffers: N_kv, or N_tot
                                 when the attention gathers the halo blocks (halo_copy 2) */
  int32_t n_halo_ops;         /* words of ultragen_plan_export_halo_ops (0 without gathering) */
  int32_t n_long_items;       /* work items of a head that are long groups, handed out first */
} ultragen_plan_info_t;

/* Human-readable name of a status code.  Never NULL. */
const char* ultragen_status_string(int status);

/*
 * ultragen_plan -- build the per-shape plan on the host: window geometry
 * ([UG-note] 关键设计 1: l x l windows, ceil(H/l) ceil(W/l) of them), the window-first
 * permutation, the block-sparse tile lists of the mask M ([UG-note] 关键设计 2, last
 * paragraph; [UG-gist] 2.B "Attention Masking"), the RoPE tables with LR positions scaled
 * by rho ([UG-note] 关键设计 2, (m,n) -> (rho m, rho n)), and the kernel schedule.
 *   H, W      HR latent rows / columns (>= 1)
 *   l         window side in latent tokens (>= 1)
 *   b         halo width in tokens, 0 <= b <= l: an HR query sees HR keys inside its
 *             window's box grown by b on each side, clipped to the image
 *   rho       LR scale (>= 1), or 0 for no LR segment; LR grid is ceil(H/rho) x ceil(W/rho)
 *   text_len  text tokens (>= 0)
 *   heads     attention heads (>= 1);  head_dim  64 or 128
 *   out       receives the plan; release it with ultragen_plan_destroy
 * Host-only: needs no GPU.  Errors: INVALID_ARG, UNSUPPORTED, OOM (host).
 */
int ultragen_plan(int H, int W, int l, int b, int rho, int text_len, int heads,
                  int head_dim, ultragen_plan_t** out);

/* RoPE split (ax0 + ax1 + ax2 == head_dim, each even) and base theta (> 0).
 * Default: head_dim 64 -> (16,24,24), 128 -> (16,56,56); theta 1e4.  Axis 0 always has
 * position 0; axis 1 takes the row (rho*m for LR), axis 2 the column (rho*n for LR). */
int ultragen_plan_set_rope(ultragen_plan_t* plan, int ax0, int ax1, int ax2, double theta);

/* Split long query groups' key lists into chunks of `chunk` key tiles, merged by a
 * log-sum-exp combine.  chunk = 0: never split.  chunk = -1: automatic (the default): no
 * split when the longest group fits one streaming multiprocessor's share of a layer of one
 * batch element (longest * 148 <= key-tile steps of all heads), since the attention hands
 * out work items longest first from a counter; otherwise chunk = the longest HR/LR group,
 * applied to groups at least 1.5x longer. */
int ultragen_plan_set_split(ultragen_plan_t* plan, int chunk);

/* Scope of the LR tokens an HR query sees.  radius = -1 (default): all LR tokens, the
 * reading of [UG-gist] 2.B ("the scaled global guidance tokens").  radius = r >= 0: the
 * "corresponding" anchors of [UG-note] 关键设计 2 (and the German summary's "entsprechenden
 * skalierten Regionen"): LR token (m, n) is visible to the HR queries of window (wr, wc) iff
 * (rho m, rho n) lies in [wr l - r, (wr+1) l + r) x [wc l - r, (wc+1) l + r).  Rebuilds the
 * tile lists; rope and split settings are kept.  INVALID_ARG for radius < -1. */
int ultragen_plan_set_lr_scope(ultragen_plan_t* plan, int radius);

/* Order of the LR segment in the permuted layout (no counterpart in the pages; the attention is
 * the same function).  mode = 0: raster order over the LR grid (h x w), padded to 128.  mode = 1:
 * blocks of 8 LR rows x 16 columns, one 128-slot tile each, row-major over the grid, raster order
 * inside a block (LR token (m, n) at off_lr + ((m/8) * ceil(w/16) + n/16) * 128 + (m%8) * 16 +
 * n%16; edge blocks keep pad slots), so the LR region an HR window sees under
 * ultragen_plan_set_lr_scope falls into a few dense tiles.  mode = -1 (the default): blocks when
 * they give fewer tile-list entries.  Blocks apply only with an LR-region scope (radius >= 0);
 * with all LR tokens visible the order stays raster.  Rebuilds the tile lists; may change
 * N_tot.  INVALID_ARG for another mode. */
int ultragen_plan_set_lr_order(ultragen_plan_t* plan, int mode);

/* Compact halo blocks in the K/V layout (no counterpart in the pages; the attention is the
 * same function).  Window w's halo -- the HR tokens of its box grown by b ([UG-note] 关键设计 1/2,
 * "adjacent boundary tokens"), outside the window itself -- forms K/V slots
 * [off_halo + w*G, off_halo + (w+1)*G) in eight pieces: the top and bottom strips (b x l), the
 * left and right strips (l x b) and the four corners (b x b), each in raster order from the
 * next multiple of 8 slots, a piece of at most 128 slots never crossing a multiple of 128;
 * piece positions outside the image are pad slots, and G is the pieces' length padded to 128.
 * An HR query of window w then reads its neighbours' tokens from that one dense block instead
 * of partial tiles of up to 8 neighbouring windows; nothing else sees the blocks.
 *   mode 1: ultragen_permute_rope copies the blocks into the K/V buffers (kv_rows = N_kv).
 *   mode 2: the blocks stay virtual: the attention assembles each halo tile itself with one
 *           tile copy per piece from the neighbours' window-first slots (kv_rows = N_tot, no
 *           copies).  It needs whole windows (H and W multiples of l), every piece within
 *           one tile, and pieces, gaps and offsets on multiples of b*b slots (at least 8),
 *           b < l <= 256 (e.g. l = 16 with b = 4 or 8); ULTRAGEN_ERR_UNSUPPORTED otherwise.
 *   mode 0: no blocks.  mode -1 (the default): mode 2 when it is possible and saves tile steps,
 *           else mode 1 when the steps saved outweigh the copies (e.g. b = 4 with l = 16), else
 *           none (always none for b = 0, and when the neighbours' tiles are all fully visible,
 *           e.g. b = l).
 * Rebuilds the tile lists; changes N_kv and kv_rows.  INVALID_ARG for another mode. */
int ultragen_plan_set_halo(ultragen_plan_t* plan, int mode);

/* Storage format of the permuted Q and K, and so the precision of the logits Q K^T (no
 * counterpart in the pages, which only place the permuted layout next to SageAttention's
 * tiling, [UG-note] 关键设计 1).
 *   format ULTRAGEN_QK_BF16 (the default): bf16 Q and K, bf16 tensor-core products.
 *   format ULTRAGEN_QK_E4M3: ultragen_permute_rope stores each RoPE'd element x of Q as the
 *     e4m3 byte nearest to x * 2^-q_exp (of K: x * 2^-k_exp), ties to even, saturating at
 *     +-448 (cvt.rn.satfinite); the attention forms Q K^T from those bytes with 8-bit
 *     tensor-core products (tcgen05 kind::f8f6f4, fp32 accumulation) and multiplies the logits
 *     by 2^(q_exp + k_exp) / sqrt(head_dim).  V, the softmax and P V keep bf16 / fp32.  Choose
 *     the exponents so that |x| * 2^-exp stays below 448 (0 suits RMS-normalised activations).
 * The permuted Q and K buffers then hold one byte per element ([batch, heads, N_tot, D] and
 * [batch, heads, N_kv, D] bytes).  The tile lists do not change.  INVALID_ARG for another
 * format or |exp| > ULTRAGEN_QK_EXP_MAX; UNSUPPORTED for E4M3 with head_dim 64. */
int ultragen_plan_set_qk_format(ultragen_plan_t* plan, int format, int q_exp, int k_exp);

int ultragen_plan_info(const ultragen_plan_t* plan, ultragen_plan_info_t* out);

/*
 * Host copies of the plan's integer tables (caller-allocated host buffers):
 *   perm     [N_tot]       raster index of each permuted slot, -1 for pad slots
 *   row_ptr  [n_qtiles+1]  CSR offsets of each query tile's entries
 *   entries  [n_entries]   key-tile index | (1u << 31 if partial), ascending per tile.
 * An entry exists iff some (real query row, key column) cell of the 128x128 block is
 * visible; it is partial iff some such cell is not.  Any pointer may be NULL to skip it.
 */
int ultragen_plan_export(const ultragen_plan_t* plan, int32_t* perm, int32_t* row_ptr,
                         int32_t* entries);

/* Host copy of the K/V slot map: kv_perm [N_kv], raster index of each K/V slot (its first
 * N_tot entries equal perm; halo-block slots follow), -1 for pad slots.  Entries of the tile
 * lists index K/V tiles of this layout. */
int ultragen_plan_export_kv(const ultragen_plan_t* plan, int32_t* kv_perm);

/* Host copy of the copy lists of gathered halo tiles (halo_copy 2): out [n_halo_ops] int32.
 * Words 0..G/128 bound the copies of each tile of a halo block (indices into out); each copy
 * is one word: bits 0-6 its first row in the tile (a multiple of 8), 7-8 the box (0: b rows
 * x l columns, 1: l x b, 2: b x b tokens), 9 zero fill, 10-11 and 12-13 the source window's
 * offset from the block's window plus one (rows, columns), 14-21 and 22-29 the box's first
 * row and column in that window.  A box lands as its tokens in raster order; a zero box, or
 * one whose window lies outside the image, lands as zeros.  The copies of a tile cover its
 * 128 rows exactly once.  n_halo_ops is 0 without gathered tiles (nothing is written). */
int ultragen_plan_export_halo_ops(const ultragen_plan_t* plan, int32_t* out);

/* Host copy of the attention's work items of one (batch, head), in the order the head-major
 * work order takes them: out [n_items][8] int32 with, per item, its query tiles qt0 and qt1
 * (-1: a single tile), the range [e0, e1) of entries of qt0's tile list it covers (qt1's list
 * is identical), its split-partial slot (-1: unsplit, written straight to the output), the
 * number of row classes of qt0 and the first window of qt0 (-1 outside the window segment), and
 * 0.  The first n_long_items items are the long groups, longest first; the split items follow;
 * then the rest in query-tile order.  No counterpart in the pages (a schedule). */
int ultragen_plan_export_items(const ultragen_plan_t* plan, int32_t* out);

/* Per-row visibility of query tile `qtile`: out[e][r][w] (uint32) for each of the tile's
 * entries e, rows r in [0,128), words w in [0,4); bit c%32 of word c/32 = key column c of
 * the entry's key tile visible to row r.  Rows of pad slots are 0.  `out` holds
 * (row_ptr[qtile+1]-row_ptr[qtile]) * 512 words. */
int ultragen_plan_export_rowmasks(const ultragen_plan_t* plan, int qtile, uint32_t* out);

int ultragen_plan_destroy(ultragen_plan_t* plan);

/*
 * ultragen_permute_rope -- raster -> window-first gather of Q, K, V fused with axial 2D
 * RoPE on Q and K ([UG-note] 关键设计 1 window-first order; 关键设计 2 position scaling).
 *   q, k, v     [batch, N_raster, heads, head_dim], in_dtype BF16 or F32 (device)
 *   qp          [batch, heads, N_tot, head_dim] BF16 (device); pad slots written as 0
 *   kp, vp      [batch, heads, N_kv, head_dim] BF16 (device): the N_tot slots, then the
 *               halo blocks (each halo token's row again, with its own RoPE position)
 * RoPE is computed in fp32 from fp32 tables and rounded to bf16 (nearest even); V and
 * text tokens are copied (F32 input: rounded to bf16).  With the plan's Q/K format set to
 * ULTRAGEN_QK_E4M3, qp and kp receive e4m3 bytes instead: the fp32 RoPE result times
 * 2^-q_exp (2^-k_exp), rounded to nearest even and saturated at +-448; vp stays BF16.
 */
int ultragen_permute_rope(const void* q, const void* k, const void* v, int in_dtype,
                          void* qp, void* kp, void* vp, int batch,
                          const ultragen_plan_t* plan, ultragen_stream_t stream);

/*
 * ultragen_hla_forward -- masked joint attention softmax(Q K^T / sqrt(d) + M) V
 * ([UG-note] 关键设计 3, the MMA equation; M additive -inf on masked pairs) over the
 * permuted layout, visiting only the key tiles of each query tile's list.
 *   qp, op  [batch, heads, N_tot, head_dim] BF16 (device); op rows of pad slots = 0
 *   kp, vp  [batch, heads, N_kv, head_dim] BF16 (device), as ultragen_permute_rope writes them
 * bf16 tensor-core products with fp32 accumulation and fp32 online softmax (with the
 * plan's Q/K format ULTRAGEN_QK_E4M3: qp and kp are e4m3 bytes and Q K^T uses 8-bit
 * products, see ultragen_plan_set_qk_format).  Uses the
 * plan's split workspace (device memory the plan allocates and keeps) when the plan
 * splits groups; a call that needs more than the plan holds grows it with stream-ordered
 * allocation on `stream` (cudaFreeAsync / cudaMallocAsync from the device's default pool),
 * so no call synchronises the device.  Errors: INVALID_ARG, NO_DEVICE, OOM, CUDA.
 */
int ultragen_hla_forward(const void* qp, const void* kp, const void* vp, void* op,
                         const ultragen_plan_t* plan, int batch, ultragen_stream_t stream);

/*
 * ultragen_hla_forward_raster -- ultragen_hla_forward with the unpermute folded into its
 * epilogue: each output row goes straight to its raster place.
 *   qp          [batch, heads, N_tot, head_dim] BF16, or e4m3 bytes (device, permuted)
 *   kp, vp      [batch, heads, N_kv, head_dim] BF16 (kp: e4m3 bytes with the E4M3 Q/K
 *               format) (device, K/V layout)
 *   o           [batch, N_raster, heads, head_dim] BF16 (device, raster); pad slots write nothing
 * Same arithmetic as ultragen_hla_forward + ultragen_unpermute (bit for bit), one pass less
 * over HBM.  Errors as ultragen_hla_forward.
 */
int ultragen_hla_forward_raster(const void* qp, const void* kp, const void* vp, void* o,
                                const ultragen_plan_t* plan, int batch, ultragen_stream_t stream);

/*
 * ultragen_unpermute -- window-first -> raster: o[b, t, h, :] = op[b, h, slot(t), :].
 *   op  [batch, heads, N_tot, head_dim] BF16 (device)
 *   o   [batch, N_raster, heads, head_dim], out_dtype BF16 (bit copy) or F32 (device)
 */
int ultragen_unpermute(const void* op, void* o, int out_dtype, int batch,
                       const ultragen_plan_t* plan, ultragen_stream_t stream);

/*
 * ultragen_hla_forward_noalloc -- the same attention as ultragen_hla_forward, for callers that
 * cannot allocate device memory when they call it: code running while a framework's caching
 * allocator owns the whole device, real-time loops that must not hit cudaMalloc's implicit
 * synchronisation, or processes held to a fixed memory budget.  The pages have no counterpart
 * of this call; it exists for those callers only.
 *   Arguments, layouts and results are those of ultragen_hla_forward.
 *   It calls no cudaMalloc, cudaFree or other allocating routine.  The split partials live in
 *   one file-scope device array of ULTRAGEN_NOALLOC_SCRATCH_BYTES that every GPU which loads
 *   the library holds until the process exits.  No part of it needs to start at zero (each
 *   partial the merge reads is written earlier in the same call), it keeps the last call's
 *   contents, and all calls share it: calls that overlap on the GPU (two streams, two
 *   threads) race on it and give wrong results.
 *   The first call on a device (and the first after that device's CUDA context was created
 *   again, e.g. after cudaDeviceReset) looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   The plan's tables must already be on the current device: any earlier device call with
 *   this plan (e.g. ultragen_permute_rope) uploads them; otherwise ULTRAGEN_ERR_PLAN_MISMATCH.
 *   ULTRAGEN_ERR_UNSUPPORTED when batch * heads * workspace_bytes_per_head (see
 *   ultragen_plan_info) exceeds ULTRAGEN_NOALLOC_SCRATCH_BYTES; a larger split chunk
 *   (ultragen_plan_set_split) or no split (0) lowers it.
 */
#define ULTRAGEN_NOALLOC_SCRATCH_BYTES (64u << 20)
int ultragen_hla_forward_noalloc(const void* qp, const void* kp, const void* vp, void* op,
                                 const ultragen_plan_t* plan, int batch, ultragen_stream_t stream);

/* Wait for `stream`, then report (and clear) a device-side error raised by this plan's
 * kernels since the last call: ULTRAGEN_ERR_TIMEOUT if a wait ran out, ULTRAGEN_ERR_BOUNDS if a
 * debug build's index check stopped a kernel. */
int ultragen_sync_status(const ultragen_plan_t* plan, ultragen_stream_t stream);

/* Diagnostics (no counterpart in the pages).  wait_limit_s (1 ms .. 60 s, default 2 s) bounds
 * every device-side wait of the attention kernel (ultragen_hla_forward, _raster, _noalloc and
 * the host runner); past it the kernel stops cleanly and
 * ultragen_sync_status reports ULTRAGEN_ERR_TIMEOUT.  fault = 1 makes the MMA warp of every
 * CTA withhold one "S ready" signal, so a wait runs out on purpose (tests of that path);
 * fault = 0 is normal operation.  INVALID_ARG outside these ranges. */
int ultragen_plan_set_diagnostics(ultragen_plan_t* plan, int fault, double wait_limit_s);

/* Launch clock record (no counterpart in the pages; measurement support).  With on = 1, every
 * attention launch of this plan adds, from its first CTA (which lives for the whole persistent
 * launch), the SM cycles (clock64) and the nanoseconds (globaltimer) from that CTA's start to
 * the issue of its last tensor-core product (the last item's epilogue, a few thousand cycles of
 * millions, is left out) to a small device record that the plan owns; on = 0 stops recording.
 * Cycles over nanoseconds is the SM clock the kernel actually ran at, which under a power cap
 * can be well below what a driver query reports.  The record is uploaded with the plan's tables
 * (any device call).  INVALID_ARG for a null plan or on not 0/1. */
int ultragen_plan_set_clock_record(ultragen_plan_t* plan, int on);

/* Copies the record to out[3] = {launches, cycles, nanoseconds} summed since the last read,
 * then clears it.  Host, synchronous (cudaMemcpy: it waits for the device); call it after the
 * launches of interest completed.  All zeros when the plan has no tables on the device yet. */
int ultragen_plan_read_clock(const ultragen_plan_t* plan, uint64_t out[3]);

/* Kernel launches the last device call of this plan issued (for launch accounting). */
int ultragen_last_launch_count(const ultragen_plan_t* plan);

/*
 * Host-buffer runner -- the whole layer for Q/K/V and O in HOST memory, with the PCIe copies
 * overlapped with the kernels (no counterpart in the pages; it serves callers whose
 * activations live on the host).  The heads are independent problems, so the layer runs as
 * units of (batch element, heads_per_chunk heads): each unit's slice is copied in with one 2D
 * copy per tensor, permuted and attended exactly as ultragen_permute_rope +
 * ultragen_hla_forward_raster would (the same kernels, bit for bit), and copied out, while the
 * next unit's copy-in and the previous unit's copy-out proceed on their own streams.
 *
 * ultragen_host_runner_create(plan, batch, heads_per_chunk, &runner)
 *   Allocates every device buffer the runner needs: double-buffered staging for 3 inputs and
 *   1 output of one unit (2 x 4 x N_raster x heads_per_chunk x head_dim x 2 bytes), permuted
 *   Q/K/V of one unit, split partials of one unit; three streams and their events.  Uploads the
 *   plan's tables.  heads_per_chunk is clamped to the plan's head count.  The plan must outlive
 *   the runner.  INVALID_ARG for a null plan / out, batch < 1, heads_per_chunk < 1;
 *   NO_DEVICE, OOM, CUDA as usual.
 * ultragen_host_runner_forward(runner, q, k, v, o, stream)
 *   q, k, v  [batch, N_raster, heads, head_dim] BF16 in HOST memory (page-locked memory lets
 *            the copies overlap the kernels; pageable memory works, serialised)
 *   o        [batch, N_raster, heads, head_dim] BF16 in HOST memory, written in full
 *   The layer follows the plan's settings at the call (Q/K format, LR scope and order, halo
 *   blocks, split schedule), exactly as the device entry points would.
 *   Asynchronous: the work is ordered after what `stream` holds at the call, and `stream`
 *   waits for all of it, so o is complete once `stream` is synchronised.  Calls on one runner
 *   must not overlap (one call at a time per runner).  PLAN_MISMATCH when called on another
 *   device than the one the runner was created on, or when the plan's split schedule, halo
 *   blocks or LR order now need more storage than was allocated.  Device-side wait timeouts are reported by
 *   ultragen_sync_status(plan, stream).
 * ultragen_host_runner_last_launch_count(runner): kernels the last forward launched.
 * ultragen_host_runner_destroy(runner): waits for the runner's streams, frees everything.
 */
typedef struct ultragen_host_runner ultragen_host_runner_t;   /* opaque */
int ultragen_host_runner_create(ultragen_plan_t* plan, int batch, int heads_per_chunk,
                                ultragen_host_runner_t** out);
int ultragen_host_runner_forward(ultragen_host_runner_t* runner, const void* q, const void* k,
                                 const void* v, void* o, ultragen_stream_t stream);
int ultragen_host_runner_last_launch_count(const ultragen_host_runner_t* runner);
int ultragen_host_runner_destroy(ultragen_host_runner_t* runner);

/*
 * ultragen_warm_start -- warm-start initialisation of the high-resolution latent
 * ([UG-note] 关键设计 4 and its blend equation; [UG-gist] 2.D "Warm-Start Initialization"):
 *     U     = bilinear upsampling of x_lr to H x W: along each axis output index i reads
 *             source coordinate max((i + 1/2) * n_in / n_out - 1/2, 0), taps floor() and the
 *             next index (both clamped to n_in - 1), weighted by the fractional part;
 *     X_ref = U + sharpen * (U - B(U)), B the 3x3 binomial blur (1 2 1)^T (1 2 1) / 16 per
 *             channel with replicated edges (sharpen = 0: plain interpolation);
 *     x_hr  = alpha * X_T + (1 - alpha) * X_ref, alpha = t / T of the starting timestep.
 *   x_lr   [batch, channels, h, w] F32 (device)
 *   noise  [batch, channels, H, W] F32 (device) X_T, or NULL: X_T is drawn in the kernel from
 *          Philox4x32-10 (key = seed, counter = (g, offset) for 4-element block g of the flat
 *          output index) and the Box-Muller transform of the words mapped to
 *          (floor(x / 2^9) + 1/2) * 2^-23; lanes 0..3 of a block are r cos, r sin of words
 *          (0, 1), then of words (2, 3).
 *   x_hr   [batch, channels, H, W] F32 (device), written in full.
 *   Pointers need 4-byte alignment; W % 4 == 0 with 16-byte aligned noise and x_hr takes the
 *   vector path.  INVALID_ARG: null x_lr / x_hr, a size < 1, a non-finite alpha or sharpen,
 *   sharpen < 0.  UNSUPPORTED: batch * channels > 65535 or H > 2,097,120.  Computed in fp32.
 *   One kernel launch; asynchronous on `stream`.
 */
int ultragen_warm_start(const float* x_lr, const float* noise, float* x_hr, int batch,
                        int channels, int h, int w, int H, int W, float alpha, float sharpen,
                        uint64_t seed, uint64_t offset, ultragen_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ULTRAGEN_H */
