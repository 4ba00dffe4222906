// Host plan builder: window geometry, window-first permutation, block-sparse tile lists with
// per-class column masks, RoPE tables and the kernel schedule.
//
// Method (page title, section):
//   "UltraGen: Efficient Ultra-High-Resolution Image Generation with Hierarchical Local
//   Attention" -- papernotes.org note, 关键设计 1 (l x l windows, window-first token order,
//   dense local blocks), 关键设计 2 (LR positions (m,n) -> (rho m, rho n); the mask M:
//   text <-> text + HR, HR -> own window + neighbouring boundary tokens + text + LR,
//   LR -> LR), 关键设计 3 (sequence [C_T; X; X_lr]); gist.science summary, 2.B.
//
// Visibility classes.  Every query row of a query tile belongs to one class: "text", "LR",
// or "HR window w" (all rows of a window share the window's halo box).  A key column is
// visible to a class by the rules above; pad slots are never visible.  For a (query tile,
// key tile) pair the plan stores, per class of the tile, a 128-bit column mask; the kernel
// only applies masks on partial entries.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "nvtx_range.h"
#include "plan_internal.h"

namespace ug {
namespace {

int64_t pad128(int64_t n) { return (n + kTile - 1) / kTile * kTile; }
int cdiv(int a, int b) { return (a + b - 1) / b; }

struct ClassDesc {
  int kind;              // SEG_TEXT, SEG_HR, SEG_LR
  int r0, r1, c0, c1;    // HR halo box [r0, r1) x [c0, c1)
  int lr0, lr1, lc0, lc1;  // scaled LR positions visible to the window (lr_radius >= 0)
  int wid;               // the window (HR classes)
};

inline bool visible(const ultragen_plan_t* p, const ClassDesc& c, int64_t s) {
  const int sg = p->seg[s];
  switch (c.kind) {
    case SEG_TEXT:
      return sg == SEG_TEXT || sg == SEG_HR;
    case SEG_LR:
      return sg == SEG_LR || sg == SEG_TEXT;
    default:
      if (sg == SEG_TEXT) return true;
      if (sg == SEG_LR) {
        if (p->lr_radius < 0) return true;
        const int pm = p->rho * p->ci[s], pn = p->rho * p->cj[s];
        return pm >= c.lr0 && pm < c.lr1 && pn >= c.lc0 && pn < c.lc1;
      }
      // with halo blocks, the window's own segment and its own halo block (R18)
      if (p->halo_copy) return (sg == SEG_HR || sg == SEG_HALO) && p->owner[s] == c.wid;
      if (sg != SEG_HR) return false;
      return p->ci[s] >= c.r0 && p->ci[s] < c.r1 && p->cj[s] >= c.c0 && p->cj[s] < c.c1;
  }
}

ClassDesc window_class(const ultragen_plan_t* p, int wid) {
  const int wr = wid / p->nWw, wc = wid % p->nWw;
  ClassDesc c;
  c.kind = SEG_HR;
  c.wid = wid;
  c.r0 = std::max(0, wr * p->l - p->b);
  c.r1 = std::min(p->H, (wr + 1) * p->l + p->b);
  c.c0 = std::max(0, wc * p->l - p->b);
  c.c1 = std::min(p->W, (wc + 1) * p->l + p->b);
  // the "corresponding" LR region: the window's l x l box grown by lr_radius
  c.lr0 = wr * p->l - p->lr_radius;
  c.lr1 = (wr + 1) * p->l + p->lr_radius;
  c.lc0 = wc * p->l - p->lr_radius;
  c.lc1 = (wc + 1) * p->l + p->lr_radius;
  return c;
}

// LR block of one tile in the block order of the LR segment (R20): 8 LR rows x 16 columns.
constexpr int kLrBH = 8, kLrBW = 16;

// Slot of LR token (m, n): raster order over the LR grid, or block order (blocks of
// kLrBH x kLrBW row-major, raster order inside a block) when the plan takes it.
int64_t lr_slot(const ultragen_plan_t* p, int m, int n) {
  if (!p->lr_block) return p->off_lr + (int64_t)m * p->w + n;
  const int nbw = cdiv(p->w, kLrBW);
  return p->off_lr + ((int64_t)(m / kLrBH) * nbw + n / kLrBW) * kTile + (m % kLrBH) * kLrBW +
         n % kLrBW;
}

void add_range(std::vector<int>& v, int64_t s_begin, int64_t s_end) {
  if (s_end <= s_begin) return;
  for (int64_t t = s_begin / kTile; t <= (s_end - 1) / kTile; ++t) v.push_back((int)t);
}

// Window w's halo block (R18): eight pieces of its grown box outside the window -- the top and
// bottom strips (b x l), the left and right strips (l x b), then the top-left, top-right,
// bottom-left and bottom-right corners (b x b) -- each in raster order, at the slot offsets of
// ug::halo_pieces.  f(slot in the block, i, j, real) for every piece position; positions
// outside the image are pad slots.
template <typename F>
void for_each_halo_slot(const ultragen_plan_t* p, int w, F&& f) {
  const int wr = w / p->nWw, wc = w % p->nWw;
  const std::array<ug::HaloPiece, 8> pc = ug::halo_pieces(p->l, p->b);
  for (const ug::HaloPiece& q : pc) {
    const int i0 = wr * p->l + q.di, j0 = wc * p->l + q.dj;
    for (int a = 0; a < q.nr; ++a)
      for (int c = 0; c < q.nc; ++c) {
        const int i = i0 + a, j = j0 + c;
        f(q.off + (int64_t)a * q.nc + c, i, j, i >= 0 && i < p->H && j >= 0 && j < p->W);
      }
  }
}

int build_tables_mode(ultragen_plan_t* p, int halo, int lr_block);

}  // namespace

// Builds the tables with compact halo blocks on or off; "auto" takes them when the tile-list
// entries they save (one entry = one 128 x 128 tile step of one query tile) outweigh the extra
// permute traffic of the copies (about 3.3 entries per copied 128-row K/V tile: written once
// and read again by the attention).
int build_tables(ultragen_plan_t* p) {
  // LR segment order (R20): blocks only serve the LR-region scope; "auto" takes them when they
  // give fewer tile-list entries (they cost no extra traffic)
  int lrb = 0;
  if (p->lr_radius >= 0 && p->rho > 0 && p->lr_order_req != 0) {
    if (p->lr_order_req == 1) {
      lrb = 1;
    } else {
      int st = build_tables_mode(p, 0, 0);
      if (st) return st;
      const size_t n_raster_order = p->entries.size();
      st = build_tables_mode(p, 0, 1);
      if (st) return st;
      lrb = p->entries.size() < n_raster_order ? 1 : 0;
    }
  }
  if (p->halo_req == 0 || p->b == 0) return build_tables_mode(p, 0, lrb);
  if (p->halo_req == 1) return build_tables_mode(p, 1, lrb);
  // gathered halo tiles read a neighbour's piece as a box of its l x l slots, which needs
  // every window whole (a partial edge window packs its tokens at the front)
  const bool gatherable = ug::halo_gather_supported(p->l, p->b, p->qk_format) &&
                          p->H % p->l == 0 && p->W % p->l == 0;
  if (p->halo_req == 2) {
    if (!gatherable) return ULTRAGEN_ERR_UNSUPPORTED;
    return build_tables_mode(p, 2, lrb);
  }
  int st = build_tables_mode(p, 0, lrb);
  if (st) return st;
  // entries the halo blocks would replace: each HR query tile's neighbour-window tiles give way
  // to its windows' halo tiles
  const int64_t l2 = (int64_t)p->l * p->l;
  const int64_t G = ug::halo_block_slots(p->l, p->b);
  std::vector<int> halo_tiles(p->nWh * p->nWw, (int)(G / kTile));
  int64_t saved = 0;
  for (int t = (int)(p->off_hr / kTile); t < (int)(p->off_lr / kTile); ++t) {
    if (p->qt_wfirst[t] < 0) continue;
    const int wf = p->qt_wfirst[t], C = p->qt_classes[t];
    for (int e = p->row_ptr[t]; e < p->row_ptr[t + 1]; ++e) {
      const int64_t k0 = (int64_t)(p->entries[e] & 0x7fffffff) * kTile;
      if (k0 < p->off_hr || k0 >= p->off_lr) continue;
      const int64_t kw = (k0 - p->off_hr) / l2;
      if (kw < wf || kw >= wf + C) ++saved;                    // another window's tile
    }
    for (int c = 0; c < C; ++c) saved -= halo_tiles[wf + c];
  }
  // gathered halo tiles cost the permute nothing: take them whenever they save entries; copied
  // blocks only when the saved entries outweigh the copies
  const bool gather = gatherable;
  const double copy_tiles = (double)p->nWh * p->nWw * (G / kTile);
  if (gather ? saved > 0 : (double)saved > 3.3 * copy_tiles)
    return build_tables_mode(p, gather ? 2 : 1, lrb);
  return ULTRAGEN_OK;
}

namespace {

int build_tables_mode(ultragen_plan_t* p, int halo, int lr_block) {
  p->nWh = cdiv(p->H, p->l);
  p->nWw = cdiv(p->W, p->l);
  p->h = p->rho > 0 ? cdiv(p->H, p->rho) : 0;
  p->w = p->rho > 0 ? cdiv(p->W, p->rho) : 0;
  p->N_hr = (int64_t)p->H * p->W;
  p->N_lr = (int64_t)p->h * p->w;
  p->N_hrp = (int64_t)p->nWh * p->nWw * p->l * p->l;
  p->off_hr = pad128(p->T);
  p->off_lr = p->off_hr + pad128(p->N_hrp);
  p->lr_block = (lr_block && p->lr_radius >= 0 && p->rho > 0) ? 1 : 0;
  const int nbw = cdiv(p->w, kLrBW);   // LR blocks per block row (R20)
  p->N_tot = p->off_lr + (p->lr_block ? (int64_t)cdiv(p->h, kLrBH) * nbw * kTile : pad128(p->N_lr));
  p->N_raster = p->T + p->N_hr + p->N_lr;
  if (p->N_tot > (int64_t)1 << 30) return ULTRAGEN_ERR_UNSUPPORTED;
  p->n_qtiles = (int)(p->N_tot / kTile);
  const int nW = p->nWh * p->nWw;
  p->halo_copy = halo;
  p->G = halo ? ug::halo_block_slots(p->l, p->b) : 0;
  p->off_halo = p->N_tot;
  p->N_kv = p->N_tot + (int64_t)nW * p->G;
  // gathered halo blocks (mode 2) exist only as tiles the attention assembles: the K/V buffers
  // hold the N_tot window-first slots
  p->kv_rows = halo == 2 ? p->N_tot : p->N_kv;
  if (p->N_kv > (int64_t)1 << 30) return ULTRAGEN_ERR_UNSUPPORTED;

  const int64_t N = p->N_kv;
  p->perm.assign(N, -1);
  p->inv_perm.assign(p->N_raster, -1);
  p->seg.assign(N, SEG_PAD);
  p->ci.assign(N, 0);
  p->cj.assign(N, 0);
  p->owner.assign(N, -1);
  p->slot_pos.assign(N, 0u);

  // window-first permutation ([UG-note] 关键设计 1)
  for (int t = 0; t < p->T; ++t) {
    p->perm[t] = t;
    p->inv_perm[t] = t;
    p->seg[t] = SEG_TEXT;
    p->ci[t] = t;
  }
  const int64_t l2 = (int64_t)p->l * p->l;
  for (int i = 0; i < p->H; ++i) {
    for (int j = 0; j < p->W; ++j) {
      const int64_t win = (int64_t)(i / p->l) * p->nWw + (j / p->l);
      // raster order inside the window's part in the image (rows of cn tokens)
      const int cn = std::min(p->l, p->W - (j / p->l) * p->l);
      const int64_t s = p->off_hr + win * l2 + (int64_t)(i % p->l) * cn + (j % p->l);
      const int64_t r = p->T + (int64_t)i * p->W + j;
      p->perm[s] = (int32_t)r;
      p->inv_perm[r] = (int32_t)s;
      p->seg[s] = SEG_HR;
      p->ci[s] = i;
      p->cj[s] = j;
      p->owner[s] = (int32_t)win;
      p->slot_pos[s] = ((uint32_t)i << 16) | (uint32_t)j;
    }
  }
  // compact halo blocks of K/V (R18): window w's block at off_halo + w * G; with copied blocks
  // (mode 1), for the permute, each window-segment slot's list of halo-block copies (CSR) and
  // the blocks' pad slots
  p->halo_ptr.clear();
  p->halo_dst.clear();
  p->halo_pad.clear();
  p->halo_ops.clear();
  if (halo == 2) p->halo_ops = ug::halo_gather_ops(p->l, p->b);
  if (halo) {
    std::vector<int32_t> count(p->N_hrp + 1, 0);
    for (int w = 0; w < nW; ++w) {
      const int64_t hb = p->off_halo + (int64_t)w * p->G;
      for_each_halo_slot(p, w, [&](int64_t k, int i, int j, bool real) {
        if (!real) return;
        const int64_t s = hb + k, r = p->T + (int64_t)i * p->W + j;
        p->perm[s] = (int32_t)r;
        p->seg[s] = SEG_HALO;
        p->ci[s] = i;
        p->cj[s] = j;
        p->owner[s] = w;
        p->slot_pos[s] = ((uint32_t)i << 16) | (uint32_t)j;
        ++count[p->inv_perm[r] - p->off_hr + 1];
      });
      if (halo == 1)
        for (int64_t k = 0; k < p->G; ++k)
          if (p->perm[hb + k] < 0) p->halo_pad.push_back((int32_t)(hb + k));
    }
    if (halo == 1) {
      for (int64_t k = 0; k < p->N_hrp; ++k) count[k + 1] += count[k];
      p->halo_ptr = count;
      p->halo_dst.assign(count[p->N_hrp], -1);
      std::vector<int32_t> fill(count.begin(), count.end() - 1);
      for (int w = 0; w < nW; ++w) {
        const int64_t hb = p->off_halo + (int64_t)w * p->G;
        for_each_halo_slot(p, w, [&](int64_t k, int i, int j, bool real) {
          if (!real) return;
          const int64_t r = p->T + (int64_t)i * p->W + j;
          p->halo_dst[fill[p->inv_perm[r] - p->off_hr]++] = (int32_t)(hb + k);
        });
      }
    }
  }
  // LR tokens at positions (rho m, rho n) ([UG-note] 关键设计 2)
  for (int m = 0; m < p->h; ++m) {
    for (int n = 0; n < p->w; ++n) {
      const int64_t s = lr_slot(p, m, n);
      const int64_t r = p->T + p->N_hr + (int64_t)m * p->w + n;
      p->perm[s] = (int32_t)r;
      p->inv_perm[r] = (int32_t)s;
      p->seg[s] = SEG_LR;
      p->ci[s] = m;
      p->cj[s] = n;
      p->slot_pos[s] = ((uint32_t)(p->rho * m) << 16) | (uint32_t)(p->rho * n);
    }
  }

  // tile lists
  const int nq = p->n_qtiles;
  p->row_ptr.assign(nq + 1, 0);
  p->entries.clear();
  p->mask_off.clear();
  p->mask_pool.clear();
  p->qt_classes.assign(nq, 1);
  p->qt_wfirst.assign(nq, -1);
  p->qt_real.assign(nq, 0);
  p->useful_pairs = 0;
  p->n_partial = 0;

  const int64_t hr_end = p->off_hr + p->N_hrp;
  std::vector<ClassDesc> classes;
  std::vector<int> class_real;
  std::vector<int> cand;
  std::vector<uint32_t> masks;

  for (int t = 0; t < nq; ++t) {
    const int64_t s0 = (int64_t)t * kTile;
    int kind = s0 < p->off_hr ? SEG_TEXT : (s0 < p->off_lr ? SEG_HR : SEG_LR);
    classes.clear();
    int wfirst = -1;
    if (kind == SEG_HR && s0 < hr_end) {
      wfirst = (int)((s0 - p->off_hr) / l2);
      const int wlast = (int)((std::min<int64_t>(s0 + kTile, hr_end) - 1 - p->off_hr) / l2);
      for (int wid = wfirst; wid <= wlast; ++wid) classes.push_back(window_class(p, wid));
    } else {
      ClassDesc c{kind, 0, 0, 0, 0, 0, 0, 0, 0, -1};
      classes.push_back(c);
      if (kind == SEG_HR) wfirst = -1;   // pad-only tile between HR and LR segments
    }
    const int C = (int)classes.size();
    p->qt_classes[t] = C;
    p->qt_wfirst[t] = wfirst;

    class_real.assign(C, 0);
    int real = 0;
    for (int r = 0; r < kTile; ++r) {
      const int64_t s = s0 + r;
      if (p->perm[s] < 0) continue;
      int c = 0;
      if (wfirst >= 0) c = std::min(C - 1, (int)((s - p->off_hr) / l2) - wfirst);
      class_real[c]++;
      real++;
    }
    p->qt_real[t] = real;
    p->row_ptr[t + 1] = p->row_ptr[t];
    if (real == 0) continue;

    // candidate key tiles
    cand.clear();
    add_range(cand, 0, p->T);
    if (kind == SEG_TEXT) add_range(cand, p->off_hr, hr_end);
    if (kind == SEG_LR || (kind == SEG_HR && p->lr_radius < 0))
      add_range(cand, p->off_lr, p->N_tot);
    if (kind == SEG_HR && p->lr_radius >= 0 && p->rho > 0) {
      for (int c = 0; c < C; ++c) {
        if (class_real[c] == 0) continue;
        const ClassDesc& cd = classes[c];
        // LR rows m with lr0 <= rho*m < lr1, columns n with lc0 <= rho*n < lc1
        const int m0 = std::max(0, cd.lr0 > 0 ? cdiv(cd.lr0, p->rho) : 0);
        const int m1 = std::min(p->h - 1, (cd.lr1 - 1) / p->rho);
        const int n0 = std::max(0, cd.lc0 > 0 ? cdiv(cd.lc0, p->rho) : 0);
        const int n1 = std::min(p->w - 1, (cd.lc1 - 1) / p->rho);
        for (int m = m0; m <= m1 && n0 <= n1; ++m) {
          if (!p->lr_block) {
            add_range(cand, p->off_lr + (int64_t)m * p->w + n0, p->off_lr + (int64_t)m * p->w + n1 + 1);
            continue;
          }
          for (int bn = n0 / kLrBW; bn <= n1 / kLrBW; ++bn) {   // the row's piece in each block
            const int a = std::max(n0, bn * kLrBW), z = std::min(n1, bn * kLrBW + kLrBW - 1);
            add_range(cand, lr_slot(p, m, a), lr_slot(p, m, z) + 1);
          }
        }
      }
    }
    if (kind == SEG_HR) {
      for (int c = 0; c < C; ++c) {
        if (class_real[c] == 0) continue;
        const ClassDesc& cd = classes[c];
        if (p->halo_copy) {   // the window itself and its halo block (R18)
          const int64_t ws = p->off_hr + (int64_t)cd.wid * l2;
          add_range(cand, ws, ws + l2);
          const int64_t hb = p->off_halo + (int64_t)cd.wid * p->G;
          add_range(cand, hb, hb + p->G);
          continue;
        }
        if (cd.r1 <= cd.r0 || cd.c1 <= cd.c0) continue;
        for (int wr = cd.r0 / p->l; wr <= (cd.r1 - 1) / p->l; ++wr)
          for (int wc = cd.c0 / p->l; wc <= (cd.c1 - 1) / p->l; ++wc) {
            const int64_t ws = p->off_hr + ((int64_t)wr * p->nWw + wc) * l2;
            add_range(cand, ws, ws + l2);
          }
      }
    }
    std::sort(cand.begin(), cand.end());
    cand.erase(std::unique(cand.begin(), cand.end()), cand.end());

    masks.assign((size_t)C * 4, 0u);
    for (int kt : cand) {
      std::fill(masks.begin(), masks.end(), 0u);
      const int64_t k0 = (int64_t)kt * kTile;
      for (int c = 0; c < C; ++c)
        for (int col = 0; col < kTile; ++col)
          if (visible(p, classes[c], k0 + col)) masks[c * 4 + col / 32] |= 1u << (col % 32);
      bool any = false, all = true;
      int64_t pairs = 0;
      for (int c = 0; c < C; ++c) {
        if (class_real[c] == 0) continue;
        int pc = 0;
        for (int wd = 0; wd < 4; ++wd) {
          pc += __builtin_popcount(masks[c * 4 + wd]);
          if (masks[c * 4 + wd] != 0xffffffffu) all = false;
        }
        if (pc) any = true;
        pairs += (int64_t)pc * class_real[c];
      }
      if (!any) continue;
      p->useful_pairs += pairs;
      if (all) {
        p->entries.push_back(kt);
        p->mask_off.push_back(-1);
      } else {
        p->entries.push_back((int32_t)((uint32_t)kt | 0x80000000u));
        p->mask_off.push_back((int32_t)p->mask_pool.size());
        p->mask_pool.insert(p->mask_pool.end(), masks.begin(), masks.end());
        p->n_partial++;
      }
      p->row_ptr[t + 1]++;
    }
  }
  build_schedule(p);
  return ULTRAGEN_OK;
}

}  // namespace

static bool same_list(const ultragen_plan_t* p, int a, int b) {
  const int na = p->row_ptr[a + 1] - p->row_ptr[a];
  const int nb = p->row_ptr[b + 1] - p->row_ptr[b];
  if (na != nb || p->qt_classes[a] != 1 || p->qt_classes[b] != 1) return false;
  if (p->qt_real[a] == 0 || p->qt_real[b] == 0) return false;
  for (int e = 0; e < na; ++e) {
    const int ea = p->row_ptr[a] + e, eb = p->row_ptr[b] + e;
    if (p->entries[ea] != p->entries[eb]) return false;
    if (p->mask_off[ea] >= 0) {
      for (int wd = 0; wd < 4; ++wd)
        if (p->mask_pool[p->mask_off[ea] + wd] != p->mask_pool[p->mask_off[eb] + wd]) return false;
    }
  }
  return true;
}

void build_schedule(ultragen_plan_t* p) {
  struct Group { int qt0, qt1, e0, n; };
  std::vector<Group> groups;
  for (int t = 0; t < p->n_qtiles;) {
    if (t + 1 < p->n_qtiles && same_list(p, t, t + 1)) {
      groups.push_back({t, t + 1, p->row_ptr[t], p->row_ptr[t + 1] - p->row_ptr[t]});
      t += 2;
    } else {
      groups.push_back({t, -1, p->row_ptr[t], p->row_ptr[t + 1] - p->row_ptr[t]});
      t += 1;
    }
  }

  // split policy
  int chunk = 0;
  double threshold = 0;
  if (p->split_req > 0) {
    chunk = p->split_req;
    threshold = chunk;
  } else if (p->split_req < 0) {
    int longest = 0, longest_all = 0;
    int64_t steps = 0;
    for (const Group& g : groups) {
      const int64_t s0 = (int64_t)g.qt0 * kTile;
      if (s0 >= p->off_hr && g.n > longest) longest = g.n;   // HR and LR groups
      longest_all = std::max(longest_all, g.n);
      steps += g.n;
    }
    // The attention hands items out from a work counter, longest first, so a group needs no
    // split unless it alone outlasts a streaming multiprocessor's share of the layer (one
    // batch element of all heads on kPlanSMs): then a split only adds partials and a merge.
    const bool fits = (double)longest_all * kPlanSMs <= (double)steps * p->heads;
    if (longest > 0 && !fits) {
      chunk = std::max(longest, 8);
      threshold = 1.5 * chunk;
    }
  }
  p->split_chunk = chunk;

  p->items.clear();
  p->combine.clear();
  p->n_split_items = 0;
  std::vector<ug::Item> rest;
  auto make = [&](const Group& g, int e0, int e1, int ws) {
    ug::Item it;
    it.v[0] = g.qt0;
    it.v[1] = g.qt1;
    it.v[2] = e0;
    it.v[3] = e1;
    it.v[4] = ws;
    it.v[5] = p->qt_classes[g.qt0];
    it.v[6] = p->qt_wfirst[g.qt0];
    it.v[7] = 0;
    return it;
  };
  std::vector<ug::Item> split_items;
  for (const Group& g : groups) {
    if (chunk > 0 && g.n > threshold && g.n > chunk) {
      const int nsplit = cdiv(g.n, chunk);
      const int cs = cdiv(g.n, nsplit);
      ug::CombineGroup cg{g.qt0, g.qt1, p->n_split_items, nsplit};
      p->combine.push_back(cg);
      for (int s = 0; s < nsplit; ++s) {
        const int e0 = g.e0 + s * cs;
        const int e1 = g.e0 + std::min(g.n, (s + 1) * cs);
        split_items.push_back(make(g, e0, e1, p->n_split_items++));
      }
    } else {
      rest.push_back(make(g, g.e0, g.e0 + g.n, -1));
    }
  }
  // Per-head item order: long groups first (longer than the longest HR / LR group, e.g.
  // unsplit text groups), longest first -- the head-major work order hands these out for all
  // heads at the start of the launch instead of as each head begins -- then the split items,
  // then the rest in query-tile order.
  int hr_longest = 0;
  for (const Group& g : groups)
    if ((int64_t)g.qt0 * kTile >= p->off_hr) hr_longest = std::max(hr_longest, g.n);
  std::stable_partition(rest.begin(), rest.end(),
                        [&](const ug::Item& it) { return it.v[3] - it.v[2] > hr_longest; });
  const auto long_end = std::find_if(rest.begin(), rest.end(), [&](const ug::Item& it) {
    return it.v[3] - it.v[2] <= hr_longest;
  });
  std::stable_sort(rest.begin(), long_end, [](const ug::Item& a, const ug::Item& b) {
    return a.v[3] - a.v[2] > b.v[3] - b.v[2];
  });
  p->n_long_items = (int)(long_end - rest.begin());
  p->items.insert(p->items.end(), rest.begin(), long_end);
  p->items.insert(p->items.end(), split_items.begin(), split_items.end());
  p->items.insert(p->items.end(), long_end, rest.end());
  // longest items first, for the item-major order small layers use (ties keep the list order)
  p->item_order.resize(p->items.size());
  for (size_t i = 0; i < p->items.size(); ++i) p->item_order[i] = (int32_t)i;
  std::stable_sort(p->item_order.begin(), p->item_order.end(), [&](int32_t a, int32_t b) {
    return p->items[a].v[3] - p->items[a].v[2] > p->items[b].v[3] - p->items[b].v[2];
  });
  p->dirty = true;
}

std::vector<float> rope_table(const ultragen_plan_t* p) {
  const int P = std::max(p->H, p->W);
  const int half = p->D / 2;
  std::vector<float> tab((size_t)P * half * 2);
  for (int q = 0; q < half; ++q) {
    int axis, k, d;
    if (q < p->axes[0] / 2) {
      axis = 0; k = q; d = p->axes[0];
    } else if (q < (p->axes[0] + p->axes[1]) / 2) {
      axis = 1; k = q - p->axes[0] / 2; d = p->axes[1];
    } else {
      axis = 2; k = q - (p->axes[0] + p->axes[1]) / 2; d = p->axes[2];
    }
    (void)axis;
    const double omega = std::pow(p->theta, -2.0 * k / d);
    for (int pos = 0; pos < P; ++pos) {
      const double phi = pos * omega;
      tab[((size_t)pos * half + q) * 2 + 0] = (float)std::cos(phi);
      tab[((size_t)pos * half + q) * 2 + 1] = (float)std::sin(phi);
    }
  }
  return tab;
}

}  // namespace ug

// ------------------------------------------------------------------------------------
// host-only C entry points
// ------------------------------------------------------------------------------------
extern "C" {

const char* ultragen_status_string(int s) {
  switch (s) {
    case ULTRAGEN_OK: return "ok";
    case ULTRAGEN_ERR_INVALID_ARG: return "invalid argument";
    case ULTRAGEN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ULTRAGEN_ERR_CUDA: return "CUDA error";
    case ULTRAGEN_ERR_OOM: return "out of memory";
    case ULTRAGEN_ERR_TIMEOUT: return "device wait timed out";
    case ULTRAGEN_ERR_PLAN_MISMATCH: return "plan does not match the call";
    case ULTRAGEN_ERR_NO_DEVICE: return "no sm_100 device";
    case ULTRAGEN_ERR_BOUNDS: return "index outside its table (debug build check)";
    default: return "unknown status";
  }
}

int ultragen_plan(int H, int W, int l, int b, int rho, int text_len, int heads, int head_dim,
                  ultragen_plan_t** out) {
  ug::NvtxRange nvtx_range("ultragen_plan");
  if (!out) return ULTRAGEN_ERR_INVALID_ARG;
  *out = nullptr;
  if (H < 1 || W < 1 || l < 1 || b < 0 || rho < 0 || text_len < 0 || heads < 1)
    return ULTRAGEN_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return ULTRAGEN_ERR_UNSUPPORTED;
  if (b > l || H > 32767 || W > 32767 || l > 4096 || text_len > (1 << 24) || heads > 4096)
    return ULTRAGEN_ERR_UNSUPPORTED;
  ultragen_plan_t* p = new (std::nothrow) ultragen_plan_t();
  if (!p) return ULTRAGEN_ERR_OOM;
  p->H = H; p->W = W; p->l = l; p->b = b; p->rho = rho; p->T = text_len;
  p->heads = heads; p->D = head_dim;
  if (head_dim == 64) { p->axes[0] = 16; p->axes[1] = 24; p->axes[2] = 24; }
  else { p->axes[0] = 16; p->axes[1] = 56; p->axes[2] = 56; }
  p->theta = 1.0e4;
  int st;
  try {
    st = ug::build_tables(p);
  } catch (const std::bad_alloc&) {
    st = ULTRAGEN_ERR_OOM;
  } catch (...) {
    st = ULTRAGEN_ERR_INVALID_ARG;
  }
  if (st != ULTRAGEN_OK) {
    delete p;
    return st;
  }
  *out = p;
  return ULTRAGEN_OK;
}

int ultragen_plan_set_rope(ultragen_plan_t* p, int a0, int a1, int a2, double theta) {
  if (!p) return ULTRAGEN_ERR_INVALID_ARG;
  if (a0 < 0 || a1 < 0 || a2 < 0 || (a0 | a1 | a2) & 1 || a0 + a1 + a2 != p->D ||
      !(theta > 0.0) || !std::isfinite(theta))
    return ULTRAGEN_ERR_INVALID_ARG;
  p->axes[0] = a0; p->axes[1] = a1; p->axes[2] = a2;
  p->theta = theta;
  p->dirty = true;
  return ULTRAGEN_OK;
}

int ultragen_plan_set_split(ultragen_plan_t* p, int chunk) {
  if (!p || chunk < -1) return ULTRAGEN_ERR_INVALID_ARG;
  p->split_req = chunk;
  try {
    ug::build_schedule(p);
  } catch (...) {
    return ULTRAGEN_ERR_OOM;
  }
  return ULTRAGEN_OK;
}

int ultragen_plan_set_lr_scope(ultragen_plan_t* p, int radius) {
  if (!p || radius < -1 || radius > (1 << 20)) return ULTRAGEN_ERR_INVALID_ARG;
  const int old = p->lr_radius;
  p->lr_radius = radius;
  int st;
  try {
    st = ug::build_tables(p);
  } catch (const std::bad_alloc&) {
    st = ULTRAGEN_ERR_OOM;
  }
  if (st != ULTRAGEN_OK) {
    p->lr_radius = old;
    ug::build_tables(p);
    return st;
  }
  p->dirty = true;
  return ULTRAGEN_OK;
}

int ultragen_plan_set_halo(ultragen_plan_t* p, int mode) {
  if (!p || mode < -1 || mode > 2) return ULTRAGEN_ERR_INVALID_ARG;
  const int old = p->halo_req;
  p->halo_req = mode;
  int st;
  try {
    st = ug::build_tables(p);
  } catch (const std::bad_alloc&) {
    st = ULTRAGEN_ERR_OOM;
  }
  if (st != ULTRAGEN_OK) {
    p->halo_req = old;
    ug::build_tables(p);
    return st;
  }
  p->dirty = true;
  return ULTRAGEN_OK;
}

int ultragen_plan_set_lr_order(ultragen_plan_t* p, int mode) {
  if (!p || mode < -1 || mode > 1) return ULTRAGEN_ERR_INVALID_ARG;
  const int old = p->lr_order_req;
  p->lr_order_req = mode;
  int st;
  try {
    st = ug::build_tables(p);
  } catch (const std::bad_alloc&) {
    st = ULTRAGEN_ERR_OOM;
  }
  if (st != ULTRAGEN_OK) {
    p->lr_order_req = old;
    ug::build_tables(p);
    return st;
  }
  p->dirty = true;
  return ULTRAGEN_OK;
}

int ultragen_plan_set_qk_format(ultragen_plan_t* p, int format, int q_exp, int k_exp) {
  if (!p || (format != ULTRAGEN_QK_BF16 && format != ULTRAGEN_QK_E4M3) ||
      q_exp < -ULTRAGEN_QK_EXP_MAX || q_exp > ULTRAGEN_QK_EXP_MAX ||
      k_exp < -ULTRAGEN_QK_EXP_MAX || k_exp > ULTRAGEN_QK_EXP_MAX)
    return ULTRAGEN_ERR_INVALID_ARG;
  if (format == ULTRAGEN_QK_E4M3 && p->D != 128) return ULTRAGEN_ERR_UNSUPPORTED;
  p->qk_format = format;
  p->q_exp = format == ULTRAGEN_QK_E4M3 ? q_exp : 0;
  p->k_exp = format == ULTRAGEN_QK_E4M3 ? k_exp : 0;
  return ULTRAGEN_OK;
}

int ultragen_plan_info(const ultragen_plan_t* p, ultragen_plan_info_t* o) {
  if (!p || !o) return ULTRAGEN_ERR_INVALID_ARG;
  std::memset(o, 0, sizeof(*o));
  o->H = p->H; o->W = p->W; o->l = p->l; o->b = p->b; o->rho = p->rho;
  o->text_len = p->T; o->heads = p->heads; o->head_dim = p->D;
  o->nWh = p->nWh; o->nWw = p->nWw; o->h = p->h; o->w = p->w;
  o->N_raster = p->N_raster; o->N_tot = p->N_tot;
  o->off_hr = p->off_hr; o->off_lr = p->off_lr;
  o->n_qtiles = p->n_qtiles;
  o->n_items = (int32_t)p->items.size();
  o->n_entries = (int64_t)p->entries.size();
  o->n_partial = p->n_partial;
  o->useful_pairs = p->useful_pairs;
  for (int i = 0; i < 3; ++i) o->rope_axes[i] = p->axes[i];
  o->rope_theta = p->theta;
  o->split_chunk = p->split_chunk;
  o->n_split_groups = (int32_t)p->combine.size();
  o->n_split_items = p->n_split_items;
  o->workspace_bytes_per_head = (int64_t)p->n_split_items * 2 * ug::kTile * (p->D + 1) * 4;
  o->lr_radius = p->lr_radius;
  o->halo_copy = p->halo_copy;
  o->kv_rows = p->kv_rows;
  o->n_halo_ops = (int32_t)p->halo_ops.size();
  o->n_long_items = p->n_long_items;
  o->halo_slots_per_window = (int32_t)p->G;
  o->N_kv = p->N_kv;
  o->off_halo = p->off_halo;
  o->lr_block = p->lr_block;
  o->qk_format = p->qk_format;
  o->q_exp = p->q_exp;
  o->k_exp = p->k_exp;
  return ULTRAGEN_OK;
}

int ultragen_plan_export(const ultragen_plan_t* p, int32_t* perm, int32_t* row_ptr,
                         int32_t* entries) {
  if (!p) return ULTRAGEN_ERR_INVALID_ARG;
  if (perm) std::memcpy(perm, p->perm.data(), (size_t)p->N_tot * sizeof(int32_t));
  if (row_ptr) std::memcpy(row_ptr, p->row_ptr.data(), p->row_ptr.size() * sizeof(int32_t));
  if (entries) std::memcpy(entries, p->entries.data(), p->entries.size() * sizeof(int32_t));
  return ULTRAGEN_OK;
}

int ultragen_plan_export_kv(const ultragen_plan_t* p, int32_t* kv_perm) {
  if (!p || !kv_perm) return ULTRAGEN_ERR_INVALID_ARG;
  std::memcpy(kv_perm, p->perm.data(), (size_t)p->N_kv * sizeof(int32_t));
  return ULTRAGEN_OK;
}

int ultragen_plan_export_items(const ultragen_plan_t* p, int32_t* out) {
  if (!p || !out) return ULTRAGEN_ERR_INVALID_ARG;
  for (size_t i = 0; i < p->items.size(); ++i)
    std::memcpy(out + i * ug::kItemInts, p->items[i].v, sizeof(p->items[i].v));
  return ULTRAGEN_OK;
}

int ultragen_plan_export_halo_ops(const ultragen_plan_t* p, int32_t* out) {
  if (!p || !out) return ULTRAGEN_ERR_INVALID_ARG;
  if (!p->halo_ops.empty())
    std::memcpy(out, p->halo_ops.data(), p->halo_ops.size() * sizeof(int32_t));
  return ULTRAGEN_OK;
}

int ultragen_plan_export_rowmasks(const ultragen_plan_t* p, int qtile, uint32_t* out) {
  if (!p || !out || qtile < 0 || qtile >= p->n_qtiles) return ULTRAGEN_ERR_INVALID_ARG;
  const int e0 = p->row_ptr[qtile], e1 = p->row_ptr[qtile + 1];
  const int64_t s0 = (int64_t)qtile * ug::kTile;
  const int64_t l2 = (int64_t)p->l * p->l;
  const int C = p->qt_classes[qtile], wfirst = p->qt_wfirst[qtile];
  for (int e = e0; e < e1; ++e) {
    for (int r = 0; r < ug::kTile; ++r) {
      uint32_t* dst = out + ((size_t)(e - e0) * ug::kTile + r) * 4;
      const int64_t s = s0 + r;
      if (p->perm[s] < 0) {
        dst[0] = dst[1] = dst[2] = dst[3] = 0u;
        continue;
      }
      if (p->mask_off[e] < 0) {
        dst[0] = dst[1] = dst[2] = dst[3] = 0xffffffffu;
        continue;
      }
      int c = 0;
      if (wfirst >= 0) c = std::min(C - 1, (int)((s - p->off_hr) / l2) - wfirst);
      for (int wd = 0; wd < 4; ++wd) dst[wd] = p->mask_pool[p->mask_off[e] + c * 4 + wd];
    }
  }
  return ULTRAGEN_OK;
}

}  // extern "C"
