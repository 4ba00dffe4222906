// C entry points that touch the device: plan table upload, tensor-map creation, launches,
// error read-back.  Host-only entry points live in plan.cpp.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "kernels.h"
#include "nvtx_range.h"
#include "warm_fused.h"
#include "plan_internal.h"

namespace ug {
namespace {


template <typename T>
int upload(T** dst, const std::vector<T>& src) {
  const size_t bytes = std::max<size_t>(src.size(), 1) * sizeof(T);
  if (cudaMalloc(reinterpret_cast<void**>(dst), bytes) != cudaSuccess) {
    cudaGetLastError();
    *dst = nullptr;
    return ULTRAGEN_ERR_OOM;
  }
  if (!src.empty() && cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess)
    return ULTRAGEN_ERR_CUDA;
  return ULTRAGEN_OK;
}

void free_device(ultragen_plan_t* p) {
  DeviceTables& d = p->dev;
  void* ptrs[] = {d.items, d.entries, d.mask_off, d.mask_pool, d.perm, d.inv_perm,
                  d.slot_pos, d.halo_ptr, d.halo_dst, d.halo_pad, d.halo_ops, d.item_order, d.rope,
                  d.combine, d.error, d.clock, d.sched, d.ws};
  for (void* q : ptrs)
    if (q) cudaFree(q);
  d = DeviceTables();
}

int check_device(int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ULTRAGEN_ERR_NO_DEVICE;
  }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return ULTRAGEN_ERR_NO_DEVICE;
  }
  if (major != 10) return ULTRAGEN_ERR_NO_DEVICE;
  *dev_out = dev;
  return ULTRAGEN_OK;
}

// Uploads (or re-uploads after a change) the plan's tables to the current device.
int ensure_device(ultragen_plan_t* p) {
  int dev;
  int st = check_device(&dev);
  if (st != ULTRAGEN_OK) return st;
  if (p->dev.valid && p->dev.device == dev && !p->dirty) return ULTRAGEN_OK;
  free_device(p);
  DeviceTables& d = p->dev;
  std::vector<int32_t> items;
  items.reserve(p->items.size() * kItemInts);
  for (const Item& it : p->items) items.insert(items.end(), it.v, it.v + kItemInts);
  std::vector<int32_t> comb;
  for (const CombineGroup& g : p->combine) {
    comb.push_back(g.qtile0);
    comb.push_back(g.qtile1);
    comb.push_back(g.ws_first);
    comb.push_back(g.nsplit);
  }
  const std::vector<float> rope = rope_table(p);
  if ((st = upload(&d.items, items)) || (st = upload(&d.entries, p->entries)) ||
      (st = upload(&d.mask_off, p->mask_off)) || (st = upload(&d.mask_pool, p->mask_pool)) ||
      (st = upload(&d.perm, p->perm)) || (st = upload(&d.inv_perm, p->inv_perm)) ||
      (st = upload(&d.slot_pos, p->slot_pos)) || (st = upload(&d.halo_ptr, p->halo_ptr)) ||
      (st = upload(&d.halo_dst, p->halo_dst)) || (st = upload(&d.halo_pad, p->halo_pad)) ||
      (st = upload(&d.halo_ops, p->halo_ops)) || (st = upload(&d.item_order, p->item_order)) ||
      (st = upload(&d.rope, rope)) ||
      (st = upload(&d.combine, comb)) || (st = upload(&d.error, std::vector<int>(1, 0))) ||
      (st = upload(&d.clock, std::vector<unsigned long long>(5, 0ull))) ||
      (st = upload(&d.sched, std::vector<int>(2, 0)))) {
    free_device(p);
    return st;
  }
  d.device = dev;
  d.valid = true;
  p->dirty = false;
  return ULTRAGEN_OK;
}

// Weights of output phase p of an axis with integer ratio rho (half-pixel centres): output
// rho k + p interpolates its cell's rows k + o, o in {-1, 0, 1}, as w[o + 1].  The source
// coordinate relative to row k is (p + 1/2) / rho - 1/2, in (-1/2, 1/2).
void phase_weights(int rho, int p, double (&w)[3]) {
  w[0] = w[1] = w[2] = 0.0;
  const double src = (p + 0.5) / rho - 0.5;
  const double f0 = std::floor(src);
  const double f = src - f0;
  const int o = (int)f0;                   // -1 or 0
  w[o + 1] += 1.0 - f;
  w[o + 2] += f;
}

// Row (ra, rb) and column (ca, cb) weights of the fused warm start: bilinear weights a_p,
// blurred ones b_p = (a_{p-1} + 2 a_p + a_{p+1}) / 4 (neighbouring phases of the adjacent
// cells shifted by one row), and the column weights scaled by the sharpening and the blend.
void warm_weights(WarmFused& a, int ry, float sharpen, float alpha) {
  auto fill = [](int rho, int p, double (&aw)[3], double (&bw)[3]) {
    double c[3], u[3], d[3];
    phase_weights(rho, p, c);
    // the row above: phase p - 1 of this cell, or phase rho - 1 of the cell above
    if (p > 0) {
      phase_weights(rho, p - 1, u);
    } else {
      double t[3];
      phase_weights(rho, rho - 1, t);
      u[0] = t[1]; u[1] = t[2]; u[2] = 0.0;
      // t[0] would sit two rows up: phase rho - 1 starts at its own row, so t[0] == 0
    }
    if (p + 1 < rho) {
      phase_weights(rho, p + 1, d);
    } else {
      double t[3];
      phase_weights(rho, 0, t);
      d[0] = 0.0; d[1] = t[0]; d[2] = t[1];
      // t[2] would sit two rows down: phase 0 ends at its own row, so t[2] == 0
    }
    for (int i = 0; i < 3; ++i) {
      aw[i] = c[i];
      bw[i] = (u[i] + 2.0 * c[i] + d[i]) / 4.0;
    }
  };
  a.ry = ry;
  for (int p = 0; p < ry; ++p) {
    double aw[3], bw[3];
    fill(ry, p, aw, bw);
    for (int i = 0; i < 3; ++i) {
      a.ra[p][i] = (float)aw[i];
      a.rb[p][i] = (float)bw[i];
    }
  }
  const double s = sharpen, beta = 1.0 - (double)alpha;
  for (int q = 0; q < 4; ++q) {
    double aw[3], bw[3];
    fill(4, q, aw, bw);
    for (int j = 0; j < 3; ++j) {
      a.ca[q][j] = (float)(beta * (1.0 + s) * aw[j]);
      a.cb[q][j] = (float)(-beta * s * bw[j]);
    }
  }
}

int grid_for(int64_t rows, int rows_per_block) {
  const int64_t need = (rows + rows_per_block - 1) / rows_per_block;
  const int64_t cap = (int64_t)sm_count() * 8;
  return (int)std::max<int64_t>(1, std::min(need, cap));
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ULTRAGEN_OK;
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? ULTRAGEN_ERR_OOM : ULTRAGEN_ERR_CUDA;
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    cudaGetLastError();
  });
  return fn;
}

// 2D view [rows, D] bf16 with [128 x 64] boxes and the 128-byte swizzle.
int make_tmap(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ULTRAGEN_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ULTRAGEN_OK : ULTRAGEN_ERR_CUDA;
}

// 2D view [rows, D] of bytes (e4m3) with [128 x 128] boxes (128-byte rows) and the 128-byte
// swizzle: the layout the 8-bit S = Q K^T products read (D = 128).
int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || D != 128) return ULTRAGEN_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ULTRAGEN_OK : ULTRAGEN_ERR_CUDA;
}

// The window segment of permuted K or V as a 5D view (element, column and row in the window,
// window, batch-head) with [inner x nc x nr] boxes and the 128-byte swizzle: one box is one
// piece of a halo block (nr x nc tokens of one window, raster order), landing as nr * nc
// consecutive 128-byte rows.  inner = 64 bf16 elements, or 128 bytes of e4m3 (bytes = 1).
int make_tmap_window(CUtensorMap* m, const void* kv, const ultragen_plan_t* p, uint64_t units,
                     int nc, int nr, int bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return ULTRAGEN_ERR_CUDA;
  const uint64_t es = bytes ? 1 : 2, row = (uint64_t)p->D * es, l = (uint64_t)p->l;
  const cuuint64_t dims[5] = {(cuuint64_t)p->D, l, l, (cuuint64_t)p->nWh * p->nWw, units};
  const cuuint64_t strides[4] = {row, l * row, l * l * row, (cuuint64_t)p->kv_rows * row};
  const cuuint32_t box[5] = {bytes ? 128u : 64u, (cuuint32_t)nc, (cuuint32_t)nr, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const void* base = static_cast<const uint8_t*>(kv) + (uint64_t)p->off_hr * row;
  CUresult r = fn(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ULTRAGEN_OK : ULTRAGEN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  return n > 0 ? n : 148;
}

int ensure_device_tables(ultragen_plan_t* p) { return ensure_device(p); }

size_t split_workspace_bytes(const ultragen_plan_t* p, int64_t units) {
  return (size_t)units * p->n_split_items * 2 * kTile * (p->D + 1) * sizeof(float);
}

// Attention over `units` (batch, head) pairs whose permuted Q/K/V start at qp/kp/vp; a raster
// output is laid out [units / heads][N_raster][heads][D].  The plan's tables must already be on
// the device and `ws` must hold split_workspace_bytes(p, units).
int launch_attention(const ultragen_plan_t* p, const void* qp, const void* kp, const void* vp,
                     void* op, int units, int heads, int raster, float* ws, cudaStream_t s,
                     int* launches) {
  const int64_t rows = (int64_t)units * p->N_tot, kv_rows = (int64_t)units * p->kv_rows;
  const int64_t items = (int64_t)units * (int64_t)p->items.size();
  alignas(64) CUtensorMap tq, tk, tv;
  const int qk8 = p->qk_format == ULTRAGEN_QK_E4M3;
  if (qk8 && p->D != 128) return ULTRAGEN_ERR_UNSUPPORTED;
  int st;
  if (qk8) {
    if ((st = make_tmap_u8(&tq, qp, rows, p->D)) || (st = make_tmap_u8(&tk, kp, kv_rows, p->D)))
      return st;
  } else if ((st = make_tmap(&tq, qp, rows, p->D)) || (st = make_tmap(&tk, kp, kv_rows, p->D))) {
    return st;
  }
  if ((st = make_tmap(&tv, vp, kv_rows, p->D))) return st;
  // gathered halo tiles: K and V window views with the three piece boxes (b x l, l x b, b x b)
  HaloMaps hm;
  std::memset(&hm, 0, sizeof(hm));
  const int gather = p->halo_copy == 2;
  if (gather) {
    const int shp[3][2] = {{p->l, p->b}, {p->b, p->l}, {p->b, p->b}};   // (nc, nr)
    for (int s = 0; s < 3; ++s)
      if ((st = make_tmap_window(&hm.m[s], kp, p, units, shp[s][0], shp[s][1], qk8)) ||
          (st = make_tmap_window(&hm.m[3 + s], vp, p, units, shp[s][0], shp[s][1], 0)))
        return st;
  }
  FwdParams f;
  f.items = p->dev.items;
  f.entries = p->dev.entries;
  f.mask_off = p->dev.mask_off;
  f.mask_pool = p->dev.mask_pool;
  f.perm = p->dev.perm;
  f.out = static_cast<__nv_bfloat16*>(op);
  f.ws = ws;
  f.err = p->dev.error;
  f.n_items_head = (int)p->items.size();
  f.n_long = p->n_long_items;
  f.total_items = (int)items;
  f.N_tot = (int)p->N_tot;
  f.N_kv = (int)p->kv_rows;
  f.n_ktiles = (int)(p->N_kv / kTile);
  if (gather) {
    f.halo_ops = p->dev.halo_ops;
    f.halo_tile0 = (int)(p->off_halo / kTile);
    f.halo_gtiles = (int)(p->G / kTile);
    f.nWh = p->nWh;
    f.nWw = p->nWw;
    f.n_halo_ops = (int)p->halo_ops.size();
  }
  f.off_hr = (int)p->off_hr;
  f.l2 = p->l * p->l;
  f.n_ws_head = p->n_split_items;
  // log2(e) / sqrt(D), times 2^(q_exp + k_exp) for the scaled e4m3 Q and K
  f.scale_log2 = (float)(std::ldexp(1.4426950408889634, p->q_exp + p->k_exp) /
                         std::sqrt((double)p->D));
  f.timeout_ns = p->wait_limit_ns;
  f.fault = p->fault;
  f.raster = raster;
  f.N_raster = (int)p->N_raster;
  f.heads = heads;
  f.n_entries = (int)p->entries.size();
  f.n_mask_words = (int)p->mask_pool.size();
  f.clock = p->clock_record ? p->dev.clock : nullptr;
  f.sched = p->dev.sched;
  const int grid = (int)std::min<int64_t>(items, sm_count());
  // few items per CTA: hand them out item-major, longest first, so that the last round holds
  // the short ones; otherwise head-major keeps one head's shared key tiles (its LR segment)
  // hot in L2 while many CTAs work on it
  f.item_major = items < 8 * (int64_t)grid ? 1 : 0;
  f.units = units;
  f.item_order = p->dev.item_order;
  *launches = 0;
  if (grid > 0) {
    st = cuda_status(launch_hla_fwd(&tq, &tk, &tv, &hm, f, p->D, qk8, grid, s));
    if (st) return st;
    ++*launches;
  }
  if (!p->combine.empty()) {
    CombineArgs c;
    c.ws = ws;
    c.out = f.out;
    c.groups = p->dev.combine;
    c.perm = p->dev.perm;
    c.n_groups = (int)p->combine.size();
    c.n_ws_head = p->n_split_items;
    c.N_tot = (int)p->N_tot;
    c.BH = units;
    c.raster = raster;
    c.N_raster = (int)p->N_raster;
    c.heads = heads;
    st = cuda_status(launch_combine(c, p->D, s));
    if (st) return st;
    ++*launches;
  }
  return ULTRAGEN_OK;
}

// permute_rope over `batch` raster blocks of `heads` heads: raster [batch][N_raster][heads][D]
// -> permuted [batch][heads][N_tot][D].  The plan's tables must already be on the device.
int launch_permute(const ultragen_plan_t* p, const void* q, const void* k, const void* v,
                   int in_dtype, void* qp, void* kp, void* vp, int batch, int heads,
                   cudaStream_t s) {
  PermuteArgs a;
  a.in[0] = q; a.in[1] = k; a.in[2] = v;
  a.out[0] = qp;
  a.out[1] = kp;
  a.out[2] = vp;
  a.qk8 = p->qk_format == ULTRAGEN_QK_E4M3;
  if (a.qk8 && p->D != 128) return ULTRAGEN_ERR_UNSUPPORTED;
  a.qk_inv[0] = std::ldexp(1.0f, -p->q_exp);
  a.qk_inv[1] = std::ldexp(1.0f, -p->k_exp);
  a.perm = p->dev.perm;
  a.slot_pos = p->dev.slot_pos;
  a.rope = p->dev.rope;
  a.err = p->dev.error;
  a.rope_rows = std::max(p->H, p->W);
  a.n_halo_dst = (int)p->halo_dst.size();
  // rows: every Q slot, then the pad slots of the halo blocks (their token slots are written
  // with their source rows)
  const int64_t n_pad = p->halo_copy == 1 ? (int64_t)p->halo_pad.size() : 0;
  a.rows_total = (int64_t)batch * heads * (p->N_tot + n_pad);
  a.N_tot = (int)p->N_tot;
  a.N_kv = (int)p->kv_rows;
  a.halo_pad = p->dev.halo_pad;
  a.div_rows = FastDiv((uint32_t)(p->N_tot + n_pad));
  a.N_raster = (int)p->N_raster;
  a.heads = heads;
  a.div_heads = FastDiv((uint32_t)heads);
  a.pair_a0 = p->axes[0] / 2;
  a.pair_a01 = (p->axes[0] + p->axes[1]) / 2;
  a.halo_ptr = p->halo_copy == 1 ? p->dev.halo_ptr : nullptr;
  a.halo_dst = p->dev.halo_dst;
  a.off_hr = (int)p->off_hr;
  a.N_hrp = (int)p->N_hrp;
  const int rows_per_block = 256 / (p->D / 8);
  return cuda_status(launch_permute_rope(a, in_dtype, p->D, grid_for(a.rows_total, rows_per_block), s));
}

}  // namespace ug

using namespace ug;

extern "C" {

int ultragen_plan_destroy(ultragen_plan_t* p) {
  if (!p) return ULTRAGEN_ERR_INVALID_ARG;
  if (p->dev.valid) free_device(p);
  delete p;
  return ULTRAGEN_OK;
}

int ultragen_permute_rope(const void* q, const void* k, const void* v, int in_dtype, void* qp,
                          void* kp, void* vp, int batch, const ultragen_plan_t* cplan,
                          ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_permute_rope");
  ultragen_plan_t* p = const_cast<ultragen_plan_t*>(cplan);
  if (!p || !q || !k || !v || !qp || !kp || !vp || batch < 1) return ULTRAGEN_ERR_INVALID_ARG;
  if (in_dtype != ULTRAGEN_BF16 && in_dtype != ULTRAGEN_F32) return ULTRAGEN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, qp, kp, vp};
  for (const void* x : ptrs)
    if (!aligned16(x)) return ULTRAGEN_ERR_INVALID_ARG;
  if ((int64_t)batch * p->heads * p->kv_rows >= ((int64_t)1 << 31) ||
      (int64_t)batch * p->heads * p->N_raster >= ((int64_t)1 << 31))
    return ULTRAGEN_ERR_UNSUPPORTED;
  int st = ensure_device(p);
  if (st) return st;
  p->last_launches = 1;
  return launch_permute(p, q, k, v, in_dtype, qp, kp, vp, batch, p->heads,
                        reinterpret_cast<cudaStream_t>(stream));
}

// The attention forward; `raster` selects the output layout (0: permuted, 1: raster).
static int hla_forward_impl(const void* qp, const void* kp, const void* vp, void* op,
                            const ultragen_plan_t* cplan, int batch, ultragen_stream_t stream,
                            int raster) {
  ultragen_plan_t* p = const_cast<ultragen_plan_t*>(cplan);
  if (!p || !qp || !kp || !vp || !op || batch < 1) return ULTRAGEN_ERR_INVALID_ARG;
  const void* ptrs[] = {qp, kp, vp, op};
  for (const void* x : ptrs)
    if (!aligned16(x)) return ULTRAGEN_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)batch * p->heads * p->kv_rows;
  const int64_t items = (int64_t)batch * p->heads * (int64_t)p->items.size();
  if (rows >= ((int64_t)1 << 31) || items >= ((int64_t)1 << 31)) return ULTRAGEN_ERR_UNSUPPORTED;
  int st = ensure_device(p);
  if (st) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // split workspace, owned by the plan and grown on demand with stream-ordered allocation (no
  // device-wide synchronisation, and capturable in a CUDA graph)
  const size_t ws_need = ug::split_workspace_bytes(p, batch * p->heads);
  if (ws_need > p->dev.ws_bytes) {
    if (p->dev.ws) {
      cudaFreeAsync(p->dev.ws, s);
      p->dev.ws = nullptr;
      p->dev.ws_bytes = 0;
    }
    if (cudaMallocAsync(reinterpret_cast<void**>(&p->dev.ws), ws_need, s) != cudaSuccess) {
      cudaGetLastError();
      p->dev.ws = nullptr;
      return ULTRAGEN_ERR_OOM;
    }
    p->dev.ws_bytes = ws_need;
  }
  int launches = 0;
  st = ug::launch_attention(p, qp, kp, vp, op, batch * p->heads, p->heads, raster, p->dev.ws, s,
                            &launches);
  p->last_launches = launches;
  return st;
}

int ultragen_hla_forward(const void* qp, const void* kp, const void* vp, void* op,
                         const ultragen_plan_t* plan, int batch, ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_hla_forward");
  return hla_forward_impl(qp, kp, vp, op, plan, batch, stream, 0);
}

int ultragen_hla_forward_raster(const void* qp, const void* kp, const void* vp, void* o,
                                const ultragen_plan_t* plan, int batch, ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_hla_forward_raster");
  if (plan && (int64_t)batch * plan->heads * plan->N_raster >= ((int64_t)1 << 31))
    return ULTRAGEN_ERR_UNSUPPORTED;
  return hla_forward_impl(qp, kp, vp, o, plan, batch, stream, 1);
}

int ultragen_unpermute(const void* op, void* o, int out_dtype, int batch,
                       const ultragen_plan_t* cplan, ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_unpermute");
  ultragen_plan_t* p = const_cast<ultragen_plan_t*>(cplan);
  if (!p || !op || !o || batch < 1) return ULTRAGEN_ERR_INVALID_ARG;
  if (out_dtype != ULTRAGEN_BF16 && out_dtype != ULTRAGEN_F32) return ULTRAGEN_ERR_INVALID_ARG;
  if (!aligned16(op) || !aligned16(o)) return ULTRAGEN_ERR_INVALID_ARG;
  if ((int64_t)batch * p->heads * p->N_tot >= ((int64_t)1 << 31)) return ULTRAGEN_ERR_UNSUPPORTED;
  int st = ensure_device(p);
  if (st) return st;
  UnpermuteArgs a;
  a.in = static_cast<const __nv_bfloat16*>(op);
  a.out = o;
  a.inv_perm = p->dev.inv_perm;
  a.rows_total = (int64_t)batch * p->N_raster * p->heads;
  a.N_tot = (int)p->N_tot;
  a.N_raster = (int)p->N_raster;
  a.heads = p->heads;
  a.div_heads = FastDiv((uint32_t)p->heads);
  a.div_nraster = FastDiv((uint32_t)p->N_raster);
  const int rows_per_block = 256 / (p->D / 8);
  p->last_launches = 1;
  return cuda_status(launch_unpermute(a, out_dtype, p->D, grid_for(a.rows_total, rows_per_block),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

int ultragen_sync_status(const ultragen_plan_t* cplan, ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_sync_status");
  ultragen_plan_t* p = const_cast<ultragen_plan_t*>(cplan);
  if (!p) return ULTRAGEN_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e);
  if (!p->dev.valid || !p->dev.error) return ULTRAGEN_OK;
  int h = 0;
  if (cudaMemcpy(&h, p->dev.error, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_status(cudaGetLastError());
  if (h != 0) {
    cudaMemset(p->dev.error, 0, sizeof(int));
    return h == ug::DEV_BOUNDS ? ULTRAGEN_ERR_BOUNDS : ULTRAGEN_ERR_TIMEOUT;
  }
  return ULTRAGEN_OK;
}

int ultragen_last_launch_count(const ultragen_plan_t* p) { return p ? p->last_launches : -1; }

int ultragen_warm_start(const float* x_lr, const float* noise, float* x_hr, int batch,
                        int channels, int h, int w, int H, int W, float alpha, float sharpen,
                        uint64_t seed, uint64_t offset, ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_warm_start");
  if (!x_lr || !x_hr || batch < 1 || channels < 1 || h < 1 || w < 1 || H < 1 || W < 1)
    return ULTRAGEN_ERR_INVALID_ARG;
  if (!std::isfinite(alpha) || !std::isfinite(sharpen) || sharpen < 0.0f)
    return ULTRAGEN_ERR_INVALID_ARG;
  const void* ptrs[] = {x_lr, noise, x_hr};
  for (const void* x : ptrs)
    if (reinterpret_cast<uintptr_t>(x) & 3u) return ULTRAGEN_ERR_INVALID_ARG;
  const int64_t planes = (int64_t)batch * channels;
  if (planes > 65535 || H > 65535 * 32 || (int64_t)h * w >= ((int64_t)1 << 31))
    return ULTRAGEN_ERR_UNSUPPORTED;
  int dev;
  int st = check_device(&dev);
  if (st) return st;
  WarmArgs a;
  a.lr = x_lr;
  a.noise = noise;
  a.out = x_hr;
  a.planes = (int)planes;
  a.h = h;
  a.w = w;
  a.H = H;
  a.W = W;
  a.sy = (float)h / (float)H;
  a.sx = (float)w / (float)W;
  a.alpha = alpha;
  a.amount = sharpen;
  a.seed = seed;
  a.offset = offset;
  a.vec = (W % 4 == 0) && aligned16(x_hr) && (!noise || aligned16(noise));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a.vec && W == 4 * w && H % h == 0 && H / h <= 8) {
    WarmFused f;
    warm_weights(f, H / h, sharpen, alpha);
    return cuda_status(launch_warm_start_fused(a, f, s));
  }
  return cuda_status(launch_warm_start(a, s));
}

int ultragen_plan_set_clock_record(ultragen_plan_t* p, int on) {
  if (!p || on < 0 || on > 1) return ULTRAGEN_ERR_INVALID_ARG;
  p->clock_record = on;
  return ULTRAGEN_OK;
}

int ultragen_plan_read_clock(const ultragen_plan_t* p, uint64_t out[3]) {
  if (!p || !out) return ULTRAGEN_ERR_INVALID_ARG;
  out[0] = out[1] = out[2] = 0;
  if (!p->dev.valid || !p->dev.clock) return ULTRAGEN_OK;
  unsigned long long h[3];   // words 3, 4 are the running launch's start (scratch)
  if (cudaMemcpy(h, p->dev.clock, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(p->dev.clock, 0, sizeof(h)) != cudaSuccess)
    return cuda_status(cudaGetLastError());
  for (int i = 0; i < 3; ++i) out[i] = h[i];
  return ULTRAGEN_OK;
}

int ultragen_plan_set_diagnostics(ultragen_plan_t* p, int fault, double wait_limit_s) {
  if (!p || fault < 0 || fault > 1 || !(wait_limit_s >= 1e-3 && wait_limit_s <= 60.0))
    return ULTRAGEN_ERR_INVALID_ARG;
  p->fault = fault;
  p->wait_limit_ns = (unsigned long long)(wait_limit_s * 1e9);
  return ULTRAGEN_OK;
}

}  // extern "C"
