// ultragen_hla_forward_noalloc: the attention forward for callers that cannot allocate device
// memory at call time -- code that runs while a framework's caching allocator owns the whole
// device, real-time loops that must not hit cudaMalloc's implicit device synchronisation, or
// hosts whose memory budget forbids a library growing its own buffers.  It runs the same
// kernels as ultragen_hla_forward, but the split partials (the only scratch the forward needs
// beyond its inputs and outputs) live in a fixed, file-scope device array instead of a
// workspace the plan allocates.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "kernels.h"
#include "plan_internal.h"

namespace {

constexpr size_t kScratchBytes = ULTRAGEN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
constexpr unsigned long long kTimeoutNs = 2000ull * 1000 * 1000;

// Split partials of the no-allocation forward.  Every GPU that loads this library holds it
// until the process exits.  All calls share it and it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};   // device address of g_scratch, per device

// Host code must not use g_scratch's name as a device address: look the address up once per
// device, with that device current.
int scratch_for_device(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return ULTRAGEN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return ULTRAGEN_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return ULTRAGEN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int ultragen_hla_forward_noalloc(const void* qp, const void* kp, const void* vp,
                                            void* op, const ultragen_plan_t* cplan, int batch,
                                            ultragen_stream_t stream) {
  ultragen_plan_t* p = const_cast<ultragen_plan_t*>(cplan);
  if (!p || !qp || !kp || !vp || !op || batch < 1) return ULTRAGEN_ERR_INVALID_ARG;
  const void* ptrs[] = {qp, kp, vp, op};
  for (const void* x : ptrs)
    if (!aligned16(x)) return ULTRAGEN_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)batch * p->heads * p->N_tot;
  const int64_t items = (int64_t)batch * p->heads * (int64_t)p->items.size();
  if (rows >= ((int64_t)1 << 31) || items >= ((int64_t)1 << 31)) return ULTRAGEN_ERR_UNSUPPORTED;

  // the scratch bound: split partials of every (batch, head)
  const size_t need = (size_t)batch * p->heads * p->n_split_items * 2 * ug::kTile * (p->D + 1) * sizeof(float);
  if (need > kScratchBytes) return ULTRAGEN_ERR_UNSUPPORTED;

  // the plan's tables must already be on this device: this call uploads nothing
  int dev = -1, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return ULTRAGEN_ERR_NO_DEVICE;
  }
  if (major != 10) return ULTRAGEN_ERR_NO_DEVICE;
  if (!p->dev.valid || p->dev.device != dev || p->dirty) return ULTRAGEN_ERR_PLAN_MISMATCH;

  float* scratch = nullptr;
  int st = scratch_for_device(dev, &scratch);
  if (st) return st;

  alignas(64) CUtensorMap tq, tk, tv;
  if ((st = ug::make_tmap(&tq, qp, rows, p->D)) || (st = ug::make_tmap(&tk, kp, rows, p->D)) ||
      (st = ug::make_tmap(&tv, vp, rows, p->D)))
    return st;

  ug::FwdParams f;
  f.items = p->dev.items;
  f.entries = p->dev.entries;
  f.mask_off = p->dev.mask_off;
  f.mask_pool = p->dev.mask_pool;
  f.perm = p->dev.perm;
  f.out = static_cast<__nv_bfloat16*>(op);
  f.ws = scratch;
  f.err = p->dev.error;
  f.n_items_head = (int)p->items.size();
  f.total_items = (int)items;
  f.N_tot = (int)p->N_tot;
  f.off_hr = (int)p->off_hr;
  f.l2 = p->l * p->l;
  f.n_ws_head = p->n_split_items;
  f.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->D));
  f.timeout_ns = kTimeoutNs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int grid = (int)std::min<int64_t>(items, ug::sm_count());
  int launches = 0;
  if (grid > 0) {
    cudaError_t e = ug::launch_hla_fwd(&tq, &tk, &tv, f, p->D, grid, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return ULTRAGEN_ERR_CUDA;
    }
    ++launches;
  }
  if (!p->combine.empty()) {
    ug::CombineArgs c;
    c.ws = scratch;
    c.out = f.out;
    c.groups = p->dev.combine;
    c.perm = p->dev.perm;
    c.n_groups = (int)p->combine.size();
    c.n_ws_head = p->n_split_items;
    c.N_tot = (int)p->N_tot;
    c.BH = batch * p->heads;
    cudaError_t e = ug::launch_combine(c, p->D, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return ULTRAGEN_ERR_CUDA;
    }
    ++launches;
  }
  p->last_launches = launches;
  return ULTRAGEN_OK;
}
