// ultragen_hla_forward_noalloc: the attention forward for callers that cannot allocate device
// memory at call time -- code that runs while a framework's caching allocator owns the whole
// device, real-time loops that must not hit cudaMalloc's implicit device synchronisation, or
// hosts whose memory budget forbids a library growing its own buffers.  It runs the same
// kernels as ultragen_hla_forward, but the split partials (the only scratch the forward needs
// beyond its inputs and outputs) live in a fixed, file-scope device array instead of a
// workspace the plan allocates.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "nvtx_range.h"
#include "plan_internal.h"

namespace {

constexpr size_t kScratchBytes = ULTRAGEN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Split partials of the no-allocation forward.  Every GPU that loads this library holds it
// until the process exits.  All calls share it and it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
// device address of g_scratch, per device, and the CUDA context it was looked up in: a context
// that was torn down and created again (cudaDeviceReset, a framework's reset) loads the module
// again at another address, so a cached address is only reused within its own context
float* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The driver's cuCtxGetCurrent, found through the runtime (the library does not link libcuda).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<CtxGetCurrentFn>(nullptr);
    }
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  return fn;
}

// Host code must not use g_scratch's name as a device address: look the address up with the
// device current, once per device and context.
int scratch_for_device(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return ULTRAGEN_ERR_UNSUPPORTED;
  CtxGetCurrentFn get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS || !ctx) return ULTRAGEN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return ULTRAGEN_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return ULTRAGEN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int ultragen_hla_forward_noalloc(const void* qp, const void* kp, const void* vp,
                                            void* op, const ultragen_plan_t* cplan, int batch,
                                            ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_hla_forward_noalloc");
  ultragen_plan_t* p = const_cast<ultragen_plan_t*>(cplan);
  if (!p || !qp || !kp || !vp || !op || batch < 1) return ULTRAGEN_ERR_INVALID_ARG;
  const void* ptrs[] = {qp, kp, vp, op};
  for (const void* x : ptrs)
    if (!aligned16(x)) return ULTRAGEN_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)batch * p->heads * p->kv_rows;
  const int64_t items = (int64_t)batch * p->heads * (int64_t)p->items.size();
  if (rows >= ((int64_t)1 << 31) || items >= ((int64_t)1 << 31)) return ULTRAGEN_ERR_UNSUPPORTED;

  // the scratch bound: split partials of every (batch, head)
  if (ug::split_workspace_bytes(p, (int64_t)batch * p->heads) > kScratchBytes)
    return ULTRAGEN_ERR_UNSUPPORTED;

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
  // the same launches as ultragen_hla_forward (tensor maps, attention, split merge): none of
  // them allocates
  int launches = 0;
  st = ug::launch_attention(p, qp, kp, vp, op, batch * p->heads, p->heads, 0, scratch, stream,
                            &launches);
  p->last_launches = launches;
  return st;
}
