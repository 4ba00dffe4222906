// Host-buffer runner: the whole layer (permute_rope -> attention with the unpermute in its
// epilogue) for Q/K/V and O that live in host memory, with the PCIe copies overlapped with
// the kernels.
//
// The heads are independent problems, so the layer is cut into units of (batch element, slice
// of `heads_per_chunk` heads).  A unit's Q/K/V slice is a 2D region of the raster host array
// (N_raster rows of heads_per_chunk * D elements, row pitch heads * D); one 2D copy per tensor
// brings it into a compact device staging buffer, where it is exactly the raster layout of a
// layer with heads_per_chunk heads, so the ordinary kernels run on it unchanged.  The output
// slice goes back the same way.  Three streams overlap the copy-in of unit u + 1, the kernels
// of unit u and the copy-out of unit u - 1; staging buffers are double-buffered and events
// order their reuse.  Every device buffer is allocated when the runner is created.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>

#include "kernels.h"
#include "nvtx_range.h"
#include "plan_internal.h"

struct ultragen_host_runner {
  ultragen_plan_t* plan = nullptr;
  int batch = 1, hpc = 1, device = -1;
  size_t stage_elems = 0;               // N_raster * hpc * D
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr},
              ev_out[2] = {nullptr, nullptr};
  void* in_stage[2][3] = {{nullptr, nullptr, nullptr}, {nullptr, nullptr, nullptr}};
  void* out_stage[2] = {nullptr, nullptr};
  void* perm_buf[3] = {nullptr, nullptr, nullptr};   // permuted Q, K, V of one unit
  float* ws = nullptr;
  size_t ws_bytes = 0;
  int64_t kv_rows = 0;                  // N_kv the permuted buffers were sized for
  int last_launches = 0;
};

namespace {

void release(ultragen_host_runner_t* r) {
  for (auto& set : r->in_stage)
    for (void*& b : set)
      if (b) cudaFree(b);
  for (void* b : r->out_stage)
    if (b) cudaFree(b);
  for (void* b : r->perm_buf)
    if (b) cudaFree(b);
  if (r->ws) cudaFree(r->ws);
  cudaEvent_t evs[] = {r->ev_start, r->ev_done, r->ev_in[0], r->ev_in[1], r->ev_comp[0],
                       r->ev_comp[1], r->ev_out[0], r->ev_out[1]};
  for (cudaEvent_t e : evs)
    if (e) cudaEventDestroy(e);
  cudaStream_t ss[] = {r->s_in, r->s_comp, r->s_out};
  for (cudaStream_t s : ss)
    if (s) cudaStreamDestroy(s);
  cudaGetLastError();
  delete r;
}

int status_of(cudaError_t e) {
  if (e == cudaSuccess) return ULTRAGEN_OK;
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? ULTRAGEN_ERR_OOM : ULTRAGEN_ERR_CUDA;
}

}  // namespace

extern "C" {

int ultragen_host_runner_create(ultragen_plan_t* p, int batch, int heads_per_chunk,
                                ultragen_host_runner_t** out) {
  if (!out) return ULTRAGEN_ERR_INVALID_ARG;
  *out = nullptr;
  if (!p || batch < 1 || heads_per_chunk < 1) return ULTRAGEN_ERR_INVALID_ARG;
  const int hpc = std::min(heads_per_chunk, p->heads);
  if ((int64_t)hpc * p->kv_rows >= ((int64_t)1 << 31) ||
      (int64_t)hpc * p->N_raster >= ((int64_t)1 << 31) ||
      (int64_t)hpc * (int64_t)p->items.size() >= ((int64_t)1 << 31))
    return ULTRAGEN_ERR_UNSUPPORTED;
  int st = ug::ensure_device_tables(p);   // checks for an sm_100 device and uploads the tables
  if (st) return st;
  ultragen_host_runner_t* r = new (std::nothrow) ultragen_host_runner_t();
  if (!r) return ULTRAGEN_ERR_OOM;
  r->plan = p;
  r->batch = batch;
  r->hpc = hpc;
  cudaGetDevice(&r->device);
  r->stage_elems = (size_t)p->N_raster * hpc * p->D;
  const size_t stage_bytes = r->stage_elems * 2;
  r->kv_rows = p->kv_rows;
  const size_t perm_bytes = (size_t)hpc * p->kv_rows * p->D * 2;   // Q uses the first N_tot rows
  r->ws_bytes = std::max<size_t>(ug::split_workspace_bytes(p, hpc), 16);
  cudaError_t e = cudaSuccess;
  for (auto& set : r->in_stage)
    for (void*& b : set)
      if (e == cudaSuccess) e = cudaMalloc(&b, stage_bytes);
  for (void*& b : r->out_stage)
    if (e == cudaSuccess) e = cudaMalloc(&b, stage_bytes);
  for (void*& b : r->perm_buf)
    if (e == cudaSuccess) e = cudaMalloc(&b, perm_bytes);
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&r->ws), r->ws_bytes);
  cudaStream_t* ss[] = {&r->s_in, &r->s_comp, &r->s_out};
  for (cudaStream_t* s : ss)
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
  cudaEvent_t* evs[] = {&r->ev_start, &r->ev_done, &r->ev_in[0], &r->ev_in[1], &r->ev_comp[0],
                        &r->ev_comp[1], &r->ev_out[0], &r->ev_out[1]};
  for (cudaEvent_t* ev : evs)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    st = status_of(e);
    release(r);
    return st;
  }
  *out = r;
  return ULTRAGEN_OK;
}

int ultragen_host_runner_forward(ultragen_host_runner_t* r, const void* q, const void* k,
                                 const void* v, void* o, ultragen_stream_t stream) {
  ug::NvtxRange nvtx_range("ultragen_host_runner_forward");
  if (!r || !q || !k || !v || !o) return ULTRAGEN_ERR_INVALID_ARG;
  ultragen_plan_t* p = r->plan;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != r->device) {
    cudaGetLastError();
    return ULTRAGEN_ERR_PLAN_MISMATCH;
  }
  int st = ug::ensure_device_tables(p);   // a no-op unless the plan changed since creation
  if (st) return st;
  // a split schedule changed after creation may need more partial storage than was allocated
  if (ug::split_workspace_bytes(p, r->hpc) > r->ws_bytes || p->kv_rows > r->kv_rows)
    return ULTRAGEN_ERR_PLAN_MISMATCH;
  const cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
  const int H = p->heads, D = p->D;
  const size_t row_bytes = (size_t)H * D * 2;             // host raster row: every head
  const int per_b = (H + r->hpc - 1) / r->hpc;
  const int units = r->batch * per_b;
  const char* src[3] = {static_cast<const char*>(q), static_cast<const char*>(k),
                        static_cast<const char*>(v)};
  char* dst = static_cast<char*>(o);
  cudaError_t e = cudaEventRecord(r->ev_start, user);
  cudaStream_t ss[] = {r->s_in, r->s_comp, r->s_out};
  for (cudaStream_t s : ss)
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, r->ev_start, 0);
  int launches = 0;
  for (int u = 0; u < units && e == cudaSuccess && st == ULTRAGEN_OK; ++u) {
    const int b = u / per_b, h0 = (u % per_b) * r->hpc;
    const int hc = std::min(r->hpc, H - h0);
    const int buf = u & 1;
    const size_t slice = (size_t)hc * D * 2;                // bytes of one raster row slice
    const size_t off = (size_t)b * p->N_raster * row_bytes + (size_t)h0 * D * 2;
    // copy-in: the staging set is free once the kernels of unit u - 2 are done with it
    if (u >= 2) e = cudaStreamWaitEvent(r->s_in, r->ev_comp[buf], 0);
    for (int x = 0; x < 3 && e == cudaSuccess; ++x)
      e = cudaMemcpy2DAsync(r->in_stage[buf][x], slice, src[x] + off, row_bytes, slice,
                            (size_t)p->N_raster, cudaMemcpyHostToDevice, r->s_in);
    if (e == cudaSuccess) e = cudaEventRecord(r->ev_in[buf], r->s_in);
    // kernels: after the copy-in, and once the copy-out of unit u - 2 has drained out_stage
    if (e == cudaSuccess) e = cudaStreamWaitEvent(r->s_comp, r->ev_in[buf], 0);
    if (e == cudaSuccess && u >= 2) e = cudaStreamWaitEvent(r->s_comp, r->ev_out[buf], 0);
    if (e != cudaSuccess) break;
    st = ug::launch_permute(p, r->in_stage[buf][0], r->in_stage[buf][1], r->in_stage[buf][2],
                            ULTRAGEN_BF16, r->perm_buf[0], r->perm_buf[1], r->perm_buf[2], 1, hc,
                            r->s_comp);
    if (st) break;
    ++launches;
    int n = 0;
    st = ug::launch_attention(p, r->perm_buf[0], r->perm_buf[1], r->perm_buf[2], r->out_stage[buf],
                              hc, hc, 1, r->ws, r->s_comp, &n);
    if (st) break;
    launches += n;
    e = cudaEventRecord(r->ev_comp[buf], r->s_comp);
    // copy-out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(r->s_out, r->ev_comp[buf], 0);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(dst + off, row_bytes, r->out_stage[buf], slice, slice,
                            (size_t)p->N_raster, cudaMemcpyDeviceToHost, r->s_out);
    if (e == cudaSuccess) e = cudaEventRecord(r->ev_out[buf], r->s_out);
  }
  // the caller's stream continues after the last copy-out, and after the other two streams
  // (so that a later call cannot overwrite staging still in use)
  cudaError_t e2 = cudaSuccess;
  for (cudaStream_t s : ss) {
    if (e2 == cudaSuccess) e2 = cudaEventRecord(r->ev_done, s);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(user, r->ev_done, 0);
  }
  r->last_launches = launches;
  if (st) return st;
  if (e != cudaSuccess) return status_of(e);
  return status_of(e2);
}

int ultragen_host_runner_last_launch_count(const ultragen_host_runner_t* r) {
  return r ? r->last_launches : -1;
}

int ultragen_host_runner_destroy(ultragen_host_runner_t* r) {
  if (!r) return ULTRAGEN_ERR_INVALID_ARG;
  if (r->s_in) cudaStreamSynchronize(r->s_in);
  if (r->s_comp) cudaStreamSynchronize(r->s_comp);
  if (r->s_out) cudaStreamSynchronize(r->s_out);
  release(r);
  return ULTRAGEN_OK;
}

}  // extern "C"
