// HBM-bound passes around the attention:
//   permute_rope   raster [B, N_raster, H, D] -> window-first [B, H, N_tot, D] bf16, with axial
//                  2D RoPE on Q and K ("UltraGen ..." papernotes note, 关键设计 1 window-first
//                  order; 关键设计 2 LR positions (rho m, rho n)); optionally Q and K as scaled
//                  e4m3 bytes (the 8-bit Q K^T format).
//   unpermute      window-first [B, H, N_tot, D] bf16 -> raster [B, N_raster, H, D].
//   split combine  log-sum-exp merge of the partial outputs of split query groups.
// Every thread moves 16-byte chunks (8 bf16) so loads and stores are full-sector.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

#ifndef ULTRAGEN_DEBUG
#define ULTRAGEN_DEBUG 0
#endif

namespace ug {

namespace {

// Index checks of debug builds (ULTRAGEN_DEBUG): a plan index outside its table is recorded in
// the device error word (DEV_BOUNDS) and the row is skipped instead of read or written.
// Release builds compile them away.
__device__ __forceinline__ bool index_ok(bool cond, int* err) {
  if (ULTRAGEN_DEBUG && !cond) {
    if (err) atomicExch(err, DEV_BOUNDS);
    return false;
  }
  return true;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ void load8(const float* src, float (&x)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Eight values times a power of two as e4m3 bytes (nearest even, saturating at +-448), element
// i in byte i.
__device__ __forceinline__ uint2 pack_e4m3x8(const float (&x)[8], float s) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = __nv_cvt_float2_to_fp8x2(make_float2(x[2 * i] * s, x[2 * i + 1] * s), __NV_SATFINITE,
                                    __NV_E4M3);
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

}  // namespace

// One thread = one 16-byte chunk of one output row, for Q, K and V together: the row's index
// decode and its cos/sin values (the same for Q and K) are shared by the three tensors, and
// three loads per row are in flight at once.  Rows are visited in (batch, slot, head) order,
// so the heads of one token -- contiguous in the raster input -- are read together while
// each output row is written whole.  The walk covers the N_tot Q slots and then only the pad
// slots of the halo blocks: a halo block's token slots are written from the source token's
// row, whose halo-copy list (CSR bounds and first target) is loaded together with the row.  (4K layer on B200: 5.9 TB/s with one row per thread,
// 4.9 TB/s with two, 2.5 TB/s with four.)  QK8: Q and K leave as 8 e4m3 bytes per thread.
template <typename Tin, int D, bool QK8>
__global__ void __launch_bounds__(256) permute_rope_kernel(PermuteArgs a) {
  constexpr int CH = D / 8;
  constexpr int ROWS = 256 / CH;
  constexpr int U = 1;                              // measured: 1 row per thread is fastest
  constexpr int HALF = D / 2;
  const Tin* __restrict__ qin = static_cast<const Tin*>(a.in[0]);
  const Tin* __restrict__ kin = static_cast<const Tin*>(a.in[1]);
  const Tin* __restrict__ vin = static_cast<const Tin*>(a.in[2]);
  const int c = threadIdx.x % CH;
  const int rsub = threadIdx.x / CH;
  const int rows_total = (int)a.rows_total;          // < 2^31, checked by the caller
  const int step = gridDim.x * ROWS * U;

  for (int row0 = blockIdx.x * ROWS * U; row0 < rows_total; row0 += step) {
    float xq[U][8], xk[U][8], xv[U][8];
    int pos_r[U], pos_c[U];
    int dst[U];                                       // K/V output row, -1 when out of range
    int dq[U];                                        // Q output row, -1 for halo-block pads
    int hb[U], he[U], h0[U];                          // halo copies: CSR range, first target
    int kvb[U];                                       // first K/V row of this (b, h)
    bool real[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = row0 + u * ROWS + rsub;         // (b, slot index, h)
      dst[u] = -1;
      dq[u] = -1;
      real[u] = false;
      hb[u] = he[u] = h0[u] = kvb[u] = 0;
      if (row >= rows_total) continue;
      const int bs = (int)a.div_heads.div((uint32_t)row);
      const int h = row - bs * a.heads;
      const int b = (int)a.div_rows.div((uint32_t)bs);
      const int idx = bs - b * (int)a.div_rows.d;
      // indices past N_tot are the halo blocks' pad slots; their token slots are written with
      // the source token's row below
      const int slot = idx < a.N_tot ? idx : __ldg(a.halo_pad + (idx - a.N_tot));
      if (!index_ok(slot >= 0 && slot < a.N_kv, a.err)) continue;
      const int r = __ldg(a.perm + slot);
      if (!index_ok(r < a.N_raster, a.err)) continue;
      kvb[u] = (b * a.heads + h) * a.N_kv;
      dst[u] = kvb[u] + slot;
      if (idx < a.N_tot) dq[u] = (b * a.heads + h) * a.N_tot + slot;
      if (r < 0) continue;
      real[u] = true;
      const uint32_t sp = __ldg(a.slot_pos + slot);
      pos_r[u] = (int)(sp >> 16);
      pos_c[u] = (int)(sp & 0xffffu);
      if (!index_ok(pos_r[u] < a.rope_rows && pos_c[u] < a.rope_rows, a.err)) {
        dst[u] = dq[u] = -1;
        real[u] = false;
        continue;
      }
      const int64_t src = ((int64_t)(b * a.N_raster + r) * a.heads + h) * D + c * 8;
      load8(qin + src, xq[u]);
      load8(kin + src, xk[u]);
      load8(vin + src, xv[u]);
      const int k = slot - a.off_hr;
      if (a.halo_ptr && k >= 0 && k < a.N_hrp) {
        hb[u] = __ldg(a.halo_ptr + k);
        he[u] = __ldg(a.halo_ptr + k + 1);
        if (!index_ok(hb[u] >= 0 && he[u] <= a.n_halo_dst, a.err)) he[u] = hb[u] = 0;
        if (he[u] > hb[u]) h0[u] = __ldg(a.halo_dst + hb[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (dst[u] < 0) continue;
      uint4 oq = make_uint4(0u, 0u, 0u, 0u), ok = oq, ov = oq;
      uint2 oq8 = make_uint2(0u, 0u), ok8 = oq8;
      if (real[u]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int q = c * 4 + k;                       // rotation pair index
          const int pos = q < a.pair_a0 ? 0 : (q < a.pair_a01 ? pos_r[u] : pos_c[u]);
          if (pos != 0) {
            const float2 cs = __ldg(reinterpret_cast<const float2*>(a.rope) + pos * HALF + q);
            const float q0 = xq[u][2 * k], q1 = xq[u][2 * k + 1];
            xq[u][2 * k] = q0 * cs.x - q1 * cs.y;
            xq[u][2 * k + 1] = q0 * cs.y + q1 * cs.x;
            const float k0 = xk[u][2 * k], k1 = xk[u][2 * k + 1];
            xk[u][2 * k] = k0 * cs.x - k1 * cs.y;
            xk[u][2 * k + 1] = k0 * cs.y + k1 * cs.x;
          }
        }
        if (QK8) {
          oq8 = pack_e4m3x8(xq[u], a.qk_inv[0]);
          ok8 = pack_e4m3x8(xk[u], a.qk_inv[1]);
        } else {
          oq = make_uint4(pack_bf16(xq[u][0], xq[u][1]), pack_bf16(xq[u][2], xq[u][3]),
                          pack_bf16(xq[u][4], xq[u][5]), pack_bf16(xq[u][6], xq[u][7]));
          ok = make_uint4(pack_bf16(xk[u][0], xk[u][1]), pack_bf16(xk[u][2], xk[u][3]),
                          pack_bf16(xk[u][4], xk[u][5]), pack_bf16(xk[u][6], xk[u][7]));
        }
        ov = make_uint4(pack_bf16(xv[u][0], xv[u][1]), pack_bf16(xv[u][2], xv[u][3]),
                        pack_bf16(xv[u][4], xv[u][5]), pack_bf16(xv[u][6], xv[u][7]));
      }
      const int64_t o = (int64_t)dst[u] * D + c * 8;   // element offset of the chunk
      __nv_bfloat16* const vout = static_cast<__nv_bfloat16*>(a.out[2]);
      if (QK8) {
        uint8_t* const qout = static_cast<uint8_t*>(a.out[0]);
        uint8_t* const kout = static_cast<uint8_t*>(a.out[1]);
        if (dq[u] >= 0) *reinterpret_cast<uint2*>(qout + (int64_t)dq[u] * D + c * 8) = oq8;
        *reinterpret_cast<uint2*>(kout + o) = ok8;
      } else {
        __nv_bfloat16* const qout = static_cast<__nv_bfloat16*>(a.out[0]);
        __nv_bfloat16* const kout = static_cast<__nv_bfloat16*>(a.out[1]);
        if (dq[u] >= 0) *reinterpret_cast<uint4*>(qout + (int64_t)dq[u] * D + c * 8) = oq;
        *reinterpret_cast<uint4*>(kout + o) = ok;
      }
      *reinterpret_cast<uint4*>(vout + o) = ov;
      if (he[u] > hb[u]) {
        // copies into the halo blocks of the neighbouring windows (the first target was loaded
        // with the row)
        for (int e = hb[u]; e < he[u]; ++e) {
          const int tgt = e == hb[u] ? h0[u] : __ldg(a.halo_dst + e);
          if (!index_ok(tgt >= 0 && tgt < a.N_kv, a.err)) continue;
          const int64_t oh = (int64_t)(kvb[u] + tgt) * D + c * 8;
          if (QK8)
            *reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.out[1]) + oh) = ok8;
          else
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out[1]) + oh) = ok;
          *reinterpret_cast<uint4*>(vout + oh) = ov;
        }
      }
    }
  }
}

template <typename Tout, int D>
__global__ void __launch_bounds__(256) unpermute_kernel(UnpermuteArgs a) {
  constexpr int CH = D / 8;
  constexpr int ROWS = 256 / CH;
  constexpr int U = 1;                              // measured: fastest (6.4 TB/s at 4K)
  const int c = threadIdx.x % CH;
  const int rsub = threadIdx.x / CH;
  const int rows_total = (int)a.rows_total;          // < 2^31, checked by the caller
  const int step = gridDim.x * ROWS * U;
  Tout* __restrict__ out = static_cast<Tout*>(a.out);
  for (int row0 = blockIdx.x * ROWS * U; row0 < rows_total; row0 += step) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = row0 + u * ROWS + rsub;          // (b, t, h) raster row
      if (row >= rows_total) continue;
      const int bt = (int)a.div_heads.div((uint32_t)row);
      const int h = row - bt * a.heads;
      const int b = (int)a.div_nraster.div((uint32_t)bt);
      const int t = bt - b * a.N_raster;
      const int slot = __ldg(a.inv_perm + t);
      v[u] = __ldg(reinterpret_cast<const uint4*>(a.in + ((int64_t)(b * a.heads + h) * a.N_tot + slot) * D + c * 8));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = row0 + u * ROWS + rsub;
      if (row >= rows_total) continue;
      if constexpr (sizeof(Tout) == 2) {
        *reinterpret_cast<uint4*>(out + row * D + c * 8) = v[u];
      } else {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        float4 f0, f1;
        f0.x = __uint_as_float(w[0] << 16); f0.y = __uint_as_float(w[0] & 0xffff0000u);
        f0.z = __uint_as_float(w[1] << 16); f0.w = __uint_as_float(w[1] & 0xffff0000u);
        f1.x = __uint_as_float(w[2] << 16); f1.y = __uint_as_float(w[2] & 0xffff0000u);
        f1.z = __uint_as_float(w[3] << 16); f1.w = __uint_as_float(w[3] & 0xffff0000u);
        reinterpret_cast<float4*>(out + row * D + c * 8)[0] = f0;
        reinterpret_cast<float4*>(out + row * D + c * 8)[1] = f1;
      }
    }
  }
}

// One warp per output row of a split group: merges nsplit partial rows (O_s normalised,
// lse_s in log2 units) as O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), M = max_s lse_s.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  constexpr int PER = D / 32;
  const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t total = (int64_t)a.BH * a.n_groups * 2 * 128;
  if (warp_id >= total) return;
  const int row = (int)(warp_id % 128);
  const int t = (int)((warp_id / 128) % 2);
  const int g = (int)((warp_id / 256) % a.n_groups);
  const int64_t bh = warp_id / (256 * (int64_t)a.n_groups);
  const int32_t* G = a.groups + 4 * g;
  const int qt = t ? G[1] : G[0];
  if (qt < 0) return;
  const int slot = qt * 128 + row;
  const int tok = __ldg(a.perm + slot);
  if (a.raster && tok < 0) return;                 // pad rows have no raster row
  __nv_bfloat16* dst =
      a.raster ? a.out + (((bh / a.heads) * a.N_raster + tok) * a.heads + bh % a.heads) * D + lane * PER
               : a.out + (bh * a.N_tot + slot) * D + lane * PER;
  const size_t item_floats = (size_t)2 * 128 * (D + 1);
  const float* base = a.ws + (size_t)(bh * a.n_ws_head) * item_floats;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float M = -INFINITY;
  if (tok >= 0) {
    for (int s = 0; s < G[3]; ++s) {
      const float* it = base + (size_t)(G[2] + s) * item_floats;
      M = fmaxf(M, __ldg(it + 2 * 128 * D + t * 128 + row));
    }
  }
  float den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < G[3]; ++s) {
      const float* it = base + (size_t)(G[2] + s) * item_floats;
      const float wgt = exp2f(__ldg(it + 2 * 128 * D + t * 128 + row) - M);
      den += wgt;
      const float* o = it + (size_t)(t * 128 + row) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] += wgt * __ldg(o + i);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint32_t pk[PER / 2];
#pragma unroll
  for (int i = 0; i < PER / 2; ++i) pk[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  if constexpr (PER == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pk[0];
  }
}

// ------------------------------------------------------------------------------ launchers
cudaError_t launch_permute_rope(const PermuteArgs& a, int in_dtype, int D, int grid_x,
                                cudaStream_t st) {
  dim3 grid(grid_x, 1);
  if (a.qk8) {
    if (D != 128) return cudaErrorInvalidValue;
    if (in_dtype == 0) permute_rope_kernel<__nv_bfloat16, 128, true><<<grid, 256, 0, st>>>(a);
    else permute_rope_kernel<float, 128, true><<<grid, 256, 0, st>>>(a);
  } else if (D == 128) {
    if (in_dtype == 0) permute_rope_kernel<__nv_bfloat16, 128, false><<<grid, 256, 0, st>>>(a);
    else permute_rope_kernel<float, 128, false><<<grid, 256, 0, st>>>(a);
  } else {
    if (in_dtype == 0) permute_rope_kernel<__nv_bfloat16, 64, false><<<grid, 256, 0, st>>>(a);
    else permute_rope_kernel<float, 64, false><<<grid, 256, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const UnpermuteArgs& a, int out_dtype, int D, int grid_x,
                             cudaStream_t st) {
  if (D == 128) {
    if (out_dtype == 0) unpermute_kernel<__nv_bfloat16, 128><<<grid_x, 256, 0, st>>>(a);
    else unpermute_kernel<float, 128><<<grid_x, 256, 0, st>>>(a);
  } else {
    if (out_dtype == 0) unpermute_kernel<__nv_bfloat16, 64><<<grid_x, 256, 0, st>>>(a);
    else unpermute_kernel<float, 64><<<grid_x, 256, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, int D, cudaStream_t st) {
  const int64_t warps = (int64_t)a.BH * a.n_groups * 2 * 128;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (D == 128) combine_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(a);
  else combine_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace ug
