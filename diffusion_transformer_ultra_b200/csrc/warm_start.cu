// Warm-start initialisation of the high-resolution latent ("UltraGen ..." papernotes note,
// 关键设计 4 and its blend equation; gist.science summary, Methodology D):
//
//   U     = bilinear upsampling of the low-resolution latent to the high-resolution grid
//           (half-pixel centres, source index clamped at 0 and at the last row/column),
//   X_ref = U + s (U - B(U)),  B = 3x3 binomial blur (1 2 1)^T (1 2 1) / 16, edges replicated,
//   X_hr  = alpha X_T + (1 - alpha) X_ref.
//
// X_T is read from the caller's buffer, or, without one, drawn in the kernel: Philox4x32-10
// (Salmon, Moraes, Dror, Shaw, SC 2011) over the flat output index, each 32-bit word mapped
// to (floor(x / 2^9) + 1/2) 2^-23 in (0, 1), then the Box-Muller transform.
//
// HBM-bound: per output element 4 bytes of noise read (none when drawn here) and 4 bytes
// written; the low-resolution latent is 1/rho^2 of that.  One CTA computes a 32 x 128 output
// tile of one (batch, channel) plane.  Each thread first issues the noise loads of its 4
// output rows (16 bytes each), so they are in flight while the CTA stages the low-resolution
// patch under the tile in shared memory (one coalesced pass) and evaluates U on the tile
// plus a one-element border from it, separably: vertical interpolation once per (U row,
// patch column), then horizontal.  Then each warp sweeps 4 rows with the vertical blur
// window held in registers, each lane owning 4 consecutive columns (16-byte loads and stores
// when the row width and the pointers allow it).
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "warm_fused.h"

namespace ug {
namespace {

constexpr int kTH = 32, kTW = 128, kWarmThreads = 256;
constexpr int kUCols = kTW + 8;   // shared columns: tile column c lives at c + 4 (c = -1 .. 128)
// low-resolution patch staged in shared memory (rows x columns); a tile whose patch is larger
// (a ratio near or below 1) reads the latent through L1/L2 instead
constexpr int kPR = 36, kPC = 132;

__device__ __forceinline__ void axis_tap(int i, float scale, int n_in, int& i0, int& i1, float& f) {
  const float src = fmaxf((static_cast<float>(i) + 0.5f) * scale - 0.5f, 0.0f);
  const int a = min(static_cast<int>(src), n_in - 1);   // src >= 0, so truncation is floor
  i0 = a;
  i1 = min(a + 1, n_in - 1);
  f = src - static_cast<float>(a);
}

// Philox4x32 with 10 rounds (the published round function and key schedule).
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k.x += 0x9E3779B9u;
      k.y += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
  }
  return c;
}

__device__ __forceinline__ float unit_open(uint32_t x) {
  return (static_cast<float>(x >> 9) + 0.5f) * 0x1p-23f;   // exact: 24 significant bits
}

__device__ __forceinline__ float2 box_muller(uint32_t a, uint32_t b) {
  const float r = sqrtf(-2.0f * logf(unit_open(a)));
  float s, c;
  sincospif(2.0f * unit_open(b), &s, &c);
  return make_float2(r * c, r * s);
}

// The four normals of Philox block g of the stream (seed, offset).
__device__ __forceinline__ float4 normals4(uint64_t g, uint64_t seed, uint64_t offset) {
  const uint4 w = philox4x32_10(
      make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32),
                 static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32)),
      make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
  const float2 z01 = box_muller(w.x, w.y), z23 = box_muller(w.z, w.w);
  return make_float4(z01.x, z01.y, z23.x, z23.y);
}

__device__ __forceinline__ float lane_of(const float4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

__global__ void __launch_bounds__(kWarmThreads) warm_start_kernel(const WarmArgs a) {
  // the low-resolution patch P is dead once V is built, so U reuses its storage
  static_assert(kPR * kPC >= (kTH + 2) * kUCols, "U must fit in the patch buffer");
  __shared__ __align__(16) float PU[kPR * kPC];
  __shared__ float V[(kTH + 2) * kPC];      // patch interpolated to the U rows
  float* P = PU;
  float(*U)[kUCols] = reinterpret_cast<float(*)[kUCols]>(PU);
  __shared__ int cx0[kTW + 2], cx1[kTW + 2], ry0[kTH + 2], ry1[kTH + 2];
  __shared__ float cfx[kTW + 2], rfy[kTH + 2];

  const int plane = blockIdx.z;
  const int ty0 = blockIdx.y * kTH, tx0 = blockIdx.x * kTW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c4 = 4 * lane;                 // tile columns c4 .. c4 + 3
  const int x = tx0 + c4;
  const int r0 = warp * (kTH / 8);        // this warp's first tile row
  // the noise of this thread's outputs, requested before anything else
  float4 nz[kTH / 8];
  if (a.vec && a.noise && x < a.W) {
#pragma unroll
    for (int o = 0; o < kTH / 8; ++o) {
      const int y = min(ty0 + r0 + o, a.H - 1);
      nz[o] = __ldcs(reinterpret_cast<const float4*>(
          a.noise + (static_cast<uint64_t>(plane) * a.H + y) * a.W + x));
    }
  }
  // bilinear taps of the U rows/columns this tile needs (HR index clamped: replicated edges)
  for (int t = threadIdx.x; t < kTW + 2; t += kWarmThreads) {
    const int xx = min(max(tx0 - 1 + t, 0), a.W - 1);
    axis_tap(xx, a.sx, a.w, cx0[t], cx1[t], cfx[t]);
  }
  for (int t = threadIdx.x; t < kTH + 2; t += kWarmThreads) {
    const int y = min(max(ty0 - 1 + t, 0), a.H - 1);
    axis_tap(y, a.sy, a.h, ry0[t], ry1[t], rfy[t]);
  }
  __syncthreads();
  const float* L = a.lr + static_cast<size_t>(plane) * a.h * a.w;
  // the taps are monotone in the output index, so the patch is [ry0[0], ry1[last]] x [cx0[0], ..]
  const int pr0 = ry0[0], pc0 = cx0[0];
  const int npr = ry1[kTH + 1] - pr0 + 1, npc = cx1[kTW + 1] - pc0 + 1;
  if (npr <= kPR && npc <= kPC) {
    // separable: stage the patch, interpolate it vertically once per (U row, patch column),
    // then horizontally with each thread holding one U column's taps
    for (int r = warp; r < npr; r += kWarmThreads / 32) {
      const float* src = L + static_cast<size_t>(pr0 + r) * a.w + pc0;
      for (int c = lane; c < npc; c += 32) P[r * kPC + c] = __ldg(src + c);
    }
    __syncthreads();
    for (int r = warp; r < kTH + 2; r += kWarmThreads / 32) {
      const float* top = P + (ry0[r] - pr0) * kPC;
      const float* bot = P + (ry1[r] - pr0) * kPC;
      const float fy = rfy[r];
      for (int c = lane; c < npc; c += 32) V[r * kPC + c] = fmaf(fy, bot[c] - top[c], top[c]);
    }
    __syncthreads();
    for (int uc = threadIdx.x & 127; uc < kTW + 2; uc += 128) {
      const int i0 = cx0[uc] - pc0, i1 = cx1[uc] - pc0;
      const float fx = cfx[uc];
      for (int r = threadIdx.x >> 7; r < kTH + 2; r += 2) {
        const float v0 = V[r * kPC + i0], v1 = V[r * kPC + i1];
        U[r][uc + 3] = fmaf(fx, v1 - v0, v0);
      }
    }
  } else {
    for (int e = threadIdx.x; e < (kTH + 2) * (kTW + 2); e += kWarmThreads) {
      const int r = e / (kTW + 2), c = e - r * (kTW + 2);
      const float* g0 = L + static_cast<size_t>(ry0[r]) * a.w;
      const float* g1 = L + static_cast<size_t>(ry1[r]) * a.w;
      const float v00 = __ldg(g0 + cx0[c]), v01 = __ldg(g0 + cx1[c]);
      const float v10 = __ldg(g1 + cx0[c]), v11 = __ldg(g1 + cx1[c]);
      const float fx = cfx[c], fy = rfy[r];
      const float top = fmaf(fx, v01 - v00, v00);
      const float bot = fmaf(fx, v11 - v10, v10);
      U[r][c + 3] = fmaf(fy, bot - top, top);
    }
  }
  __syncthreads();

  if (x >= a.W) return;
  const float amount = a.amount, alpha = a.alpha, beta = 1.0f - alpha;
  // horizontal (1 2 1) sums and centre values of U rows, a sliding window of three
  float hb[3][4], mid[3][4];
  auto load_row = [&](int ur, float (&h)[4], float (&m)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(&U[ur][c4 + 4]);
    const float l = U[ur][c4 + 3], rgt = U[ur][c4 + 8];
    m[0] = v.x; m[1] = v.y; m[2] = v.z; m[3] = v.w;
    h[0] = l + 2.0f * v.x + v.y;
    h[1] = v.x + 2.0f * v.y + v.z;
    h[2] = v.y + 2.0f * v.z + v.w;
    h[3] = v.z + 2.0f * v.w + rgt;
  };
  const uint64_t row0 = (static_cast<uint64_t>(plane) * a.H + ty0 + r0) * a.W + x;   // flat index, row r0
  load_row(r0, hb[0], mid[0]);
  load_row(r0 + 1, hb[1], mid[1]);
#pragma unroll
  for (int o = 0; o < kTH / 8; ++o) {
    const int y = ty0 + r0 + o;
    load_row(r0 + o + 2, hb[(o + 2) % 3], mid[(o + 2) % 3]);
    if (y >= a.H) break;
    const float(&hu)[4] = hb[o % 3];
    const float(&hc)[4] = hb[(o + 1) % 3];
    const float(&hd)[4] = hb[(o + 2) % 3];
    const float(&u)[4] = mid[(o + 1) % 3];
    float ref[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float blur = (hu[q] + 2.0f * hc[q] + hd[q]) * 0.0625f;
      ref[q] = fmaf(amount, u[q] - blur, u[q]);
    }
    const uint64_t flat = row0 + static_cast<uint64_t>(o) * a.W;
    const int nq = min(4, a.W - x);
    if (a.vec) {   // W % 4 == 0 and 16-byte aligned buffers: flat is a multiple of 4
      const float4 n = a.noise ? nz[o] : normals4(flat >> 2, a.seed, a.offset);
      float4 out;
      out.x = fmaf(alpha, n.x, beta * ref[0]);
      out.y = fmaf(alpha, n.y, beta * ref[1]);
      out.z = fmaf(alpha, n.z, beta * ref[2]);
      out.w = fmaf(alpha, n.w, beta * ref[3]);
      __stcs(reinterpret_cast<float4*>(a.out + flat), out);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q >= nq) break;
        const uint64_t f = flat + q;
        const float n = a.noise ? __ldcs(a.noise + f) : lane_of(normals4(f >> 2, a.seed, a.offset),
                                                                static_cast<int>(f & 3));
        a.out[f] = fmaf(alpha, n, beta * ref[q]);
      }
    }
  }
}

// Integer ratios (W = 4 w, H = ry h): upsampling, blur, sharpening and the blend are linear
// and separable, so output (ry k + p, 4 l + q) is
//   alpha X_T + sum_j ca[q][j] Ra[j] + sum_j cb[q][j] Rb[j],
//   Ra[j] = sum_i ra[p][i] X(k + i - 1, l + j - 1),  Rb[j] = sum_i rb[p][i] X(k + i - 1, l + j - 1),
// with X read at clamped indices.  Clamping reproduces both edge rules: a source coordinate
// clamped at 0 (or a second tap clamped at the last row) reads one value with weights summing
// to 1, and the blur's replicated edge row equals the upsampled edge row, which is that value.
// One thread per low-resolution cell: its 3 x 3 neighbourhood, then ry rows of 4 outputs (one
// 16-byte load of noise and one 16-byte store each); a warp covers 32 cells of one row, so
// loads and stores are 512-byte runs.
template <int RY>
__global__ void __launch_bounds__(kWarmThreads) warm_start_fused_kernel(const WarmArgs a,
                                                                        const WarmFused wf) {
  const int plane = blockIdx.z;
  const int l = blockIdx.x * 32 + (threadIdx.x & 31);
  const int k = blockIdx.y * (kWarmThreads / 32) + (threadIdx.x >> 5);
  if (l >= a.w || k >= a.h) return;
  const int x = 4 * l;
  // first output row of the cell; rows of one plane step by W elements
  const size_t first = (static_cast<size_t>(plane) * a.H + static_cast<size_t>(k) * RY) * a.W + x;
  float* out = a.out + first;
  // the noise of the cell's outputs first, so the loads are in flight during the arithmetic
  float4 nz[RY];
  if (a.noise) {
    const float* nzp = a.noise + first;
#pragma unroll
    for (int p = 0; p < RY; ++p)
      nz[p] = __ldcs(reinterpret_cast<const float4*>(nzp + static_cast<size_t>(p) * a.W));
  }
  const float* L = a.lr + static_cast<size_t>(plane) * a.h * a.w;
  const int c0 = max(l - 1, 0), c2 = min(l + 1, a.w - 1);
  float X[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const float* row = L + static_cast<size_t>(min(max(k + i - 1, 0), a.h - 1)) * a.w;
    X[i][0] = __ldg(row + c0);
    X[i][1] = __ldg(row + l);
    X[i][2] = __ldg(row + c2);
  }
  const float alpha = a.alpha;
#pragma unroll
  for (int p = 0; p < RY; ++p) {
    float Ra[3], Rb[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      Ra[j] = fmaf(wf.ra[p][2], X[2][j], fmaf(wf.ra[p][1], X[1][j], wf.ra[p][0] * X[0][j]));
      Rb[j] = fmaf(wf.rb[p][2], X[2][j], fmaf(wf.rb[p][1], X[1][j], wf.rb[p][0] * X[0][j]));
    }
    float r[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float acc = wf.ca[q][0] * Ra[0];
      acc = fmaf(wf.ca[q][1], Ra[1], acc);
      acc = fmaf(wf.ca[q][2], Ra[2], acc);
      acc = fmaf(wf.cb[q][0], Rb[0], acc);
      acc = fmaf(wf.cb[q][1], Rb[1], acc);
      r[q] = fmaf(wf.cb[q][2], Rb[2], acc);
    }
    const float4 n = a.noise ? nz[p]
                             : normals4((first + static_cast<size_t>(p) * a.W) >> 2, a.seed, a.offset);
    __stcs(reinterpret_cast<float4*>(out + static_cast<size_t>(p) * a.W),
           make_float4(fmaf(alpha, n.x, r[0]), fmaf(alpha, n.y, r[1]), fmaf(alpha, n.z, r[2]),
                       fmaf(alpha, n.w, r[3])));
  }
}

}  // namespace

cudaError_t launch_warm_start(const WarmArgs& a, cudaStream_t st) {
  const dim3 grid((a.W + kTW - 1) / kTW, (a.H + kTH - 1) / kTH, a.planes);
  warm_start_kernel<<<grid, kWarmThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_warm_start_fused(const WarmArgs& a, const WarmFused& f, cudaStream_t st) {
  const dim3 grid((a.w + 31) / 32, (a.h + kWarmThreads / 32 - 1) / (kWarmThreads / 32), a.planes);
  switch (f.ry) {   // the row ratio as a constant: fully unrolled rows, no bounds checks
    case 1: warm_start_fused_kernel<1><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 2: warm_start_fused_kernel<2><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 3: warm_start_fused_kernel<3><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 4: warm_start_fused_kernel<4><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 5: warm_start_fused_kernel<5><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 6: warm_start_fused_kernel<6><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 7: warm_start_fused_kernel<7><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    case 8: warm_start_fused_kernel<8><<<grid, kWarmThreads, 0, st>>>(a, f); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ug
