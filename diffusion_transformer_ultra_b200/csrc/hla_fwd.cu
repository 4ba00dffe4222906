// Block-sparse masked attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes softmax(Q K^T / sqrt(d) + M) V over the window-first layout ("UltraGen ..."
// papernotes note, 关键设计 3, the MMA equation, with M read as an additive -inf on masked
// pairs), visiting for each query tile only the key tiles its plan list names; masks are
// applied per element on partial tiles only.
//
// CTA organisation (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warps 0-3   softmax group 0: owns query tile slot 0 (thread = row, TMEM lane = row)
//   warps 4-7   softmax group 1: owns query tile slot 1
//   warp  8     producer: TMA loads of Q (per item) and of K, V tiles in stages
//   warp  9     MMA issuer: tcgen05.mma for S = Q K^T (both operands in shared memory) and
//               O += P V (P read from TMEM, V from shared memory); owns TMEM allocation
//   warps 10-11 idle
// The kernel is compiled for 168 registers per thread (384 x 168 = 64,512); the control
// warpgroup gives registers back (setmaxnreg 56) so the softmax groups can hold a whole
// 128-column S row in registers (setmaxnreg 224): 2 x 128 x 224 + 128 x 56 = 64,512.
// A work item is one or two query tiles with the same key list (the two 128-row halves of
// a 16x16 window, two text tiles, two LR tiles), so each K/V tile is loaded once per two
// query tiles.  The issue order S0(j) / S1(j) / [P0 V(j)] / S0(j+1) ... lets one softmax
// group work on its tile while the tensor core runs the other group's products.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D, 256+2D).
// P (bf16, packed in pairs) overwrites the first 64 columns of its S block.
// Shared memory: Q0, Q1, and NS K/V tile slots, each [128 rows x D] bf16 stored as D/64 boxes
// of [128 x 64] with the 128-byte swizzle (TMA writes it, the MMA descriptors read it).  K/V
// tiles travel in stages of two: stage j of an item with n key tiles holds V(j-1) (j > 0) and
// K(j) (j < n), exactly what step j of the MMA loop reads, so the MMA warp waits on one full
// barrier per key tile and releases both slots with one commit.
// With 8-bit Q K^T (QK8, D = 128) Q and K tiles are e4m3 bytes, one [128 x 128] box of 128-byte
// rows at the start of their slot, and S = Q K^T takes 4 kind::f8f6f4 products of 32
// K-elements instead of 8 kind::f16 products of 16; V, P and O are unchanged.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "exp2_poly.h"
#include "kernels.h"
#include "ptx.cuh"

#ifndef ULTRAGEN_DEBUG
#define ULTRAGEN_DEBUG 0
#endif

namespace ug {

// Index checks of debug builds (ULTRAGEN_DEBUG): a plan index or tile coordinate outside its
// table or tensor stops the CTA before the access, the way a timed-out wait does (abort flag,
// DEV_BOUNDS in the error word).  Release builds compile them away.
__device__ __forceinline__ bool bounds_fail(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicExch(err, DEV_BOUNDS);
  return false;
}
#if ULTRAGEN_DEBUG
#define UG_CHECK(cond) ((cond) || bounds_fail(abort_flag, p.err))
#else
#define UG_CHECK(cond) true
#endif

template <int D>
struct FwdCfg {
  static constexpr int BOXES = D / 64;
  static constexpr int BOX_BYTES = 128 * 64 * 2;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NS = D == 128 ? 4 : 8;      // tile slots
  static constexpr int NSTG = NS / 2;               // stages in flight (two tiles each)
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NS * TILE_BYTES;
  // barrier indices
  // B_KVF / B_KVE + g: stage slot g full / empty (g < NSTG)
  // B_IF / B_IE + s: item ring slot s full / empty (s < NIR)
  static constexpr int NIR = 4;                     // item ring slots
  static constexpr int B_QF = 0, B_QE = 1, B_KVF = 2, B_KVE = 2 + NSTG, B_SF = 2 + 2 * NSTG,
                       B_PF = 4 + 2 * NSTG, B_OF = 6 + 2 * NSTG, B_DRAIN = 8 + 2 * NSTG,
                       B_IF = 9 + 2 * NSTG, B_IE = 9 + 2 * NSTG + NIR;
  static constexpr int NBAR = 9 + 2 * NSTG + 2 * NIR;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  // misc words: 0 TMEM base, 1 abort flag, 2-3 unused, 4.. the item ring
  static constexpr int RING_OFF = MISC_OFF + 16;
  static constexpr int SMEM_BYTES = RING_OFF + 4 * NIR + 1024;   // + slack for 1024-B alignment
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA exceeds 227 KB");
  // the tile slots of stage slot g: V at 2 g, K at 2 g + 1
  static __device__ __forceinline__ uint32_t v_slot(uint32_t g) { return 2 * g; }
  static __device__ __forceinline__ uint32_t k_slot(uint32_t g) { return 2 * g + 1; }
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL = 256;
};

constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;      // per thread at launch: 65536 / 384, rounded down to 8
constexpr int kRegsSoftmax = 224;
constexpr int kRegsControl = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr uint64_t kDrainNs = 50ull * 1000 * 1000;   // bounded drain on the abort path

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// 2^x for a pair of arguments on the FMA pipe (Cody-Waite range reduction + minimax
// polynomial): n = round(x) by the 1.5 * 2^23 shifter, f = x - n in [-1/2, 1/2],
// 2^x = 2^n * p(f), with n added to the exponent field as an integer.  x is clamped at -125
// so the result stays a normal float; 2^-125 then stands for 0 (masked entries), far below
// any visible weight.
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 u = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = ffma2(u, make_float2(-1.0f, -1.0f), x);
  float2 p = ffma2(f, make_float2(UG_EXP2_C3, UG_EXP2_C3), make_float2(UG_EXP2_C2, UG_EXP2_C2));
  p = ffma2(f, p, make_float2(UG_EXP2_C1, UG_EXP2_C1));
  p = ffma2(f, p, make_float2(UG_EXP2_C0, UG_EXP2_C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Which exponential pairs (of the 64 in a row of a tile) go to ex2_fma2 instead of the SFU.
#ifndef UG_FMA_EXP_MASK
#define UG_FMA_EXP_MASK 0
#endif
__device__ __forceinline__ constexpr bool pair_on_fma(int c2) {
  return ((UG_FMA_EXP_MASK >> (c2 & 7)) & 1) != 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Work items reach the roles of a CTA through a ring of NIR slots in shared memory.  The
// producer thread takes the next item of the launch -- from the work counter (one atomic add
// per item, so a CTA that finishes early takes more), or from the round-robin sequence
// blockIdx.x, blockIdx.x + gridDim.x, ... without one -- writes its index, or -1 after the
// last, into slot k % NIR and arrives on that slot's "full" barrier; the MMA thread and the
// eight softmax warps read the slot and arrive on its "empty" barrier.
constexpr int kRingReaders = 1 + 8;     // the MMA thread and one arrive per softmax warp

// The i-th work item of the launch: its 8-int record and its (batch, head) index.
__device__ __forceinline__ const int32_t* item_at(const FwdParams& p, int it, int& bh) {
  if (p.item_major) {
    const int k = it / p.units;
    bh = it - k * p.units;
    return p.items + __ldg(p.item_order + k) * 8;
  }
  const int nl = p.n_long * p.units;
  if (it < nl) {
    const int k = it / p.units;
    bh = it - k * p.units;
    return p.items + k * 8;
  }
  it -= nl;
  const int nr = p.n_items_head - p.n_long;
  bh = it / nr;
  return p.items + (p.n_long + it - bh * nr) * 8;
}

// ------------------------------------------------------------------------ producer warp
template <int D, bool QK8>
__device__ void producer_role(const CUtensorMap* tmQ, const CUtensorMap* tmK,
                              const CUtensorMap* tmV, const HaloMaps* hm, const FwdParams& p,
                              uint32_t sbase, volatile int* abort_flag) {
  using C = FwdCfg<D>;
  constexpr int QK_BYTES = QK8 ? 128 * D : C::TILE_BYTES;   // one Q or K tile
  const uint32_t sQ = sbase + C::Q_OFF, sKV = sbase + C::KV_OFF, bar = sbase + C::BAR_OFF;
  uint32_t st = 0, qi = 0, ik = 0;                          // stages, Q loads, items published
  bool ok = true;
  // one tile: e4m3 Q or K is a single [128 x 128]-byte box, bf16 D / 64 boxes of [128 x 64]
  auto load_tile = [&](const CUtensorMap* tm, bool bytes, uint32_t dst, int y, uint32_t b) {
    if (bytes) {
      tma_load_2d(dst, tm, 0, y, b);
    } else {
#pragma unroll
      for (int bx = 0; bx < C::BOXES; ++bx) tma_load_2d(dst + bx * C::BOX_BYTES, tm, bx * 64, y, b);
    }
  };
  // key (isv = 0) or value (1) tile kt of (batch, head) bh: a window-first tile, or a tile of a
  // window's halo block assembled from its neighbours' window-first slots, one box per piece
  // (b x l, l x b or b x b tokens of one window, raster order) and zero-filled boxes for the
  // gaps.  Every box lands at a multiple of 8 rows (1 KB) of the 128-byte-swizzled slot, so
  // the tile reads exactly as if its 128 rows had been copied there.
  auto load_kv = [&](bool isv, uint32_t dst, int kt, int bh, uint32_t b) {
    if (p.halo_ops == nullptr || kt < p.halo_tile0) {
      load_tile(isv ? tmV : tmK, !isv && QK8, dst, bh * p.N_kv + kt * 128, b);
      return true;
    }
    const int v = kt - p.halo_tile0;
    const int w = v / p.halo_gtiles, tb = v - w * p.halo_gtiles;
    const int wr = w / p.nWw, wc = w - wr * p.nWw;
    const int o0 = __ldg(p.halo_ops + tb), o1 = __ldg(p.halo_ops + tb + 1);
    if (!UG_CHECK(o0 > p.halo_gtiles && o0 <= o1 && o1 <= p.n_halo_ops)) return false;
    for (int o = o0; o < o1; ++o) {
      const uint32_t c = (uint32_t)__ldg(p.halo_ops + o);
      const int row = c & 127, shape = (c >> 7) & 3;
      const int sr = wr + (int)((c >> 10) & 3) - 1, sc = wc + (int)((c >> 12) & 3) - 1;
      const int i0 = (c >> 14) & 255, j0 = (c >> 22) & 255;
      if (!UG_CHECK(shape <= 2 && row % 8 == 0)) return false;
      // a zero box, or a piece of a window outside the image, reads window -1: out of bounds
      // as a whole, it lands as zeros
      const bool zero = ((c >> 9) & 1) || sr < 0 || sr >= p.nWh || sc < 0 || sc >= p.nWw;
      const int win = zero ? -1 : sr * p.nWw + sc;
      const CUtensorMap* tm = &hm->m[(isv ? 3 : 0) + shape];
      if (!isv && QK8) {
        tma_load_5d(dst + row * 128, tm, 0, j0, i0, win, bh, b);
      } else {
#pragma unroll
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_load_5d(dst + bx * C::BOX_BYTES + row * 128, tm, bx * 64, j0, i0, win, bh, b);
      }
    }
    return true;
  };
  while (ok) {
    // the ik-th item of this CTA: from the counter, or round-robin
    int it = p.sched != nullptr ? atomicAdd(p.sched, 1) : (int)(blockIdx.x + ik * gridDim.x);
    if (it >= p.total_items) it = -1;
    {
      const uint32_t s = ik % C::NIR;
      if (!mbar_wait(bar + 8 * (C::B_IE + s), ((ik / C::NIR) & 1) ^ 1, abort_flag, p.err,
                     DEV_TIMEOUT_PRODUCER, p.timeout_ns)) {
        ok = false;
        break;
      }
      st_shared_s32(sbase + C::RING_OFF + 4 * s, it);
      mbar_arrive(bar + 8 * (C::B_IF + s));
      ++ik;
    }
    if (it < 0) break;
    int bh;
    const int32_t* I = item_at(p, it, bh);
    const int qt0 = I[0], qt1 = I[1], e0 = I[2], n = I[3] - I[2];
    if (!UG_CHECK(bh >= 0 && bh < p.units && e0 >= 0 && n >= 0 && e0 + n <= p.n_entries &&
                  qt0 >= 0 && qt0 * 128 < p.N_tot &&
                  (qt1 == -1 || (qt1 >= 0 && qt1 * 128 < p.N_tot)))) {
      ok = false;
      break;
    }
    if (n == 0) continue;
    if (!mbar_wait(bar + 8 * C::B_QE, (qi & 1) ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER,
                   p.timeout_ns)) {
      ok = false;
      break;
    }
    const int ntile = qt1 >= 0 ? 2 : 1;
    mbar_expect_tx(bar + 8 * C::B_QF, ntile * QK_BYTES);
    for (int t = 0; t < ntile; ++t)
      load_tile(tmQ, QK8, sQ + t * C::TILE_BYTES, bh * p.N_tot + (t ? qt1 : qt0) * 128,
                bar + 8 * C::B_QF);
    ++qi;
    for (int j = 0; j <= n; ++j) {   // stage j: V(j - 1) if j > 0, K(j) if j < n
      const uint32_t g = st % C::NSTG, ph = (st / C::NSTG) & 1;
      if (!mbar_wait(bar + 8 * (C::B_KVE + g), ph ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER,
                     p.timeout_ns)) {
        ok = false;
        break;
      }
      const uint32_t fb = bar + 8 * (C::B_KVF + g);
      const int kv = j > 0 ? (__ldg(p.entries + e0 + j - 1) & 0x7fffffff) : 0;
      const int kk = j < n ? (__ldg(p.entries + e0 + j) & 0x7fffffff) : 0;
      if (!UG_CHECK(kv < p.n_ktiles && kk < p.n_ktiles)) {
        ok = false;
        break;
      }
      mbar_expect_tx(fb, (j > 0 ? C::TILE_BYTES : 0) + (j < n ? QK_BYTES : 0));
      ++st;
      if (j > 0 && !load_kv(true, sKV + C::v_slot(g) * C::TILE_BYTES, kv, bh, fb)) {
        ok = false;
        break;
      }
      if (j < n && !load_kv(false, sKV + C::k_slot(g) * C::TILE_BYTES, kk, bh, fb)) {
        ok = false;
        break;
      }
    }
  }
  if (!ok) {
    // Abort: wait (bounded) until the copies this thread issued have landed, so that no TMA
    // write targets this CTA's shared memory after it exits.
    for (uint32_t g = st >= (uint32_t)C::NSTG ? st - C::NSTG : 0; g < st; ++g)
      mbar_wait(bar + 8 * (C::B_KVF + g % C::NSTG), (g / C::NSTG) & 1, nullptr, p.err,
                DEV_TIMEOUT_DRAIN, kDrainNs);
    if (qi > 0) mbar_wait(bar + 8 * C::B_QF, (qi - 1) & 1, nullptr, p.err, DEV_TIMEOUT_DRAIN, kDrainNs);
  }
  // The work counter resets itself for the next launch: each CTA's producer counts itself out
  // once it will take no more items (on the abort path too), and the last one clears both
  // words, when no producer of this launch can take another item.
  if (p.sched != nullptr && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
    atomicExch(p.sched, 0);
    atomicExch(p.sched + 1, 0);
  }
}

// ------------------------------------------------------------------------ MMA warp
template <int D, bool QK8>
__device__ __forceinline__ void issue_s(uint32_t tmem_d, uint32_t sQt, uint32_t sK) {
  using C = FwdCfg<D>;
  constexpr uint32_t hi = desc_hi_sw128(1024);
  const uint32_t qlo = desc_lo(sQt, 16), klo = desc_lo(sK, 16);
  if (QK8) {
    // e4m3 rows of 128 bytes: each product takes the next 32 bytes (32 K-elements) of the row
    constexpr uint32_t idS = idesc_e4m3(128, 128);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk)
      mma_ss_f8_w(tmem_d, qlo + kk * 2, klo + kk * 2, hi, idS, kk > 0 ? 1u : 0u);
  } else {
    constexpr uint32_t idS = idesc_bf16(128, 128, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
      mma_ss_w(tmem_d, qlo + off, klo + off, hi, idS, kk > 0 ? 1u : 0u);
    }
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t tmem_d, uint32_t tmem_p, uint32_t sV,
                                         bool accumulate) {
  using C = FwdCfg<D>;
  constexpr uint32_t idO = idesc_bf16(128, D, 1);
  constexpr uint32_t hi = desc_hi_sw128(1024);
  const uint32_t vlo = desc_lo(sV, C::BOX_BYTES);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_w(tmem_d, tmem_p + kk * 8, vlo + kk * (2048 >> 4), hi, idO,
             (accumulate || kk > 0) ? 1u : 0u);
}

template <int D, bool QK8>
__device__ void mma_role(const FwdParams& p, uint32_t sbase, uint32_t tbase,
                         volatile int* abort_flag) {
  using C = FwdCfg<D>;
  const uint32_t sQ = sbase + C::Q_OFF, sKV = sbase + C::KV_OFF, bar = sbase + C::BAR_OFF;
  uint32_t st = 0, qi = 0, pc0 = 0, pc1 = 0;   // stages, Q loads, P phases consumed
  bool withhold = p.fault == 1;   // injected fault: drop the first item's first "S ready"
  auto wait = [&](int b, uint32_t par) {
    return mbar_wait(bar + 8 * b, par, abort_flag, p.err, DEV_TIMEOUT_MMA, p.timeout_ns);
  };
  uint32_t ik = 0;
  bool ok = true;
  while (ok) {
    const uint32_t s = ik % C::NIR;
    if (!wait(C::B_IF + s, (ik / C::NIR) & 1)) { ok = false; break; }
    const int it = ld_shared_s32(sbase + C::RING_OFF + 4 * s);
    mbar_arrive(bar + 8 * (C::B_IE + s));
    ++ik;
    if (it < 0) break;
    int bh;
    const int32_t* I = item_at(p, it, bh);
    (void)bh;
    const int qt1 = I[1], n = I[3] - I[2];
    if (n == 0) continue;
    const int ntile = qt1 >= 0 ? 2 : 1;
    if (!wait(C::B_QF, qi & 1)) { ok = false; break; }
    ++qi;
    tc_fence_after();
    // step j of the item reads stage j: S_t(j) = Q_t K(j)^T needs K(j) (j < n), and
    // O_t += P_t(j - 1) V(j - 1) (j > 0) needs V(j - 1) and the softmax's P_t(j - 1)
    for (int j = 0; j <= n && ok; ++j) {
      const uint32_t g = st % C::NSTG;
      if (!wait(C::B_KVF + g, (st / C::NSTG) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sV = sKV + C::v_slot(g) * C::TILE_BYTES, sK = sKV + C::k_slot(g) * C::TILE_BYTES;
      for (int t = 0; t < ntile; ++t) {
        if (j > 0) {
          uint32_t& pc = t ? pc1 : pc0;
          if (!wait(C::B_PF + t, pc & 1)) { ok = false; break; }
          ++pc;
          tc_fence_after();
          issue_pv<D>(tbase + C::O_COL + D * t, tbase + 128 * t, sV, j > 1);
        }
        if (j < n) {
          issue_s<D, QK8>(tbase + 128 * t, sQ + t * C::TILE_BYTES, sK);
          if (withhold && t == 0) {
            withhold = false;     // nothing completes this barrier: its waiters time out
          } else {
            mma_commit(bar + 8 * (C::B_SF + t));
          }
        } else {
          mma_commit(bar + 8 * (C::B_OF + t));
        }
      }
      if (!ok) break;
      mma_commit(bar + 8 * (C::B_KVE + g));     // both tiles of the stage are read
      if (j == n - 1) mma_commit(bar + 8 * C::B_QE);   // all products that read Q are issued
      ++st;
    }
  }
  if (p.clock != nullptr && blockIdx.x == 0) {
    volatile unsigned long long* start = p.clock + 3;   // written by thread 0 at entry
    atomicAdd(p.clock, 1ull);
    atomicAdd(p.clock + 1, (unsigned long long)clock64() - start[0]);
    atomicAdd(p.clock + 2, globaltimer_ns() - start[1]);
  }
  if (!ok) {
    // Abort: let the products already issued finish before TMEM is released.
    mma_commit(bar + 8 * C::B_DRAIN);
    mbar_wait(bar + 8 * C::B_DRAIN, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN, kDrainNs);
  }
}

// ------------------------------------------------------------------------ softmax groups
// Exponentials of one S row at the running max mu (log2 units): the pair (s[2c], s[2c+1]) is
// replaced by its packed bf16 P in s[c].  Returns the row sum of this tile's P.
__device__ __forceinline__ float exp_row(uint32_t (&s)[128], float scale, float mu) {
  const float2 scale2 = make_float2(scale, scale), nmu2 = make_float2(-mu, -mu);
  float2 ls[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c2 = 0; c2 < 64; ++c2) {
    const float2 x =
        ffma2(make_float2(__uint_as_float(s[2 * c2]), __uint_as_float(s[2 * c2 + 1])), scale2, nmu2);
    float2 pp;
    if (pair_on_fma(c2)) {
      pp = ex2_fma2(x);
    } else {
      pp.x = ex2(x.x);
      pp.y = ex2(x.y);
    }
    ls[c2 & 3] = fadd2(ls[c2 & 3], pp);
    s[c2] = pack_bf16x2(pp.x, pp.y);
  }
  const float2 l2 = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
  return l2.x + l2.y;
}

// Multiplies the O accumulator row (TMEM) by f, 32 columns at a time.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float f) {
#pragma unroll 1
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t o[32];
    tmem_ld32_sync(tO + ch * 32, o);
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
    tmem_st32(tO + ch * 32, o);
  }
}

template <int D>
__device__ void softmax_role(const FwdParams& p, uint32_t sbase, uint32_t tbase,
                             volatile int* abort_flag) {
  using C = FwdCfg<D>;
  const uint32_t bar = sbase + C::BAR_OFF;
  const int t = threadIdx.x >> 7;                 // query tile slot 0 / 1
  const int r = threadIdx.x & 127;                // row inside the tile = TMEM lane
  const uint32_t lane_off = (uint32_t)((threadIdx.x >> 5) & 3) * 32u << 16;
  const uint32_t tS = tbase + lane_off + (uint32_t)(t * 128);
  const uint32_t tO = tbase + lane_off + C::O_COL + (uint32_t)(t * D);
  const float scale = p.scale_log2;
  uint32_t sc = 0, oc = 0, ik = 0;

  for (;;) {
    int it;
    {
      const uint32_t s = ik % C::NIR;
      const bool ok = mbar_wait(bar + 8 * (C::B_IF + s), (ik / C::NIR) & 1, abort_flag, p.err,
                                DEV_TIMEOUT_SOFTMAX, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) return;
      it = ld_shared_s32(sbase + C::RING_OFF + 4 * s);
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bar + 8 * (C::B_IE + s));
      ++ik;
    }
    if (it < 0) break;
    int bh;
    const int32_t* I = item_at(p, it, bh);
    const int qt = t ? I[1] : I[0];
    if (qt < 0) continue;
    const int e0 = I[2], n = I[3] - I[2], ws_slot = I[4], ncls = I[5], wfirst = I[6];
    const int slot = qt * 128 + r;
    const bool real = __ldg(p.perm + slot) >= 0;
    int cls = 0;
    if (ncls > 1 && wfirst >= 0) {
      cls = (slot - p.off_hr) / p.l2 - wfirst;
      cls = cls < 0 ? 0 : (cls > ncls - 1 ? ncls - 1 : cls);
    }
    // output row: permuted [bh][slot], or raster [b][token][h] (pad rows have no raster row)
    __nv_bfloat16* orow;
    if (!UG_CHECK(slot < p.N_tot && ws_slot < p.n_ws_head)) return;
    if (p.raster) {
      const int tok = __ldg(p.perm + slot);
      if (!UG_CHECK(tok < p.N_raster)) return;
      const int b = bh / p.heads, hh = bh - (bh / p.heads) * p.heads;
      orow = tok >= 0 ? p.out + (((size_t)b * p.N_raster + tok) * p.heads + hh) * D : nullptr;
    } else {
      orow = p.out + ((size_t)bh * p.N_tot + slot) * D;
    }
    if (n == 0) {
      if (!orow) continue;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
      continue;
    }
    float m = neg_inf(), lsum = 0.f;
    for (int j = 0; j < n; ++j) {
      const int ent = __ldg(p.entries + e0 + j);
      uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};
      if (ent < 0) {
        if (!UG_CHECK(__ldg(p.mask_off + e0 + j) >= 0 &&
                      __ldg(p.mask_off + e0 + j) + cls * 4 + 4 <= p.n_mask_words))
          return;
        const uint32_t* mp = p.mask_pool + __ldg(p.mask_off + e0 + j) + cls * 4;
#pragma unroll
        for (int w = 0; w < 4; ++w) mw[w] = __ldg(mp + w);
      }
      bool ok = mbar_wait(bar + 8 * (C::B_SF + t), sc & 1, abort_flag, p.err, DEV_TIMEOUT_SOFTMAX,
                          p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) return;
      ++sc;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld128_sync(tS, s);
      if (ent < 0) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = 0xff800000u;   // -inf
      }
      if (__any_sync(0xffffffffu, m == neg_inf())) {
        // A row without a running max yet (its first tile, or only masked scores so far):
        // take the tile max first (thread-local row, 4 chains of three-input max).
        float mx4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx4[i] = neg_inf();
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            mx4[i] = fmax3(mx4[i], __uint_as_float(s[c + 2 * i]), __uint_as_float(s[c + 2 * i + 1]));
        }
        const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]);
        const float mnew = fmaxf(m, mx * scale);
        // Lazy rescale: a row with a running max keeps it unless it grew by more than 2^8 (the
        // final division by the matching row sum makes the result exact either way); a row
        // without one takes the tile max (its O and sum are still zero).
        const bool need = m != neg_inf() && mnew > m + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2(m - mnew) : 1.0f;
          if (need) lsum *= f;
          __syncwarp();
          rescale_o<D>(tO, f);
        }
        if (m == neg_inf() || need) m = mnew;
        lsum += exp_row(s, scale, (m == neg_inf()) ? 0.f : m);
      } else {
        // Every row has a running max: take the exponentials at it, with no tile max at all.
        // The final division by the row sum makes the result exact for any max, and only
        // overflow must be excluded: a tile sum above 2^12 (also inf or NaN) means some score
        // may have risen far above the running max, so the tile is redone from S (still in
        // TMEM) at its exact max, with O and the sum rescaled to it (rare).
        float part = exp_row(s, scale, m);
        if (__any_sync(0xffffffffu, !(part <= 4096.0f))) {
          float mx = neg_inf();
#pragma unroll 1
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t c32[32];
            tmem_ld32_sync(tS + ch * 32, c32);
            const uint32_t mwc = ch == 0 ? mw[0] : (ch == 1 ? mw[1] : (ch == 2 ? mw[2] : mw[3]));
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float a = ((mwc >> c) & 1u) ? __uint_as_float(c32[c]) : neg_inf();
              const float b = ((mwc >> (c + 1)) & 1u) ? __uint_as_float(c32[c + 1]) : neg_inf();
              mx = fmax3(mx, a, b);
            }
          }
          const float mnew = fmaxf(m, mx * scale);
          const float f = ex2(m - mnew);
          lsum *= f;
          m = mnew;
          __syncwarp();
          rescale_o<D>(tO, f);
          tmem_ld128_sync(tS, s);
          if (ent < 0) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = 0xff800000u;
          }
          part = exp_row(s, scale, m);
        }
        lsum += part;
      }
      __syncwarp();
      tmem_st64(tS, s);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bar + 8 * (C::B_PF + t));
    }
    bool ok = mbar_wait(bar + 8 * (C::B_OF + t), oc & 1, abort_flag, p.err, DEV_TIMEOUT_SOFTMAX,
                        p.timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) return;
    ++oc;
    tc_fence_after();
    __syncwarp();
    const float inv = (lsum > 0.f) ? 1.0f / lsum : 0.f;
    if (ws_slot < 0) {
      // every lane loads (tcgen05.ld is warp-wide); rows without a raster row store nothing
      const float f = real ? inv : 0.f;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld32_sync(tO + ch * 32, o);
        if (orow) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * f, __uint_as_float(o[8 * q + 1]) * f);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * f, __uint_as_float(o[8 * q + 3]) * f);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * f, __uint_as_float(o[8 * q + 5]) * f);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * f, __uint_as_float(o[8 * q + 7]) * f);
            dst[q] = v;
          }
        }
      }
    } else {
      float* wsb = p.ws + ((size_t)bh * p.n_ws_head + ws_slot) * ((size_t)2 * 128 * (D + 1));
      float* wo = wsb + (size_t)(t * 128 + r) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32_sync(tO + ch * 32, o);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 v = make_float4(__uint_as_float(o[4 * q + 0]) * inv, __uint_as_float(o[4 * q + 1]) * inv,
                                 __uint_as_float(o[4 * q + 2]) * inv, __uint_as_float(o[4 * q + 3]) * inv);
          reinterpret_cast<float4*>(wo + ch * 32)[q] = v;
        }
      }
      wsb[2 * 128 * D + t * 128 + r] = (lsum > 0.f) ? m + log2f(lsum) : neg_inf();
    }
    tc_fence_before();
  }
}

// ------------------------------------------------------------------------ kernel
template <int D, bool QK8>
__global__ void __launch_bounds__(kThreads, 1)
    hla_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ HaloMaps hm,
                   const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + C::BAR_OFF;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // launch clock record: the first CTA lives for the whole persistent launch (the start values
  // wait in shared memory, not in registers the softmax roles need)

  if (threadIdx.x == 0) {
    // launch clock record: the first CTA lives for the whole persistent launch; its start goes
    // to the record's scratch words, its end is taken when its MMA warp has issued its last
    // product (the last item's epilogue, a few thousand cycles of millions, is left out)
    if (p.clock != nullptr && blockIdx.x == 0) {
      p.clock[3] = (unsigned long long)clock64();
      p.clock[4] = globaltimer_ns();
    }
    mbar_init(bar + 8 * C::B_QF, 1);
    mbar_init(bar + 8 * C::B_QE, 1);
    for (int s = 0; s < C::NSTG; ++s) {
      mbar_init(bar + 8 * (C::B_KVF + s), 1);
      mbar_init(bar + 8 * (C::B_KVE + s), 1);
    }
    for (int s = 0; s < C::NIR; ++s) {
      mbar_init(bar + 8 * (C::B_IF + s), 1);
      mbar_init(bar + 8 * (C::B_IE + s), kRingReaders);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar + 8 * (C::B_SF + t), 1);
      mbar_init(bar + 8 * (C::B_PF + t), 4);      // one arrive per softmax warp
      mbar_init(bar + 8 * (C::B_OF + t), 1);
    }
    mbar_init(bar + 8 * C::B_DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  if (warp >= 8) {
    regs_shrink<kRegsControl>();
    if (warp == kWarpProducer) {
      if (lane == 0) producer_role<D, QK8>(&tmQ, &tmK, &tmV, &hm, p, sbase, abort_flag);
    } else if (warp == kWarpMma) {
      if (lane == 0) mma_role<D, QK8>(p, sbase, tbase, abort_flag);
    }
  } else {
    regs_grow<kRegsSoftmax>();
    softmax_role<D>(p, sbase, tbase, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) {
    __syncwarp();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

template <int D, bool QK8>
static cudaError_t launch_d(const void* tmQ, const void* tmK, const void* tmV,
                            const HaloMaps* hm, const FwdParams& p, int grid, cudaStream_t st) {
  // The shared-memory size attribute belongs to the kernel on each device: set it once per
  // device (one process may drive several GPUs, from several threads).
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static bool attr_set[kMaxDev] = {};
  const int smem = FwdCfg<D>::SMEM_BYTES;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      // The register split above is only sound if the kernel really launches with
      // kRegsLaunch registers per thread; refuse to launch otherwise.
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, hla_fwd_kernel<D, QK8>);
      if (e != cudaSuccess) return e;
      if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
      e = cudaFuncSetAttribute(hla_fwd_kernel<D, QK8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  hla_fwd_kernel<D, QK8><<<grid, kThreads, smem, st>>>(*static_cast<const CUtensorMap*>(tmQ),
                                                        *static_cast<const CUtensorMap*>(tmK),
                                                        *static_cast<const CUtensorMap*>(tmV), *hm,
                                                        p);
  return cudaGetLastError();
}

cudaError_t launch_hla_fwd(const void* tmQ, const void* tmK, const void* tmV, const HaloMaps* hm,
                           const FwdParams& p, int D, int qk8, int grid, cudaStream_t st) {
  if (qk8) {
    if (D != 128) return cudaErrorInvalidValue;
    return launch_d<128, true>(tmQ, tmK, tmV, hm, p, grid, st);
  }
  return D == 128 ? launch_d<128, false>(tmQ, tmK, tmV, hm, p, grid, st)
                  : launch_d<64, false>(tmQ, tmK, tmV, hm, p, grid, st);
}

}  // namespace ug
