// Weights of the warm start's fused path for integer ratios (W = 4 w, H = ry h, ry <= 8):
// every output is a fixed combination of the 3 x 3 low-resolution neighbourhood of its cell
// (indices clamped at the edges), with weights that depend only on the output's phase inside
// the cell.  Host side: api.cu; device side: warm_start.cu.
#pragma once

#include <cuda_runtime.h>

#include "kernels.h"

namespace ug {

struct WarmFused {
  int ry;                          // H / h
  float ra[8][3], rb[8][3];        // row phase p: bilinear, and blurred bilinear, weights of
                                   //   low-resolution rows k-1, k, k+1
  float ca[4][3], cb[4][3];        // column phase q: (1-alpha)(1+s) x bilinear and
                                   //   -(1-alpha) s x blurred bilinear weights of l-1, l, l+1
};

cudaError_t launch_warm_start_fused(const WarmArgs& a, const WarmFused& f, cudaStream_t st);

}  // namespace ug
