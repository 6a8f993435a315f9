// Block-wide scan shared by the hybrid-format kernels.
#pragma once

#include "sge_common.cuh"

namespace sge {

// Exclusive prefix sum of v over the CTA (blockDim.x a multiple of 32, at
// most 1024): shuffles within warps, then one warp over the warp totals.
// *total gets the CTA's sum.  Every thread of the CTA must call it.  wsum:
// 33 ints of shared memory.
SGE_DEV int block_scan_exclusive(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < nw ? wsum[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < nw) wsum[lane] = wi - w;
    if (lane == 31) wsum[32] = wi;  // the total
  }
  __syncthreads();
  const int r = wsum[warp] + incl - v;
  *total = wsum[32];
  __syncthreads();  // wsum may be reused after the return
  return r;
}

}  // namespace sge
