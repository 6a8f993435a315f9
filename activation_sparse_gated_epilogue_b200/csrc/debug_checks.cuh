// Index checks of the debug build.  Compiled with SGE_DEBUG (libsge_debug.so),
// every checked index that falls outside its range sets SGE_FLAG_BOUNDS in
// the translation unit's debug word (read and cleared by sge_debug_flags)
// and is replaced by an index inside the range, so the kernel goes on
// without touching memory it does not own; nothing traps.  In the release
// build checked_index is the identity and clamp_index the plain clamp the
// kernels always apply to stored TwELL columns.
#pragma once

#include "sge_common.cuh"
#include "sge_host.h"

namespace sge {

#ifdef SGE_DEBUG
static __device__ int g_debug_word;

SGE_DEV void debug_flag() { atomicOr(&g_debug_word, SGE_FLAG_BOUNDS); }

// i if 0 <= i < n, else 0 (flagged)
SGE_DEV int64_t checked_index(int64_t i, int64_t n) {
  if (i >= 0 && i < n) return i;
  debug_flag();
  return 0;
}

// a stored local column k of a tile of width n, kept inside the tile
SGE_DEV int clamp_index(int k, int n) {
  if (k < 0 || k >= n) debug_flag();
  return max(0, min(k, n - 1));
}

static int read_debug_word(bool clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_debug_word, sizeof(int)) != cudaSuccess) return -1;
  if (clear) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_debug_word, &z, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}
static const bool g_debug_registered = register_debug_reader(&read_debug_word);
#else
SGE_DEV int64_t checked_index(int64_t i, int64_t) { return i; }
SGE_DEV int clamp_index(int k, int n) { return min(k, n - 1); }
#endif

}  // namespace sge
