// Self-test of the failure handling of the tcgen05 GEMM engines (a
// test-only library, libsge_selftest.so, not part of libsge.so).
//
// Every wait of the engines is bounded: a wait that runs out sets
// SGE_FLAG_TIMEOUT in the caller's diag word, raises the CTA's abort flag,
// and the CTA drains its in-flight loads and MMAs (again with bounded waits),
// frees its tensor memory and returns, leaving the context usable.  This
// library builds the engines with a 20 ms deadline and runs them on a tile
// pipeline whose stage barriers can never complete: the B operand's tensor
// map has a box half as tall as the stage the producer arms for, so every
// stage receives fewer bytes than it expects.  The copies themselves are in
// bounds; only the barriers' transaction counts stay above zero.  The MMA
// issuer's first wait then runs out, and the abort and drain paths run.
#define SGE_WAIT_NS 20000000ull

#include "../../../include/sge_selftest.h"
#include "../tc_launch.cuh"

namespace sge {

// Counts the output tiles whose accumulators reached the epilogue (none may).
struct EpiCountTiles {
  int* tiles_done;
  template <int BN>
  __device__ __forceinline__ void run(uint32_t, int64_t, int, int lane) const {
    if (lane == 0) atomicAdd(tiles_done, 1);
  }
};

}  // namespace sge

using namespace sge;

extern "C" int sge_selftest_wait_timeout(int pair, const void* a, const void* b, int64_t m, int64_t n,
                                         int64_t k, int32_t* diag, int32_t* tiles_done, void* stream) {
  clear_error();
  if (!a || !b || !diag || !tiles_done || m < 1 || n < 1 || k < 64 || m > (1 << 20) || n > (1 << 20) ||
      k > (1 << 20) || !aligned16(a) || !aligned16(b))
    return fail(SGE_ERR_ARG, "sge_selftest_wait_timeout: bad arguments");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  EpiCountTiles epi{tiles_done};
  CUtensorMap ma, mb;
  if (pair) {
    using S = TcPairShape<256, 1>;
    int rc = make_tmap_bf16(&ma, a, m, k, k, kBM);
    // half the rows the stage expects: its barrier is never satisfied
    if (!rc) rc = make_tmap_bf16(&mb, b, n, k, k, S::BN / 4);
    if (rc) return rc;
    return launch_tc_gemm_pair<S>(ma, mb, mb, m, n, k, epi, diag, st, "selftest (pair engine)");
  }
  using S = TcShape<128, 1>;
  int rc = make_tmap_bf16(&ma, a, m, k, k, a_box_rows(m));
  if (!rc) rc = make_tmap_bf16(&mb, b, n, k, k, S::BN / 2);
  if (rc) return rc;
  return launch_tc_gemm<S>(ma, mb, mb, m, n, k, epi, diag, st, "selftest (single-CTA engine)");
}
