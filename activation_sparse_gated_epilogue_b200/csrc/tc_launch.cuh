// Host launchers of the tcgen05 GEMM engines (single CTA and CTA pair).
#pragma once

#include "sge_host.h"
#include "tc_gemm.cuh"

namespace sge {

template <class Shape, class Epi>
int launch_tc_gemm(const CUtensorMap& ma, const CUtensorMap& mb0, const CUtensorMap& mb1,
                   int64_t m, int64_t n, int64_t k, const Epi& epi, int32_t* diag,
                   cudaStream_t st, const char* what) {
  auto kern = tc_gemm_kernel<Shape, Epi>;
  int rc = set_smem_limit(reinterpret_cast<const void*>(kern), Shape::SMEM_BYTES);
  if (rc) return rc;
  const int64_t tiles = ((m + kBM - 1) / kBM) * ((n + Shape::BN - 1) / Shape::BN);
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  return launch_pdl(kern, dim3(grid), dim3(Shape::THREADS), Shape::SMEM_BYTES, st, what, ma, mb0, mb1,
                    static_cast<int>(m), static_cast<int>(n), static_cast<int>(k), epi, diag);
}

// Number of CTA pairs that can be resident at once (cached per kernel).
template <class Shape, class Epi>
int max_resident_pairs() {
  static int cached = 0;
  if (cached) return cached;
  auto kern = tc_gemm_pair_kernel<Shape, Epi>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2));
  cfg.blockDim = dim3(Shape::THREADS);
  cfg.dynamicSmemBytes = Shape::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kern), &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  cached = n;
  return n;
}

// `splits`: the K splits the epilogue asks for (Epi::splits), for the grid size.
template <class Shape, class Epi>
int launch_tc_gemm_pair(const CUtensorMap& ma, const CUtensorMap& mb0, const CUtensorMap& mb1,
                        int64_t m, int64_t n, int64_t k, const Epi& epi, int32_t* diag,
                        cudaStream_t st, const char* what, int splits = 1) {
  auto kern = tc_gemm_pair_kernel<Shape, Epi>;
  int rc = set_smem_limit(reinterpret_cast<const void*>(kern), Shape::SMEM_BYTES);
  if (rc) return rc;
  const int64_t tiles = ((m + Shape::BM - 1) / Shape::BM) * ((n + Shape::BN - 1) / Shape::BN) * splits;
  const int64_t resident = max_resident_pairs<Shape, Epi>();
  const int pairs = static_cast<int>(tiles < resident ? tiles : resident);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(Shape::THREADS);
  cfg.dynamicSmemBytes = Shape::SMEM_BYTES;
  cfg.stream = st;
  // programmatic dependent launch: the kernel's set-up (barriers, TMEM,
  // descriptors) overlaps the end of the previous kernel in the stream
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb0, mb1, static_cast<int>(m),
                                     static_cast<int>(n), static_cast<int>(k), epi, diag);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

}  // namespace sge
