// Host-side helpers shared by the library's .cu files: error reporting,
// argument checks, device properties and TMA descriptor encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <string>

#include "../../include/sge.h"

namespace sge {

// Debug builds: each translation unit registers the reader of its device
// debug word (read, optionally cleared; -1 on a CUDA error) at load time.
using DebugReader = int (*)(bool clear);
bool register_debug_reader(DebugReader reader);

// Records a message for sge_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
void clear_error();

// SGE_OK, or SGE_ERR_CUDA with the message of the pending launch error.
int check_launch(const char* what);

// An NVTX range over a library call on the calling host thread (names the
// call in profiler timelines; next to free when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// Multiprocessor count of the current device (cached per device).
int sm_count();

// Sets the dynamic shared memory limit of a kernel once per device.
int set_smem_limit(const void* kernel, int bytes);

// Asks for the largest shared-memory carveout for a kernel, once per device.
int prefer_max_shared(const void* kernel);

// The calling thread's current CUDA context (nullptr if none), via the
// driver entry point; CUDA_SUCCESS or the driver's error.
CUresult current_context(CUcontext* ctx);

// Launch with programmatic stream serialization: the kernel may start
// while its predecessor in the stream finishes and must call grid_dep_wait()
// before touching global memory.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               const char* what, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix with row pitch
// `pitch_elems`, box [box_rows][64] (64 bf16 = one 128-byte swizzle row),
// 128-byte swizzle, out-of-bounds elements read as zero.
int make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint64_t pitch_elems, uint32_t box_rows);

}  // namespace sge
