// Host-side helpers: error strings, device properties, TMA descriptors.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "sge_host.h"

namespace sge {

static thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_err[0] = 0; }

static DebugReader g_debug_readers[32];
static int g_debug_reader_count = 0;

bool register_debug_reader(DebugReader reader) {
  if (g_debug_reader_count < 32) g_debug_readers[g_debug_reader_count++] = reader;
  return true;
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SGE_OK;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// The dynamic shared-memory limit of each (device, kernel) is set once and
// only raised afterwards: setting the attribute on every launch is not free.
int set_smem_limit(const void* kernel, int bytes) {
  struct Entry {
    int dev;
    const void* kernel;
    int bytes;
  };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  std::lock_guard<std::mutex> lock(mu);
  Entry* hit = nullptr;
  for (int i = 0; i < used; ++i)
    if (table[i].dev == dev && table[i].kernel == kernel) hit = &table[i];
  if (hit && hit->bytes >= bytes) return SGE_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess)
    return fail(SGE_ERR_CUDA, "cudaFuncSetAttribute(smem=%d): %s", bytes, cudaGetErrorString(e));
  if (hit) hit->bytes = bytes;
  else if (used < 256) table[used++] = Entry{dev, kernel, bytes};
  return SGE_OK;
}

int prefer_max_shared(const void* kernel) {
  struct Entry {
    int dev;
    const void* kernel;
  };
  static Entry table[64];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (table[i].dev == dev && table[i].kernel == kernel) return SGE_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "cudaFuncSetAttribute(carveout): %s", cudaGetErrorString(e));
  if (used < 64) table[used++] = Entry{dev, kernel};
  return SGE_OK;
}

CUresult current_context(CUcontext* ctx) {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  return fn(ctx);
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint64_t pitch_elems, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(SGE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(SGE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%llu cols=%llu box=%u", (int)r,
                (unsigned long long)rows, (unsigned long long)cols, box_rows);
  return SGE_OK;
}

}  // namespace sge

extern "C" int sge_version(void) { return 100; }

extern "C" int sge_debug_flags(int clear) {
#ifdef SGE_DEBUG
  int flags = 0;
  for (int i = 0; i < sge::g_debug_reader_count; ++i) {
    const int v = sge::g_debug_readers[i](clear != 0);
    if (v < 0) {
      sge::fail(SGE_ERR_CUDA, "sge_debug_flags: %s", cudaGetErrorString(cudaGetLastError()));
      return -2;
    }
    flags |= v;
  }
  return flags;
#else
  (void)clear;
  return -1;
#endif
}

extern "C" const char* sge_last_error(void) { return sge::g_err; }
