// C entry points of the fused up/down projections over TwELL nonzeros (the
// kernels and their planning are in fused_kernels.cuh): the workspace entry
// point, the allocation-free variant and the interleaved weight layout.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 02, last paragraph: one custom kernel performs the up and the down
// projection in a single traversal, without writing h to global memory.
#include <mutex>

#include "fused_kernels.cuh"

using namespace sge;

extern "C" size_t twell_fused_up_down_workspace_bytes(int64_t n_tokens, int64_t d_model) {
  if (n_tokens < 0 || d_model < 1) return 0;
  return WsLayout(n_tokens, d_model, pool_slots_for(kPoolBytes, d_model)).total;
}

extern "C" int twell_fused_up_down(const void* x, const uint8_t* count, const uint8_t* idx,
                                   const void* val, const void* wu_t, const void* wd, int64_t ldw,
                                   void* y, int64_t n_tokens, int64_t d_model, int64_t d_ff,
                                   int dtype, int tile, int cap, void* workspace,
                                   size_t workspace_bytes, int32_t* diag, void* stream) {
  NvtxRange nvtx_range("twell_fused_up_down");
  static const char* kName = "twell_fused_up_down";
  clear_error();
  int rc = check_args(kName, n_tokens, d_model, d_ff, ldw, tile, cap);
  if (rc) return rc;
  if (n_tokens == 0) return SGE_OK;
  if (!x || !count || !idx || !val || !wu_t || !wd || !y || !workspace)
    return fail(SGE_ERR_ARG, "%s: null pointer", kName);
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) || !aligned16(val) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(SGE_ERR_ARG, "%s: pointer not 16-byte aligned (workspace: 256)", kName);
  const size_t need = twell_fused_up_down_workspace_bytes(n_tokens, d_model);
  if (workspace_bytes < need)
    return fail(SGE_ERR_ARG, "%s: workspace of %zu bytes, %zu needed", kName, workspace_bytes, need);
  return run_fused(kName, x, count, idx, val, wu_t, wd, ldw, y, n_tokens, d_model, d_ff, dtype, tile, cap,
                   workspace, pool_slots_for(kPoolBytes, d_model), diag,
                   static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Allocation-free variant.
//
// Some callers cannot allocate device memory for a workspace: code that runs
// where no allocator may be called (an embedding runtime that forbids
// cudaMalloc after start-up, a memory-capped inference server that has
// handed all device memory to its own pools, a plugin that receives only the
// tensors it works on).  For them the workspace of twell_fused_up_down lives
// in this file-scope device array instead, sized for at most
// kNoAllocMaxTokens tokens and a smaller pool for the partial outputs of
// split heavy tokens; every GPU that loads the library holds it until the
// process exits.  In host code `g_fused_scratch` names a host-side stand-in,
// not a device address, so its device address is looked up per device with
// cudaGetSymbolAddress, once, with that device current.

constexpr int64_t kNoAllocMaxTokens = 65536;
constexpr int64_t kNoAllocPoolSlots = 1024;
constexpr size_t kNoAllocPoolBytes = size_t(4) << 20;
constexpr size_t kNoAllocScratchBytes =
    kHdrBytes + ((8 * static_cast<size_t>((kNoAllocMaxTokens + 255) / 256) + 255) & ~size_t(255)) +
    4 * static_cast<size_t>(kNoAllocMaxTokens) + 8 * kLightClasses * static_cast<size_t>(kNoAllocMaxTokens) +
    static_cast<size_t>(kNoAllocPoolSlots) * (32 + 4) + kNoAllocPoolBytes + 1024;

static __device__ __align__(256) uint8_t g_fused_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
// Per device: the context the address was looked up in, and the address.  A
// device reset or a new primary context maps the array afresh, so the
// address is looked up again whenever the current context differs.
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_fused_scratch in the current device's current context
// (looked up once per context).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "twell_fused_up_down_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down_noalloc: device %d beyond %d", dev, kMaxDevices);
  // Before the runtime has set up this thread no context is current; the
  // symbol lookup then makes the device's primary context current.
  CUcontext ctx = nullptr;
  if (current_context(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fused_scratch);
    if (e != cudaSuccess || !p)
      return fail(SGE_ERR_CUDA, "twell_fused_up_down_noalloc: cudaGetSymbolAddress: %s",
                  cudaGetErrorString(e));
    if (current_context(&ctx) != CUDA_SUCCESS || !ctx)
      return fail(SGE_ERR_CUDA, "twell_fused_up_down_noalloc: no current CUDA context");
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return SGE_OK;
}

}  // namespace

extern "C" int64_t twell_fused_up_down_noalloc_max_tokens(void) { return kNoAllocMaxTokens; }

extern "C" int twell_fused_up_down_noalloc(const void* x, const uint8_t* count, const uint8_t* idx,
                                           const void* val, const void* wu_t, const void* wd,
                                           int64_t ldw, void* y, int64_t n_tokens, int64_t d_model,
                                           int64_t d_ff, int dtype, int tile, int cap,
                                           int32_t* diag, void* stream) {
  static const char* kName = "twell_fused_up_down_noalloc";
  clear_error();
  if (n_tokens > kNoAllocMaxTokens)
    return fail(SGE_ERR_UNSUPPORTED,
                "%s: %lld tokens exceed the built-in scratch limit of %lld; "
                "use twell_fused_up_down with a workspace",
                kName, (long long)n_tokens, (long long)kNoAllocMaxTokens);
  int rc = check_args(kName, n_tokens, d_model, d_ff, ldw, tile, cap);
  if (rc) return rc;
  void* scratch = nullptr;
  // a call without tokens only sets up the array's address (start-up)
  if (n_tokens == 0) return scratch_address(&scratch);
  if (!x || !count || !idx || !val || !wu_t || !wd || !y)
    return fail(SGE_ERR_ARG, "%s: null pointer", kName);
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) || !aligned16(val))
    return fail(SGE_ERR_ARG, "%s: pointer not 16-byte aligned", kName);
  int64_t slots = pool_slots_for(kNoAllocPoolBytes, d_model);
  if (slots > kNoAllocPoolSlots) slots = kNoAllocPoolSlots;
  if (WsLayout(n_tokens, d_model, slots).total > kNoAllocScratchBytes)
    return fail(SGE_ERR_UNSUPPORTED, "%s: built-in scratch too small for this shape", kName);
  rc = scratch_address(&scratch);
  if (rc) return rc;
  // The array keeps the previous call's contents; the planning kernels reset
  // every counter the call relies on (job counters and cursor, and the
  // completion counter of each split token).
  return run_fused(kName, x, count, idx, val, wu_t, wd, ldw, y, n_tokens, d_model, d_ff, dtype, tile, cap,
                   scratch, slots, diag, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// The interleaved weight layout: row j of w_ud is wu_t[j] then wd[j].

extern "C" int sge_interleave_up_down(const void* wu_t, const void* wd, void* w_ud, int64_t d_ff,
                                      int64_t d_model, int dtype, void* stream) {
  NvtxRange nvtx_range("sge_interleave_up_down");
  static const char* kName = "sge_interleave_up_down";
  clear_error();
  if (dtype != SGE_BF16 && dtype != SGE_F32) return fail(SGE_ERR_UNSUPPORTED, "%s: dtype %d", kName, dtype);
  if (d_ff < 0 || d_model < 1 || d_model >= (1LL << 31) || d_ff >= (1LL << 31))
    return fail(SGE_ERR_ARG, "%s: bad sizes", kName);
  if (d_ff == 0) return SGE_OK;
  if (!wu_t || !wd || !w_ud) return fail(SGE_ERR_ARG, "%s: null pointer", kName);
  const size_t rb = static_cast<size_t>(d_model) * (dtype == SGE_BF16 ? 2 : 4);
  const size_t n = rb * static_cast<size_t>(d_ff);
  const char* o = static_cast<const char*>(w_ud);
  auto overlaps = [&](const void* a, size_t na) {
    const char* c = static_cast<const char*>(a);
    return c < o + 2 * n && o < c + na;
  };
  if (overlaps(wu_t, n) || overlaps(wd, n)) return fail(SGE_ERR_ARG, "%s: w_ud overlaps an input", kName);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpy2DAsync(w_ud, 2 * rb, wu_t, rb, rb, static_cast<size_t>(d_ff),
                                    cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(static_cast<char*>(w_ud) + rb, 2 * rb, wd, rb, rb, static_cast<size_t>(d_ff),
                          cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: %s", kName, cudaGetErrorString(e));
  return SGE_OK;
}
