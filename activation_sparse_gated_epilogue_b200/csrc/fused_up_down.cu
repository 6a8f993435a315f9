// Fused up and down projections over the TwELL nonzeros.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 02, last paragraph: one custom kernel performs the up and the down
// projection in a single traversal, fusing the two products so that the
// intermediate h is never written to global memory.  For every stored entry
// (t, j, a) of the TwELL gate activations:
//     u = x[t] . W_up[:, j]      h = a * u      y[t] += h * W_down[j, :]
//
// Work is per token, and per-token work is heavy-tailed (a few tokens carry
// tens of times the mean number of entries), so:
//   * a classify kernel marks tokens with more than kHeavyEntries entries and
//     lists them in the caller's workspace;
//   * one persistent kernel (one CTA per SM made of three 128-thread
//     groups) first takes the heavy tokens, one per CTA, the groups
//     splitting the token's TwELL tiles and summing their partial y in a
//     fixed order in shared memory; then each group pulls light tokens one at
//     a time from a global cursor.
// Inside a group a token is processed in chunks of at most kMaxEntries
// entries gathered into shared memory (ascending column order):
//   * the d-vector is split across the group's threads in 16-byte vectors,
//     so each thread keeps a few elements of x[t] and of the fp32 y[t]
//     accumulator in registers;
//   * phase U: every thread loads its 16-byte slice of row j of W_up for a
//     batch of entries (two batches in flight: register double buffering),
//     forms exact bf16 x bf16 products accumulated in fp32, the warp reduces a
//     batch with a halving shuffle tree and the per-warp partials go to
//     shared memory;
//   * h_e = a_e * (sum of the per-warp partials, fixed order), rounded to the
//     activation dtype (the precision the dense FFN gives h);
//   * phase D: every thread streams its slice of row j of W_down and
//     accumulates h_e * W_down[j] into its y registers.
// h lives only in shared memory.  Results do not depend on which CTA or
// group processes a token: no atomics touch data.
#include <mutex>

#include "sge_host.h"
#include "sparse_common.cuh"

namespace sge {

constexpr int kGroupThreads = 128;  // threads processing one token
constexpr int kGroupWarps = kGroupThreads / 32;
constexpr int kMaxEntries = 512;    // entries per chunk in a group's shared list
constexpr int kMaxTiles = 512;      // TwELL tiles per chunk
constexpr int kHeavyEntries = 384;  // tokens with more entries use a whole CTA

// Per row width (NV 16-byte vectors per thread): groups per CTA and entries
// per load batch (two batches in flight), chosen so that the double-buffered
// rows fit in registers at one CTA per SM.
template <int NV>
struct UdTune {
  static constexpr int kGroups = 3;
  static constexpr int kBatch = NV == 1 ? 8 : (NV == 2 ? 4 : 2);
  static constexpr int kThreads = kGroups * kGroupThreads;
};

// Workspace: int header[4] = {heavy count, heavy cursor, light cursor, 0},
// int heavy_list[N], uint8 heavy_flag[N].
constexpr size_t kWsHeader = 16;

__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;" ::"r"(g + 1), "r"(kGroupThreads) : "memory");
}

struct UdParams {
  const void* x;
  const uint8_t* count;
  const uint8_t* idx;
  const void* val;
  const void* wu_t;
  const void* wd;
  void* y;
  int* ws;             // header + heavy list
  const uint8_t* heavy_flag;
  int64_t n_rows;
  int d;
  int n_cols;
  int tile;
  int cap;
};

// Shared memory of one group.
struct GroupSmem {
  int2 jh[kMaxEntries];                 // (column j, a bits) -> (j, h bits)
  float upart[kGroupWarps][kMaxEntries];
  int tile_off[kMaxTiles + 1];
  int chunk[2];
  int token;
};

template <int NV, bool BF16>
struct Group {
  static constexpr int kBatch = UdTune<NV>::kBatch;
  using E = Elem<BF16>;
  static constexpr int VEC = E::VEC;
  static constexpr int ESZ = BF16 ? 2 : 4;

  const UdParams& p;
  GroupSmem& sm;
  const int g, gtid, gwarp, lane, nvec;
  const int64_t row_bytes;

  __device__ Group(const UdParams& p_, GroupSmem& sm_, int g_, int gtid_)
      : p(p_), sm(sm_), g(g_), gtid(gtid_), gwarp(gtid_ >> 5), lane(gtid_ & 31),
        nvec(p_.d / E::VEC), row_bytes(static_cast<int64_t>(p_.d) * ESZ) {}

  __device__ __forceinline__ void load_x(int64_t t, uint4 (&xv)[NV]) const {
    const uint4* xrow = reinterpret_cast<const uint4*>(static_cast<const char*>(p.x) + t * row_bytes);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int v = gtid + k * kGroupThreads;
      xv[k] = v < nvec ? __ldg(xrow + v) : make_uint4(0, 0, 0, 0);
    }
  }

  __device__ __forceinline__ void load_rows(const void* base, int e0, int n_e, uint4 (&w)[kBatch][NV]) const {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = e0 + u;
      const int j = e < n_e ? sm.jh[e].x : -1;
      const uint4* row = reinterpret_cast<const uint4*>(static_cast<const char*>(base) + static_cast<int64_t>(j) * row_bytes);
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int v = gtid + k * kGroupThreads;
        w[u][k] = (j >= 0 && v < nvec) ? __ldg(row + v) : make_uint4(0, 0, 0, 0);
      }
    }
  }

  __device__ __forceinline__ void reduce_u(const uint4 (&xv)[NV], const uint4 (&w)[kBatch][NV], int e0, int n_e) const {
    float part[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      float s = 0.0f;
#pragma unroll
      for (int k = 0; k < NV; ++k) s = E::dot(xv[k], w[u][k], s);
      part[u] = s;
    }
    const float tot = warp_reduce_multi<kBatch>(part, lane);
    if ((lane & (32 / kBatch - 1)) == 0) {
      const int e = e0 + multi_entry<kBatch>(lane);
      if (e < n_e) sm.upart[gwarp][e] = tot;
    }
  }

  __device__ __forceinline__ void apply_d(const uint4 (&w)[kBatch][NV], int e0, int n_e,
                                          float (&acc)[NV][VEC]) const {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = e0 + u;
      const typename E::HType h = E::h_from_bits(e < n_e ? sm.jh[e].y : 0);
#pragma unroll
      for (int k = 0; k < NV; ++k) E::axpy(h, w[u][k], acc[k]);
    }
  }

  // Accumulate into acc the entries of token t in tiles b_first, b_first +
  // stride, ... (ascending).
  __device__ void run(int64_t t, int b_first, int stride, const uint4 (&xv)[NV],
                      float (&acc)[NV][VEC]) const {
    const int nt = p.n_cols / p.tile;
    const uint8_t* cnt = p.count + t * nt;
    const int nk = b_first < nt ? (nt - b_first + stride - 1) / stride : 0;
    int k0 = 0;
    while (k0 < nk) {
      // ---- chunk: tiles k0 .. k1 (in units of stride) holding <= kMaxEntries
      if (gwarp == 0) {
        int k = k0, total = 0, n_tiles = 0;
        if (lane == 0) sm.tile_off[0] = 0;
        while (true) {
          const int kk = k + lane;
          const int c = kk < nk ? min(static_cast<int>(cnt[b_first + kk * stride]), p.cap) : 0;
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int nb = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nb;
          }
          // all three conditions are monotone in the lane: the fitting lanes form a prefix
          const bool fits = kk < nk && total + incl <= kMaxEntries && n_tiles + lane < kMaxTiles;
          const int take = __popc(__ballot_sync(0xffffffffu, fits));
          if (lane < take) sm.tile_off[n_tiles + lane + 1] = total + incl;
          if (take > 0) total += __shfl_sync(0xffffffffu, incl, take - 1);
          n_tiles += take;
          k += take;
          if (take < 32) break;
        }
        if (lane == 0) {
          sm.chunk[0] = k;
          sm.chunk[1] = total;
        }
      }
      group_sync(g);
      const int k1 = sm.chunk[0];
      const int n_e = sm.chunk[1];
      const int n_tiles = k1 - k0;

      // ---- gather the chunk's entries, one thread per entry
      for (int e = gtid; e < n_e; e += kGroupThreads) {
        int lo = 0, hi = n_tiles;  // tile_off[lo] <= e < tile_off[lo + 1]
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (sm.tile_off[mid] <= e) lo = mid; else hi = mid;
        }
        const int b = b_first + (k0 + lo) * stride;
        const int s = e - sm.tile_off[lo];
        const int64_t seg = t * nt + b;
        sm.jh[e] = make_int2(b * p.tile + p.idx[seg * p.cap + s],
                             __float_as_int(E::load_val(p.val, seg * p.cap + s)));
      }
      group_sync(g);

      // ---- phase U: partial dot products, two batches of rows in flight
      {
        uint4 wa[kBatch][NV], wb[kBatch][NV];
        if (n_e > 0) load_rows(p.wu_t, 0, n_e, wa);
        for (int e0 = 0; e0 < n_e; e0 += 2 * kBatch) {
          if (e0 + kBatch < n_e) load_rows(p.wu_t, e0 + kBatch, n_e, wb);
          reduce_u(xv, wa, e0, n_e);
          if (e0 + kBatch >= n_e) break;
          if (e0 + 2 * kBatch < n_e) load_rows(p.wu_t, e0 + 2 * kBatch, n_e, wa);
          reduce_u(xv, wb, e0 + kBatch, n_e);
        }
      }
      group_sync(g);

      // ---- h = a * u, rounded as phase D consumes it
      for (int e = gtid; e < n_e; e += kGroupThreads) {
        float u = 0.0f;
#pragma unroll
        for (int w = 0; w < kGroupWarps; ++w) u += sm.upart[w][e];
        sm.jh[e].y = E::h_bits(E::h_of(__int_as_float(sm.jh[e].y) * u));
      }
      group_sync(g);

      // ---- phase D: y += h * W_down[j], two batches of rows in flight
      {
        uint4 wa[kBatch][NV], wb[kBatch][NV];
        if (n_e > 0) load_rows(p.wd, 0, n_e, wa);
        for (int e0 = 0; e0 < n_e; e0 += 2 * kBatch) {
          if (e0 + kBatch < n_e) load_rows(p.wd, e0 + kBatch, n_e, wb);
          apply_d(wa, e0, n_e, acc);
          if (e0 + kBatch >= n_e) break;
          if (e0 + 2 * kBatch < n_e) load_rows(p.wd, e0 + 2 * kBatch, n_e, wa);
          apply_d(wb, e0 + kBatch, n_e, acc);
        }
      }
      group_sync(g);  // the next chunk rewrites the shared lists
      k0 = k1;
    }
  }

  __device__ __forceinline__ void store_y(int64_t t, const float (&acc)[NV][VEC]) const {
    uint4* yrow = reinterpret_cast<uint4*>(static_cast<char*>(p.y) + t * row_bytes);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int v = gtid + k * kGroupThreads;
      if (v < nvec) yrow[v] = E::pack(acc[k]);
    }
  }
};

// Marks tokens whose stored entry count exceeds kHeavyEntries and lists them.
__global__ void __launch_bounds__(256) classify_kernel(const uint8_t* __restrict__ count,
                                                       int64_t n_rows, int nt, int cap, int* ws,
                                                       uint8_t* heavy_flag) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= n_rows) return;
  const uint8_t* cnt = count + t * nt;
  int s = 0;
  for (int b = lane; b < nt; b += 32) s += min(static_cast<int>(cnt[b]), cap);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const bool heavy = s > kHeavyEntries;
    heavy_flag[t] = heavy ? 1 : 0;
    if (heavy) ws[4 + atomicAdd(&ws[0], 1)] = static_cast<int>(t);
  }
}

template <int NV, bool BF16>
__global__ void __launch_bounds__(UdTune<NV>::kThreads, 1) fused_up_down_kernel(UdParams p) {
  using G = Group<NV, BF16>;
  constexpr int VEC = G::VEC;
  constexpr int kGroups = UdTune<NV>::kGroups;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  GroupSmem* gsm = reinterpret_cast<GroupSmem*>(smem_raw);
  float* red = reinterpret_cast<float*>(smem_raw + kGroups * sizeof(GroupSmem));  // [3][128][NV*VEC]
  __shared__ int s_heavy;

  const int g = threadIdx.x / kGroupThreads;
  const int gtid = threadIdx.x % kGroupThreads;
  const G grp(p, gsm[g], g, gtid);
  const int n_heavy = *reinterpret_cast<volatile int*>(&p.ws[0]);

  // ---- heavy tokens: the whole CTA, tiles split across the groups
  while (true) {
    if (threadIdx.x == 0) {
      const int k = atomicAdd(&p.ws[1], 1);
      s_heavy = k < n_heavy ? p.ws[4 + k] : -1;
    }
    __syncthreads();
    const int64_t t = s_heavy;
    __syncthreads();
    if (t < 0) break;
    uint4 xv[NV];
    float acc[NV][VEC];
    grp.load_x(t, xv);
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
    grp.run(t, g, kGroups, xv, acc);
    // fixed-order sum of the groups' partial accumulators
    if (g > 0) {
      float* dst = red + ((g - 1) * kGroupThreads + gtid) * (NV * VEC);
#pragma unroll
      for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int q = 0; q < VEC; ++q) dst[k * VEC + q] = acc[k][q];
    }
    __syncthreads();
    if (g == 0) {
#pragma unroll
      for (int r = 0; r < kGroups - 1; ++r) {
        const float* src = red + (r * kGroupThreads + gtid) * (NV * VEC);
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
          for (int q = 0; q < VEC; ++q) acc[k][q] += src[k * VEC + q];
      }
      grp.store_y(t, acc);
    }
    __syncthreads();
  }

  // ---- light tokens: each group pulls one token at a time
  while (true) {
    if (gtid == 0) gsm[g].token = atomicAdd(&p.ws[2], 1);
    group_sync(g);
    const int64_t t = gsm[g].token;
    group_sync(g);
    if (t >= p.n_rows) break;
    if (p.heavy_flag[t]) continue;
    uint4 xv[NV];
    float acc[NV][VEC];
    grp.load_x(t, xv);
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
    grp.run(t, 0, 1, xv, acc);
    grp.store_y(t, acc);
  }
}

template <int NV, bool BF16>
static int launch_ud(const UdParams& prm, cudaStream_t st) {
  constexpr int VEC = Elem<BF16>::VEC;
  constexpr int kGroups = UdTune<NV>::kGroups;
  const int smem = static_cast<int>(kGroups * sizeof(GroupSmem) +
                                    (kGroups - 1) * kGroupThreads * NV * VEC * sizeof(float));
  auto kern = fused_up_down_kernel<NV, BF16>;
  int rc = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (rc) return rc;
  const int nt = prm.n_cols / prm.tile;
  const int64_t cblocks = (prm.n_rows + 7) / 8;
  classify_kernel<<<static_cast<unsigned>(cblocks), 256, 0, st>>>(
      prm.count, prm.n_rows, nt, prm.cap, prm.ws, const_cast<uint8_t*>(prm.heavy_flag));
  rc = check_launch("twell_fused_up_down (classify)");
  if (rc) return rc;
  const int64_t want = (prm.n_rows + kGroups - 1) / kGroups;
  const int grid = static_cast<int>(want < sm_count() ? want : sm_count());
  kern<<<grid, UdTune<NV>::kThreads, smem, st>>>(prm);
  return check_launch("twell_fused_up_down");
}

template <bool BF16>
static int dispatch_ud(const UdParams& prm, cudaStream_t st) {
  constexpr int VEC = Elem<BF16>::VEC;
  const int64_t nvec = prm.d / VEC;
  if (nvec <= 1 * kGroupThreads) return launch_ud<1, BF16>(prm, st);
  if (nvec <= 2 * kGroupThreads) return launch_ud<2, BF16>(prm, st);
  if (nvec <= 3 * kGroupThreads) return launch_ud<3, BF16>(prm, st);
  if (nvec <= 4 * kGroupThreads) return launch_ud<4, BF16>(prm, st);
  return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: d_model %d too large (max %d)", prm.d,
              4 * kGroupThreads * VEC);
}

}  // namespace sge

using namespace sge;

extern "C" size_t twell_fused_up_down_workspace_bytes(int64_t n_tokens) {
  if (n_tokens < 0) return 0;
  return (kWsHeader + 5 * static_cast<size_t>(n_tokens) + 15) & ~static_cast<size_t>(15);
}

extern "C" int twell_fused_up_down(const void* x, const uint8_t* count, const uint8_t* idx,
                                   const void* val, const void* wu_t, const void* wd, void* y,
                                   int64_t n_tokens, int64_t d_model, int64_t d_ff, int dtype,
                                   int tile, int cap, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  clear_error();
  if (n_tokens < 0 || d_model < 1 || d_ff < 1)
    return fail(SGE_ERR_ARG, "twell_fused_up_down: bad sizes");
  if (d_model % 8) return fail(SGE_ERR_ARG, "twell_fused_up_down: d_model %% 8 != 0");
  if (tile < 1 || tile > 255 || d_ff % tile)
    return fail(SGE_ERR_ARG, "twell_fused_up_down: tile must divide d_ff and be <= 255");
  if (cap < 1 || cap > tile) return fail(SGE_ERR_ARG, "twell_fused_up_down: cap outside [1, tile]");
  if (d_ff >= (1LL << 31) || n_tokens >= (1LL << 31))
    return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: size beyond 2^31");
  if (n_tokens == 0) return SGE_OK;
  if (!x || !count || !idx || !val || !wu_t || !wd || !y || !workspace)
    return fail(SGE_ERR_ARG, "twell_fused_up_down: null pointer");
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) || !aligned16(val) ||
      !aligned16(workspace))
    return fail(SGE_ERR_ARG, "twell_fused_up_down: pointer not 16-byte aligned");
  if (workspace_bytes < twell_fused_up_down_workspace_bytes(n_tokens))
    return fail(SGE_ERR_ARG, "twell_fused_up_down: workspace of %zu bytes, %zu needed", workspace_bytes,
                twell_fused_up_down_workspace_bytes(n_tokens));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  UdParams prm;
  prm.x = x;
  prm.count = count;
  prm.idx = idx;
  prm.val = val;
  prm.wu_t = wu_t;
  prm.wd = wd;
  prm.y = y;
  prm.ws = static_cast<int*>(workspace);
  prm.heavy_flag = static_cast<const uint8_t*>(workspace) + kWsHeader + 4 * static_cast<size_t>(n_tokens);
  prm.n_rows = n_tokens;
  prm.d = static_cast<int>(d_model);
  prm.n_cols = static_cast<int>(d_ff);
  prm.tile = tile;
  prm.cap = cap;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "twell_fused_up_down: %s", cudaGetErrorString(e));
  if (dtype == SGE_BF16) return dispatch_ud<true>(prm, st);
  if (dtype == SGE_F32) return dispatch_ud<false>(prm, st);
  return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: dtype %d", dtype);
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
// kNoAllocMaxTokens tokens; every GPU that loads the library holds it until
// the process exits.  In host code `g_fused_scratch` names a host-side stand-in,
// not a device address, so its device address is looked up per device with
// cudaGetSymbolAddress, once, with that device current.

constexpr int64_t kNoAllocMaxTokens = 262144;
constexpr size_t kNoAllocScratchBytes =
    (kWsHeader + 5 * static_cast<size_t>(kNoAllocMaxTokens) + 15) & ~static_cast<size_t>(15);

static __device__ __align__(256) uint8_t g_fused_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_fused_scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "twell_fused_up_down_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down_noalloc: device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fused_scratch);
    if (e != cudaSuccess || !p)
      return fail(SGE_ERR_CUDA, "twell_fused_up_down_noalloc: cudaGetSymbolAddress: %s",
                  cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SGE_OK;
}

}  // namespace

extern "C" int64_t twell_fused_up_down_noalloc_max_tokens(void) { return kNoAllocMaxTokens; }

extern "C" int twell_fused_up_down_noalloc(const void* x, const uint8_t* count, const uint8_t* idx,
                                           const void* val, const void* wu_t, const void* wd,
                                           void* y, int64_t n_tokens, int64_t d_model,
                                           int64_t d_ff, int dtype, int tile, int cap,
                                           void* stream) {
  clear_error();
  if (n_tokens < 0 || d_model < 1 || d_ff < 1)
    return fail(SGE_ERR_ARG, "twell_fused_up_down_noalloc: bad sizes");
  if (n_tokens > kNoAllocMaxTokens)
    return fail(SGE_ERR_UNSUPPORTED,
                "twell_fused_up_down_noalloc: %lld tokens exceed the built-in scratch limit of %lld; "
                "use twell_fused_up_down with a workspace",
                (long long)n_tokens, (long long)kNoAllocMaxTokens);
  if (d_model % 8) return fail(SGE_ERR_ARG, "twell_fused_up_down_noalloc: d_model %% 8 != 0");
  if (tile < 1 || tile > 255 || d_ff % tile)
    return fail(SGE_ERR_ARG, "twell_fused_up_down_noalloc: tile must divide d_ff and be <= 255");
  if (cap < 1 || cap > tile)
    return fail(SGE_ERR_ARG, "twell_fused_up_down_noalloc: cap outside [1, tile]");
  if (d_ff >= (1LL << 31)) return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down_noalloc: d_ff beyond 2^31");
  if (n_tokens == 0) return SGE_OK;
  if (!x || !count || !idx || !val || !wu_t || !wd || !y)
    return fail(SGE_ERR_ARG, "twell_fused_up_down_noalloc: null pointer");
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) || !aligned16(val))
    return fail(SGE_ERR_ARG, "twell_fused_up_down_noalloc: pointer not 16-byte aligned");
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  UdParams prm;
  prm.x = x;
  prm.count = count;
  prm.idx = idx;
  prm.val = val;
  prm.wu_t = wu_t;
  prm.wd = wd;
  prm.y = y;
  prm.ws = static_cast<int*>(scratch);
  prm.heavy_flag = static_cast<const uint8_t*>(scratch) + kWsHeader + 4 * static_cast<size_t>(n_tokens);
  prm.n_rows = n_tokens;
  prm.d = static_cast<int>(d_model);
  prm.n_cols = static_cast<int>(d_ff);
  prm.tile = tile;
  prm.cap = cap;
  // the array keeps the previous call's contents: the cursors start at zero
  cudaError_t e = cudaMemsetAsync(scratch, 0, kWsHeader, st);
  if (e != cudaSuccess)
    return fail(SGE_ERR_CUDA, "twell_fused_up_down_noalloc: %s", cudaGetErrorString(e));
  if (dtype == SGE_BF16) return dispatch_ud<true>(prm, st);
  if (dtype == SGE_F32) return dispatch_ud<false>(prm, st);
  return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down_noalloc: dtype %d", dtype);
}
