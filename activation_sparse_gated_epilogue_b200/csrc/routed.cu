// Routed forward: up and down projections from TwELL with the heavy tokens
// on tensor cores.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 03 and figure "基于混合格式的稀疏矩阵算子路由计算逻辑": tokens with few
// active gates take the sparse path, the occasional highly active token a
// dense backup path on tensor cores; the kongchang.com page ("核心思路")
// describes the same split as a fast path plus a dense fallback.  Here the
// split serves inference straight from the gate GEMM's TwELL output, with no
// ELL repack and nothing saved for a backward pass:
//
//   plan    stored entries per token; tokens with more than K stored entries
//           are heavy and ranked in ascending token order; the first S_max
//           go to the spill list (fused_kernels.cuh's planning kernels)
//   light   on a stream of the library's own, at the same time as the spill:
//           every other token through CUDA cores (light_fwd_kernel below),
//           y = 0 for tokens without stored entries
//   prep    per spill row: its x row into X_s, its stored activations
//           scattered into a dense row of A_s (zeros elsewhere)
//   GEMM 1  U = X_s W_up on tcgen05 (CTA pairs), epilogue H_s = bf16(A_s (.) U)
//   GEMM 2  Y_s = H_s W_down on tcgen05, epilogue scatters row r to y[token r]
//
// Every token's y is written exactly once, by GEMM 2 or by the light-token
// kernel; results do not depend on scheduling.  Per row the arithmetic is
// that of the dense FFN restricted to the stored entries: fp32 accumulation,
// h rounded to bf16 before the down projection, as in twell_fused_up_down.
#include <mutex>

#include "fused_kernels.cuh"
#include "spill_gemm.cuh"
#include "tc_launch.cuh"

namespace sge {

// Exclusive prefix over the first nt (<= 256) capped tile counts of token t,
// into pre[0 .. nt] (pre[nt] = the token's stored entries), by the `nthr`
// threads of a group (thread index gt; 128 or 256 threads, which share the
// named barrier `bar`; wsum holds nthr / 32 ints).  The caller synchronises
// the group before pre[] is read.
__device__ __forceinline__ void tile_prefix(const uint8_t* __restrict__ count, int64_t t, int nt, int cap,
                                            int gt, int nthr, int bar, int* pre, int* wsum) {
  const int lane = gt & 31, gw = gt >> 5, nw = nthr >> 5;
  // each thread owns tiles 2 gt and 2 gt + 1 (nt <= 256 = 2 x 128)
  int c0 = 0, c1 = 0;
  const int b0 = 2 * gt;
  if (b0 < nt) c0 = min(static_cast<int>(__ldg(count + t * nt + b0)), cap);
  if (b0 + 1 < nt) c1 = min(static_cast<int>(__ldg(count + t * nt + b0 + 1)), cap);
  int incl = c0 + c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[gw] = incl;
  named_sync(bar, nthr);
  int base = 0;
  for (int w = 0; w < gw; ++w) base += wsum[w];
  const int ex = base + incl - c0 - c1;
  if (b0 < nt) pre[b0] = ex;
  if (b0 + 1 < nt) pre[b0 + 1] = ex + c0;
  if (gt == nthr - 1) {
    int tot = 0;
    for (int w = 0; w < nw; ++w) tot += wsum[w];
    pre[nt] = tot;
  }
}

// X_s and A_s rows of the kept spill tokens, a CTA per row (grid-stride over
// the spill ranks): the x row is copied, the dense row of a is zeroed, then
// every stored entry is written by its own thread (its tile found by a
// binary search over the row's tile prefix).
constexpr int kPrepThreads = 256;
constexpr int kPrepCtas = 2048;  // about two rows per CTA for the largest spills

__global__ void __launch_bounds__(kPrepThreads) spill_prep_kernel(const uint16_t* __restrict__ x,
                                                                  const uint8_t* __restrict__ count,
                                                                  const uint8_t* __restrict__ idx,
                                                                  const uint16_t* __restrict__ val,
                                                                  const int* __restrict__ spill_rows,
                                                                  const int* __restrict__ n_heavy,
                                                                  int s_max, int d, int f, int nt,
                                                                  int tile, int cap,
                                                                  uint16_t* __restrict__ xs,
                                                                  uint16_t* __restrict__ as) {
  __shared__ int pre[257];
  __shared__ int wsum[kPrepThreads / 32];
  const int tid = threadIdx.x;
  const int kept = min(*n_heavy, s_max);
  for (int r = blockIdx.x; r < kept; r += gridDim.x) {
    const int64_t t = spill_rows[r];
    const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
    uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<int64_t>(r) * d);
    for (int v = tid; v < d / 8; v += kPrepThreads) dst[v] = __ldg(src + v);
    uint16_t* arow = as + static_cast<int64_t>(r) * f;
    for (int v = tid; v < f / 8; v += kPrepThreads) reinterpret_cast<uint4*>(arow)[v] = make_uint4(0, 0, 0, 0);
    tile_prefix(count, t, nt, cap, tid, kPrepThreads, 0, pre, wsum);
    __syncthreads();  // the prefix is complete and the zeros have landed
    const int n = pre[nt];
    for (int e = tid; e < n; e += kPrepThreads) {
      int b = 0;  // the last tile whose prefix is <= e
      for (int step = 128; step > 0; step >>= 1)
        if (b + step < nt && pre[b + step] <= e) b += step;
      const int64_t at = (t * nt + b) * cap + (e - pre[b]);
      // a stored index is < T; kept inside its tile even if it is not
      const int j = b * tile + min(static_cast<int>(__ldg(idx + at)), tile - 1);
      arow[j] = __ldg(val + at);
    }
    __syncthreads();  // pre[] is rewritten for the next row
  }
}

// ------------------------------------------------------ light tokens
//
// Every token not on the spill, straight from TwELL.  A group of four
// warps takes one token at a time (tokens in a static stride over the batch,
// so no queue); it resolves the token's entries from the tile counts (up to
// kLightMaxK at a time), then runs them in batches of kLightBatch: the W_up
// and W_down rows of a batch are loaded together (one memory round trip per
// batch), u is summed over the group's warps in warp order, h = bf16(a u),
// and h W_down[j] is accumulated into the fp32 y row held in registers.  The
// group also stores y = 0 for the tokens of its stride without stored
// entries.  Light tokens have at most K <= kLightMaxK entries; heavy tokens
// past S_max (only when the caller's S_max is too small) take as many rounds
// of kLightMaxK entries as they need.  Few registers and little shared
// memory per CTA, one CTA per SM: it runs beside the spill GEMMs' CTAs.
constexpr int kLightBatch = 4;
constexpr int kLightMaxK = 512;  // the largest K of a routed call

struct LightParams {
  const uint16_t* x;
  const uint8_t* count;
  const uint8_t* idx;
  const uint16_t* val;
  const char* wu;  // row j at wu + j * w_ld bytes
  const char* wd;
  int64_t w_ld;
  uint16_t* y;
  const int* ntok;
  int64_t n_rows;
  int d, nt, tile, cap, k;
};

// Registers per thread: with G groups of 128 threads the CTA stays within
// the 64 K registers an SM has minus the ~15 K of a spill GEMM CTA.
template <int G>
struct LightRegs {
  static constexpr int kMax = G >= 3 ? 128 : 192;
};

template <int NV, int G>
__global__ void __launch_bounds__(G * 128) __maxnreg__(LightRegs<G>::kMax)
    light_fwd_kernel(const LightParams p) {
  using E = Elem<true>;
  constexpr int VEC = E::VEC;
  __shared__ int s_pre[G][257];
  __shared__ int s_wsum[G][4];
  __shared__ int s_j[G][kLightMaxK];
  __shared__ float s_a[G][kLightMaxK];
  __shared__ float s_part[G][4][kLightBatch];
  __shared__ uint16_t s_h[G][kLightBatch];
  const int g = threadIdx.x >> 7, gt = threadIdx.x & 127, lane = gt & 31, gw = gt >> 5;
  const int nvec = p.d / VEC;
  const int64_t groups = static_cast<int64_t>(gridDim.x) * G;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * G + g; t < p.n_rows; t += groups) {
    const int n = p.ntok[t];
    uint4* yrow = reinterpret_cast<uint4*>(p.y + t * p.d);
    if (n == 0) {
      for (int v = gt; v < nvec; v += 128) yrow[v] = make_uint4(0, 0, 0, 0);
      continue;
    }
    if (n < 0) continue;  // spill token
    uint4 xv[NV];
    const uint4* xrow = reinterpret_cast<const uint4*>(p.x + t * p.d);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int v = gt + k * 128;
      xv[k] = v < nvec ? __ldg(xrow + v) : make_uint4(0, 0, 0, 0);
    }
    tile_prefix(p.count, t, p.nt, p.cap, gt, 128, 1 + g, s_pre[g], s_wsum[g]);
    float acc[NV][VEC];
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
    for (int c0 = 0; c0 < n; c0 += kLightMaxK) {
    const int cn = min(kLightMaxK, n - c0);  // entries of this round
    named_sync(1 + g, 128);  // the prefix (first round) or the last round's batches are done
    for (int e = gt; e < cn; e += 128) {
      const int eg = c0 + e;
      int b = 0;
      for (int step = 128; step > 0; step >>= 1)
        if (b + step < p.nt && s_pre[g][b + step] <= eg) b += step;
      const int64_t at = (t * p.nt + b) * p.cap + (eg - s_pre[g][b]);
      s_j[g][e] = b * p.tile + min(static_cast<int>(__ldg(p.idx + at)), p.tile - 1);
      s_a[g][e] = E::from_raw(__ldg(p.val + at));
    }
    named_sync(1 + g, 128);
    for (int e0 = 0; e0 < cn; e0 += kLightBatch) {
      uint4 wu[kLightBatch][NV], wdv[kLightBatch][NV];
#pragma unroll
      for (int u = 0; u < kLightBatch; ++u) {
        const int e = e0 + u;
        const int j = e < cn ? s_j[g][e] : 0;
        const uint4* ur = reinterpret_cast<const uint4*>(p.wu + static_cast<int64_t>(j) * p.w_ld);
        const uint4* dr = reinterpret_cast<const uint4*>(p.wd + static_cast<int64_t>(j) * p.w_ld);
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const int v = gt + k * 128;
          const bool in = e < cn && v < nvec;
          wu[u][k] = in ? __ldg(ur + v) : make_uint4(0, 0, 0, 0);
          wdv[u][k] = in ? __ldg(dr + v) : make_uint4(0, 0, 0, 0);
        }
      }
      float part[kLightBatch];
#pragma unroll
      for (int u = 0; u < kLightBatch; ++u) {
        float s = 0.0f;
#pragma unroll
        for (int k = 0; k < NV; ++k) s = E::dot(xv[k], wu[u][k], s);
        part[u] = s;
      }
      const float tot = warp_reduce_multi<kLightBatch>(part, lane);
      if ((lane & (32 / kLightBatch - 1)) == 0) s_part[g][gw][multi_entry<kLightBatch>(lane)] = tot;
      named_sync(1 + g, 128);
      if (gt < kLightBatch) {
        const int e = e0 + gt;
        // u summed over the group's warps in warp order
        const float u = ((s_part[g][0][gt] + s_part[g][1][gt]) + s_part[g][2][gt]) + s_part[g][3][gt];
        s_h[g][gt] = e < cn ? E::h_of(s_a[g][e] * u) : 0;
      }
      named_sync(1 + g, 128);
#pragma unroll
      for (int u = 0; u < kLightBatch; ++u) {
        const uint16_t hb = s_h[g][u];
#pragma unroll
        for (int k = 0; k < NV; ++k) E::axpy(hb, wdv[u][k], acc[k]);
      }
    }
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int v = gt + k * 128;
      if (v < nvec) yrow[v] = E::pack(acc[k]);
    }
    named_sync(1 + g, 128);  // s_pre / s_j / s_h are rewritten for the next token
  }
}

// Workspace: the planning kernels' (fused_kernels.cuh), then the per-block
// heavy counts, the spill list and the spill operands X_s [S_max][d], A_s
// and H_s [S_max][F] (bf16, 1024-byte aligned offsets).
constexpr int kSpillBN = 256;

struct RoutedLayout {
  WsLayout fused;
  size_t heavy, rows, xs, as, hs, total;
  RoutedLayout(int64_t n, int64_t d, int64_t f, int64_t s_max, int64_t pool_slots)
      : fused(n, d, pool_slots) {
    auto up = [](size_t v, size_t a) { return (v + a - 1) / a * a; };
    const size_t nblk = static_cast<size_t>((n + 255) / 256);
    const size_t sm = static_cast<size_t>(s_max);
    size_t o = up(fused.total, 1024);
    heavy = o;     o = up(o + 8 * nblk, 256);
    rows = o;      o = up(o + 4 * sm, 1024);
    xs = o;        o = up(o + 2 * sm * static_cast<size_t>(d), 1024);
    as = o;        o = up(o + 2 * sm * static_cast<size_t>(f), 1024);
    hs = o;        o = up(o + 2 * sm * static_cast<size_t>(f), 1024);
    total = o;
  }
};

template <int NV, int G>
static int launch_light(const LightParams& p, cudaStream_t st) {
  // kernels beside the spill GEMMs ask for the largest shared-memory
  // carveout: an SM configured for a small one cannot take a GEMM CTA (about
  // 197 KB) until it has drained
  const int rc = prefer_max_shared(reinterpret_cast<const void*>(light_fwd_kernel<NV, G>));
  if (rc) return rc;
  light_fwd_kernel<NV, G><<<sm_count(), G * 128, 0, st>>>(p);
  return check_launch("twell_hybrid_up_down (light tokens)");
}

static int launch_light_nv(const LightParams& p, cudaStream_t st) {
  const int nvec = p.d / 8;
  if (nvec <= 128) return launch_light<1, 3>(p, st);
  if (nvec <= 256) return launch_light<2, 3>(p, st);
  if (nvec <= 384) return launch_light<3, 2>(p, st);
  return launch_light<4, 2>(p, st);
}

// The light-token kernel runs on a stream of the library's own, beside the
// spill work on the caller's stream: the caller's stream forks into it after
// planning and joins it before the call's last kernel.  One such stream and
// its two events per device and context, created on first use; the mutex
// keeps the record / wait sequences of concurrent calls apart.
namespace {
constexpr int kMaxDevices = 64;
struct SideStream {
  CUcontext ctx = nullptr;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
SideStream g_side[kMaxDevices];
std::mutex g_side_mutex;

int side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "twell_hybrid_up_down: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(SGE_ERR_UNSUPPORTED, "twell_hybrid_up_down: device %d beyond %d", dev, kMaxDevices);
  CUcontext ctx = nullptr;
  if (current_context(&ctx) != CUDA_SUCCESS || !ctx)
    return fail(SGE_ERR_CUDA, "twell_hybrid_up_down: no current CUDA context");
  SideStream& sd = g_side[dev];
  if (sd.ctx != ctx) {  // first use, or a new context (the old handles died with the old one)
    sd = SideStream{};
    if ((e = cudaStreamCreateWithFlags(&sd.s, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming)) != cudaSuccess) {
      sd = SideStream{};
      return fail(SGE_ERR_CUDA, "twell_hybrid_up_down: side stream: %s", cudaGetErrorString(e));
    }
    sd.ctx = ctx;
  }
  *out = &sd;
  return SGE_OK;
}
}  // namespace

}  // namespace sge

using namespace sge;

extern "C" size_t twell_hybrid_up_down_workspace_bytes(int64_t n_tokens, int64_t d_model, int64_t d_ff,
                                                       int s_max) {
  if (n_tokens < 0 || d_model < 1 || d_ff < 1 || s_max < 0) return 0;
  return RoutedLayout(n_tokens, d_model, d_ff, s_max, pool_slots_for(kPoolBytes, d_model)).total;
}

extern "C" int twell_hybrid_up_down(const void* x, const uint8_t* count, const uint8_t* idx,
                                    const void* val, const void* wu_t, const void* wd, int64_t ldw,
                                    const void* wd_t, void* y, int64_t n_tokens, int64_t d_model,
                                    int64_t d_ff, int tile, int cap, int ell_cap, int s_max,
                                    void* workspace, size_t workspace_bytes, int32_t* diag,
                                    void* stream) {
  static const char* kName = "twell_hybrid_up_down";
  clear_error();
  int rc = check_args(kName, n_tokens, d_model, d_ff, ldw, tile, cap);
  if (rc) return rc;
  if (ell_cap < 0 || s_max < 0)
    return fail(SGE_ERR_ARG, "%s: negative ELL capacity K (%d) or spill capacity S_max (%d)", kName,
                ell_cap, s_max);
  if (ell_cap > kLightMaxK)
    return fail(SGE_ERR_UNSUPPORTED, "%s: ELL capacity K = %d beyond %d", kName, ell_cap, kLightMaxK);
  if (d_ff % 8) return fail(SGE_ERR_ARG, "%s: d_ff %% 8 != 0", kName);
  if (n_tokens == 0) return SGE_OK;
  if (!x || !count || !idx || !val || !wu_t || !wd || !y || !workspace || (s_max > 0 && !wd_t))
    return fail(SGE_ERR_ARG, "%s: null pointer", kName);
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) || !aligned16(val) ||
      (wd_t && !aligned16(wd_t)) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(SGE_ERR_ARG, "%s: pointer not 16-byte aligned (workspace: 256)", kName);
  const int64_t pool_slots = pool_slots_for(kPoolBytes, d_model);
  const RoutedLayout L(n_tokens, d_model, d_ff, s_max, pool_slots);
  if (workspace_bytes < L.total)
    return fail(SGE_ERR_ARG, "%s: workspace of %zu bytes, %zu needed", kName, workspace_bytes, L.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FusedCall c;
  rc = fused_prepare(c, kName, x, count, idx, val, wu_t, wd, ldw, y, n_tokens, d_model, d_ff, SGE_BF16,
                     tile, cap, workspace, pool_slots, diag, true);
  if (rc) return rc;
  // Few tokens: every spill GEMM would stream all of W_up and W_down for a
  // handful of rows; the per-entry path streams only the rows it uses.
  if (c.small || s_max == 0) {
    if (c.small) return run_small(c.prm, c.L, c.ws, pool_slots, c.nv, true, st);
    if ((rc = fused_launch_plan(c, no_route(), st))) return rc;
    return fused_launch_main(c, st);
  }
  SideStream* side = nullptr;
  if ((rc = side_stream(&side))) return rc;
  if ((rc = prefer_max_shared(reinterpret_cast<const void*>(spill_prep_kernel)))) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* spill_rows = reinterpret_cast<int*>(ws + L.rows);
  int* n_heavy = c.prm.hdr + kHHeavy;
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  uint16_t* as = reinterpret_cast<uint16_t*>(ws + L.as);
  uint16_t* hs = reinterpret_cast<uint16_t*>(ws + L.hs);
  const RouteArgs route{ell_cap, s_max, 1, reinterpret_cast<int2*>(ws + L.heavy), spill_rows, diag};
  if ((rc = fused_launch_plan(c, route, st))) return rc;

  const int f = static_cast<int>(d_ff), d = static_cast<int>(d_model);
  LightParams lp{static_cast<const uint16_t*>(x), count, idx, static_cast<const uint16_t*>(val),
                 static_cast<const char*>(wu_t), static_cast<const char*>(wd), ldw * 2,
                 static_cast<uint16_t*>(y), c.prm.ntok, n_tokens, d, f / tile, tile, cap, ell_cap};
  std::lock_guard<std::mutex> lock(g_side_mutex);
  cudaError_t e = cudaEventRecord(side->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s, side->fork, 0);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: fork: %s", kName, cudaGetErrorString(e));
  rc = launch_light_nv(lp, side->s);
  e = cudaEventRecord(side->join, side->s);  // recorded even after a failed launch
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: join: %s", kName, cudaGetErrorString(e));

  // the spill on the caller's stream, beside the light tokens
  if (!rc) {
    const int prep_grid = s_max < kPrepCtas ? s_max : kPrepCtas;
    spill_prep_kernel<<<prep_grid, kPrepThreads, 0, st>>>(
        static_cast<const uint16_t*>(x), count, idx, static_cast<const uint16_t*>(val), spill_rows,
        n_heavy, s_max, d, f, f / tile, tile, cap, xs, as);
    rc = check_launch("twell_hybrid_up_down (spill prep)");
  }
  using S = TcPairShape<kSpillBN, 1>;
  CUtensorMap ma, mb, mh, md;
  if (!rc) rc = make_tmap_bf16(&ma, xs, s_max, d_model, d_model, kBM);
  if (!rc) rc = make_tmap_bf16(&mb, wu_t, d_ff, d_model, ldw, S::BN / 2);
  if (!rc) {
    EpiSpillUp e1{as, nullptr, hs, n_heavy, s_max, f};
    rc = launch_tc_gemm_pair<S>(ma, mb, mb, s_max, d_ff, d_model, e1, diag, st,
                                "twell_hybrid_up_down (spill up)");
  }
  if (!rc) rc = make_tmap_bf16(&mh, hs, s_max, d_ff, d_ff, kBM);
  if (!rc) rc = make_tmap_bf16(&md, wd_t, d_model, d_ff, d_ff, S::BN / 2);
  if (!rc) {
    EpiScatterRows e2{static_cast<uint16_t*>(y), spill_rows, n_heavy, s_max, d};
    rc = launch_tc_gemm_pair<S>(mh, md, md, s_max, d_model, d_ff, e2, diag, st,
                                "twell_hybrid_up_down (spill down)");
  }
  // join: the caller's stream continues once the light tokens are done too
  e = cudaStreamWaitEvent(st, side->join, 0);
  if (rc) return rc;
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "%s: join: %s", kName, cudaGetErrorString(e));
  return SGE_OK;
}
