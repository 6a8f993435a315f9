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
//           go to the spill list, every other non-empty token to a size
//           class of the light lists (fused_kernels.cuh's planning kernels)
//   prep    per spill row: its x row into X_s, its stored activations
//           scattered into a dense row of A_s (zeros elsewhere)
//   GEMM 1  U = X_s W_up on tcgen05 (CTA pairs), epilogue H_s = bf16(A_s (.) U)
//   light   the light tokens (and heavy ones past S_max) through CUDA
//           cores, one warp per token, its entries' W_up and W_down rows
//           streamed through a ring of shared-memory slots filled by bulk
//           copies (light_ring_kernel below); y = 0 for tokens without
//           stored entries.  Its CTAs start while GEMM 1's last wave runs.
//   GEMM 2  Y_s = H_s W_down on tcgen05, epilogue scatters row r to y[token r]
//           (with split-K and a part-sum kernel when the spill rows make
//           few output tiles)
//
// Consecutive launches use programmatic dependent launch: each kernel's
// set-up overlaps the end of the previous one.
// Every token's y is written exactly once, by GEMM 2 or by the light-token
// kernel; results do not depend on scheduling.  Per row the arithmetic is
// that of the dense FFN restricted to the stored entries: fp32 accumulation,
// h rounded to bf16 before the down projection, as in twell_fused_up_down.
#include <algorithm>

#include "fused_kernels.cuh"
#include "spill_gemm.cuh"
#include "tc_launch.cuh"

namespace sge {

// X_s and A_s rows of the kept spill tokens, a CTA per row (grid-stride over
// the spill ranks): the x row is copied while the tile counts load; the dense
// row of a is assembled in shared memory (zeroed, then every stored entry
// written by its own thread, which finds its tile by a binary search over the
// row's tile prefix) and stored with whole 16-byte vectors, so global memory
// sees each row written once, in full lines.
constexpr int kPrepThreads = 256;

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
  extern __shared__ __align__(16) uint8_t prep_smem[];
  grid_dep_launch();
  grid_dep_wait();
  uint16_t* row = reinterpret_cast<uint16_t*>(prep_smem);              // f bf16
  int* pre = reinterpret_cast<int*>(prep_smem + ((2 * f + 15) & ~15));  // nt + 1
  int* wsum = pre + 260;                                                // warps
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kept = min(*n_heavy, s_max);
  for (int r = blockIdx.x; r < kept; r += gridDim.x) {
    const int64_t t = spill_rows[r];
    const int c = tid < nt ? min(static_cast<int>(__ldg(count + t * nt + tid)), cap) : 0;
    const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
    uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<int64_t>(r) * d);
    for (int v = tid; v < d / 8; v += kPrepThreads) dst[v] = __ldg(src + v);
    for (int v = tid; v < f / 8; v += kPrepThreads) reinterpret_cast<uint4*>(row)[v] = make_uint4(0, 0, 0, 0);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kPrepThreads / 32; ++w) {
      base += w < warp ? wsum[w] : 0;
      total += wsum[w];
    }
    if (tid < nt) pre[tid] = base + incl - c;
    __syncthreads();  // the prefix is complete, the row is zero
    for (int e = tid; e < total; e += kPrepThreads) {
      int b = 0;  // the last tile whose prefix is <= e
      for (int step = 128; step > 0; step >>= 1)
        if (b + step < nt && pre[b + step] <= e) b += step;
      const int64_t at = (t * nt + b) * cap + (e - pre[b]);
      // a stored index is < T; kept inside its tile even if it is not
      row[b * tile + clamp_index(__ldg(idx + at), tile)] = __ldg(val + at);
    }
    __syncthreads();  // the row is assembled
    uint4* arow = reinterpret_cast<uint4*>(as + static_cast<int64_t>(r) * f);
    for (int v = tid; v < f / 8; v += kPrepThreads) arow[v] = reinterpret_cast<const uint4*>(row)[v];
    __syncthreads();  // row[], pre[] and wsum[] are rewritten for the next row
  }
}

// Shared memory of the prep kernel for F hidden units.
inline int prep_smem_bytes(int64_t f) { return static_cast<int>(((2 * f + 15) & ~15) + 4 * (260 + 8)); }

// ------------------------------------------------------ light tokens
//
// Every token not on the spill, straight from TwELL, one warp per token: the
// warps pull tokens from the planning kernel's size-class lists (largest
// class first) through a global cursor.  A warp keeps x[t] (bf16) and the
// fp32 y[t] in registers and streams the token's entries through its own
// ring of S (2 to 4) shared-memory slots filled by cp.async.bulk: a slot
// holds an entry's W_up row in its first half and its W_down row in the
// second (one 8 KB copy when the caller interleaves the two matrices row by
// row with rows of a multiple of 512 bytes, two copies otherwise).  Per
// entry: u = x . W_up[:, j] (exact bf16 products, fp32 sums, reduced over the
// lanes), h = bf16(a u), y += h W_down[j].  Entries are resolved from the
// tile counts 32 at a time, one round ahead of the copies.  The warps first
// store y = 0 for the tokens without stored entries, each an equal share of
// the batch.  Light tokens have at most K entries; heavy tokens past S_max
// (when the caller's S_max is too small) take the same path, entry by
// entry.  Every wait is bounded: a wait that runs out sets SGE_FLAG_TIMEOUT
// and stops the CTA after its copies in flight have landed.
constexpr int kRingMaxWarps = 8;
constexpr int kRingMaxSlots = 4;
constexpr int kRingSmem = 220 * 1024;  // slots of all warps

struct RingParams {
  const uint16_t* x;
  const uint8_t* count;
  const uint8_t* idx;
  const uint16_t* val;
  const char* wu;  // row j at wu + j * w_ld bytes
  const char* wd;
  int64_t w_ld;
  uint16_t* y;
  const int* ntok;
  const int* hdr;       // job counts per class (kHLight), cursor (kHCursor)
  int* cursor;
  const int2* lights;   // [kLightClasses][n_rows]: (token, entries)
  int32_t* diag;
  int64_t n_rows;
  int nt, tile, cap;
  int row_bytes;   // d * 2
  int slot_bytes;  // two halves of NV * 512 bytes
  int slots;       // S, slots per warp
  int w_one;       // one copy brings both rows of an entry
};

template <int NV, int NTR>
__device__ __forceinline__ void light_ring_body(const RingParams& p) {
  using E = Elem<true>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5, S = p.slots;
  const int half = p.slot_bytes / 2;
  uint8_t* ring = smem + warp * S * p.slot_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + warps * S * p.slot_bytes);
  uint64_t* full = bars + warp * S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + warps * S);
  const int pieces = p.row_bytes / 16;

  // slot bytes past a row stay zero for the whole kernel (loads need no test)
  if (p.row_bytes < half)
    for (int q = 0; q < 2 * S; ++q)
      for (int o = p.row_bytes + lane * 16; o < half; o += 32 * 16)
        *reinterpret_cast<uint4*>(ring + q * half + o) = make_uint4(0, 0, 0, 0);
  if (lane == 0)
    for (int q = 0; q < S; ++q) mbar_init(full + q, 1);
  if (threadIdx.x == 0) *abort_flag = 0;
  fence_mbar_init();
  __syncthreads();

  // y = 0 for the tokens without stored entries, an equal share per warp
  {
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * warps + warp;
    const int64_t ngw = static_cast<int64_t>(gridDim.x) * warps;
    const int64_t per = (p.n_rows + ngw - 1) / ngw;
    const int64_t t0 = gw * per, t1 = min(p.n_rows, t0 + per);
    for (int64_t tb = t0; tb < t1; tb += 32) {
      unsigned m = __ballot_sync(0xffffffffu, tb + lane < t1 && p.ntok[tb + lane] == 0);
      while (m) {
        const int i = __ffs(m) - 1;
        m &= m - 1;
        uint4* row = reinterpret_cast<uint4*>(p.y + (tb + i) * (p.row_bytes / 2));
        for (int pc = lane; pc < pieces; pc += 32) row[pc] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  int n_light[kLightClasses];
#pragma unroll
  for (int c = 0; c < kLightClasses; ++c) n_light[c] = p.hdr[kHLight + c];

  uint32_t parity = 0;  // bit q: phase parity of slot q's next completion
  bool ok = true;
  int issued_total = 0, consumed_total = 0;  // copies issued / consumed by this warp
  while (ok) {
    // ---- next token (largest class first)
    int k = 0;
    if (lane == 0) k = atomicAdd(p.cursor, 1);
    k = __shfl_sync(0xffffffffu, k, 0);
    int t = -1, n = 0;
#pragma unroll
    for (int c = 0; c < kLightClasses; ++c) {
      if (t < 0 && k < n_light[c]) {
        const int2 j = p.lights[c * p.n_rows + k];
        t = static_cast<int>(checked_index(j.x, p.n_rows));
        n = j.y;
      }
      k -= n_light[c];
    }
    if (t < 0) break;
    // ---- x row and the tile prefix of the token's counts
    uint4 xr[NV];
    const uint4* xrow = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(t) * (p.row_bytes / 2));
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int pc = lane + 32 * q;
      xr[q] = pc < pieces ? __ldg(xrow + pc) : make_uint4(0, 0, 0, 0);
    }
    int pre[NTR];
    {
      const uint8_t* cnt = p.count + static_cast<int64_t>(t) * p.nt;
      int c[NTR];
#pragma unroll
      for (int r = 0; r < NTR; ++r) {
        const int b = lane + 32 * r;
        c[r] = b < p.nt ? min(static_cast<int>(__ldg(cnt + b)), p.cap) : 0;
      }
      int carry = 0;
#pragma unroll
      for (int r = 0; r < NTR; ++r) {
        int incl = c[r];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        pre[r] = carry + incl - c[r];
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    // entry e of round e / 32 lives in lane e % 32: its column and raw value
    auto resolve = [&](int round, int& jcol, uint32_t& araw) {
      const int e = round * 32 + lane;
      jcol = 0;
      araw = 0;
      int b = 0;
#pragma unroll
      for (int step = 16 * NTR; step > 0; step >>= 1) {
        const int cand = b + step;
        const int v = prefix_at<NTR>(pre, cand < p.nt ? cand : 0);
        if (cand < p.nt && v <= e) b = cand;
      }
      const int s = e - prefix_at<NTR>(pre, b);
      if (e < n) {
        const int64_t at = (static_cast<int64_t>(t) * p.nt + b) * p.cap + s;
        jcol = b * p.tile + clamp_index(__ldg(p.idx + at), p.tile);
        araw = __ldg(p.val + at);
      }
    };
    int cur_j, nxt_j;
    uint32_t cur_a, nxt_a;
    resolve(0, cur_j, cur_a);
    resolve(1, nxt_j, nxt_a);
    // ---- the ring: entry e goes to slot (first + e) % S
    const int first = issued_total % S;
    float acc[NV][8];
#pragma unroll
    for (int q = 0; q < NV; ++q)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q][i] = 0.0f;
    // copies of the first min(n, slots) entries
    int round_base = 0;  // first entry of the round held in cur_*
    int next_issue = 0;
    auto issue_next = [&]() {
      const int e = next_issue;
      const int jc = __shfl_sync(0xffffffffu, e - round_base < 32 ? cur_j : nxt_j, e & 31);
      if (lane == 0) {
        const int q = (first + e) % S;
        uint8_t* dst = ring + q * p.slot_bytes;
        fence_proxy_async_smem();  // the slot's earlier reads come before the copy
        mbar_arrive_expect_tx(full + q, 2 * static_cast<uint32_t>(p.row_bytes));
        if (p.w_one) {
          bulk_load(dst, p.wu + static_cast<int64_t>(jc) * p.w_ld, 2 * p.row_bytes, full + q);
        } else {
          bulk_load(dst, p.wu + static_cast<int64_t>(jc) * p.w_ld, p.row_bytes, full + q);
          bulk_load(dst + half, p.wd + static_cast<int64_t>(jc) * p.w_ld, p.row_bytes, full + q);
        }
      }
      ++next_issue;
      ++issued_total;
    };
    while (next_issue < n && next_issue < S) issue_next();
    for (int e = 0; e < n; ++e) {
      const int q = (first + e) % S;
      const float a = E::from_raw(__shfl_sync(0xffffffffu, cur_a, e & 31));
      if (!(ok = ud_wait_or_abort(full + q, (parity >> q) & 1u, abort_flag, p.diag))) break;
      parity ^= 1u << q;
      ++consumed_total;
      const uint32_t sa = smem_u32(ring + q * p.slot_bytes);
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k2 = 0; k2 < NV; ++k2)
        E::dot2(xr[k2], lds128(sa + (lane + 32 * k2) * 16), s8[2 * (k2 & 3)], s8[2 * (k2 & 3) + 1]);
      float u = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
      const uint16_t h = E::h_of(a * u);
#pragma unroll
      for (int k2 = 0; k2 < NV; ++k2) E::axpy(h, lds128(sa + half + (lane + 32 * k2) * 16), acc[k2]);
      __syncwarp();  // every lane has read the slot
      if ((e & 31) == 31) {  // the next round becomes current; resolve the one after
        cur_j = nxt_j;
        cur_a = nxt_a;
        round_base += 32;
        resolve((e >> 5) + 2, nxt_j, nxt_a);
      }
      if (next_issue < n) issue_next();
    }
    if (!ok) break;
    uint4* yrow = reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(t) * (p.row_bytes / 2));
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int pc = lane + 32 * q;
      if (pc < pieces) yrow[pc] = E::pack(acc[q]);
    }
  }
  // copies still in flight (only after a give-up) land before the CTA exits
  for (int i = consumed_total; i < issued_total; ++i) {
    const int q = i % S;
    mbar_wait(full + q, (parity >> q) & 1u, p.diag);
    parity ^= 1u << q;
  }
}

// Workspace: the planning kernels' (fused_kernels.cuh), then the per-block
// heavy counts, the spill list and the spill operands X_s [S_max][d], A_s
// and H_s [S_max][F] (bf16, 1024-byte aligned offsets).
constexpr int kSpillBN = 256;

struct RoutedLayout {
  WsLayout fused;
  size_t heavy, rows, xs, as, hs, part, total;
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
    part = o;      o = up(o + (sm > 0 ? kSplitPartBytes : 0), 1024);
    total = o;
  }
};

// The light-token kernel runs after the spill up GEMM in the stream but does
// not wait for it: it needs only the planning kernels' lists, complete once
// the up GEMM has passed its own dependency wait (the GEMM engine lets its
// successor launch only after that wait), and it touches nothing the GEMM
// writes.  So its CTAs start on the SMs the GEMM's last wave of tiles leaves
// idle.  It waits for the GEMM before exiting, so that the down GEMM, which
// waits for this kernel, also finds H_s complete.
template <int NV, int NTR>
__global__ void __launch_bounds__(kRingMaxWarps * 32, 1) light_ring_kernel(const RingParams p) {
  grid_dep_launch();
  light_ring_body<NV, NTR>(p);
  grid_dep_wait();
}

template <int NV, int NTR>
static int launch_ring(const RingParams& p, int warps, int smem, cudaStream_t st) {
  auto kern = light_ring_kernel<NV, NTR>;
  const int rc = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (rc) return rc;
  return launch_pdl(kern, dim3(sm_count()), dim3(warps * 32), smem, st, "twell_hybrid_up_down (light tokens)", p);
}

template <int NV>
static int ring_ntr(const RingParams& p, int warps, int smem, cudaStream_t st) {
  if (p.nt <= 32) return launch_ring<NV, 1>(p, warps, smem, st);
  if (p.nt <= 64) return launch_ring<NV, 2>(p, warps, smem, st);
  if (p.nt <= 128) return launch_ring<NV, 4>(p, warps, smem, st);
  return launch_ring<NV, 8>(p, warps, smem, st);
}

// The light-token kernel: slots of two halves of nv * 512 bytes, as many
// warps (at most kRingMaxWarps) and slots (2 to kRingMaxSlots, 3 preferred)
// as the shared memory holds.
static int run_ring(RingParams p, int nv, cudaStream_t st) {
  p.slot_bytes = 2 * nv * 512;
  int warps = kRingMaxWarps, slots = 3;
  while (warps * slots * p.slot_bytes > kRingSmem) {
    if (slots > 2) --slots;
    else --warps;
  }
  if (warps < 1) return fail(SGE_ERR_UNSUPPORTED, "twell_hybrid_up_down: rows of %d bytes", p.row_bytes);
  p.slots = slots;
  p.w_one = p.w_one && 2 * p.row_bytes == p.slot_bytes;
  const int smem = warps * slots * p.slot_bytes + warps * slots * 8 + 16;
  switch (nv) {
    case 2: return ring_ntr<2>(p, warps, smem, st);
    case 4: return ring_ntr<4>(p, warps, smem, st);
    case 8: return ring_ntr<8>(p, warps, smem, st);
    case 12: return ring_ntr<12>(p, warps, smem, st);
    default: return ring_ntr<16>(p, warps, smem, st);
  }
}

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
  NvtxRange nvtx_range("twell_hybrid_up_down");
  static const char* kName = "twell_hybrid_up_down";
  clear_error();
  int rc = check_args(kName, n_tokens, d_model, d_ff, ldw, tile, cap);
  if (rc) return rc;
  if (ell_cap < 0 || s_max < 0)
    return fail(SGE_ERR_ARG, "%s: negative ELL capacity K (%d) or spill capacity S_max (%d)", kName,
                ell_cap, s_max);
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
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* spill_rows = reinterpret_cast<int*>(ws + L.rows);
  int* n_heavy = c.prm.hdr + kHHeavy;
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  uint16_t* as = reinterpret_cast<uint16_t*>(ws + L.as);
  uint16_t* hs = reinterpret_cast<uint16_t*>(ws + L.hs);
  float* part = reinterpret_cast<float*>(ws + L.part);
  const RouteArgs route{ell_cap, s_max, 1, reinterpret_cast<int2*>(ws + L.heavy), spill_rows, diag};
  if ((rc = fused_launch_plan(c, route, st))) return rc;

  // the spill prep, the up GEMM, the light tokens, the down GEMM
  const int f = static_cast<int>(d_ff), d = static_cast<int>(d_model);
  RingParams rp{static_cast<const uint16_t*>(x), count, idx, static_cast<const uint16_t*>(val),
                static_cast<const char*>(wu_t), static_cast<const char*>(wd), ldw * 2,
                static_cast<uint16_t*>(y), c.prm.ntok, c.prm.hdr, c.prm.hdr + kHCursor, c.prm.lights,
                diag, n_tokens, f / tile, tile, cap, d * 2, 0, 0, 0};
  // one copy per entry when each wd row directly follows its wu_t row
  // (run_ring also needs a row to fill half a slot exactly)
  rp.w_one = static_cast<const char*>(wd) == static_cast<const char*>(wu_t) + 2 * d_model &&
             ldw == 2 * d_model;
  {
    const int smem = prep_smem_bytes(d_ff);
    if ((rc = set_smem_limit(reinterpret_cast<const void*>(spill_prep_kernel), smem))) return rc;
    const int prep_grid = static_cast<int>(std::min<int64_t>(s_max, 8 * static_cast<int64_t>(sm_count())));
    if ((rc = launch_pdl(spill_prep_kernel, dim3(prep_grid), dim3(kPrepThreads), smem, st,
                         "twell_hybrid_up_down (spill prep)", static_cast<const uint16_t*>(x), count, idx,
                         static_cast<const uint16_t*>(val), spill_rows, n_heavy, s_max, d, f, f / tile,
                         tile, cap, xs, as)))
      return rc;
  }
  using S = TcPairShape<kSpillBN, 1, 2>;
  CUtensorMap ma, mb, mh, md;
  if ((rc = make_tmap_bf16(&ma, xs, s_max, d_model, d_model, kBM))) return rc;
  if ((rc = make_tmap_bf16(&mb, wu_t, d_ff, d_model, ldw, S::BN / 2))) return rc;
  EpiSpillUp e1{as, nullptr, hs, n_heavy, s_max, f};
  if ((rc = launch_tc_gemm_pair<S>(ma, mb, mb, s_max, d_ff, d_model, e1, diag, st,
                                   "twell_hybrid_up_down (spill up)")))
    return rc;
  // the light tokens, overlapping the up GEMM's last wave (see light_ring_kernel)
  if ((rc = run_ring(rp, c.nv, st))) return rc;
  if ((rc = make_tmap_bf16(&mh, hs, s_max, d_ff, d_ff, kBM))) return rc;
  if ((rc = make_tmap_bf16(&md, wd_t, d_model, d_ff, d_ff, S::BN / 2))) return rc;
  const int tiles_n = (d + S::BN - 1) / S::BN;
  EpiScatterRows e2{static_cast<uint16_t*>(y), spill_rows, n_heavy, s_max, d, part, tiles_n, S::BN};
  if ((rc = launch_tc_gemm_pair<S>(mh, md, md, s_max, d_model, d_ff, e2, diag, st,
                                   "twell_hybrid_up_down (spill down)", kSplitMax)))
    return rc;
  return launch_split_scatter(part, spill_rows, n_heavy, s_max, d, tiles_n * S::BN, static_cast<uint16_t*>(y),
                              st, "twell_hybrid_up_down (split sum)");
}
