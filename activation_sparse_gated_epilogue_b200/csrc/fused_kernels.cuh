// Fused up and down projections over the TwELL nonzeros.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 02, last paragraph: one custom kernel performs the up and the down
// projection in a single traversal, fusing the two products so that the
// intermediate h is never written to global memory.  For every stored entry
// (t, j, a) of the TwELL gate activations:
//     u = x[t] . W_up[:, j]      h = a * u      y[t] += h * W_down[j, :]
//
// At the densities the method runs at (about 1% of d_ff) two tokens rarely
// share a column, so every entry streams one row of W_up and one of W_down
// from L2 with little reuse: the kernel is bound by how many row bytes it
// keeps in flight between L2 and the SMs, by the copies and waits per byte,
// and by its instructions per row.
//
// Warps.  Each warp streams its entries through its own ring of
// shared-memory slots with cp.async.bulk: one slot holds an entry's W_up row
// and its W_down row (one copy when the caller interleaves the two matrices
// row by row, two copies on the same mbarrier otherwise); its lanes issue the
// copies of several slots in parallel, ahead of consumption.  It keeps x[t]
// (bf16) and the fp32 y[t] of its job in registers.  For each entry it forms
// the dot product x[t] . W_up[:, j] with exact bf16 x bf16 products
// accumulated in fp32, reduces it over the lanes, rounds h = a * u to the
// activation dtype (what the dense FFN gives h), and accumulates
// h * W_down[j] into y.  h lives only in registers.  Entries are resolved in
// chunks of 32, one per lane.
//
// Teams.  A team of kTeam warps shares one job (a token, or a unit of a heavy
// token): warp w takes the job's entries w, w + kTeam, ...  At the end of the
// job the warps add their fp32 partial y, one after the other in warp order,
// into a row buffer in shared memory; the last warp stores the sum.
//
// Entries.  Each warp resolves its own entries straight from the TwELL
// (exclusive prefix of the token's tile counts in registers, a binary search
// per lane, one load of idx and of val) one chunk ahead of consumption, so
// its copies run ahead across chunk and job boundaries.
//
// Jobs.  Two small kernels plan the work: stored entries per token; then the
// unit length U (a multiple of 32: heavy tokens split into units of about a
// quarter of a team's average share, whose fp32 partial outputs fit the
// pool) and the job lists: units of heavy tokens first, then the other
// non-empty tokens in four classes of decreasing size, so that the last jobs
// are short.  The main kernel's warps first store y = 0 for the empty tokens
// of an equal share of the batch each.  The team leader pulls jobs from a
// global cursor and queues them two jobs ahead.  A unit stores its fp32
// partial in the pool; the team that completes a split token's last unit (a
// counter per token) sums the units' partials in unit order and stores y.  No
// atomics touch data, so results do not depend on scheduling.
//
// Every wait is bounded: a wait that runs out of time sets SGE_FLAG_TIMEOUT in
// diag and stops the CTA, after each warp has waited (again bounded) for its
// own copies in flight.
#pragma once

#include "sge_host.h"
#include "debug_checks.cuh"
#include "sparse_common.cuh"

namespace sge {

constexpr int kTeam = 4;        // warps per job
constexpr int kChunk = 32;      // entries per chunk, one per lane
constexpr int kMaxSlots = 8;    // ring slots per warp
constexpr int kSmemBudget = 232448;
constexpr int kUnitMin = 32;
constexpr int kMaxCtas = 256;   // the grid is clamped to this many CTAs
constexpr int kLightClasses = 4;
// Per-team shared memory before the row buffer: the job queue (4 entries and
// a staging entry), then the barriers tbar, tfree and chain[kTeam - 1].
constexpr int kTeamHdr = (5 * 32 + 8 * (2 + kTeam - 1) + 15) & ~15;

constexpr size_t kPoolBytes = size_t(64) << 20;

// Warps per CTA for NV pieces per lane: registers hold NV pieces of x and
// the fp32 y of NV pieces per lane.
template <int NV>
struct UdLaunch {
  static constexpr int kWarps = NV <= 2 ? 24 : (NV <= 4 ? 16 : (NV <= 8 ? 12 : 8));
};

inline int warps_for_nv(int nv) {
  return nv <= 2 ? UdLaunch<2>::kWarps
                 : (nv <= 4 ? UdLaunch<4>::kWarps : (nv <= 8 ? UdLaunch<8>::kWarps : UdLaunch<16>::kWarps));
}

// Pieces per lane (2, 4, 8, 12 or 16) for rows of row_bytes; 0 if too long.
inline int nv_for(int64_t row_bytes) {
  const int64_t need = (row_bytes / 16 + 31) / 32;
  if (need <= 2) return 2;
  if (need <= 4) return 4;
  if (need <= 8) return 8;
  if (need <= 12) return 12;
  if (need <= 16) return 16;
  return 0;
}

// Header of the workspace (int32 words).
constexpr int kHTotal = 0;     // stored entries (int64, words 0..1)
constexpr int kHUnit = 2;      // unit length U
constexpr int kHUnits = 3;     // unit jobs
constexpr int kHLight = 4;     // unsplit non-empty tokens per size class (4 words)
constexpr int kHSplit = 8;     // split tokens
constexpr int kHCursor = 9;    // job cursor
constexpr int kHOverflow = 10; // units that did not fit the pool (stays 0)
constexpr int kHHeavy = 11;    // routed calls: tokens with more than K stored entries
constexpr size_t kHdrBytes = 256;

// Routing of heavy tokens to the tensor-core spill (routed calls only): a
// token with more than k stored entries is a heavy token; heavy tokens are
// ranked in ascending token order and the first s_max of them go to the
// spill (spill_rows[rank] = token, and the token's entry count is replaced
// by -1 so that the per-entry kernel neither runs nor zeroes it); heavy
// tokens ranked s_max or later stay per-entry jobs.  k < 0: no routing.
struct RouteArgs {
  int k;
  int s_max;
  int light_apart;   // job lists for the light-token kernel: every token not on the
                     // spill, unsplit, in size classes
  int2* blk_heavy;   // per count block: heavy tokens, their stored entries
  int* spill_rows;   // [s_max]
  int32_t* diag;     // nullable: gains the number of heavy tokens
};

inline RouteArgs no_route() { return RouteArgs{-1, 0, 0, nullptr, nullptr, nullptr}; }

struct Job {  // 32 bytes
  int t;      // token; -1 ends the work
  int e0;     // first entry of the job among the token's entries
  int n;      // entries
  int nu;     // units of the token (1: not split)
  int u;      // this unit
  int base;   // first pool slot of the token's units
  int sid;    // split-token index (completion counters)
  int pad;
};

// Workspace layout for n tokens and pool_slots pool slots of d floats.
struct WsLayout {
  size_t blk, ntok, lights, units, done, pool, total;
  WsLayout(int64_t n, int64_t d, int64_t pool_slots) {
    const size_t nblk = static_cast<size_t>((n + 255) / 256);
    const size_t ps = static_cast<size_t>(pool_slots);
    size_t o = kHdrBytes;
    blk = o;     o += (8 * nblk + 255) & ~size_t(255);
    ntok = o;    o += (4 * static_cast<size_t>(n) + 255) & ~size_t(255);
    lights = o;  o += (8 * kLightClasses * static_cast<size_t>(n) + 255) & ~size_t(255);
    units = o;   o += 32 * ps;
    done = o;    o += (4 * ps + 255) & ~size_t(255);
    pool = o;    o += 4 * ps * static_cast<size_t>(d);
    total = o;
  }
};

inline int64_t pool_slots_for(size_t pool_bytes, int64_t d) {
  const int64_t s = static_cast<int64_t>(pool_bytes / (4 * static_cast<size_t>(d)));
  return s < (1 << 28) ? s : (1 << 28);
}

struct UdParams {
  const void* x;
  const uint8_t* count;
  const uint8_t* idx;
  const void* val;
  const void* wu_t;
  const void* wd;
  void* y;
  int* hdr;
  const int* ntok;
  const int2* lights;  // [kLightClasses][n_rows]
  const Job* units;
  int* done;
  float* pool;
  int32_t* diag;
  int64_t n_rows;
  int d;
  int nt;
  int tile;
  int cap;
  int row_bytes;
  int teams;       // teams per CTA
  int slots;       // ring slots per warp
  int slot_bytes;  // one ring slot: two halves of NV * 512 bytes (a row, then zeros)
  int64_t w_ld;    // row stride of wu_t and wd in bytes
  int w_one;       // each wd row directly follows its wu_t row and fills a half: one copy per entry
  int off_full;    // shared-memory offsets: per-warp slot barriers,
  int off_team;    // per-team job queue, barriers and row buffer,
  int team_bytes;
  int off_abort;   // CTA-wide abort flag
  int zero_empty;  // store y = 0 for tokens without stored entries (routed calls leave it to
                   // the light-token kernel)
};

// ------------------------------------------------------------- planning

// Stored entries of every token (counts capped at C) and per-block sums;
// block 0 also zeroes the job counters that the job-list kernel fills.
static __global__ void __launch_bounds__(256) ud_count_kernel(const uint8_t* __restrict__ count,
                                                       int64_t n_rows, int nt, int cap,
                                                       int* __restrict__ ntok,
                                                       long long* __restrict__ blk_sum, int* hdr,
                                                       RouteArgs route) {
  __shared__ long long wsum[8];
  __shared__ int2 wheavy[8];
  grid_dep_launch();
  grid_dep_wait();  // the counts come from the gate GEMM (no-op for a plain launch)
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (blockIdx.x == 0 && threadIdx.x < 16) {
    const int w = threadIdx.x;
    if (w >= kHUnits && w <= kHOverflow) hdr[w] = 0;
  }
  int s = 0;
  if (t < n_rows) {
    const uint8_t* c = count + t * nt;
    if ((nt & 3) == 0 && (reinterpret_cast<uintptr_t>(count) & 3) == 0) {
      const uint32_t* c4 = reinterpret_cast<const uint32_t*>(c);
      for (int b = 0; b < nt / 4; ++b) {
        const uint32_t v = __ldg(c4 + b);
#pragma unroll
        for (int k = 0; k < 4; ++k) s += min(static_cast<int>((v >> (8 * k)) & 255u), cap);
      }
    } else {
      for (int b = 0; b < nt; ++b) s += min(static_cast<int>(__ldg(c + b)), cap);
    }
    ntok[t] = s;
  }
  // routed calls: heavy tokens count apart (rows, entries) from the others
  const bool heavy = route.k >= 0 && s > route.k;
  long long v = heavy ? 0 : s;
  int hr = heavy ? 1 : 0, he = heavy ? s : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v += __shfl_xor_sync(0xffffffffu, v, o);
    hr += __shfl_xor_sync(0xffffffffu, hr, o);
    he += __shfl_xor_sync(0xffffffffu, he, o);
  }
  if ((threadIdx.x & 31) == 0) {
    wsum[threadIdx.x >> 5] = v;
    wheavy[threadIdx.x >> 5] = make_int2(hr, he);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    int2 h = make_int2(0, 0);
    for (int w = 0; w < 8; ++w) {
      tot += wsum[w];
      h.x += wheavy[w].x;
      h.y += wheavy[w].y;
    }
    blk_sum[blockIdx.x] = tot;
    if (route.k >= 0) route.blk_heavy[blockIdx.x] = h;
  }
}

// Total entries (summed from the per-block sums by the calling CTA; every
// CTA gets the same value) and the unit length U.  All threads must call it.
static __device__ int plan_unit(const long long* __restrict__ blk_sum, int64_t nblk, int64_t pool_slots,
                         int64_t n_teams, long long extra, long long* total) {
  __shared__ long long wsum[8];
  __shared__ int u_sh;
  __shared__ long long tot_sh;
  long long s = threadIdx.x == 0 ? extra : 0;
  for (int64_t b = threadIdx.x; b < nblk; b += blockDim.x) s += blk_sum[b];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += wsum[w];
    // Units of about a quarter of a team's average share (measured on the 1B
    // workload: an eighth costs more job overhead, a half more imbalance);
    // split tokens must fit the pool (a token of n > U entries takes
    // ceil(n / U) <= 2n / U slots).
    long long u = (tot + 4 * n_teams - 1) / (4 * n_teams);
    const long long u_pool = pool_slots > 0 ? (2 * tot + pool_slots - 1) / pool_slots : (1LL << 30);
    if (u < u_pool) u = u_pool;
    if (u < kUnitMin) u = kUnitMin;
    u = (u + kChunk - 1) / kChunk * kChunk;
    if (u > (1LL << 30)) u = 1LL << 30;
    u_sh = static_cast<int>(u);
    tot_sh = tot;
  }
  __syncthreads();
  *total = tot_sh;
  return u_sh;
}

// Size class of an unsplit token of n entries (0: largest).
__device__ __forceinline__ int light_class(int n, int U) {
  return n > U / 2 ? 0 : (n > U / 8 ? 1 : (n > U / 32 ? 2 : 3));
}

// Job lists: every split token's units, every other non-empty token in its
// size class.  Each CTA first derives the unit length from the count
// kernel's per-block sums (CTA 0 records it).  Slots in the lists come from
// warp-aggregated atomics: the job order may vary between calls, the results
// do not.
static __global__ void __launch_bounds__(256) ud_jobs_kernel(int* __restrict__ ntok, int64_t n_rows,
                                                      const long long* __restrict__ blk_sum,
                                                      int64_t nblk, int64_t n_teams,
                                                      int* hdr, int2* __restrict__ lights,
                                                      Job* __restrict__ units, int* __restrict__ done,
                                                      int64_t pool_slots, RouteArgs route) {
  grid_dep_launch();
  grid_dep_wait();
  __shared__ long long hsum[3][8];
  __shared__ int wrank[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const unsigned lt = (1u << lane) - 1u;
  // routed calls: heavy tokens in all blocks and in the blocks before this one
  long long h_rows = 0, h_entries = 0, h_before = 0;
  if (route.k >= 0) {
    long long a = 0, b = 0, c = 0;
    for (int64_t k = threadIdx.x; k < nblk; k += blockDim.x) {
      const int2 h = route.blk_heavy[k];
      a += h.x;
      b += h.y;
      if (k < blockIdx.x) c += h.x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
      c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    if (lane == 0) {
      hsum[0][warp] = a;
      hsum[1][warp] = b;
      hsum[2][warp] = c;
    }
    __syncthreads();
    for (int w = 0; w < 8; ++w) {
      h_rows += hsum[0][w];
      h_entries += hsum[1][w];
      h_before += hsum[2][w];
    }
  }
  long long total = 0;
  // heavy tokens past s_max stay per-entry jobs: then their entries count
  // (all heavy entries: an upper bound, which only coarsens the units)
  const int U = plan_unit(blk_sum, nblk, pool_slots, n_teams, h_rows > route.s_max ? h_entries : 0,
                          &total);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *reinterpret_cast<long long*>(hdr + kHTotal) = total;
    hdr[kHUnit] = U;
    if (route.k >= 0) {
      hdr[kHHeavy] = static_cast<int>(h_rows);
      if (route.diag) atomicAdd(reinterpret_cast<int*>(route.diag + SGE_DIAG_SPILL_ROWS), static_cast<int>(h_rows));
    }
  }
  int n = t < n_rows ? ntok[t] : -1;
  if (route.k >= 0) {
    // ascending rank among the heavy tokens: blocks before, warps before, lanes before
    const bool heavy = n > route.k;
    const unsigned mh = __ballot_sync(0xffffffffu, heavy);
    if (lane == 0) wrank[warp] = __popc(mh);
    __syncthreads();
    long long rank = h_before + __popc(mh & lt);
    for (int w = 0; w < warp; ++w) rank += wrank[w];
    if (heavy && rank < route.s_max) {
      route.spill_rows[rank] = static_cast<int>(t);
      ntok[t] = -1;
      n = -1;
    }
  }
  // routed calls list every token left off the spill, unsplit, in four size
  // classes (more than 32, 8, 2 entries, the rest) for the light-token kernel
  const bool routed_lists = route.k >= 0 && route.light_apart;
  const bool split = !routed_lists && n > U;
  // split tokens: ceil(n / U) units each
  const int k = split ? (n + U - 1) / U : 0;
  int incl = k;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int ktot = __shfl_sync(0xffffffffu, incl, 31);
  const unsigned ms = __ballot_sync(0xffffffffu, split);
  int ubase = 0, sbase = 0;
  if (ms && lane == 0) {
    ubase = atomicAdd(&hdr[kHUnits], ktot);
    sbase = atomicAdd(&hdr[kHSplit], __popc(ms));
  }
  ubase = __shfl_sync(0xffffffffu, ubase, 0);
  sbase = __shfl_sync(0xffffffffu, sbase, 0);
  bool light = n > 0 && (routed_lists || n <= U);
  if (split) {
    const int first = ubase + incl - k;
    const int sid = sbase + __popc(ms & lt);
    if (static_cast<int64_t>(first) + k > pool_slots) {
      atomicAdd(&hdr[kHOverflow], 1);  // cannot happen with the planned U; run it unsplit
      light = true;
    } else {
      for (int u = 0; u < k; ++u) {
        Job j;
        j.t = static_cast<int>(t);
        j.e0 = u * U;
        j.n = min(U, n - u * U);
        j.nu = k;
        j.u = u;
        j.base = first;
        j.sid = sid;
        j.pad = 0;
        units[first + u] = j;
      }
      done[sid] = 0;
    }
  }
  const int cls = light ? light_class(n, routed_lists ? 64 : U) : -1;
#pragma unroll
  for (int c = 0; c < kLightClasses; ++c) {
    const unsigned ml = __ballot_sync(0xffffffffu, cls == c);
    int lbase = 0;
    if (ml && lane == 0) lbase = atomicAdd(&hdr[kHLight + c], __popc(ml));
    lbase = __shfl_sync(0xffffffffu, lbase, 0);
    if (cls == c) lights[c * n_rows + lbase + __popc(ml & lt)] = make_int2(static_cast<int>(t), n);
  }
}

// v += the VEC floats at src + u * stride for u = 0 .. nu - 1, in unit order
// (the fp32 partial rows of a split token's units); the loads of eight units
// are issued together, then added in order.
template <int VEC>
__device__ __forceinline__ void sum_partials(const float* src, int64_t stride, int nu, float (&v)[VEC]) {
  constexpr int B = 8;
  for (int u0 = 0; u0 < nu; u0 += B) {
    float4 f[B][VEC / 4];
#pragma unroll
    for (int b = 0; b < B; ++b)
#pragma unroll
      for (int q = 0; q < VEC / 4; ++q)
        f[b][q] = u0 + b < nu ? __ldcg(reinterpret_cast<const float4*>(src + (u0 + b) * stride) + q)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int b = 0; b < B; ++b) {
      if (u0 + b >= nu) break;
#pragma unroll
      for (int q = 0; q < VEC / 4; ++q) {
        v[4 * q] += f[b][q].x;
        v[4 * q + 1] += f[b][q].y;
        v[4 * q + 2] += f[b][q].z;
        v[4 * q + 3] += f[b][q].w;
      }
    }
  }
}

// -------------------------------------------------------------- main kernel

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bounded wait that also gives up as soon as another warp of the CTA has.
__device__ __forceinline__ bool ud_wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int32_t* diag) {
  uint64_t t0 = 0;  // the clock is read only once a wait has lasted kWaitSpins tries
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31) == 0) {
      if (*abort_flag) return false;
      if ((i & (kWaitSpins - 1)) == 0) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        else if (now - t0 > kWaitNs) break;
      }
    }
  }
  *abort_flag = 1;
  if (diag) atomicOr(reinterpret_cast<int*>(diag + SGE_DIAG_FLAGS), SGE_FLAG_TIMEOUT);
  return false;
}

// Exclusive prefix of tile c's capped count, from the lane-distributed copy
// (tile b lives in lane b % 32, register b / 32).  All lanes must call it.
template <int NTR>
__device__ __forceinline__ int prefix_at(const int (&pre)[NTR], int c) {
  int v = 0;
#pragma unroll
  for (int r = 0; r < NTR; ++r) {
    const int x = __shfl_sync(0xffffffffu, pre[r], c & 31);
    if ((c >> 5) == r) v = x;
  }
  return v;
}

constexpr int kFirst = 1;  // chunk flags: first chunk of its job for this warp
constexpr int kLast = 2;   //              last chunk of its job for this warp
constexpr int kHasX = 4;   //              the x row leads the chunk's stream

// The main kernel: teams of kTeam warps, one job at a time per team, each
// warp streaming whole rows of its own entries through its own ring of
// p.slots slots (see the file comment).
template <bool BF16, int NTR, int NV>
__global__ void __launch_bounds__(UdLaunch<NV>::kWarps * 32, 1) ud_main_kernel(const UdParams p) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  using E = Elem<BF16>;
  constexpr int VEC = E::VEC;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int team = warp / kTeam, w = warp - team * kTeam;
  const int S = p.slots;
  uint8_t* ring = smem + warp * S * p.slot_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_full) + warp * S;
  uint8_t* tb = smem + p.off_team + team * p.team_bytes;
  Job* jobq = reinterpret_cast<Job*>(tb);  // [4] + a staging entry
  uint64_t* tbar = reinterpret_cast<uint64_t*>(tb + 5 * sizeof(Job));
  uint64_t* tfree = tbar + 1;  // the row buffer may be written again
  uint64_t* chain = tbar + 2;  // chain[w - 1]: warp w - 1 has added its partial row
  static_assert(5 * sizeof(Job) + 8 * (2 + kTeam - 1) <= kTeamHdr, "team header overlaps the row buffer");
  float* tbuf = reinterpret_cast<float*>(tb + kTeamHdr);  // the team's row buffer, d floats
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.off_abort);
  const bool leader = w == 0;
  const int pieces = p.row_bytes / 16;

  // the bytes of each half slot past the row stay zero for the whole kernel
  const int half = p.slot_bytes / 2;
  if (p.row_bytes < half) {
    for (int q = 0; q < 2 * S; ++q)
      for (int o = p.row_bytes + lane * 16; o < half; o += 32 * 16)
        *reinterpret_cast<uint4*>(ring + q * half + o) = make_uint4(0, 0, 0, 0);
  }
  if (lane == 0) {
    for (int q = 0; q < S; ++q) mbar_init(full + q, 1);
    if (leader) {
      mbar_init(tbar, kTeam);
      mbar_init(tfree, 1);
      for (int q = 0; q < kTeam - 1; ++q) mbar_init(chain + q, 1);
    }
  }
  if (threadIdx.x == 0) *abort_flag = 0;
  fence_mbar_init();
  __syncthreads();

  // y = 0 for tokens without stored entries: each warp takes an equal share
  // of the tokens; its stores drain while it starts its first job
  {
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * warps + warp;
    const int64_t ngw = static_cast<int64_t>(gridDim.x) * warps;
    const int64_t per = (p.n_rows + ngw - 1) / ngw;
    const int64_t t0 = gw * per, t1 = min(p.n_rows, t0 + per);
    for (int64_t tb = t0; tb < t1; tb += 32) {
      unsigned m = __ballot_sync(0xffffffffu, p.zero_empty && tb + lane < t1 && p.ntok[tb + lane] == 0);
      while (m) {
        const int i = __ffs(m) - 1;
        m &= m - 1;
        uint4* row = reinterpret_cast<uint4*>(static_cast<char*>(p.y) + (tb + i) * p.row_bytes);
        for (int pc = lane; pc < pieces; pc += 32) row[pc] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  const int n_units = *reinterpret_cast<volatile int*>(p.hdr + kHUnits);
  int n_light[kLightClasses];
#pragma unroll
  for (int c = 0; c < kLightClasses; ++c) n_light[c] = *reinterpret_cast<volatile int*>(p.hdr + kHLight + c);
  const int64_t rb = p.row_bytes, wl = p.w_ld;
  const char* xb = static_cast<const char*>(p.x);
  const char* ub = static_cast<const char*>(p.wu_t);
  const char* db = static_cast<const char*>(p.wd);

  // ---- team barrier (also publishes the leader's job-queue writes)
  uint32_t tpar = 0;
  auto team_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(tbar);
    const bool ok = ud_wait_or_abort(tbar, tpar, abort_flag, p.diag);
    tpar ^= 1;
    return ok;
  };

  // ---- jobs: the leader keeps the queue two jobs ahead of consumption; the
  // job after that is fetched early into a staging entry (jobq[4]) with
  // cp.async, so that no registers wait on its load.
  int pf_kind = 0;  // leader lane 0: 0 unit, 1 unsplit token, 2 none
  auto prefetch_job = [&]() {
    int k = atomicAdd(&p.hdr[kHCursor], 1);
    const uint32_t dst = smem_u32(jobq + 4);
    if (k < n_units) {
      pf_kind = 0;
      const char* src = reinterpret_cast<const char*>(p.units + k);
      asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
      asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(dst + 16), "l"(src + 16) : "memory");
    } else {
      k -= n_units;
      pf_kind = 2;
#pragma unroll
      for (int c = 0; c < kLightClasses; ++c) {
        if (pf_kind == 2 && k < n_light[c]) {
          pf_kind = 1;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst),
                       "l"(p.lights + c * p.n_rows + k) : "memory");
        }
        k -= n_light[c];
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  auto publish_job = [&](int at) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    Job j;
    if (pf_kind == 0) {
      j = jobq[4];
    } else {
      const int2 l = *reinterpret_cast<const int2*>(jobq + 4);
      j.t = pf_kind == 1 ? l.x : -1;
      j.e0 = 0;
      j.n = pf_kind == 1 ? l.y : 0;
      j.nu = 1;
      j.u = 0;
      j.base = -1;
      j.sid = -1;
      j.pad = 0;
    }
    jobq[at] = j;
  };
  if (leader && lane == 0) {
    prefetch_job();
    publish_job(0);
    prefetch_job();
    publish_job(1);
    prefetch_job();
  }
  bool ok = team_sync();

  // ---- entry resolution: this warp's entries of a job are w, w + kTeam, ...
  int rk = 0, rci = 0;  // job sequence number and next chunk of the job being resolved
  struct {
    int t, e0, n;
  } rj = {jobq[0].t, jobq[0].e0, jobq[0].n};
  auto own_count = [&](int n) { return n > w ? (n - w + kTeam - 1) / kTeam : 0; };
  int pre[NTR];
  auto load_prefix = [&](int t) {
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
  };
  if (rj.t >= 0) load_prefix(rj.t);
  // A chunk: token (-1: none), own entries in it (may be 0 when the job has
  // fewer entries than the team has warps), flags (bits 0..2) and the job
  // sequence number (the bits above); per
  // lane, for entry `lane`, the first column of its tile, its index in the
  // tile and its activation as loaded (raw bits).  The raw loads are first
  // used a chunk later, so their latency hides behind the current chunk.
  struct Chunk {
    int t, n, flags, jb, ji;
    uint32_t a;
  };
  auto resolve = [&](Chunk& c) {
    c.t = -1;
    c.n = 0;
    c.flags = 0;
    if (rj.t < 0) return;
    if (rci > 0 && rci * kChunk >= own_count(rj.n)) {
      ++rk;
      rj.t = jobq[rk & 3].t;
      rj.e0 = jobq[rk & 3].e0;
      rj.n = jobq[rk & 3].n;
      rci = 0;
      if (rj.t < 0) return;
      load_prefix(rj.t);
    }
    const int own = own_count(rj.n);
    c.t = rj.t;
    c.n = max(0, min(kChunk, own - rci * kChunk));
    c.flags = (rci == 0 ? kFirst : 0) | ((rci + 1) * kChunk >= own ? kLast : 0) |
              (rci == 0 && own > 0 ? kHasX : 0) | (rk << 3);
    const int e = rj.e0 + w + kTeam * (rci * kChunk + lane);
    int b = 0;
#pragma unroll
    for (int step = 16 * NTR; step > 0; step >>= 1) {
      const int cand = b + step;
      const int v = prefix_at<NTR>(pre, cand < p.nt ? cand : 0);
      if (cand < p.nt && v <= e) b = cand;
    }
    const int s = e - prefix_at<NTR>(pre, b);
    c.jb = b * p.tile;
    c.ji = 0;
    c.a = 0;
    if (lane < c.n) {
      const int64_t at = (static_cast<int64_t>(c.t) * p.nt + b) * p.cap + s;
      c.ji = clamp_index(__ldg(p.idx + at), p.tile);
      c.a = E::load_raw(p.val, at);
    }
    ++rci;
  };
  auto stream_len = [](const Chunk& c) {
    return c.t < 0 ? 0 : ((c.flags & kHasX) ? 1 : 0) + c.n;
  };
  Chunk cur, nxt;
  resolve(cur);
  resolve(nxt);

  // ---- this warp's ring: positions are the x row (first chunk of a job),
  // then one per entry of each chunk (its W_up row in the first half of the
  // slot, its W_down row in the second)
  uint32_t issued = 0, consumed = 0;
  int is = 0, cs = 0;   // slots of the next issue and the next consumption
  uint32_t cph = 0;     // phase parity of the slot being consumed
  int ich = 0, iq = 0;  // issuing in cur (0) or nxt (1), at position iq of its stream
  auto pump = [&]() {
    __syncwarp();
    while (true) {
      const int room = S - static_cast<int>(issued - consumed);
      if (room <= 0) break;
      const Chunk& c = ich ? nxt : cur;
      if (c.t < 0) break;
      const int len = stream_len(c);
      if (iq >= len) {
        if (ich == 0) {
          ich = 1;
          iq = 0;
          continue;
        }
        break;
      }
      const int m = min(room, len - iq);
      const int hx = (c.flags & kHasX) ? 1 : 0;
      const int q = iq + lane;
      // the column, kept in bounds even if a stored index is >= T
      const int jv = min(__shfl_sync(0xffffffffu, c.jb + c.ji, (q - hx) & 31), p.nt * p.tile - 1);
      if (lane < m) {
        int slot = is + lane;
        if (slot >= S) slot -= S;
        uint8_t* dst = ring + slot * p.slot_bytes;
        const uint32_t rb32 = static_cast<uint32_t>(p.row_bytes);
        // a W row slot's earlier contents were consumed by FMAs that have
        // issued, so its reads are complete; an x slot is fenced when read
        if (hx && q == 0) {
          mbar_arrive_expect_tx(full + slot, rb32);
          bulk_load(dst, xb + static_cast<int64_t>(c.t) * rb, rb32, full + slot);
        } else {
          mbar_arrive_expect_tx(full + slot, 2 * rb32);
          if (p.w_one) {
            bulk_load(dst, ub + static_cast<int64_t>(jv) * wl, 2 * rb32, full + slot);
          } else {
            bulk_load(dst, ub + static_cast<int64_t>(jv) * wl, rb32, full + slot);
            bulk_load(dst + half, db + static_cast<int64_t>(jv) * wl, rb32, full + slot);
          }
        }
      }
      issued += m;
      is += m;
      if (is >= S) is -= S;
      iq += m;
    }
  };
  // waits for the next position and gives its slot's shared-memory address
  auto acquire = [&](uint32_t& a) -> bool {
    if (!ud_wait_or_abort(full + cs, cph, abort_flag, p.diag)) return false;
    a = smem_u32(ring + cs * p.slot_bytes);
    return true;
  };
  // piece k of this lane; past the end of the row a slot holds zeros, which
  // the copies never overwrite, so no bounds test is needed
  auto piece = [&](uint32_t a, int k) -> uint4 { return lds128(a + (lane + 32 * k) * 16); };
  // the warp is done with the slot; the pump may refill it
  auto release = [&]() {
    __syncwarp();
    ++consumed;
    if (++cs == S) {
      cs = 0;
      cph ^= 1;
    }
  };

  // ---- consume chunks
  uint4 xr[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) xr[k] = make_uint4(0, 0, 0, 0);
  float acc[NV][VEC];
  const int rq = (pieces + kTeam - 1) / kTeam;  // pieces each warp reduces at a job's end
  const int q0 = w * rq, q1 = min(pieces, q0 + rq);
  while (ok && cur.t >= 0) {
    pump();
    if (cur.flags & kFirst) {
#pragma unroll
      for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
    }
    if (cur.flags & kHasX) {
      uint32_t a;
      if (!(ok = acquire(a))) break;
#pragma unroll
      for (int k = 0; k < NV; ++k) xr[k] = piece(a, k);
      // x stays unused for a while: order these reads before the slot's
      // next copy
      fence_proxy_async_smem();
      release();
      pump();
    }
    // each entry: u = x . W_up[:, j] reduced over the lanes, h = a * u
    // rounded as the down projection uses it, y += h * W_down[j]
    for (int e = 0; e < cur.n; ++e) {
      const float ae = E::from_raw(__shfl_sync(0xffffffffu, cur.a, e & 31));
      uint32_t a;
      if (!(ok = acquire(a))) break;
      // eight independent accumulator chains
      float s[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int k = 0; k < NV; ++k) E::dot2(xr[k], piece(a, k), s[2 * (k & 3)], s[2 * (k & 3) + 1]);
      float u = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
      const typename E::HType h = E::h_of(ae * u);
#pragma unroll
      for (int k = 0; k < NV; ++k) E::axpy(h, piece(a + half, k), acc[k]);
      release();
      pump();
    }
    if (!ok) break;
    if (cur.flags & kLast) {
      const int ck = cur.flags >> 3;  // the job's sequence number
      // ---- job done: the warps add their partial rows into the team's row
      // buffer one after the other (warp order), each waiting only for its
      // predecessor; the last one stores the sum.  Warp 0 queues the job
      // after next before it hands the buffer on.
      uint64_t* wait_bar = w == 0 ? tfree : chain + (w - 1);
      const uint32_t wait_par = w == 0 ? ((ck - 1) & 1) : (ck & 1);
      if ((w > 0 || ck > 0) && !(ok = ud_wait_or_abort(wait_bar, wait_par, abort_flag, p.diag))) break;
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int pc = lane + 32 * k;
        if (pc < pieces) {
          float4* b4 = reinterpret_cast<float4*>(tbuf + pc * VEC);
#pragma unroll
          for (int q = 0; q < VEC / 4; ++q) {
            float4 v = make_float4(acc[k][4 * q], acc[k][4 * q + 1], acc[k][4 * q + 2], acc[k][4 * q + 3]);
            if (w > 0) {
              const float4 o = b4[q];
              v.x = o.x + v.x;
              v.y = o.y + v.y;
              v.z = o.z + v.z;
              v.w = o.w + v.w;
            }
            if (w < kTeam - 1) {
              b4[q] = v;
            } else {
              acc[k][4 * q] = v.x;
              acc[k][4 * q + 1] = v.y;
              acc[k][4 * q + 2] = v.z;
              acc[k][4 * q + 3] = v.w;
            }
          }
        }
      }
      if (w < kTeam - 1) {
        if (leader && lane == 0) publish_job((ck + 2) & 3);
        __syncwarp();
        if (lane == 0) mbar_arrive(chain + w);
        if (leader && lane == 0) prefetch_job();
      }
      if (w == kTeam - 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(tfree);  // the buffer has been read
        const Job jb = jobq[ck & 3];
        char* yrow = static_cast<char*>(p.y) + static_cast<int64_t>(jb.t) * rb;
        if (jb.nu <= 1) {
#pragma unroll
          for (int k = 0; k < NV; ++k) {
            const int pc = lane + 32 * k;
            if (pc < pieces) reinterpret_cast<uint4*>(yrow)[pc] = E::pack(acc[k]);
          }
        } else {
          // a unit of a split token: its partial goes to the pool; the team
          // that completes the token's last unit sums the partials in unit order
          float* mine = p.pool + static_cast<int64_t>(jb.base + jb.u) * p.d;
#pragma unroll
          for (int k = 0; k < NV; ++k) {
            const int pc = lane + 32 * k;
            if (pc < pieces)
#pragma unroll
              for (int q = 0; q < VEC / 4; ++q)
                reinterpret_cast<float4*>(mine + pc * VEC)[q] =
                    make_float4(acc[k][4 * q], acc[k][4 * q + 1], acc[k][4 * q + 2], acc[k][4 * q + 3]);
          }
          __threadfence();
          __syncwarp();
          int last = 0;
          if (lane == 0) last = atomicAdd(p.done + jb.sid, 1) == jb.nu - 1;
          if (__shfl_sync(0xffffffffu, last, 0)) {
            __threadfence();
#pragma unroll
            for (int k = 0; k < NV; ++k) {
              const int pc = lane + 32 * k;
              if (pc < pieces) {
                float v[VEC];
#pragma unroll
                for (int q = 0; q < VEC; ++q) v[q] = 0.0f;
                for (int u = 0; u < jb.nu; ++u) {
                  const float4* src =
                      reinterpret_cast<const float4*>(p.pool + static_cast<int64_t>(jb.base + u) * p.d + pc * VEC);
#pragma unroll
                  for (int q = 0; q < VEC / 4; ++q) {
                    const float4 f = __ldcg(src + q);
                    v[4 * q] += f.x;
                    v[4 * q + 1] += f.y;
                    v[4 * q + 2] += f.z;
                    v[4 * q + 3] += f.w;
                  }
                }
                reinterpret_cast<uint4*>(yrow)[pc] = E::pack(v);
              }
            }
          }
        }
      }
    }
    // the next chunk becomes current; the issuer moves with it
    cur = nxt;
    if (ich == 1) {
      ich = 0;
    } else {
      iq = 0;
    }
    resolve(nxt);
  }
  // Copies still in flight (only after a give-up) land before the CTA exits.
  while (consumed != issued) {
    mbar_wait(full + cs, cph, p.diag);
    ++consumed;
    if (++cs == S) {
      cs = 0;
      cph ^= 1;
    }
  }
}

// ---------------------------------------------------------- small batches
//
// With few tokens (decode-sized batches) the persistent kernel's per-warp row
// streams are short and its latency chain (three launches, the job queue, a
// ring a few rows deep) dominates.  The small-batch path splits every token
// into units of E entries (E = 8, doubled until there is at most one unit
// per CTA and the split tokens' partial outputs fit the pool), gives each
// unit one CTA of kSmWarps warps and each
// warp one entry at a time: the warp loads x[t], the W_up row and the W_down
// row with plain 16-byte loads issued together, so a unit costs one memory
// round trip.  The warps' partial rows are summed in warp order in shared
// memory; a token of one unit stores y directly, the others store fp32
// partials in the pool and the CTA that completes a token's last unit (a
// counter per token) sums them in unit order.  Results do not depend on
// scheduling.

constexpr int kSmallTokens = 64;   // tokens at most for the small-batch path (measured: it
                                   // loses to the persistent kernel from about 128 tokens)
constexpr int kSmWarps = 8;        // warps per CTA (the smallest unit length)

// Exclusive prefix sum over the kSmallTokens threads of one CTA; returns the
// exclusive value of this thread and writes the total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int w = 0; w < kSmallTokens / 32; ++w) {
      const int c = tmp[w];
      tmp[w] = s;
      s += c;
    }
    tmp[kSmallTokens / 32] = s;
  }
  __syncthreads();
  const int r = tmp[warp] + incl - v;
  *total = tmp[kSmallTokens / 32];
  __syncthreads();
  return r;
}

// Entries per token, the unit length E, every token's first unit (ufirst,
// n_rows + 1 entries) and first pool slot (pbase), zeroed completion
// counters.  One CTA of kSmallTokens threads, a thread per token.
static __global__ void __launch_bounds__(kSmallTokens) us_plan_kernel(const uint8_t* __restrict__ count,
                                                              int64_t n_rows, int nt, int cap,
                                                              int64_t pool_slots, int n_cta, int* hdr,
                                                              int* __restrict__ ntok,
                                                              int* __restrict__ ufirst,
                                                              int* __restrict__ pbase,
                                                              int* __restrict__ done) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  __shared__ int tmp[kSmallTokens / 32 + 1];
  const int t = threadIdx.x;
  int n = 0;
  if (t < n_rows) {
    const uint8_t* c = count + static_cast<int64_t>(t) * nt;
    if ((nt & 15) == 0 && (reinterpret_cast<uintptr_t>(count) & 15) == 0) {
      // 16 counts per load, all loads in flight together
      for (int b = 0; b < nt; b += 16) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(c + b));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int k = 0; k < 4; ++k) n += min(static_cast<int>((w[q] >> (8 * k)) & 255u), cap);
      }
    } else {
      for (int b = 0; b < nt; ++b) n += min(static_cast<int>(__ldg(c + b)), cap);
    }
    ntok[t] = n;
    done[t] = 0;
  }
  // the smallest E (kSmWarps times a power of two) that gives at most one
  // unit per CTA of the launch and whose split tokens fit the pool: each
  // unit pays a fixed chain of dependent round trips and a cross-warp sum,
  // so fewer, longer units are faster once every CTA has one (64 tokens of
  // the 1B workload: E = 8 -> 32 took the kernel from 39.6 to 23.7 us)
  int E = kSmWarps;
  for (;;) {
    const int nu = t < n_rows ? max(1, (n + E - 1) / E) : 0;
    int split = 0, all = 0;
    block_exclusive_scan(nu > 1 ? nu : 0, tmp, &split);
    block_exclusive_scan(nu, tmp, &all);
    if ((split <= pool_slots && all <= n_cta) || E >= (1 << 24)) break;
    E *= 2;
  }
  const int nu = t < n_rows ? max(1, (n + E - 1) / E) : 0;
  int units = 0, split = 0;
  const int uf = block_exclusive_scan(nu, tmp, &units);
  const int pb = block_exclusive_scan(nu > 1 ? nu : 0, tmp, &split);
  if (t < n_rows) {
    ufirst[t] = uf;
    pbase[t] = pb;
  }
  if (t == 0) {
    ufirst[n_rows] = units;
    hdr[kHUnit] = E;
    hdr[kHUnits] = units;
    hdr[kHOverflow] = split > pool_slots ? 1 : 0;
  }
}

struct UsParams {
  const void* x;
  const uint8_t* count;
  const uint8_t* idx;
  const void* val;
  const void* wu_t;
  const void* wd;
  void* y;
  const int* hdr;
  const int* ntok;
  const int* ufirst;
  const int* pbase;
  int* done;
  float* pool;
  int64_t n_rows;
  int d;
  int nt;
  int tile;
  int cap;
  int pieces;    // 16-byte pieces per row
  int64_t w_ld;  // row stride of wu_t and wd in bytes
};

// One CTA per unit (grid-stride over the units), kSmWarps warps; NV pieces
// of a row per lane.
template <bool BF16, int NTR, int NV>
__global__ void __launch_bounds__(kSmWarps * 32, 1) us_main_kernel(const UsParams p) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  using E = Elem<BF16>;
  constexpr int VEC = E::VEC;
  extern __shared__ __align__(1024) uint8_t smem[];
  float* red = reinterpret_cast<float*>(smem);  // [kSmWarps][d]
  int* uf = reinterpret_cast<int*>(smem + kSmWarps * p.d * 4);  // [n_rows + 1]
  __shared__ int last_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i <= p.n_rows; i += blockDim.x) uf[i] = p.ufirst[i];
  __syncthreads();
  const int EU = p.hdr[kHUnit];
  const int n_units = p.hdr[kHUnits];
  const int64_t rb = static_cast<int64_t>(p.pieces) * 16;
  for (int k = blockIdx.x; k < n_units; k += gridDim.x) {
    // the unit's token: the last t with uf[t] <= k
    int lo = 0, hi = static_cast<int>(p.n_rows) - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (uf[mid] <= k) lo = mid; else hi = mid - 1;
    }
    const int t = lo;
    const int u = k - uf[t];
    const int nu = uf[t + 1] - uf[t];
    const int n = p.ntok[t];
    const int e_end = min(n, (u + 1) * EU);
    float acc[NV][VEC];
#pragma unroll
    for (int q = 0; q < NV; ++q)
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[q][v] = 0.0f;
    int e = u * EU + warp;
    if (e < e_end) {
      // exclusive prefix of the token's capped tile counts (tile b: lane b % 32, register b / 32)
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
      uint4 xr[NV];
      const uint4* xrow = reinterpret_cast<const uint4*>(static_cast<const char*>(p.x) + t * rb);
#pragma unroll
      for (int q = 0; q < NV; ++q) {
        const int pc = lane + 32 * q;
        xr[q] = pc < p.pieces ? __ldg(xrow + pc) : make_uint4(0, 0, 0, 0);
      }
      // this warp's entries e, e + kSmWarps, ...: 32 resolved at a time, one per lane
      for (; e < e_end; e += 32 * kSmWarps) {
        const int my = e + kSmWarps * lane;
        const int er = my < e_end ? my : e;
        int b = 0;
#pragma unroll
        for (int step = 16 * NTR; step > 0; step >>= 1) {
          const int cand = b + step;
          const int v = prefix_at<NTR>(pre, cand < p.nt ? cand : 0);
          if (cand < p.nt && v <= er) b = cand;
        }
        const int s = er - prefix_at<NTR>(pre, b);
        int j = 0;
        float a = 0.0f;
        if (my < e_end) {
          const int64_t at = (static_cast<int64_t>(t) * p.nt + b) * p.cap + s;
          j = b * p.tile + clamp_index(__ldg(p.idx + at), p.tile);
          a = E::load_val(p.val, at);
        }
        const int cnt = min(32, (e_end - e + kSmWarps - 1) / kSmWarps);
        for (int i = 0; i < cnt; ++i) {
          const int ji = __shfl_sync(0xffffffffu, j, i);
          const float ai = __shfl_sync(0xffffffffu, a, i);
          const uint4* ur = reinterpret_cast<const uint4*>(static_cast<const char*>(p.wu_t) + ji * p.w_ld);
          const uint4* dr = reinterpret_cast<const uint4*>(static_cast<const char*>(p.wd) + ji * p.w_ld);
          uint4 wu[NV], wdv[NV];
#pragma unroll
          for (int q = 0; q < NV; ++q) {
            const int pc = lane + 32 * q;
            wu[q] = pc < p.pieces ? __ldg(ur + pc) : make_uint4(0, 0, 0, 0);
            wdv[q] = pc < p.pieces ? __ldg(dr + pc) : make_uint4(0, 0, 0, 0);
          }
          float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int q = 0; q < NV; ++q) s4[q & 3] = E::dot(xr[q], wu[q], s4[q & 3]);
          float dot = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          const typename E::HType h = E::h_of(ai * dot);
#pragma unroll
          for (int q = 0; q < NV; ++q) E::axpy(h, wdv[q], acc[q]);
        }
      }
    }
    // the warps' partial rows, summed in warp order
    float* mine = red + warp * p.d;
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int pc = lane + 32 * q;
      if (pc < p.pieces)
#pragma unroll
        for (int v = 0; v < VEC / 4; ++v)
          reinterpret_cast<float4*>(mine + pc * VEC)[v] =
              make_float4(acc[q][4 * v], acc[q][4 * v + 1], acc[q][4 * v + 2], acc[q][4 * v + 3]);
    }
    __syncthreads();
    char* yrow = static_cast<char*>(p.y) + static_cast<int64_t>(t) * rb;
    float* slot = nu > 1 ? p.pool + static_cast<int64_t>(p.pbase[t] + u) * p.d : nullptr;
    for (int pc = threadIdx.x; pc < p.pieces; pc += blockDim.x) {
      float v[VEC];
#pragma unroll
      for (int q = 0; q < VEC; ++q) v[q] = 0.0f;
      for (int w = 0; w < kSmWarps; ++w)
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q) {
          const float4 f = reinterpret_cast<const float4*>(red + w * p.d + pc * VEC)[q];
          v[4 * q] += f.x;
          v[4 * q + 1] += f.y;
          v[4 * q + 2] += f.z;
          v[4 * q + 3] += f.w;
        }
      if (nu == 1) {
        reinterpret_cast<uint4*>(yrow)[pc] = E::pack(v);
      } else {
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q)
          reinterpret_cast<float4*>(slot + pc * VEC)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
    }
    if (nu > 1) {
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) last_flag = atomicAdd(p.done + t, 1) == nu - 1;
      __syncthreads();
      if (last_flag) {
        __threadfence();
        const float* base = p.pool + static_cast<int64_t>(p.pbase[t]) * p.d;
        for (int pc = threadIdx.x; pc < p.pieces; pc += blockDim.x) {
          float v[VEC];
#pragma unroll
          for (int q = 0; q < VEC; ++q) v[q] = 0.0f;
          sum_partials<VEC>(base + pc * VEC, p.d, nu, v);
          reinterpret_cast<uint4*>(yrow)[pc] = E::pack(v);
        }
      }
    }
    __syncthreads();  // red is written again by the next unit
  }
}

template <bool BF16, int NTR, int NV>
static int launch_small(const UsParams& prm, int smem, int grid, cudaStream_t st) {
  auto kern = us_main_kernel<BF16, NTR, NV>;
  const int rc = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (rc) return rc;
  return launch_pdl(kern, dim3(grid), dim3(kSmWarps * 32), smem, st, "twell_fused_up_down (small batch)", prm);
}

template <bool BF16, int NV>
static int small_ntr(const UsParams& prm, int smem, int grid, cudaStream_t st) {
  if (prm.nt <= 32) return launch_small<BF16, 1, NV>(prm, smem, grid, st);
  if (prm.nt <= 64) return launch_small<BF16, 2, NV>(prm, smem, grid, st);
  if (prm.nt <= 128) return launch_small<BF16, 4, NV>(prm, smem, grid, st);
  return launch_small<BF16, 8, NV>(prm, smem, grid, st);
}

template <bool BF16>
static int small_nv(const UsParams& prm, int nv, int smem, int grid, cudaStream_t st) {
  switch (nv) {
    case 2: return small_ntr<BF16, 2>(prm, smem, grid, st);
    case 4: return small_ntr<BF16, 4>(prm, smem, grid, st);
    default: return small_ntr<BF16, 8>(prm, smem, grid, st);
  }
}

// ------------------------------------------------------------------ host

// Teams per CTA, ring depth and shared-memory layout for rows of
// p.row_bytes with nv pieces per lane; false if the rows are too long.
static bool make_geometry(UdParams& p, int nv, int* smem_bytes) {
  int warps = warps_for_nv(nv);
  p.slot_bytes = 2 * nv * 512;
  p.team_bytes = kTeamHdr + ((p.d * 4 + 15) & ~15);
  for (;; warps -= kTeam) {
    if (warps < kTeam) return false;
    p.teams = warps / kTeam;
    const int fixed = p.teams * p.team_bytes + 16 + 16;
    int slots = (kSmemBudget - fixed) / (warps * (p.slot_bytes + 8));
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots < 2) continue;  // one slot in flight while the other is read
    p.slots = slots;
    p.off_full = warps * slots * p.slot_bytes;
    p.off_team = (p.off_full + warps * slots * 8 + 15) & ~15;
    p.off_abort = p.off_team + p.teams * p.team_bytes;
    *smem_bytes = p.off_abort + 16;
    return *smem_bytes <= kSmemBudget;
  }
}

template <bool BF16, int NTR, int NV>
static int launch_main(const UdParams& prm, int smem, int grid, cudaStream_t st) {
  auto kern = ud_main_kernel<BF16, NTR, NV>;
  const int rc = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (rc) return rc;
  return launch_pdl(kern, dim3(grid), dim3(prm.teams * kTeam * 32), smem, st, "twell_fused_up_down", prm);
}

template <bool BF16, int NV>
static int dispatch_ntr(const UdParams& prm, int smem, int grid, cudaStream_t st) {
  if (prm.nt <= 32) return launch_main<BF16, 1, NV>(prm, smem, grid, st);
  if (prm.nt <= 64) return launch_main<BF16, 2, NV>(prm, smem, grid, st);
  if (prm.nt <= 128) return launch_main<BF16, 4, NV>(prm, smem, grid, st);
  return launch_main<BF16, 8, NV>(prm, smem, grid, st);
}

template <bool BF16>
static int dispatch_main(const UdParams& prm, int nv, int smem, int grid, cudaStream_t st) {
  switch (nv) {
    case 2: return dispatch_ntr<BF16, 2>(prm, smem, grid, st);
    case 4: return dispatch_ntr<BF16, 4>(prm, smem, grid, st);
    case 8: return dispatch_ntr<BF16, 8>(prm, smem, grid, st);
    case 12: return dispatch_ntr<BF16, 12>(prm, smem, grid, st);
    default: return dispatch_ntr<BF16, 16>(prm, smem, grid, st);
  }
}

// The small-batch path: its planning kernel and its main kernel.
static int run_small(const UdParams& prm, const WsLayout& L, uint8_t* ws, int64_t pool_slots, int nv,
                     bool bf16, cudaStream_t st) {
  UsParams up;
  up.x = prm.x;
  up.count = prm.count;
  up.idx = prm.idx;
  up.val = prm.val;
  up.wu_t = prm.wu_t;
  up.wd = prm.wd;
  up.y = prm.y;
  up.hdr = prm.hdr;
  up.ntok = prm.ntok;
  int* ufirst = reinterpret_cast<int*>(ws + L.lights);  // n + 1 words, then pbase (n words)
  int* pbase = ufirst + prm.n_rows + 1;
  up.ufirst = ufirst;
  up.pbase = pbase;
  up.done = prm.done;
  up.pool = prm.pool;
  up.n_rows = prm.n_rows;
  up.d = prm.d;
  up.nt = prm.nt;
  up.tile = prm.tile;
  up.cap = prm.cap;
  up.pieces = prm.row_bytes / 16;
  up.w_ld = prm.w_ld;
  const int rc = launch_pdl(us_plan_kernel, dim3(1), dim3(kSmallTokens), 0, st,
                            "twell_fused_up_down (small-batch plan)", prm.count, prm.n_rows, prm.nt, prm.cap,
                            pool_slots, sm_count(), prm.hdr, const_cast<int*>(prm.ntok), ufirst, pbase, prm.done);
  if (rc) return rc;
  const int smem = (kSmWarps * prm.d * 4 + 4 * static_cast<int>(prm.n_rows + 1) + 15) & ~15;
  return bf16 ? small_nv<true>(up, nv, smem, sm_count(), st) : small_nv<false>(up, nv, smem, sm_count(), st);
}

// Host-side set-up of one call of the fused kernels: parameters, workspace
// layout, kernel geometry, and which path runs.
struct FusedCall {
  UdParams prm;
  WsLayout L{0, 8, 0};
  uint8_t* ws = nullptr;
  long long* blk = nullptr;
  int64_t pool_slots = 0;
  int64_t nblk = 0;
  int nv = 0, smem = 0, grid = 0;
  bool bf16 = true;
  bool small = false;  // the small-batch path (at most kSmallTokens tokens)
};

static int fused_prepare(FusedCall& c, const char* name, const void* x, const uint8_t* count,
                         const uint8_t* idx, const void* val, const void* wu_t, const void* wd,
                         int64_t ldw, void* y, int64_t n_tokens, int64_t d_model, int64_t d_ff,
                         int dtype, int tile, int cap, void* workspace, int64_t pool_slots,
                         int32_t* diag, bool allow_small) {
  if (dtype != SGE_BF16 && dtype != SGE_F32) return fail(SGE_ERR_UNSUPPORTED, "%s: dtype %d", name, dtype);
  const int64_t esz = dtype == SGE_BF16 ? 2 : 4;
  UdParams& prm = c.prm;
  prm.x = x;
  prm.count = count;
  prm.idx = idx;
  prm.val = val;
  prm.wu_t = wu_t;
  prm.wd = wd;
  prm.y = y;
  c.L = WsLayout(n_tokens, d_model, pool_slots);
  c.ws = static_cast<uint8_t*>(workspace);
  c.pool_slots = pool_slots;
  c.bf16 = dtype == SGE_BF16;
  prm.hdr = reinterpret_cast<int*>(c.ws);
  c.blk = reinterpret_cast<long long*>(c.ws + c.L.blk);
  prm.ntok = reinterpret_cast<const int*>(c.ws + c.L.ntok);
  prm.lights = reinterpret_cast<const int2*>(c.ws + c.L.lights);
  prm.units = reinterpret_cast<const Job*>(c.ws + c.L.units);
  prm.done = reinterpret_cast<int*>(c.ws + c.L.done);
  prm.pool = reinterpret_cast<float*>(c.ws + c.L.pool);
  prm.diag = diag;
  prm.n_rows = n_tokens;
  prm.d = static_cast<int>(d_model);
  prm.nt = static_cast<int>(d_ff / tile);
  prm.tile = tile;
  prm.cap = cap;
  prm.row_bytes = static_cast<int>(d_model * esz);
  prm.w_ld = ldw * esz;
  prm.zero_empty = 1;
  c.nv = nv_for(prm.row_bytes);
  if (!c.nv || !make_geometry(prm, c.nv, &c.smem))
    return fail(SGE_ERR_UNSUPPORTED, "%s: d_model too large: rows of %d bytes (max 8192)", name, prm.row_bytes);
  // one copy per entry brings both rows when each wd row directly follows
  // its wu_t row and a row fills half a slot exactly
  prm.w_one = static_cast<const char*>(wd) == static_cast<const char*>(wu_t) + prm.row_bytes &&
              prm.w_ld == 2 * static_cast<int64_t>(prm.row_bytes) && 2 * prm.row_bytes == prm.slot_bytes;
  if (prm.nt > 256)
    return fail(SGE_ERR_UNSUPPORTED, "%s: %d TwELL tiles per row (max 256)", name, prm.nt);
  c.small = allow_small && n_tokens <= kSmallTokens && c.nv <= 8 && pool_slots >= n_tokens;
  // every SM gets a CTA (small batches split their tokens into more units)
  int64_t grid = sm_count();
  if (grid > kMaxCtas) grid = kMaxCtas;
  c.grid = static_cast<int>(grid);
  c.nblk = (n_tokens + 255) / 256;
  return SGE_OK;
}

// The persistent path's planning launches: entries per token (and, for a
// routed call, the heavy tokens' ranks and the spill list), then the job
// lists.
static int fused_launch_plan(const FusedCall& c, const RouteArgs& route, cudaStream_t st) {
  const UdParams& prm = c.prm;
  int rc = launch_pdl(ud_count_kernel, dim3(static_cast<unsigned>(c.nblk)), dim3(256), 0, st,
                      "fused up/down (count)", prm.count, prm.n_rows, prm.nt, prm.cap,
                      const_cast<int*>(prm.ntok), c.blk, prm.hdr, route);
  if (rc) return rc;
  return launch_pdl(ud_jobs_kernel, dim3(static_cast<unsigned>(c.nblk)), dim3(256), 0, st,
                    "fused up/down (jobs)", const_cast<int*>(prm.ntok), prm.n_rows, c.blk, c.nblk,
                    static_cast<int64_t>(c.grid) * prm.teams, prm.hdr, const_cast<int2*>(prm.lights),
                    const_cast<Job*>(prm.units), prm.done, c.pool_slots, route);
}

static int fused_launch_main(const FusedCall& c, cudaStream_t st) {
  return c.bf16 ? dispatch_main<true>(c.prm, c.nv, c.smem, c.grid, st)
                : dispatch_main<false>(c.prm, c.nv, c.smem, c.grid, st);
}

// Planning kernels and the main kernel (or the small-batch path), shared by
// the workspace and the allocation-free entry points.
static int run_fused(const char* name, const void* x, const uint8_t* count, const uint8_t* idx,
                     const void* val, const void* wu_t, const void* wd, int64_t ldw, void* y, int64_t n_tokens,
                     int64_t d_model, int64_t d_ff, int dtype, int tile, int cap, void* workspace,
                     int64_t pool_slots, int32_t* diag, cudaStream_t st) {
  FusedCall c;
  int rc = fused_prepare(c, name, x, count, idx, val, wu_t, wd, ldw, y, n_tokens, d_model, d_ff, dtype,
                         tile, cap, workspace, pool_slots, diag, true);
  if (rc) return rc;
  if (c.small) return run_small(c.prm, c.L, c.ws, pool_slots, c.nv, c.bf16, st);
  if ((rc = fused_launch_plan(c, no_route(), st))) return rc;
  return fused_launch_main(c, st);
}

static int check_args(const char* name, int64_t n_tokens, int64_t d_model, int64_t d_ff, int64_t ldw,
                      int tile, int cap) {
  if (n_tokens < 0 || d_model < 1 || d_ff < 1) return fail(SGE_ERR_ARG, "%s: bad sizes", name);
  if (d_model % 8) return fail(SGE_ERR_ARG, "%s: d_model %% 8 != 0", name);
  if (ldw < d_model || ldw % 8 || ldw >= (1LL << 40))
    return fail(SGE_ERR_ARG, "%s: ldw %lld must be a multiple of 8 and >= d_model", name, (long long)ldw);
  if (tile < 1 || tile > 255 || d_ff % tile)
    return fail(SGE_ERR_ARG, "%s: tile must divide d_ff and be <= 255", name);
  if (cap < 1 || cap > tile) return fail(SGE_ERR_ARG, "%s: cap outside [1, tile]", name);
  if (d_ff >= (1LL << 31) || n_tokens >= (1LL << 31))
    return fail(SGE_ERR_UNSUPPORTED, "%s: size beyond the supported range", name);
  return SGE_OK;
}

}  // namespace sge
