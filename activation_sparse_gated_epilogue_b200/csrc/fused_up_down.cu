// Fused up and down projections over the TwELL nonzeros.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 02, last paragraph: one custom kernel performs the up and the down
// projection in a single traversal, fusing the two products so that the
// intermediate h is never written to global memory.  For every stored entry
// (t, j, a) of the TwELL gate activations:
//     u = x[t] . W_up[:, j]      h = a * u      y[t] += h * W_down[j, :]
//
// Design (one CTA per token; the hardware block scheduler balances the
// heavy-tailed per-token work across SMs):
//   * the token's d-vector is split across the CTA's threads in 16-byte
//     vectors, so every thread holds a few elements of x[t] and of the fp32
//     y[t] accumulator in registers (small footprint: several CTAs per SM);
//   * the token's entries are gathered from TwELL into a shared-memory list
//     (in chunks of at most kMaxEntries, in ascending column order);
//   * phase U: for each entry, every thread loads its 16-byte slice of row j
//     of W_up (8 entries in flight per thread), forms its partial dot product
//     with exact bf16 x bf16 products accumulated in fp32, the warp reduces 8
//     entries at once with a halving shuffle tree, and the per-warp partials
//     go to shared memory;
//   * h_e = a_e * sum of the per-warp partials (fixed order);
//   * phase D: every thread streams its slice of row j of W_down and
//     accumulates h_e * W_down[j] into its y registers.
// h lives only in shared memory.  No atomics on data: deterministic results.
#include "sge_host.h"
#include "sge_common.cuh"

namespace sge {

constexpr int kMaxEntries = 512;  // entries per chunk held in shared memory
constexpr int kUnroll = 8;        // entries per reduction group
constexpr int kMaxTiles = 512;    // TwELL tiles per chunk

template <bool BF16>
struct Elem;

template <>
struct Elem<true> {
  static constexpr int VEC = 8;  // elements per 16-byte vector
  using Acc = float;
  // partial += sum_k x_k * w_k with exact products (fma.rn.f32.bf16)
  __device__ __forceinline__ static float dot(const uint4& x, const uint4& w, float acc) {
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
          "mov.b32 {xl, xh}, %1;\n\t"
          "mov.b32 {wl, wh}, %2;\n\t"
          "fma.rn.f32.bf16 %0, xl, wl, %0;\n\t"
          "fma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
          : "+f"(acc)
          : "r"(xs[i]), "r"(ws[i]));
    return acc;
  }
  // y += h * w with h already rounded to bf16 (hb), exact products
  __device__ __forceinline__ static void axpy(uint16_t hb, const uint4& w, float (&y)[8]) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm("{\n\t.reg .b16 wl, wh;\n\t"
          "mov.b32 {wl, wh}, %2;\n\t"
          "fma.rn.f32.bf16 %0, %3, wl, %0;\n\t"
          "fma.rn.f32.bf16 %1, %3, wh, %1;\n\t}"
          : "+f"(y[2 * i]), "+f"(y[2 * i + 1])
          : "r"(ws[i]), "h"(hb));
  }
  using HType = uint16_t;
  __device__ __forceinline__ static HType h_of(float h) { return f32_to_bf16_bits(h); }
  __device__ __forceinline__ static float load_val(const void* p, int64_t i) {
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16);
  }
  __device__ __forceinline__ static uint4 pack(const float (&o)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = static_cast<uint32_t>(f32_to_bf16_bits(o[2 * i])) |
             (static_cast<uint32_t>(f32_to_bf16_bits(o[2 * i + 1])) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

template <>
struct Elem<false> {
  static constexpr int VEC = 4;
  __device__ __forceinline__ static float dot(const uint4& x, const uint4& w, float acc) {
    acc = fmaf(__uint_as_float(x.x), __uint_as_float(w.x), acc);
    acc = fmaf(__uint_as_float(x.y), __uint_as_float(w.y), acc);
    acc = fmaf(__uint_as_float(x.z), __uint_as_float(w.z), acc);
    acc = fmaf(__uint_as_float(x.w), __uint_as_float(w.w), acc);
    return acc;
  }
  __device__ __forceinline__ static void axpy(float h, const uint4& w, float (&y)[4]) {
    y[0] = fmaf(h, __uint_as_float(w.x), y[0]);
    y[1] = fmaf(h, __uint_as_float(w.y), y[1]);
    y[2] = fmaf(h, __uint_as_float(w.z), y[2]);
    y[3] = fmaf(h, __uint_as_float(w.w), y[3]);
  }
  using HType = float;
  __device__ __forceinline__ static HType h_of(float h) { return h; }
  __device__ __forceinline__ static float load_val(const void* p, int64_t i) {
    return static_cast<const float*>(p)[i];
  }
  __device__ __forceinline__ static uint4 pack(const float (&o)[4]) {
    return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                      __float_as_uint(o[3]));
  }
};

// Sum of v[0..7] over the 32 lanes of a warp with 5 + 4 shuffles: after the
// call, lane l holds the total of entry (l >> 2) & 7 (valid in every lane).
__device__ __forceinline__ float warp_reduce8(float (&v)[8], int lane) {
  // xor 16: keep 4 of 8 (upper half of the warp keeps entries 4..7)
  const bool hi16 = lane & 16;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float send = hi16 ? v[k] : v[k + 4];
    const float keep = hi16 ? v[k + 4] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  const bool hi8 = lane & 8;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float send = hi8 ? v[k] : v[k + 2];
    const float keep = hi8 ? v[k + 2] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const bool hi4 = lane & 4;
  {
    const float send = hi4 ? v[0] : v[1];
    const float keep = hi4 ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  float s = v[0];
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  // entry held: bit4 selects +4, bit3 selects +2, bit2 selects +1
  return s;
}

__device__ __forceinline__ int reduce8_entry(int lane) {
  return ((lane & 16) ? 4 : 0) + ((lane & 8) ? 2 : 0) + ((lane & 4) ? 1 : 0);
}

template <int THREADS, int NV, bool BF16>
__global__ void __launch_bounds__(THREADS, THREADS == 256 ? 2 : (NV == 1 ? 6 : (NV == 2 ? 5 : (NV == 3 ? 4 : 3))))
    fused_up_down_kernel(const void* __restrict__ x, const uint8_t* __restrict__ count,
                         const uint8_t* __restrict__ idx, const void* __restrict__ val,
                         const void* __restrict__ wu_t, const void* __restrict__ wd,
                         void* __restrict__ y, int d, int n_cols, int tile, int cap) {
  using E = Elem<BF16>;
  constexpr int VEC = E::VEC;
  constexpr int ESZ = BF16 ? 2 : 4;
  constexpr int kUdThreads = THREADS;
  constexpr int kUdWarps = THREADS / 32;
  __shared__ int2 s_jh[kMaxEntries];  // (column j, a bits); after phase U: (j, h bits)
  __shared__ float s_upart[kUdWarps][kMaxEntries];
  __shared__ int s_tile_off[kMaxTiles + 1];
  __shared__ int s_chunk[2];  // [0] first tile after the chunk, [1] entries in the chunk

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t = blockIdx.x;
  const int nvec = d / VEC;  // 16-byte vectors per row
  const int64_t row_bytes = static_cast<int64_t>(d) * ESZ;

  // this thread's vectors: v = tid + k * kUdThreads
  uint4 xv[NV];
  float acc[NV][VEC];
  const char* xrow = static_cast<const char*>(x) + t * row_bytes;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kUdThreads;
    xv[k] = v < nvec ? __ldg(reinterpret_cast<const uint4*>(xrow) + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
  }

  const int nt = n_cols / tile;
  const uint8_t* cnt = count + t * nt;
  int b0 = 0;
  while (b0 < nt) {
    // ---- chunk: tiles [b0, b1) holding at most kMaxEntries entries and at
    // most kMaxTiles tiles (one tile always fits: cap <= 255 < kMaxEntries)
    if (warp == 0) {
      int b = b0, total = 0, n_tiles = 0;
      if (lane == 0) s_tile_off[0] = 0;
      while (true) {
        const int bb = b + lane;
        const int c = bb < nt ? min(static_cast<int>(cnt[bb]), cap) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int nb = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += nb;
        }
        // every condition is monotone in the lane, so the fitting lanes form a prefix
        const bool fits = bb < nt && total + incl <= kMaxEntries && n_tiles + lane < kMaxTiles;
        const int take = __popc(__ballot_sync(0xffffffffu, fits));
        if (lane < take) s_tile_off[n_tiles + lane + 1] = total + incl;
        if (take > 0) total += __shfl_sync(0xffffffffu, incl, take - 1);
        n_tiles += take;
        b += take;
        if (take < 32) break;
      }
      if (lane == 0) {
        s_chunk[0] = b;
        s_chunk[1] = total;
      }
    }
    __syncthreads();
    const int b1 = s_chunk[0];
    const int n_e = s_chunk[1];
    const int n_tiles = b1 - b0;

    // ---- gather the chunk's entries, one thread per entry
    for (int e = tid; e < n_e; e += kUdThreads) {
      int lo = 0, hi = n_tiles;  // find i with s_tile_off[i] <= e < s_tile_off[i + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_tile_off[mid] <= e) lo = mid; else hi = mid;
      }
      const int b = b0 + lo;
      const int s = e - s_tile_off[lo];
      const int64_t seg = t * nt + b;
      s_jh[e] = make_int2(b * tile + idx[seg * cap + s], __float_as_int(E::load_val(val, seg * cap + s)));
    }
    __syncthreads();

    // ---- phase U: per-warp partial dot products of 8 entries at a time
    const char* wub = static_cast<const char*>(wu_t);
    for (int e0 = 0; e0 < n_e; e0 += kUnroll) {
      float part[kUnroll];
      uint4 w[kUnroll][NV];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = e0 + u;
        const int j = e < n_e ? s_jh[e].x : -1;
        const uint4* row = reinterpret_cast<const uint4*>(wub + static_cast<int64_t>(j) * row_bytes);
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const int v = tid + k * kUdThreads;
          w[u][k] = (j >= 0 && v < nvec) ? __ldg(row + v) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        float p = 0.0f;
#pragma unroll
        for (int k = 0; k < NV; ++k) p = E::dot(xv[k], w[u][k], p);
        part[u] = p;
      }
      const float tot = warp_reduce8(part, lane);
      if ((lane & 3) == 0) {
        const int e = e0 + reduce8_entry(lane);
        if (e < n_e) s_upart[warp][e] = tot;
      }
    }
    __syncthreads();

    // ---- h = a * u (fixed-order sum over warps), rounded as phase D uses it
    for (int e = tid; e < n_e; e += kUdThreads) {
      float u = 0.0f;
#pragma unroll
      for (int w8 = 0; w8 < kUdWarps; ++w8) u += s_upart[w8][e];
      const typename E::HType hq = E::h_of(__int_as_float(s_jh[e].y) * u);
      int bits;
      if constexpr (BF16) bits = static_cast<int>(hq); else bits = __float_as_int(hq);
      s_jh[e].y = bits;
    }
    __syncthreads();

    // ---- phase D: y += h * W_down[j]
    const char* wdb = static_cast<const char*>(wd);
    for (int e0 = 0; e0 < n_e; e0 += kUnroll) {
      uint4 w[kUnroll][NV];
      typename E::HType hv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = e0 + u;
        const int2 jh = e < n_e ? s_jh[e] : make_int2(-1, 0);
        if constexpr (BF16) hv[u] = static_cast<uint16_t>(jh.y); else hv[u] = __int_as_float(jh.y);
        const uint4* row = reinterpret_cast<const uint4*>(wdb + static_cast<int64_t>(jh.x) * row_bytes);
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const int v = tid + k * kUdThreads;
          w[u][k] = (jh.x >= 0 && v < nvec) ? __ldg(row + v) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
#pragma unroll
        for (int k = 0; k < NV; ++k) E::axpy(hv[u], w[u][k], acc[k]);
    }
    b0 = b1;
    __syncthreads();  // the next chunk rewrites the shared lists
  }

  char* yrow = static_cast<char*>(y) + t * row_bytes;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kUdThreads;
    if (v < nvec) reinterpret_cast<uint4*>(yrow)[v] = E::pack(acc[k]);
  }
}

template <int THREADS, int NV, bool BF16>
static int launch_ud(const void* x, const uint8_t* count, const uint8_t* idx, const void* val,
                     const void* wu_t, const void* wd, void* y, int64_t n, int64_t d, int64_t f,
                     int tile, int cap, cudaStream_t st) {
  if (n > 0x7fffffff) return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: too many rows");
  fused_up_down_kernel<THREADS, NV, BF16><<<static_cast<unsigned>(n), THREADS, 0, st>>>(
      x, count, idx, val, wu_t, wd, y, static_cast<int>(d), static_cast<int>(f), tile, cap);
  return check_launch("twell_fused_up_down");
}

// A row is covered by THREADS x NV 16-byte vectors: 128 threads with 1..4
// vectors each, 256 threads with 4 for the widest rows.
template <bool BF16>
static int dispatch_ud(const void* x, const uint8_t* count, const uint8_t* idx, const void* val,
                       const void* wu_t, const void* wd, void* y, int64_t n, int64_t d, int64_t f,
                       int tile, int cap, cudaStream_t st) {
  constexpr int VEC = Elem<BF16>::VEC;
  const int64_t nvec = d / VEC;
#define SGE_UD(TH, NV) \
  if (nvec <= (TH) * (NV)) return launch_ud<TH, NV, BF16>(x, count, idx, val, wu_t, wd, y, n, d, f, tile, cap, st);
  SGE_UD(128, 1)
  SGE_UD(128, 2)
  SGE_UD(128, 3)
  SGE_UD(128, 4)
  SGE_UD(256, 4)
#undef SGE_UD
  return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: d_model %lld too large (max %d)",
              (long long)d, 256 * 4 * VEC);
}

}  // namespace sge

using namespace sge;

extern "C" int twell_fused_up_down(const void* x, const uint8_t* count, const uint8_t* idx,
                                   const void* val, const void* wu_t, const void* wd, void* y,
                                   int64_t n_tokens, int64_t d_model, int64_t d_ff, int dtype,
                                   int tile, int cap, void* stream) {
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
  if (!x || !count || !idx || !val || !wu_t || !wd || !y)
    return fail(SGE_ERR_ARG, "twell_fused_up_down: null pointer");
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) || !aligned16(val))
    return fail(SGE_ERR_ARG, "twell_fused_up_down: pointer not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SGE_BF16)
    return dispatch_ud<true>(x, count, idx, val, wu_t, wd, y, n_tokens, d_model, d_ff, tile, cap, st);
  if (dtype == SGE_F32)
    return dispatch_ud<false>(x, count, idx, val, wu_t, wd, y, n_tokens, d_model, d_ff, tile, cap, st);
  return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: dtype %d", dtype);
}
