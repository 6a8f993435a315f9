// Fused up and down projections over the TwELL nonzeros.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 02, last paragraph: one custom kernel performs the up and the down
// projection in a single traversal, fusing the two products so that the
// intermediate h is never written to global memory.  For every stored entry
// (t, j, a) of the TwELL gate activations:
//     u = x[t] . W_up[:, j]      h = a * u      y[t] += h * W_down[j, :]
//
// One warp per token.  x[t] lives in registers as fp32, the y[t]
// accumulator too; for each entry the warp streams row j of wu_t and row j
// of wd (both contiguous d-vectors) with coalesced 16-byte loads, both issued
// before any arithmetic so that their latencies overlap, reduces the dot
// product with warp shuffles and accumulates h * W_down[j] in fp32.  No
// atomics: each y row is owned by one warp, so results are deterministic.
#include "sge_host.h"
#include "sge_common.cuh"

namespace sge {

template <bool BF16>
struct Elem;
template <>
struct Elem<true> {
  static constexpr int VEC = 8;  // elements per 16-byte load
  __device__ __forceinline__ static void unpack(const uint4& v, float (&o)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
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
  __device__ __forceinline__ static void unpack(const uint4& v, float (&o)[4]) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static float load_val(const void* p, int64_t i) {
    return static_cast<const float*>(p)[i];
  }
  __device__ __forceinline__ static uint4 pack(const float (&o)[4]) {
    return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                      __float_as_uint(o[3]));
  }
};

constexpr int kUdWarps = 8;

template <int NCH, bool BF16>
__global__ void __launch_bounds__(kUdWarps * 32)
    fused_up_down_kernel(const void* __restrict__ x, const uint8_t* __restrict__ count,
                         const uint8_t* __restrict__ idx, const void* __restrict__ val,
                         const void* __restrict__ wu_t, const void* __restrict__ wd,
                         void* __restrict__ y, int64_t n_rows, int d, int n_cols, int tile,
                         int cap) {
  using E = Elem<BF16>;
  constexpr int VEC = E::VEC;
  constexpr int CH = 32 * VEC;  // elements covered by one warp-wide 16-byte load
  constexpr int ESZ = BF16 ? 2 : 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kUdWarps + warp;
  if (t >= n_rows) return;

  const char* xrow = static_cast<const char*>(x) + t * d * ESZ;
  float xf[NCH][VEC], acc[NCH][VEC];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int e = c * CH + lane * VEC;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (e < d) v = __ldg(reinterpret_cast<const uint4*>(xrow + e * ESZ));
    E::unpack(v, xf[c]);
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[c][k] = 0.0f;
  }

  const int64_t nt = n_cols / tile;
  const uint8_t* cnt = count + t * nt;
  for (int64_t b0 = 0; b0 < nt; b0 += 32) {
    const int64_t b = b0 + lane;
    const int cl = b < nt ? min(static_cast<int>(cnt[b]), cap) : 0;
    uint32_t mask = __ballot_sync(0xffffffffu, cl > 0);
    while (mask) {
      const int l = __ffs(mask) - 1;
      mask &= mask - 1;
      const int c_tile = __shfl_sync(0xffffffffu, cl, l);
      const int64_t seg = t * nt + b0 + l;
      const int64_t jbase = (b0 + l) * tile;
      for (int s0 = 0; s0 < c_tile; s0 += 32) {
        int my_j = 0;
        float my_a = 0.0f;
        if (s0 + lane < c_tile) {
          my_j = idx[seg * cap + s0 + lane];
          my_a = E::load_val(val, seg * cap + s0 + lane);
        }
        const int n_e = min(32, c_tile - s0);
        for (int e = 0; e < n_e; ++e) {
          const int64_t j = jbase + __shfl_sync(0xffffffffu, my_j, e);
          const float a = __shfl_sync(0xffffffffu, my_a, e);
          const char* wur = static_cast<const char*>(wu_t) + j * d * ESZ;
          const char* wdr = static_cast<const char*>(wd) + j * d * ESZ;
          uint4 vu[NCH], vd[NCH];
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const int ee = c * CH + lane * VEC;
            vu[c] = make_uint4(0, 0, 0, 0);
            vd[c] = make_uint4(0, 0, 0, 0);
            if (ee < d) {
              vu[c] = __ldg(reinterpret_cast<const uint4*>(wur + ee * ESZ));
              vd[c] = __ldg(reinterpret_cast<const uint4*>(wdr + ee * ESZ));
            }
          }
          float u = 0.0f;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            float w[VEC];
            E::unpack(vu[c], w);
#pragma unroll
            for (int k = 0; k < VEC; ++k) u = fmaf(xf[c][k], w[k], u);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
          const float h = a * u;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            float w[VEC];
            E::unpack(vd[c], w);
#pragma unroll
            for (int k = 0; k < VEC; ++k) acc[c][k] = fmaf(h, w[k], acc[c][k]);
          }
        }
      }
    }
  }

  char* yrow = static_cast<char*>(y) + t * d * ESZ;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int e = c * CH + lane * VEC;
    if (e < d) *reinterpret_cast<uint4*>(yrow + e * ESZ) = E::pack(acc[c]);
  }
}

template <int NCH, bool BF16>
static int launch_ud(const void* x, const uint8_t* count, const uint8_t* idx, const void* val,
                     const void* wu_t, const void* wd, void* y, int64_t n, int64_t d, int64_t f,
                     int tile, int cap, cudaStream_t st) {
  const int64_t blocks = (n + kUdWarps - 1) / kUdWarps;
  if (blocks > 0x7fffffff) return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: too many rows");
  fused_up_down_kernel<NCH, BF16><<<static_cast<unsigned>(blocks), kUdWarps * 32, 0, st>>>(
      x, count, idx, val, wu_t, wd, y, n, static_cast<int>(d), static_cast<int>(f), tile, cap);
  return check_launch("twell_fused_up_down");
}

template <bool BF16>
static int dispatch_ud(const void* x, const uint8_t* count, const uint8_t* idx, const void* val,
                       const void* wu_t, const void* wd, void* y, int64_t n, int64_t d, int64_t f,
                       int tile, int cap, cudaStream_t st) {
  constexpr int CH = 32 * Elem<BF16>::VEC;
  const int64_t nch = (d + CH - 1) / CH;
#define SGE_UD(K) \
  if (nch <= K) return launch_ud<K, BF16>(x, count, idx, val, wu_t, wd, y, n, d, f, tile, cap, st);
  SGE_UD(1)
  SGE_UD(2)
  SGE_UD(4)
  SGE_UD(8)
  SGE_UD(10)
#undef SGE_UD
  return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: d_model %lld too large (max %d)",
              (long long)d, 10 * CH);
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
  if (d_ff >= (1LL << 31) || n_tokens >= (1LL << 40))
    return fail(SGE_ERR_UNSUPPORTED, "twell_fused_up_down: size too large");
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
