// Helpers shared by the sparse CUDA-core kernels (fused up/down, hybrid
// forward and backward): element access for 16-byte vectors of bf16 or fp32,
// exact-product dot and axpy with fp32 accumulation, and a multi-value warp
// reduction.
#pragma once

#include "sge_common.cuh"

namespace sge {

template <bool BF16>
struct Elem;

template <>
struct Elem<true> {
  static constexpr int VEC = 8;  // elements per 16-byte vector
  using HType = uint16_t;
  // acc += sum_k x_k * w_k with exact products (fma.rn.f32.bf16)
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
  // two accumulators: acc0 += the products of even elements, acc1 += the odd ones
  __device__ __forceinline__ static void dot2(const uint4& x, const uint4& w, float& acc0, float& acc1) {
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
          "mov.b32 {xl, xh}, %2;\n\t"
          "mov.b32 {wl, wh}, %3;\n\t"
          "fma.rn.f32.bf16 %0, xl, wl, %0;\n\t"
          "fma.rn.f32.bf16 %1, xh, wh, %1;\n\t}"
          : "+f"(acc0), "+f"(acc1)
          : "r"(xs[i]), "r"(ws[i]));
  }
  // y += h * w with h already rounded to bf16, exact products
  __device__ __forceinline__ static void axpy(HType hb, const uint4& w, float (&y)[8]) {
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
  __device__ __forceinline__ static HType h_of(float h) { return f32_to_bf16_bits(h); }
  __device__ __forceinline__ static int h_bits(HType h) { return static_cast<int>(h); }
  __device__ __forceinline__ static HType h_from_bits(int b) { return static_cast<uint16_t>(b); }
  __device__ __forceinline__ static float load_val(const void* p, int64_t i) {
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16);
  }
  // the stored bits of value i, and the value they encode
  __device__ __forceinline__ static uint32_t load_raw(const void* p, int64_t i) {
    return static_cast<const uint16_t*>(p)[i];
  }
  __device__ __forceinline__ static float from_raw(uint32_t r) { return __uint_as_float(r << 16); }
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
  using HType = float;
  __device__ __forceinline__ static float dot(const uint4& x, const uint4& w, float acc) {
    acc = fmaf(__uint_as_float(x.x), __uint_as_float(w.x), acc);
    acc = fmaf(__uint_as_float(x.y), __uint_as_float(w.y), acc);
    acc = fmaf(__uint_as_float(x.z), __uint_as_float(w.z), acc);
    acc = fmaf(__uint_as_float(x.w), __uint_as_float(w.w), acc);
    return acc;
  }
  __device__ __forceinline__ static void dot2(const uint4& x, const uint4& w, float& acc0, float& acc1) {
    acc0 = fmaf(__uint_as_float(x.x), __uint_as_float(w.x), acc0);
    acc1 = fmaf(__uint_as_float(x.y), __uint_as_float(w.y), acc1);
    acc0 = fmaf(__uint_as_float(x.z), __uint_as_float(w.z), acc0);
    acc1 = fmaf(__uint_as_float(x.w), __uint_as_float(w.w), acc1);
  }
  __device__ __forceinline__ static void axpy(HType h, const uint4& w, float (&y)[4]) {
    y[0] = fmaf(h, __uint_as_float(w.x), y[0]);
    y[1] = fmaf(h, __uint_as_float(w.y), y[1]);
    y[2] = fmaf(h, __uint_as_float(w.z), y[2]);
    y[3] = fmaf(h, __uint_as_float(w.w), y[3]);
  }
  __device__ __forceinline__ static HType h_of(float h) { return h; }
  __device__ __forceinline__ static int h_bits(HType h) { return __float_as_int(h); }
  __device__ __forceinline__ static HType h_from_bits(int b) { return __int_as_float(b); }
  __device__ __forceinline__ static float load_val(const void* p, int64_t i) {
    return static_cast<const float*>(p)[i];
  }
  __device__ __forceinline__ static uint32_t load_raw(const void* p, int64_t i) {
    return static_cast<const uint32_t*>(p)[i];
  }
  __device__ __forceinline__ static float from_raw(uint32_t r) { return __uint_as_float(r); }
  __device__ __forceinline__ static uint4 pack(const float (&o)[4]) {
    return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                      __float_as_uint(o[3]));
  }
};

// Sum of v[0..K) over the 32 lanes of a warp with a halving shuffle tree
// (K - 1 + log2(32 / K) shuffles).  Every lane returns the total of entry
// multi_entry<K>(lane).
template <int K>
__device__ __forceinline__ float warp_reduce_multi(float (&v)[K], int lane) {
  static_assert(K >= 1 && K <= 32 && (K & (K - 1)) == 0, "power of two");
  int off = 16;
#pragma unroll
  for (int cnt = K; cnt > 1; cnt >>= 1, off >>= 1) {
    const bool hi = lane & off;
#pragma unroll
    for (int k = 0; k < cnt / 2; ++k) {
      const float send = hi ? v[k] : v[k + cnt / 2];
      const float keep = hi ? v[k + cnt / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float s = v[0];
#pragma unroll
  for (; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  return s;
}

template <int K>
__device__ __forceinline__ int multi_entry(int lane) {
  int e = 0;
#pragma unroll
  for (int cnt = K, off = 16, bit = K / 2; cnt > 1; cnt >>= 1, off >>= 1, bit >>= 1)
    if (lane & off) e += bit;
  return e;
}

}  // namespace sge
