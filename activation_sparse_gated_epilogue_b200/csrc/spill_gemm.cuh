// Tensor-core spill of the hybrid format: the pieces the hybrid forward and
// the routed forward share.  Heavy rows (many active gates) are gathered into
// a dense block and run as two tcgen05 GEMMs, U = X_s W_up with an epilogue
// forming h = a (.) u, then Y_s = H_s W_down with an epilogue scattering the
// rows back into y ("Sparser, Faster, Lighter Transformer Language Models",
// pwwt.cn summary, section 03 and figure "基于混合格式的稀疏矩阵算子路由计算逻辑":
// the dense backup path on tensor cores).
#pragma once

#include "tc_gemm.cuh"

namespace sge {

// X_s[r] = x[spill_rows[r]] for the kept spill rows, zero rows after them.
static __global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ src,
                                                          const int32_t* __restrict__ rows,
                                                          const int32_t* __restrict__ n_rows_dev,
                                                          int cap_rows, int d, uint16_t* dst) {
  const int r = blockIdx.x;
  const int kept = min(*n_rows_dev, cap_rows);
  uint4* out = reinterpret_cast<uint4*>(dst + static_cast<int64_t>(r) * d);
  const int nvec = d / 8;
  if (r < kept) {
    const uint4* in = reinterpret_cast<const uint4*>(src + static_cast<int64_t>(rows[r]) * d);
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) out[v] = __ldg(in + v);
  } else {
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) out[v] = make_uint4(0, 0, 0, 0);
  }
}

// Epilogue of U = X_s W_up: spill_u = bf16(u) (when spill_u is not null),
// h = bf16(a u) -> hs.  Rows past the kept spill rows are left untouched
// (their outputs are ignored).
struct EpiSpillUp {
  const uint16_t* spill_a;
  uint16_t* spill_u;
  uint16_t* hs;
  const int32_t* n_spill;
  int s_max;
  int n_cols;

  // only the kept spill rows are computed
  __device__ __forceinline__ int m_limit(int m) const { return min(m, min(*n_spill, s_max)); }

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
    constexpr int CH = BN / 32;
    const int kept = min(*n_spill, s_max);
    const bool live = row < kept;
    // the row's activations for the whole tile, all loads in flight at once
    // (one thread per row: each load is a separate line, so issuing them
    // chunk by chunk would cost a memory round trip per chunk)
    uint4 av[CH][4];
#pragma unroll
    for (int ch = 0; ch < CH; ++ch)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = n_blk * BN + ch * 32 + q * 8;
        av[ch][q] = live && col + 8 <= n_cols
                        ? *reinterpret_cast<const uint4*>(spill_a + row * n_cols + col)
                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
    for (int ch = 0; ch < CH; ++ch) {
      uint32_t r[32];
      tmem_ld32(taddr + ch * 32, r);
      tmem_ld_wait();
      const int col0 = n_blk * BN + ch * 32;
      if (!live) continue;
      const int64_t off = row * n_cols + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col0 + q * 8 + 8 > n_cols) break;
        const uint32_t aw[4] = {av[ch][q].x, av[ch][q].y, av[ch][q].z, av[ch][q].w};
        uint32_t uw[4], hw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float u0 = __uint_as_float(r[q * 8 + 2 * i]);
          const float u1 = __uint_as_float(r[q * 8 + 2 * i + 1]);
          const float a0 = __uint_as_float(aw[i] << 16), a1 = __uint_as_float(aw[i] & 0xFFFF0000u);
          uw[i] = static_cast<uint32_t>(f32_to_bf16_bits(u0)) | (static_cast<uint32_t>(f32_to_bf16_bits(u1)) << 16);
          hw[i] = static_cast<uint32_t>(f32_to_bf16_bits(a0 * u0)) |
                  (static_cast<uint32_t>(f32_to_bf16_bits(a1 * u1)) << 16);
        }
        if (spill_u)
          *reinterpret_cast<uint4*>(spill_u + off + q * 8) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
        *reinterpret_cast<uint4*>(hs + off + q * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      }
    }
  }
};

// Epilogue of [G | U] = X_s [W_gate | W_up] (two B operands): the spill
// rows' activations recomputed from the gate, a = bf16(ReLU(g)) -> spill_a,
// spill_u = bf16(u), h = bf16(a u) -> hs (the same roundings as the packed
// path).  Rows past the kept spill rows are left untouched.
struct EpiSpillGateUp {
  uint16_t* spill_a;
  uint16_t* spill_u;
  uint16_t* hs;
  const int32_t* n_spill;
  int s_max;
  int n_cols;

  __device__ __forceinline__ int m_limit(int m) const { return min(m, min(*n_spill, s_max)); }

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
    const int kept = min(*n_spill, s_max);
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      uint32_t g[32], u[32];
      tmem_ld32(taddr + ch * 32, g);
      tmem_ld32(taddr + BN + ch * 32, u);
      tmem_ld_wait();
      const int col0 = n_blk * BN + ch * 32;
      if (row >= kept) continue;
      const int64_t off = row * n_cols + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col0 + q * 8 + 8 > n_cols) break;
        uint32_t aw[4], uw[4], hw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = q * 8 + 2 * i;
          const uint16_t a0b = f32_to_bf16_bits(fmaxf(__uint_as_float(g[k]), 0.0f));
          const uint16_t a1b = f32_to_bf16_bits(fmaxf(__uint_as_float(g[k + 1]), 0.0f));
          const float a0 = __uint_as_float(static_cast<uint32_t>(a0b) << 16);
          const float a1 = __uint_as_float(static_cast<uint32_t>(a1b) << 16);
          const float u0 = __uint_as_float(u[k]), u1 = __uint_as_float(u[k + 1]);
          aw[i] = static_cast<uint32_t>(a0b) | (static_cast<uint32_t>(a1b) << 16);
          uw[i] = static_cast<uint32_t>(f32_to_bf16_bits(u0)) | (static_cast<uint32_t>(f32_to_bf16_bits(u1)) << 16);
          hw[i] = static_cast<uint32_t>(f32_to_bf16_bits(a0 * u0)) |
                  (static_cast<uint32_t>(f32_to_bf16_bits(a1 * u1)) << 16);
        }
        *reinterpret_cast<uint4*>(spill_a + off + q * 8) = make_uint4(aw[0], aw[1], aw[2], aw[3]);
        *reinterpret_cast<uint4*>(spill_u + off + q * 8) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
        *reinterpret_cast<uint4*>(hs + off + q * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      }
    }
  }
};

// Epilogue of Y_s = H_s W_down: row r of the tile goes to y[spill_rows[r]].
struct EpiScatterRows {
  uint16_t* y;
  const int32_t* rows;
  const int32_t* n_spill;
  int s_max;
  int n_cols;

  // only the kept spill rows are computed
  __device__ __forceinline__ int m_limit(int m) const { return min(m, min(*n_spill, s_max)); }

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
    const int kept = min(*n_spill, s_max);
    const int64_t t = row < kept ? rows[row] : -1;
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      uint32_t r[32];
      tmem_ld32(taddr + ch * 32, r);
      tmem_ld_wait();
      const int col0 = n_blk * BN + ch * 32;
      if (t < 0) continue;
      uint16_t* o = y + t * n_cols + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col0 + q * 8 + 8 > n_cols) break;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[q * 8 + 2 * i]))) |
                 (static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[q * 8 + 2 * i + 1]))) << 16);
        *reinterpret_cast<uint4*>(o + q * 8) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
};

}  // namespace sge
