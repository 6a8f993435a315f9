// Tensor-core spill of the hybrid format: the pieces the hybrid forward and
// the routed forward share.  Heavy rows (many active gates) are gathered into
// a dense block and run as two tcgen05 GEMMs, U = X_s W_up with an epilogue
// forming h = a (.) u, then Y_s = H_s W_down with an epilogue scattering the
// rows back into y ("Sparser, Faster, Lighter Transformer Language Models",
// pwwt.cn summary, section 03 and figure "基于混合格式的稀疏矩阵算子路由计算逻辑":
// the dense backup path on tensor cores).
#pragma once

#include "sge_host.h"
#include "tc_gemm.cuh"

namespace sge {

// X_s[r] = x[spill_rows[r]] for the kept spill rows, zero rows after them.
static __global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ src,
                                                          const int32_t* __restrict__ rows,
                                                          const int32_t* __restrict__ n_rows_dev,
                                                          int cap_rows, int d, uint16_t* dst) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
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

// Split-K of the spill GEMMs.  With few spill rows the output has fewer
// tiles than there are CTA pairs (130 spill rows and d = 2048: 8 tiles of
// 256 x 256 for 74 pairs), so the GEMM would stream the weights through a
// few SMs only, each a long chain of k-blocks.  An epilogue with a `part`
// area then asks for K to be cut into up to kSplitMax parts, so that tiles x
// parts fill the pairs; each part stores its fp32 product in
// part[split][row][col] (rows padded to the launch's 256-row tiles, columns
// to its n_tiles_n tiles of tile_n), the number of parts goes to the word
// after the area, and a kernel of the epilogue's own adds the parts in part
// order and applies the epilogue's arithmetic: results do not depend on
// timing.
constexpr int kSplitMax = 16;
// capacity of the partial-product area in 256 x 256 fp32 tiles (at least
// the number of CTA pairs that can be resident)
constexpr int kSplitTiles = 80;
constexpr size_t kSplitPartBytes = static_cast<size_t>(kSplitTiles) * 256 * 256 * 4 + 256;

// Parts to ask for when `rows` rows (device-side count) make the launch's
// row tiles and n_tiles_n column tiles.
SGE_DEV int split_count(int rows, int n_tiles_n) {
  const int units = ((rows + 255) / 256) * n_tiles_n;
  if (units == 0) return 1;
  const int pairs = min(static_cast<int>(cluster_count_x()), kSplitTiles);
  return max(1, min(kSplitMax, pairs / units));
}

// The word after the part area: the number of parts of the last launch.
SGE_DEV int* split_word(float* part) { return reinterpret_cast<int*>(part) + kSplitTiles * 256 * 256; }
SGE_DEV int split_word_read(const float* part) {
  return reinterpret_cast<const int*>(part)[kSplitTiles * 256 * 256];
}

// One epilogue thread's row of a tile (BN columns from TMEM) stored as part
// `split`; rows >= rows_used are not stored.
template <int BN>
SGE_DEV void store_part(float* part, int rows_used, int64_t ncp, int split, int64_t row, int n_blk,
                        uint32_t taddr) {
  const int64_t rows_pad = static_cast<int64_t>((rows_used + 255) / 256) * 256;
  float* dst = part + (split * rows_pad + row) * ncp + n_blk * BN;
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    uint32_t r[32];
    tmem_ld32(taddr + ch * 32, r);
    tmem_ld_wait();
    if (row >= rows_used) continue;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      __stcg(reinterpret_cast<float4*>(dst + ch * 32) + q,
             make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                         __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])));
  }
}

// v[0..8) = the sum in part order of the 8 columns at (row, col) of nsplit
// parts (loads of four parts in flight at once).
SGE_DEV void sum_parts8(const float* part, int nsplit, int64_t rows_pad, int64_t ncp, int64_t row, int64_t col,
                        float (&v)[8]) {
  const float* src = part + row * ncp + col;
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = 0.0f;
  for (int s0 = 0; s0 < nsplit; s0 += 4) {
    float4 f[4][2];
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        f[b][h] = s0 + b < nsplit ? __ldcg(reinterpret_cast<const float4*>(src + (s0 + b) * rows_pad * ncp) + h)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (s0 + b >= nsplit) break;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        v[4 * h] += f[b][h].x;
        v[4 * h + 1] += f[b][h].y;
        v[4 * h + 2] += f[b][h].z;
        v[4 * h + 3] += f[b][h].w;
      }
    }
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
  float* part = nullptr;  // split-K parts (split_spill_up_kernel finishes them)
  int n_tiles_n = 1;
  int tile_n = 256;

  // only the kept spill rows are computed
  __device__ __forceinline__ int m_limit(int m) const { return min(m, min(*n_spill, s_max)); }

  __device__ __forceinline__ int splits() const {
    return part == nullptr ? 1 : split_count(min(*n_spill, s_max), n_tiles_n);
  }

  template <int BN>
  __device__ __forceinline__ void run_split(uint32_t taddr, int64_t row, int n_blk, int split, int nsplit,
                                            int lane) const {
    if (part != nullptr && row == 0 && n_blk == 0 && split == 0) *split_word(part) = nsplit;
    if (nsplit == 1) {
      run<BN>(taddr, row, n_blk, lane);
      return;
    }
    store_part<BN>(part, min(*n_spill, s_max), static_cast<int64_t>(n_tiles_n) * tile_n, split, row, n_blk,
                   taddr);
  }

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

// Finishes a split U = X_s W_up: u = the parts summed in part order,
// spill_u = bf16(u) (when not null), h = bf16(a u) -> hs, for the kept rows;
// nothing when the GEMM did not split.  A thread per 8 columns of a row.
static __global__ void __launch_bounds__(256) split_spill_up_kernel(const float* __restrict__ part,
                                                                    const uint16_t* __restrict__ spill_a,
                                                                    uint16_t* spill_u, uint16_t* hs,
                                                                    const int32_t* __restrict__ n_spill,
                                                                    int s_max, int n_cols, int ncp) {
  grid_dep_wait();  // the parts come from the GEMM before
  grid_dep_launch();
  const int nsplit = split_word_read(part);
  const int kept = min(*n_spill, s_max);
  if (nsplit <= 1 || kept <= 0) return;
  const int64_t rows_pad = static_cast<int64_t>((kept + 255) / 256) * 256;
  const int per_row = n_cols / 8;
  const int64_t total = static_cast<int64_t>(kept) * per_row;
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t r = i / per_row;
    const int c = static_cast<int>(i % per_row) * 8;
    float u[8];
    sum_parts8(part, nsplit, rows_pad, ncp, r, c, u);
    const uint4 av = *reinterpret_cast<const uint4*>(spill_a + r * n_cols + c);
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
    uint32_t uw[4], hw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a0 = __uint_as_float(aw[k] << 16), a1 = __uint_as_float(aw[k] & 0xFFFF0000u);
      uw[k] = static_cast<uint32_t>(f32_to_bf16_bits(u[2 * k])) |
              (static_cast<uint32_t>(f32_to_bf16_bits(u[2 * k + 1])) << 16);
      hw[k] = static_cast<uint32_t>(f32_to_bf16_bits(a0 * u[2 * k])) |
              (static_cast<uint32_t>(f32_to_bf16_bits(a1 * u[2 * k + 1])) << 16);
    }
    if (spill_u) *reinterpret_cast<uint4*>(spill_u + r * n_cols + c) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
    *reinterpret_cast<uint4*>(hs + r * n_cols + c) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  }
}

// Grid of a part-sum kernel over `rows` rows of n_cols columns (8 per thread).
static inline int split_grid(int64_t rows, int n_cols) {
  const int64_t work = (rows * (n_cols / 8) + 255) / 256;
  return static_cast<int>(work < 4 * sm_count() ? (work > 0 ? work : 1) : 4 * sm_count());
}

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

// Epilogue of Y_s = H_s W (W's rows K-major): row r of the product goes to
// y[rows[r]] (bf16) for the kept spill rows r < min(*n_spill, s_max).  With
// `part` (kSplitPartBytes) K may be split; split_scatter_kernel then adds
// the parts and scatters the rows.
struct EpiScatterRows {
  uint16_t* y;
  const int32_t* rows;
  const int32_t* n_spill;
  int s_max;
  int n_cols;
  float* part = nullptr;
  int n_tiles_n = 1;  // output column tiles of the launch (N / Shape::BN rounded up)
  int tile_n = 256;   // Shape::BN

  // only the kept spill rows are computed
  __device__ __forceinline__ int m_limit(int m) const { return min(m, min(*n_spill, s_max)); }

  __device__ __forceinline__ int splits() const {
    return part == nullptr ? 1 : split_count(min(*n_spill, s_max), n_tiles_n);
  }

  template <int BN>
  __device__ __forceinline__ void run_split(uint32_t taddr, int64_t row, int n_blk, int split, int nsplit,
                                            int lane) const {
    const int kept = min(*n_spill, s_max);
    if (part != nullptr && row == 0 && n_blk == 0 && split == 0) *split_word(part) = nsplit;
    const int64_t t = row < kept ? rows[row] : -1;
    if (nsplit == 1) {
      uint16_t* o = t >= 0 ? y + t * n_cols : nullptr;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(taddr + ch * 32, r);
        tmem_ld_wait();
        const int col0 = n_blk * BN + ch * 32;
        if (t < 0) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (col0 + q * 8 + 8 > n_cols) break;
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            w[i] = static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[q * 8 + 2 * i]))) |
                   (static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[q * 8 + 2 * i + 1]))) << 16);
          *reinterpret_cast<uint4*>(o + col0 + q * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      return;
    }
    store_part<BN>(part, kept, static_cast<int64_t>(n_tiles_n) * tile_n, split, row, n_blk, taddr);
  }
};

// Finishes a split scatter GEMM: y[rows[r]][c] = bf16(sum over parts, in
// part order, of part[s][r][c]) for the kept rows; nothing when the GEMM
// did not split (it wrote y itself).  A thread per 8 columns of a row, the
// loads of four parts in flight at once.
static __global__ void __launch_bounds__(256) split_scatter_kernel(const float* __restrict__ part,
                                                                   const int32_t* __restrict__ rows,
                                                                   const int32_t* __restrict__ n_spill,
                                                                   int s_max, int n_cols, int ncp,
                                                                   uint16_t* __restrict__ y) {
  grid_dep_launch();
  grid_dep_wait();  // the parts come from the GEMM before
  const int nsplit = split_word_read(part);
  const int kept = min(*n_spill, s_max);
  if (nsplit <= 1 || kept <= 0) return;
  const int64_t rows_pad = static_cast<int64_t>((kept + 255) / 256) * 256;
  const int per_row = n_cols / 8;
  const int64_t total = static_cast<int64_t>(kept) * per_row;
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<int64_t>(gridDim.x) * 256) {
    const int r = static_cast<int>(i / per_row);
    const int c = static_cast<int>(i % per_row) * 8;
    float v[8];
    sum_parts8(part, nsplit, rows_pad, ncp, r, c, v);
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[k] = static_cast<uint32_t>(f32_to_bf16_bits(v[2 * k])) |
             (static_cast<uint32_t>(f32_to_bf16_bits(v[2 * k + 1])) << 16);
    *reinterpret_cast<uint4*>(y + static_cast<int64_t>(rows[r]) * n_cols + c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Launches split_scatter_kernel after a scatter GEMM launched with `part`
// (ncp = the GEMM's n_tiles_n * tile_n).
static inline int launch_split_scatter(const float* part, const int32_t* rows, const int32_t* n_spill,
                                       int s_max, int n_cols, int ncp, uint16_t* y, cudaStream_t st,
                                       const char* what) {
  return launch_pdl(split_scatter_kernel, dim3(split_grid(s_max, n_cols)), dim3(256), 0, st, what, part, rows,
                    n_spill, s_max, n_cols, ncp, y);
}

}  // namespace sge
