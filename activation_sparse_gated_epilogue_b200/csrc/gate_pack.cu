// Gate projection with the TwELL pack in its epilogue.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 02 and figure "gate projection with TwELL storage generation": the
// gate activations are written in TwELL directly by the gate GEMM's epilogue,
// so no dense gate activation reaches global memory and no conversion kernel
// runs.  TwELL (figure "TwELL cuts the column direction into tiles") keeps,
// per row and per 1-D column tile of width T, a count, the values and the
// local column indices of the nonzeros.
//
// bf16: the tcgen05 engine (tc_gemm.cuh) with N = 256 per tile; each epilogue
// thread owns one accumulator row (one TMEM lane), so compaction of a row's
// tile is a sequential in-thread scan over its columns in ascending order.
// fp32: a CUDA-core FMA GEMM (64 x 128 tiles) with the same pack from a
// shared-memory copy of the tile.
#include "tc_launch.cuh"

namespace sge {

// Epilogue: ReLU + TwELL pack of one 128 x BN accumulator tile.  Each thread
// owns one row.  Per 32-column chunk it builds the bit mask of active
// columns (g > 0; NaN and -0 are inactive), then visits only the set bits in
// ascending order, so the cost is ~2 instructions per column plus a few
// dozen per stored entry.
template <int T>
struct EpiTwell {
  uint8_t* count;
  uint8_t* idx;
  uint16_t* val;  // bf16 bits
  int64_t n_rows;
  int n_cols;
  int cap;
  int32_t* diag;

  // r[jj] for a run-time jj in [0, 32) without local memory: a 5-level
  // select tree over the 32 registers.
  __device__ __forceinline__ static uint32_t pick(const uint32_t (&r)[32], int jj) {
    uint32_t a[16], b[8], c4[4], d2[2];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = (jj & 16) ? r[i + 16] : r[i];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = (jj & 8) ? a[i + 8] : a[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) c4[i] = (jj & 4) ? b[i + 4] : b[i];
#pragma unroll
    for (int i = 0; i < 2; ++i) d2[i] = (jj & 2) ? c4[i + 2] : c4[i];
    return (jj & 1) ? d2[1] : d2[0];
  }

  // Store the active columns of `m` (bits of r) as entries of tile `seg`,
  // local index = bit + idx_off; c counts every active column.
  __device__ __forceinline__ void emit(uint32_t m, const uint32_t (&r)[32], int& c, int64_t seg,
                                       bool ok, int idx_off) const {
    while (m) {
      const int jj = __ffs(m) - 1;
      m &= m - 1;
      if (ok && c < cap) {
        idx[seg * cap + c] = static_cast<uint8_t>(jj + idx_off);
        val[seg * cap + c] = f32_to_bf16_bits(__uint_as_float(pick(r, jj)));
      }
      ++c;
    }
  }

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
    static_assert(BN % T == 0 && BN % 32 == 0, "tile must divide the GEMM N block");
    static_assert(T == 16 || T % 32 == 0, "tile width");
    const bool row_ok = row < n_rows;
    const int64_t nt = n_cols / T;
    int overflow = 0;
    int c = 0;
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      uint32_t r[32];
      tmem_ld32(taddr + ch * 32, r);
      tmem_ld_wait();
      uint32_t m = 0;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) m |= (__uint_as_float(r[jj]) > 0.0f ? 1u : 0u) << jj;
      const int col0 = n_blk * BN + ch * 32;  // global column of bit 0
      if constexpr (T == 16) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int gcol = col0 + 16 * half;
          const bool ok = row_ok && gcol < n_cols;
          const int64_t seg = row * nt + gcol / T;
          c = 0;
          emit(half ? (m & 0xFFFF0000u) : (m & 0xFFFFu), r, c, seg, ok, -16 * half);
          if (ok) {
            count[seg] = static_cast<uint8_t>(c);
            overflow += c > cap;
          }
        }
      } else {
        const int off = (ch * 32) % T;  // offset of this chunk inside its tile
        if (off == 0) c = 0;
        const bool ok = row_ok && col0 < n_cols;
        const int64_t seg = row * nt + col0 / T;
        emit(m, r, c, seg, ok, off);
        if (off + 32 == T && ok) {
          count[seg] = static_cast<uint8_t>(c);
          overflow += c > cap;
        }
      }
    }
    if (overflow && diag) atomicAdd(reinterpret_cast<int*>(diag + SGE_DIAG_OVERFLOW_TILES), overflow);
  }
};

// ---------------------------------------------------------- fp32 (SIMT)

template <int T>
__global__ void __launch_bounds__(256) gate_pack_f32_kernel(const float* __restrict__ x,
                                                            const float* __restrict__ w,
                                                            int64_t n_rows, int d, int n_cols,
                                                            int cap, uint8_t* count, uint8_t* idx,
                                                            float* val, int32_t* diag) {
  constexpr int BM = 64, BN = 128, BK = 16;
  __shared__ float xs[BK][BM + 4];
  __shared__ float ws[BK][BN + 4];
  __shared__ float gs[BM][BN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int n0 = blockIdx.x * BN;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < d; k0 += BK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + 256 * i, r = e >> 4, kk = e & 15;
      xs[kk][r] = (m0 + r < n_rows && k0 + kk < d) ? x[(m0 + r) * d + k0 + kk] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = tid + 256 * i, r = e >> 4, kk = e & 15;
      ws[kk][r] = (n0 + r < n_cols && k0 + kk < d) ? w[static_cast<int64_t>(n0 + r) * d + k0 + kk] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) gs[ty * 4 + i][tx + 16 * j] = acc[i][j];
  __syncthreads();

  constexpr int TPB = BN / T;  // TwELL tiles per block row
  const int64_t nt = n_cols / T;
  int overflow = 0;
  for (int s = tid; s < BM * TPB; s += 256) {
    const int r = s / TPB, tb = s % TPB;
    const int64_t row = m0 + r;
    const int col0 = n0 + tb * T;
    if (row >= n_rows || col0 >= n_cols) continue;
    const int64_t seg = row * nt + col0 / T;
    int c = 0;
    for (int jj = 0; jj < T; ++jj) {
      const float v = gs[r][tb * T + jj];
      if (v > 0.0f) {
        if (c < cap) {
          idx[seg * cap + c] = static_cast<uint8_t>(jj);
          val[seg * cap + c] = v;
        }
        ++c;
      }
    }
    count[seg] = static_cast<uint8_t>(c);
    overflow += c > cap;
  }
  if (overflow && diag) atomicAdd(reinterpret_cast<int*>(diag + SGE_DIAG_OVERFLOW_TILES), overflow);
}

// ----------------------------------------------------------- launchers

// Batches of at most this many tokens run on single-CTA 128 x 128 tiles:
// with few rows, the CTA pair's 256-row tiles are mostly padding, and the
// tensor-core time of that padding (not the W_gate bytes) sets the time.
constexpr int64_t kSmallGateRows = 256;

template <int T>
static int launch_bf16(const void* x, const void* wg_t, int64_t n, int64_t d, int64_t f, int cap,
                       uint8_t* count, uint8_t* idx, void* val, int32_t* diag, cudaStream_t st) {
  using Shape = TcPairShape<256, 1, 2>;
  CUtensorMap ma, mb;
  int rc = make_tmap_bf16(&ma, x, n, d, d, kBM);
  if (rc) return rc;
  if (n <= kSmallGateRows) {
    using Small = TcShape<128, 1>;
    rc = make_tmap_bf16(&ma, x, n, d, d, a_box_rows(n));  // the engine loads a_box_rows(n) rows of A
    if (!rc) rc = make_tmap_bf16(&mb, wg_t, f, d, d, Small::BN);
    if (rc) return rc;
    EpiTwell<T> epi{count, idx, static_cast<uint16_t*>(val), n, static_cast<int>(f), cap, diag};
    return launch_tc_gemm<Small>(ma, mb, mb, n, f, d, epi, diag, st,
                                 "twell_gate_pack (bf16 tcgen05, small batch)");
  }
  rc = make_tmap_bf16(&mb, wg_t, f, d, d, Shape::BN / 2);
  if (rc) return rc;
  EpiTwell<T> epi{count, idx, static_cast<uint16_t*>(val), n, static_cast<int>(f), cap, diag};
  return launch_tc_gemm_pair<Shape>(ma, mb, mb, n, f, d, epi, diag, st,
                                    "twell_gate_pack (bf16 tcgen05 pair)");
}

template <int T>
static int launch_f32(const void* x, const void* wg_t, int64_t n, int64_t d, int64_t f, int cap,
                      uint8_t* count, uint8_t* idx, void* val, int32_t* diag, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((f + 127) / 128), static_cast<unsigned>((n + 63) / 64));
  if (grid.y > 65535) return fail(SGE_ERR_UNSUPPORTED, "fp32 gate GEMM: too many rows (%lld)", (long long)n);
  gate_pack_f32_kernel<T><<<grid, 256, 0, st>>>(static_cast<const float*>(x),
                                                static_cast<const float*>(wg_t), n,
                                                static_cast<int>(d), static_cast<int>(f), cap,
                                                count, idx, static_cast<float*>(val), diag);
  return check_launch("twell_gate_pack (fp32)");
}

}  // namespace sge

using namespace sge;

extern "C" int twell_gate_pack(const void* x, const void* wg_t, int64_t n_tokens, int64_t d_model,
                               int64_t d_ff, int dtype, int tile, int cap, uint8_t* count,
                               uint8_t* idx, void* val, int32_t* diag, void* stream) {
  NvtxRange nvtx_range("twell_gate_pack");
  clear_error();
  if (n_tokens < 0 || d_model < 1 || d_ff < 1)
    return fail(SGE_ERR_ARG, "twell_gate_pack: bad sizes N=%lld d=%lld F=%lld", (long long)n_tokens,
                (long long)d_model, (long long)d_ff);
  if (d_model % 8) return fail(SGE_ERR_ARG, "twell_gate_pack: d_model %% 8 != 0");
  if (tile != 16 && tile != 32 && tile != 64 && tile != 128)
    return fail(SGE_ERR_UNSUPPORTED, "twell_gate_pack: tile %d not in {16,32,64,128}", tile);
  if (d_ff % tile) return fail(SGE_ERR_ARG, "twell_gate_pack: d_ff %% tile != 0");
  if (cap < 1 || cap > tile) return fail(SGE_ERR_ARG, "twell_gate_pack: cap %d outside [1, tile]", cap);
  if (d_ff >= (1LL << 31) || d_model >= (1LL << 31) || n_tokens >= (1LL << 31))
    return fail(SGE_ERR_UNSUPPORTED, "twell_gate_pack: size beyond 2^31");
  if (n_tokens == 0) return SGE_OK;
  if (!x || !wg_t || !count || !idx || !val)
    return fail(SGE_ERR_ARG, "twell_gate_pack: null pointer");
  if (!aligned16(x) || !aligned16(wg_t) || !aligned16(count) || !aligned16(idx) || !aligned16(val) ||
      (diag && !aligned16(diag)))
    return fail(SGE_ERR_ARG, "twell_gate_pack: pointer not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SGE_BF16) {
    switch (tile) {
      case 16: return launch_bf16<16>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
      case 32: return launch_bf16<32>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
      case 64: return launch_bf16<64>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
      default: return launch_bf16<128>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
    }
  }
  if (dtype == SGE_F32) {
    switch (tile) {
      case 16: return launch_f32<16>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
      case 32: return launch_f32<32>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
      case 64: return launch_f32<64>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
      default: return launch_f32<128>(x, wg_t, n_tokens, d_model, d_ff, cap, count, idx, val, diag, st);
    }
  }
  return fail(SGE_ERR_UNSUPPORTED, "twell_gate_pack: dtype %d", dtype);
}
