// Dense bf16 gated FFN on tcgen05 tensor cores: the baseline the sparse path
// is measured against ("Sparser, Faster, Lighter Transformer Language
// Models", pwwt.cn summary: speed-ups are quoted against the dense model).
//
//   GEMM 1 (two accumulators, shared A tile):  G = x W_gate, U = x W_up,
//          epilogue h = bf16(ReLU(G) * U) -> h [N][F]
//   GEMM 2:  y = bf16(h W_down) with W_down given transposed (K-major).
#include "tc_launch.cuh"

namespace sge {

// Epilogue of GEMM 1: h = ReLU(g) * u, rounded to bf16, row-major [M][ldh].
struct EpiGated {
  uint16_t* h;
  int64_t n_rows;
  int n_cols;

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      uint32_t g[32], u[32];
      tmem_ld32(taddr + ch * 32, g);
      tmem_ld32(taddr + BN + ch * 32, u);
      tmem_ld_wait();
      const int col0 = n_blk * BN + ch * 32;
      if (row >= n_rows) continue;
      uint16_t* out = h + row * n_cols + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col0 + q * 8 + 8 > n_cols) break;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = q * 8 + 2 * i;
          const float h0 = fmaxf(__uint_as_float(g[k]), 0.0f) * __uint_as_float(u[k]);
          const float h1 = fmaxf(__uint_as_float(g[k + 1]), 0.0f) * __uint_as_float(u[k + 1]);
          w[i] = static_cast<uint32_t>(f32_to_bf16_bits(h0)) |
                 (static_cast<uint32_t>(f32_to_bf16_bits(h1)) << 16);
        }
        *reinterpret_cast<uint4*>(out + q * 8) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
};

// Plain epilogue: D rounded to bf16, row-major [M][ldo].
struct EpiStoreBf16 {
  uint16_t* out;
  int64_t n_rows;
  int n_cols;

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      uint32_t r[32];
      tmem_ld32(taddr + ch * 32, r);
      tmem_ld_wait();
      const int col0 = n_blk * BN + ch * 32;
      if (row >= n_rows) continue;
      uint16_t* o = out + row * n_cols + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col0 + q * 8 + 8 > n_cols) break;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = q * 8 + 2 * i;
          w[i] = static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[k]))) |
                 (static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[k + 1]))) << 16);
        }
        *reinterpret_cast<uint4*>(o + q * 8) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
};

}  // namespace sge

using namespace sge;

extern "C" int dense_ffn_fwd(const void* x, const void* wg_t, const void* wu_t, const void* wd_t,
                             void* h, void* y, int64_t n_tokens, int64_t d_model, int64_t d_ff,
                             int32_t* diag, void* stream) {
  NvtxRange nvtx_range("dense_ffn_fwd");
  clear_error();
  if (n_tokens < 0 || d_model < 1 || d_ff < 1) return fail(SGE_ERR_ARG, "dense_ffn_fwd: bad sizes");
  if (d_model % 8 || d_ff % 8) return fail(SGE_ERR_ARG, "dense_ffn_fwd: d_model and d_ff must be multiples of 8");
  if (d_ff >= (1LL << 31) || d_model >= (1LL << 31) || n_tokens >= (1LL << 31))
    return fail(SGE_ERR_UNSUPPORTED, "dense_ffn_fwd: size beyond 2^31");
  if (n_tokens == 0) return SGE_OK;
  if (!x || !wg_t || !wu_t || !wd_t || !h || !y) return fail(SGE_ERR_ARG, "dense_ffn_fwd: null pointer");
  if (!aligned16(x) || !aligned16(wg_t) || !aligned16(wu_t) || !aligned16(wd_t) || !aligned16(h) ||
      !aligned16(y))
    return fail(SGE_ERR_ARG, "dense_ffn_fwd: pointer not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  using S1 = TcPairShape<128, 2>;
  using S2 = TcPairShape<256, 1>;
  CUtensorMap mx, mg, mu, mh, md;
  int rc;
  if ((rc = make_tmap_bf16(&mx, x, n_tokens, d_model, d_model, kBM))) return rc;
  if ((rc = make_tmap_bf16(&mg, wg_t, d_ff, d_model, d_model, S1::BN / 2))) return rc;
  if ((rc = make_tmap_bf16(&mu, wu_t, d_ff, d_model, d_model, S1::BN / 2))) return rc;
  if ((rc = make_tmap_bf16(&mh, h, n_tokens, d_ff, d_ff, kBM))) return rc;
  if ((rc = make_tmap_bf16(&md, wd_t, d_model, d_ff, d_ff, S2::BN / 2))) return rc;
  EpiGated e1{static_cast<uint16_t*>(h), n_tokens, static_cast<int>(d_ff)};
  if ((rc = launch_tc_gemm_pair<S1>(mx, mg, mu, n_tokens, d_ff, d_model, e1, diag, st, "dense_ffn_fwd gate/up")))
    return rc;
  EpiStoreBf16 e2{static_cast<uint16_t*>(y), n_tokens, static_cast<int>(d_model)};
  return launch_tc_gemm_pair<S2>(mh, md, md, n_tokens, d_model, d_ff, e2, diag, st, "dense_ffn_fwd down");
}
