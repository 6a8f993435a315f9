// Hybrid sparse format for training: compact ELL rows plus a dense spill.
//
// "Sparser, Faster, Lighter Transformer Language Models": the pwwt.cn summary,
// section 03 and figure "基于混合格式的稀疏矩阵算子路由计算逻辑", routes tokens
// with few active gates to a highly compressed ELL matrix and the occasional
// highly active token to a dense backup path run on tensor cores; the
// kongchang.com page ("定制CUDA内核：融合与压缩") adds that TwELL is compressed
// into this hybrid form to minimise activation storage.
//
//   hybrid_pack     TwELL -> row nnz, routing (nnz <= K and no tile past its
//                   capacity: ELL row, else spill row, spill rows numbered in
//                   ascending token order), ELL columns and values, dense
//                   spill rows of a.
//   hybrid_ffn_fwd  ELL rows: the fused sparse up/down (u saved for the
//                   backward pass); spill rows: gathered and run as tcgen05
//                   GEMMs, U = X_s W_up (u saved, h = a (.) u), Y_s = H_s W_down,
//                   the rows scattered back into y.
#include "block_scan.cuh"
#include "debug_checks.cuh"
#include "sparse_common.cuh"
#include "spill_gemm.cuh"
#include "tc_launch.cuh"

namespace sge {

constexpr uint16_t kEllPad = 0xFFFF;
constexpr int kPackThreads = 1024;

struct HybridView {
  int64_t n;
  int f, k, s_max;
  int32_t* row_nnz;
  int32_t* spill_slot;
  int32_t* spill_rows;
  int32_t* n_spill;
  uint16_t* ell_idx;
  uint16_t* ell_a;
  uint16_t* ell_u;
  uint16_t* spill_a;
  uint16_t* spill_u;
};

// ---------------------------------------------------------------- pack

// Stored entries per row (counts capped at C), one thread per row.  A row
// that lost entries to the capacity (a tile with count > C) and would fit
// the ELL gets K + 1: it goes to the spill, where the forward can recompute
// it from the gate.
__global__ void __launch_bounds__(256) hybrid_nnz_kernel(const uint8_t* __restrict__ count, int nt,
                                                         int cap, HybridView hv) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (t >= hv.n) return;
  const uint8_t* c = count + t * nt;
  int nnz = 0;
  bool over = false;
  if ((nt & 3) == 0 && (reinterpret_cast<uintptr_t>(count) & 3) == 0) {
    const uint32_t* c4 = reinterpret_cast<const uint32_t*>(c);
    for (int b = 0; b < nt / 4; ++b) {
      const uint32_t v = __ldg(c4 + b);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int cb = static_cast<int>((v >> (8 * k)) & 255u);
        nnz += min(cb, cap);
        over |= cb > cap;
      }
    }
  } else {
    for (int b = 0; b < nt; ++b) {
      const int cb = __ldg(c + b);
      nnz += min(cb, cap);
      over |= cb > cap;
    }
  }
  hv.row_nnz[t] = over && nnz <= hv.k ? hv.k + 1 : nnz;
}

// One CTA: routing and the ascending ranks of the spill rows (block-wide
// exclusive scan over contiguous row ranges of the per-row counts; up to
// kRouteRegs rows per thread have their counts loaded together).
constexpr int kRouteRegs = 16;
__global__ void __launch_bounds__(kPackThreads) hybrid_route_kernel(HybridView hv, int32_t* diag) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  __shared__ int wsum[33];
  const int tid = threadIdx.x;
  const int64_t per = (hv.n + kPackThreads - 1) / kPackThreads;
  const int64_t r0 = min(hv.n, tid * per), r1 = min(hv.n, r0 + per);
  int total = 0;
  if (per <= kRouteRegs) {
    // up to kRouteRegs rows per thread: their counts loaded together
    bool heavy[kRouteRegs];
    int local = 0;
#pragma unroll
    for (int i = 0; i < kRouteRegs; ++i) {
      heavy[i] = r0 + i < r1 && hv.row_nnz[r0 + i] > hv.k;
      local += heavy[i];
    }
    int rank = block_scan_exclusive(local, wsum, &total);
#pragma unroll
    for (int i = 0; i < kRouteRegs; ++i) {
      if (r0 + i >= r1) break;
      int slot = -1;
      if (heavy[i]) {
        if (rank < hv.s_max) {
          slot = rank;
          hv.spill_rows[rank] = static_cast<int32_t>(r0 + i);
        }
        ++rank;
      }
      hv.spill_slot[r0 + i] = slot;
    }
  } else {
    int local = 0;
    for (int64_t t = r0; t < r1; ++t) local += hv.row_nnz[t] > hv.k;
    int rank = block_scan_exclusive(local, wsum, &total);
    for (int64_t t = r0; t < r1; ++t) {
      int slot = -1;
      if (hv.row_nnz[t] > hv.k) {
        if (rank < hv.s_max) {
          slot = rank;
          hv.spill_rows[rank] = static_cast<int32_t>(t);
        }
        ++rank;
      }
      hv.spill_slot[t] = slot;
    }
  }
  if (tid == kPackThreads - 1) {
    *hv.n_spill = total;
    if (diag) {
      atomicAdd(reinterpret_cast<int*>(diag + SGE_DIAG_SPILL_ROWS), total);
      if (total > hv.s_max) atomicAdd(reinterpret_cast<int*>(diag + SGE_DIAG_DROPPED_ROWS), total - hv.s_max);
    }
  }
}

// One warp per row: ELL rows get their entries in ascending column order
// (padding kEllPad / 0); kept spill rows get a dense row of a.
__global__ void __launch_bounds__(256) hybrid_fill_kernel(const uint8_t* __restrict__ count,
                                                          const uint8_t* __restrict__ idx,
                                                          const uint16_t* __restrict__ val,
                                                          int nt, int tile, int cap, HybridView hv) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= hv.n) return;
  const int nnz = hv.row_nnz[t];
  const bool ell = nnz <= hv.k;
  const int slot = hv.spill_slot[t];
  if (!ell && slot < 0) return;  // dropped
  uint16_t* dense = ell ? nullptr : hv.spill_a + static_cast<int64_t>(slot) * hv.f;
  if (!ell) {
    for (int j = lane * 8; j < hv.f; j += 32 * 8) *reinterpret_cast<uint4*>(dense + j) = make_uint4(0, 0, 0, 0);
    __syncwarp();
  }
  const uint8_t* c = count + t * nt;
  int base = 0;
  for (int b0 = 0; b0 < nt; b0 += 32) {
    const int b = b0 + lane;
    const int cb = b < nt ? min(static_cast<int>(c[b]), cap) : 0;
    int incl = cb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int off = base + incl - cb;
    const int64_t seg = t * nt + b;
    for (int s = 0; s < cb; ++s) {
      const int j = b * tile + clamp_index(idx[seg * cap + s], tile);
      const uint16_t a = val[seg * cap + s];
      if (ell) {
        hv.ell_idx[t * hv.k + off + s] = static_cast<uint16_t>(j);
        hv.ell_a[t * hv.k + off + s] = a;
      } else {
        dense[j] = a;
      }
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (ell)
    for (int e = nnz + lane; e < hv.k; e += 32) {
      hv.ell_idx[t * hv.k + e] = kEllPad;
      hv.ell_a[t * hv.k + e] = 0;
    }
}

// ------------------------------------------------------- ELL forward

constexpr int kEllThreads = 128;
constexpr int kEllWarps = kEllThreads / 32;
constexpr int kEllMaxK = 512;
constexpr int kEllBatch = 4;

struct EllFwdParams {
  const uint16_t* x;
  const uint16_t* wu_t;
  const uint16_t* wd;
  uint16_t* y;
  HybridView hv;
  int d;
};

// One CTA per token.  ELL rows: u for every entry (saved to ell_u, rounded
// to bf16), h = bf16(a u), y = sum h W_down[j].  Dropped rows: y = 0.  Spill
// rows are left to the spill GEMMs.
template <int NV>
__global__ void __launch_bounds__(kEllThreads) hybrid_ell_fwd_kernel(EllFwdParams p) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  using E = Elem<true>;
  constexpr int VEC = E::VEC;
  __shared__ int s_j[kEllMaxK];
  __shared__ float s_h[kEllMaxK];
  __shared__ float s_up[kEllWarps][kEllMaxK];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t = blockIdx.x;
  const int nvec = p.d / VEC;
  const int64_t row_bytes = static_cast<int64_t>(p.d) * 2;
  const int nnz = p.hv.row_nnz[t];
  uint4* yrow = reinterpret_cast<uint4*>(p.y + t * p.d);
  if (nnz > p.hv.k) {
    if (p.hv.spill_slot[t] < 0)
      for (int v = tid; v < nvec; v += kEllThreads) yrow[v] = make_uint4(0, 0, 0, 0);
    return;
  }
  uint4 xv[NV];
  float acc[NV][VEC];
  const uint4* xrow = reinterpret_cast<const uint4*>(p.x + t * p.d);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kEllThreads;
    xv[k] = v < nvec ? __ldg(xrow + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
  }
  for (int e = tid; e < nnz; e += kEllThreads) {
    s_j[e] = static_cast<int>(checked_index(p.hv.ell_idx[t * p.hv.k + e], p.hv.f));
    s_h[e] = __uint_as_float(static_cast<uint32_t>(p.hv.ell_a[t * p.hv.k + e]) << 16);
  }
  __syncthreads();
  // batches of kEllBatch entries: the W_up and the W_down rows of a batch are
  // loaded together (one memory round trip per batch), u is summed over the
  // warps' parts of d, then h = bf16(a u) feeds the down projection
  for (int e0 = 0; e0 < nnz; e0 += kEllBatch) {
    uint4 wu[kEllBatch][NV], wdv[kEllBatch][NV];
#pragma unroll
    for (int u = 0; u < kEllBatch; ++u) {
      const int e = e0 + u;
      const int j = e < nnz ? s_j[e] : -1;
      const int64_t off = static_cast<int64_t>(j) * row_bytes;
      const uint4* ur = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.wu_t) + off);
      const uint4* dr = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.wd) + off);
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int v = tid + k * kEllThreads;
        const bool in = j >= 0 && v < nvec;
        wu[u][k] = in ? __ldg(ur + v) : make_uint4(0, 0, 0, 0);
        wdv[u][k] = in ? __ldg(dr + v) : make_uint4(0, 0, 0, 0);
      }
    }
    float part[kEllBatch];
#pragma unroll
    for (int u = 0; u < kEllBatch; ++u) {
      float s = 0.0f;
#pragma unroll
      for (int k = 0; k < NV; ++k) s = E::dot(xv[k], wu[u][k], s);
      part[u] = s;
    }
    const float tot = warp_reduce_multi<kEllBatch>(part, lane);
    if ((lane & (32 / kEllBatch - 1)) == 0) {
      const int e = e0 + multi_entry<kEllBatch>(lane);
      if (e < nnz) s_up[warp][e] = tot;
    }
    __syncthreads();
    if (tid < kEllBatch && e0 + tid < nnz) {
      const int e = e0 + tid;
      float u = 0.0f;
#pragma unroll
      for (int w8 = 0; w8 < kEllWarps; ++w8) u += s_up[w8][e];
      p.hv.ell_u[t * p.hv.k + e] = f32_to_bf16_bits(u);
      s_h[e] = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_bits(s_h[e] * u)) << 16);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kEllBatch; ++u) {
      const int e = e0 + u;
      const uint16_t hb = e < nnz ? static_cast<uint16_t>(__float_as_uint(s_h[e]) >> 16) : 0;
#pragma unroll
      for (int k = 0; k < NV; ++k) E::axpy(hb, wdv[u][k], acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kEllThreads;
    if (v < nvec) yrow[v] = E::pack(acc[k]);
  }
}

// ------------------------------------------------------ spill forward

static HybridView view_of(const sge_hybrid* h) {
  HybridView v;
  v.n = h->n_tokens;
  v.f = static_cast<int>(h->d_ff);
  v.k = h->ell_cap;
  v.s_max = h->s_max;
  v.row_nnz = h->row_nnz;
  v.spill_slot = h->spill_slot;
  v.spill_rows = h->spill_rows;
  v.n_spill = h->n_spill;
  v.ell_idx = h->ell_idx;
  v.ell_a = static_cast<uint16_t*>(h->ell_a);
  v.ell_u = static_cast<uint16_t*>(h->ell_u);
  v.spill_a = static_cast<uint16_t*>(h->spill_a);
  v.spill_u = static_cast<uint16_t*>(h->spill_u);
  return v;
}

static int check_hybrid(const sge_hybrid* h, const char* fn) {
  if (!h) return fail(SGE_ERR_ARG, "%s: null hybrid descriptor", fn);
  if (h->n_tokens < 0 || h->d_ff < 1 || h->d_ff > 65535 || h->d_ff % 8)
    return fail(SGE_ERR_ARG, "%s: d_ff must be in [8, 65535] and a multiple of 8", fn);
  if (h->ell_cap < 0 || h->ell_cap > kEllMaxK)
    return fail(SGE_ERR_UNSUPPORTED, "%s: ELL capacity %d outside [0, %d]", fn, h->ell_cap, kEllMaxK);
  if (h->s_max < 0) return fail(SGE_ERR_ARG, "%s: negative spill capacity", fn);
  if (h->dtype != SGE_BF16) return fail(SGE_ERR_UNSUPPORTED, "%s: the hybrid path is bf16 only", fn);
  if (h->n_tokens == 0) return SGE_OK;
  if (!h->row_nnz || !h->spill_slot || !h->n_spill || !h->ell_idx || !h->ell_a ||
      (h->s_max > 0 && (!h->spill_rows || !h->spill_a)))
    return fail(SGE_ERR_ARG, "%s: null hybrid buffer", fn);
  if (!aligned16(h->spill_a) || !aligned16(h->spill_u))
    return fail(SGE_ERR_ARG, "%s: spill buffers must be 16-byte aligned", fn);
  return SGE_OK;
}

}  // namespace sge

using namespace sge;

extern "C" int hybrid_pack(const uint8_t* count, const uint8_t* idx, const void* val, int tile,
                           int cap, sge_hybrid* hy, int32_t* diag, void* stream) {
  NvtxRange nvtx_range("hybrid_pack");
  clear_error();
  int rc = check_hybrid(hy, "hybrid_pack");
  if (rc) return rc;
  if (tile < 1 || tile > 255 || hy->d_ff % tile || cap < 1 || cap > tile)
    return fail(SGE_ERR_ARG, "hybrid_pack: bad TwELL tile %d / capacity %d", tile, cap);
  if (hy->n_tokens == 0) return SGE_OK;
  if (!count || !idx || !val) return fail(SGE_ERR_ARG, "hybrid_pack: null TwELL buffer");
  if (hy->s_max > 0 && !aligned16(hy->spill_a))
    return fail(SGE_ERR_ARG, "hybrid_pack: spill_a must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const HybridView hv = view_of(hy);
  const int nt = static_cast<int>(hy->d_ff / tile);
  if ((rc = launch_pdl(hybrid_nnz_kernel, dim3(static_cast<unsigned>((hy->n_tokens + 255) / 256)), dim3(256), 0, st,
                       "hybrid_pack (counts)", count, nt, cap, hv)))
    return rc;
  if ((rc = launch_pdl(hybrid_route_kernel, dim3(1), dim3(kPackThreads), 0, st, "hybrid_pack (route)", hv, diag)))
    return rc;
  return launch_pdl(hybrid_fill_kernel, dim3(static_cast<unsigned>((hy->n_tokens + 7) / 8)), dim3(256), 0, st,
                    "hybrid_pack (fill)", count, idx, static_cast<const uint16_t*>(val), nt, tile, cap, hv);
}

extern "C" size_t hybrid_ffn_fwd_workspace_bytes(int64_t d_model, int64_t d_ff, int s_max) {
  if (d_model < 0 || d_ff < 0 || s_max < 0) return 0;
  if (s_max == 0) return 256;
  // X_s and H_s in bf16, then the split-K partial products and counters
  return align256(static_cast<size_t>(s_max) * static_cast<size_t>(d_model + d_ff) * 2) + kSplitPartBytes + 256;
}

template <int NV>
static int launch_ell_fwd(const EllFwdParams& p, int64_t n, cudaStream_t st) {
  return launch_pdl(hybrid_ell_fwd_kernel<NV>, dim3(static_cast<unsigned>(n)), dim3(kEllThreads), 0, st,
                    "hybrid_ffn_fwd (ELL rows)", p);
}

extern "C" int hybrid_ffn_fwd(const void* x, const sge_hybrid* hy, const void* wu_t, const void* wd,
                              const void* wd_t, const void* wg_t, void* y, int64_t d_model,
                              void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("hybrid_ffn_fwd");
  clear_error();
  int rc = check_hybrid(hy, "hybrid_ffn_fwd");
  if (rc) return rc;
  if (d_model < 8 || d_model % 8) return fail(SGE_ERR_ARG, "hybrid_ffn_fwd: d_model %% 8 != 0");
  if (hy->n_tokens == 0) return SGE_OK;
  if (!x || !wu_t || !wd || !y || !hy->ell_u || (hy->s_max > 0 && (!wd_t || !hy->spill_u)))
    return fail(SGE_ERR_ARG, "hybrid_ffn_fwd: null pointer");
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y) ||
      (wd_t && !aligned16(wd_t)) || (wg_t && !aligned16(wg_t)))
    return fail(SGE_ERR_ARG, "hybrid_ffn_fwd: pointer not 16-byte aligned");
  const size_t need = hybrid_ffn_fwd_workspace_bytes(d_model, hy->d_ff, hy->s_max);
  if (hy->s_max > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(SGE_ERR_ARG, "hybrid_ffn_fwd: workspace of %zu bytes, %zu needed (16-byte aligned)",
                workspace_bytes, need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const HybridView hv = view_of(hy);
  EllFwdParams p{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(wu_t),
                 static_cast<const uint16_t*>(wd), static_cast<uint16_t*>(y), hv,
                 static_cast<int>(d_model)};
  const int64_t nvec = d_model / 8;
  if (nvec <= kEllThreads) rc = launch_ell_fwd<1>(p, hy->n_tokens, st);
  else if (nvec <= 2 * kEllThreads) rc = launch_ell_fwd<2>(p, hy->n_tokens, st);
  else if (nvec <= 3 * kEllThreads) rc = launch_ell_fwd<3>(p, hy->n_tokens, st);
  else if (nvec <= 4 * kEllThreads) rc = launch_ell_fwd<4>(p, hy->n_tokens, st);
  else return fail(SGE_ERR_UNSUPPORTED, "hybrid_ffn_fwd: d_model %lld > 4096", (long long)d_model);
  if (rc || hy->s_max == 0) return rc;

  // spill rows: X_s gathered, U = X_s W_up (epilogue: u saved, h = a u),
  // Y_s = H_s W_down scattered to y.
  uint16_t* xs = static_cast<uint16_t*>(workspace);
  uint16_t* hs = xs + static_cast<size_t>(hy->s_max) * d_model;
  if ((rc = launch_pdl(gather_rows_kernel, dim3(hy->s_max), dim3(256), 0, st, "hybrid_ffn_fwd (gather)",
                       static_cast<const uint16_t*>(x), hy->spill_rows, hy->n_spill, hy->s_max,
                       static_cast<int>(d_model), xs)))
    return rc;
  using S = TcPairShape<256, 1, 2>;
  CUtensorMap ma, mb, mh, md;
  if ((rc = make_tmap_bf16(&ma, xs, hy->s_max, d_model, d_model, kBM))) return rc;
  if (wg_t) {
    // the gate recomputed with the up projection: [G | U] = X_s [W_gate | W_up]
    using S1 = TcPairShape<128, 2>;
    CUtensorMap mg;
    if ((rc = make_tmap_bf16(&mg, wg_t, hy->d_ff, d_model, d_model, S1::BN / 2))) return rc;
    if ((rc = make_tmap_bf16(&mb, wu_t, hy->d_ff, d_model, d_model, S1::BN / 2))) return rc;
    EpiSpillGateUp e1{static_cast<uint16_t*>(hy->spill_a), static_cast<uint16_t*>(hy->spill_u), hs,
                      hy->n_spill, hy->s_max, static_cast<int>(hy->d_ff)};
    if ((rc = launch_tc_gemm_pair<S1>(ma, mg, mb, hy->s_max, hy->d_ff, d_model, e1, nullptr, st,
                                      "hybrid_ffn_fwd (spill gate and up)")))
      return rc;
  } else {
    if ((rc = make_tmap_bf16(&mb, wu_t, hy->d_ff, d_model, d_model, S::BN / 2))) return rc;
    // few spill rows: K (= d) split over the CTA pairs, the parts finished by
    // split_spill_up_kernel (which shares the down GEMM's part area)
    float* part_up = reinterpret_cast<float*>(
        reinterpret_cast<char*>(workspace) +
        align256(static_cast<size_t>(hy->s_max) * static_cast<size_t>(d_model + hy->d_ff) * 2));
    const int tiles_up = static_cast<int>((hy->d_ff + S::BN - 1) / S::BN);
    EpiSpillUp e1{static_cast<const uint16_t*>(hy->spill_a), static_cast<uint16_t*>(hy->spill_u), hs,
                  hy->n_spill, hy->s_max, static_cast<int>(hy->d_ff), part_up, tiles_up, S::BN};
    if ((rc = launch_tc_gemm_pair<S>(ma, mb, mb, hy->s_max, hy->d_ff, d_model, e1, nullptr, st,
                                     "hybrid_ffn_fwd (spill up)", kSplitMax)))
      return rc;
    if ((rc = launch_pdl(split_spill_up_kernel, dim3(split_grid(hy->s_max, static_cast<int>(hy->d_ff))), dim3(256),
                         0, st, "hybrid_ffn_fwd (spill up part sums)", static_cast<const float*>(part_up),
                         static_cast<const uint16_t*>(hy->spill_a), static_cast<uint16_t*>(hy->spill_u), hs,
                         static_cast<const int32_t*>(hy->n_spill), hy->s_max, static_cast<int>(hy->d_ff),
                         tiles_up * S::BN)))
      return rc;
  }
  if ((rc = make_tmap_bf16(&mh, hs, hy->s_max, hy->d_ff, hy->d_ff, kBM))) return rc;
  if ((rc = make_tmap_bf16(&md, wd_t, d_model, hy->d_ff, hy->d_ff, S::BN / 2))) return rc;
  char* split_base = reinterpret_cast<char*>(workspace) +
                     align256(static_cast<size_t>(hy->s_max) * static_cast<size_t>(d_model + hy->d_ff) * 2);
  float* part = reinterpret_cast<float*>(split_base);
  const int tiles_n = static_cast<int>((d_model + S::BN - 1) / S::BN);
  EpiScatterRows e2{static_cast<uint16_t*>(y), hy->spill_rows, hy->n_spill, hy->s_max,
                    static_cast<int>(d_model), part, tiles_n, S::BN};
  if ((rc = launch_tc_gemm_pair<S>(mh, md, md, hy->s_max, d_model, hy->d_ff, e2, nullptr, st,
                                   "hybrid_ffn_fwd (spill down)", kSplitMax)))
    return rc;
  return launch_split_scatter(part, hy->spill_rows, hy->n_spill, hy->s_max, static_cast<int>(d_model),
                              tiles_n * S::BN, static_cast<uint16_t*>(y), st, "hybrid_ffn_fwd (split sum)");
}
