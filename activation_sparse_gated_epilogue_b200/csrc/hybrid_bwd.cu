// Backward pass of the gated FFN from the hybrid format.
//
// "Sparser, Faster, Lighter Transformer Language Models", pwwt.cn summary,
// section 03: training routes low-activity tokens to the compact ELL matrix
// and heavy tokens to a dense path on tensor cores, cutting dense compute and
// activation storage.  The pages print no backward formulas; these are the
// derivatives of y = sum_j a_j u_j W_down[j] with a_j = ReLU(g_j) > 0 at every
// stored entry (so dReLU = 1 there and entries not stored contribute 0):
//   dh_j = dy . W_down[j]     du_j = dh_j a_j     dg_j = dh_j u_j
//   dx   = sum_j du_j W_up[:, j] + dg_j W_gate[:, j]
//   dW_down[j] += a_j u_j dy   dW_up[:, j] += du_j x   dW_gate[:, j] += dg_j x
//
// ELL rows: one CTA per token computes dh (dot products with rows of
// W_down), du, dg (kept in fp32 for the weight gradients) and dx.  Spill
// rows: dH = dY_s W_down^T on tcgen05 (gathered rows; epilogue: dU = dH a,
// dG = dH u [a > 0], both bf16), then dX_s = [dU | dG] [W_up ; W_gate]^T on
// tcgen05, scattered to dx.  Weight gradients: every stored entry, of ELL and
// of spill rows alike (a spill row's entries are its active columns, a > 0),
// is bucketed by hidden unit (counting sort) and each unit's bucket ordered
// by token; one CTA per unit then sums its entries in ascending token order
// and writes the unit's three fp32 gradient rows once.  The result is
// deterministic.
#include "block_scan.cuh"
#include "debug_checks.cuh"
#include "sparse_common.cuh"
#include "spill_gemm.cuh"
#include "tc_launch.cuh"

namespace sge {

constexpr int kBwdThreads = 128;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdMaxK = 512;
constexpr int kBwdBatch = 4;

struct BwdHybrid {
  int64_t n;
  int f, k, s_max;
  const int32_t* row_nnz;
  const int32_t* spill_slot;
  const int32_t* spill_rows;
  const int32_t* n_spill;
  const uint16_t* ell_idx;
  const uint16_t* ell_a;
  const uint16_t* ell_u;
  const uint16_t* spill_a;
  const uint16_t* spill_u;
};

// Workspace carve-up (each piece 256-byte aligned).
struct BwdWs {
  float* du;         // [N][K]
  float* dg;         // [N][K]
  int* col_count;    // [F]
  int* col_start;    // [F + 1]
  int* col_cursor;   // [F]
  int2* csc;         // [N * K + S_max * F] (token, slot), bucketed by column; a spill
                     // row's entry has slot -(spill rank + 1)
  int2* csc_sorted;  // same, ascending token within a column
  uint16_t* dys;     // [Sp][d]   gathered dy of the kept spill rows
  uint16_t* acat;    // [Sp][2F]  dU | dG
  uint16_t* bcat;    // [d][2F]   W_up | W_gate (row i = row i of W_up, W_gate), when the
                     //           caller passes none
  float* part;       // split-K partial products of the dX GEMM
  size_t bytes;
};


static BwdWs carve(void* base, int64_t n, int64_t d, int64_t f, int k, int s_max) {
  BwdWs w{};
  const int64_t sp = (s_max + 63) / 64 * 64;  // spill rows padded for 16-byte TMA pitches
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = p ? p + off : nullptr;
    off += align256(bytes);
    return q;
  };
  const size_t nk = static_cast<size_t>(n) * static_cast<size_t>(k > 0 ? k : 1);
  const size_t ne = nk + static_cast<size_t>(s_max) * static_cast<size_t>(f);
  w.du = reinterpret_cast<float*>(take(nk * 4));
  w.dg = reinterpret_cast<float*>(take(nk * 4));
  w.col_count = reinterpret_cast<int*>(take(f * 4));
  w.col_start = reinterpret_cast<int*>(take((f + 1) * 4));
  w.col_cursor = reinterpret_cast<int*>(take(f * 4));
  w.csc = reinterpret_cast<int2*>(take(ne * 8));
  w.csc_sorted = reinterpret_cast<int2*>(take(ne * 8));
  if (s_max > 0) {
    w.dys = reinterpret_cast<uint16_t*>(take(sp * d * 2));
    w.acat = reinterpret_cast<uint16_t*>(take(sp * 2 * f * 2));
    w.bcat = reinterpret_cast<uint16_t*>(take(d * 2 * f * 2));
    w.part = reinterpret_cast<float*>(take(kSplitPartBytes));
  }
  w.bytes = off;
  return w;
}

// ---------------------------------------------------------- ELL rows

struct EllBwdParams {
  const uint16_t* x;
  const uint16_t* dy;
  const uint16_t* wg_t;
  const uint16_t* wu_t;
  const uint16_t* wd;
  uint16_t* dx;
  BwdHybrid hv;
  BwdWs ws;
  int d;
};

template <int NV>
__global__ void __launch_bounds__(kBwdThreads) ell_bwd_kernel(EllBwdParams p) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  using E = Elem<true>;
  constexpr int VEC = E::VEC;
  __shared__ int s_j[kBwdMaxK];
  __shared__ float s_c[2][kBwdMaxK];  // (a, u) -> (du, dg) rounded for dx
  __shared__ float s_part[kBwdWarps][kBwdMaxK];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t = blockIdx.x;
  const int nvec = p.d / VEC;
  const int64_t row_bytes = static_cast<int64_t>(p.d) * 2;
  const int nnz = p.hv.row_nnz[t];
  uint4* dxrow = reinterpret_cast<uint4*>(p.dx + t * p.d);
  if (nnz > p.hv.k) {  // spill rows: dx from the spill GEMMs; dropped rows: 0
    if (p.hv.spill_slot[t] < 0)
      for (int v = tid; v < nvec; v += kBwdThreads) dxrow[v] = make_uint4(0, 0, 0, 0);
    return;
  }
  uint4 dyv[NV];
  float acc[NV][VEC];
  const uint4* dyrow = reinterpret_cast<const uint4*>(p.dy + t * p.d);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kBwdThreads;
    dyv[k] = v < nvec ? __ldg(dyrow + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[k][q] = 0.0f;
  }
  const int64_t rk = t * p.hv.k;
  for (int e = tid; e < nnz; e += kBwdThreads) {
    s_j[e] = static_cast<int>(checked_index(p.hv.ell_idx[rk + e], p.hv.f));
    s_c[0][e] = __uint_as_float(static_cast<uint32_t>(p.hv.ell_a[rk + e]) << 16);
    s_c[1][e] = __uint_as_float(static_cast<uint32_t>(p.hv.ell_u[rk + e]) << 16);
  }
  __syncthreads();
  // batches of kBwdBatch entries: the W_down, W_up and W_gate rows of a
  // batch are loaded together (one memory round trip per batch);
  // dh_e = dy . W_down[j_e] is summed over the warps' parts of d, then
  // du = dh a, dg = dh u and dx += du W_up[:, j] + dg W_gate[:, j]
  // (coefficients rounded to bf16)
  for (int e0 = 0; e0 < nnz; e0 += kBwdBatch) {
    uint4 wdv[kBwdBatch][NV], wu[kBwdBatch][NV], wg[kBwdBatch][NV];
#pragma unroll
    for (int u = 0; u < kBwdBatch; ++u) {
      const int e = e0 + u;
      const int j = e < nnz ? s_j[e] : -1;
      const int64_t off = static_cast<int64_t>(j) * row_bytes;
      const uint4* rd = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.wd) + off);
      const uint4* ru = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.wu_t) + off);
      const uint4* rg = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.wg_t) + off);
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int v = tid + k * kBwdThreads;
        const bool ok = j >= 0 && v < nvec;
        wdv[u][k] = ok ? __ldg(rd + v) : make_uint4(0, 0, 0, 0);
        wu[u][k] = ok ? __ldg(ru + v) : make_uint4(0, 0, 0, 0);
        wg[u][k] = ok ? __ldg(rg + v) : make_uint4(0, 0, 0, 0);
      }
    }
    float part[kBwdBatch];
#pragma unroll
    for (int u = 0; u < kBwdBatch; ++u) {
      float s = 0.0f;
#pragma unroll
      for (int k = 0; k < NV; ++k) s = E::dot(dyv[k], wdv[u][k], s);
      part[u] = s;
    }
    const float tot = warp_reduce_multi<kBwdBatch>(part, lane);
    if ((lane & (32 / kBwdBatch - 1)) == 0) {
      const int e = e0 + multi_entry<kBwdBatch>(lane);
      if (e < nnz) s_part[warp][e] = tot;
    }
    __syncthreads();
    if (tid < kBwdBatch && e0 + tid < nnz) {
      const int e = e0 + tid;
      float dh = 0.0f;
#pragma unroll
      for (int w8 = 0; w8 < kBwdWarps; ++w8) dh += s_part[w8][e];
      const float du = dh * s_c[0][e], dg = dh * s_c[1][e];
      p.ws.du[rk + e] = du;
      p.ws.dg[rk + e] = dg;
      s_c[0][e] = du;
      s_c[1][e] = dg;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kBwdBatch; ++u) {
      const int e = e0 + u;
      const uint16_t cu = e < nnz ? f32_to_bf16_bits(s_c[0][e]) : 0;
      const uint16_t cg = e < nnz ? f32_to_bf16_bits(s_c[1][e]) : 0;
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        E::axpy(cu, wu[u][k], acc[k]);
        E::axpy(cg, wg[u][k], acc[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kBwdThreads;
    if (v < nvec) dxrow[v] = E::pack(acc[k]);
  }
}

// ------------------------------------------------- column buckets (CSC)

__global__ void __launch_bounds__(256) csc_count_kernel(BwdHybrid hv, int* col_count) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= hv.n) return;
  const int nnz = hv.row_nnz[t];
  if (nnz > hv.k) return;
  for (int e = lane; e < nnz; e += 32) atomicAdd(&col_count[checked_index(hv.ell_idx[t * hv.k + e], hv.f)], 1);
}

// One CTA: exclusive scan of the column counts.
// Bucket starts: an exclusive scan of the column counts, 1024 threads with
// `per` consecutive columns each.  Up to kScanRegs columns per thread are
// loaded together into registers (one memory round trip), then scanned.
constexpr int kScanRegs = 16;

__global__ void __launch_bounds__(1024) csc_scan_kernel(const int* col_count, int f, int* col_start,
                                                        int* col_cursor) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  __shared__ int wsum[33];
  const int tid = threadIdx.x;
  const int per = (f + 1023) / 1024;  // consecutive columns per thread
  const int c0 = min(f, tid * per), c1 = min(f, c0 + per);
  int total = 0;
  if (per <= kScanRegs) {
    int v[kScanRegs];
#pragma unroll
    for (int i = 0; i < kScanRegs; ++i) v[i] = c0 + i < c1 ? __ldg(col_count + c0 + i) : 0;
    int local = 0;
#pragma unroll
    for (int i = 0; i < kScanRegs; ++i) local += v[i];
    int run = block_scan_exclusive(local, wsum, &total);
#pragma unroll
    for (int i = 0; i < kScanRegs; ++i)
      if (c0 + i < c1) {
        col_start[c0 + i] = run;
        col_cursor[c0 + i] = run;
        run += v[i];
      }
  } else {
    int local = 0;
    for (int c = c0; c < c1; ++c) local += __ldg(col_count + c);
    int run = block_scan_exclusive(local, wsum, &total);
    for (int c = c0; c < c1; ++c) {
      col_start[c] = run;
      col_cursor[c] = run;
      run += __ldg(col_count + c);
    }
  }
  if (tid == 1023) col_start[f] = total;
}

__global__ void __launch_bounds__(256) csc_scatter_kernel(BwdHybrid hv, int* col_cursor, int2* csc) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= hv.n) return;
  const int nnz = hv.row_nnz[t];
  if (nnz > hv.k) return;
  for (int e = lane; e < nnz; e += 32) {
    const int pos = atomicAdd(&col_cursor[checked_index(hv.ell_idx[t * hv.k + e], hv.f)], 1);
    csc[pos] = make_int2(static_cast<int>(t), e);
  }
}

// Entries of the kept spill rows (their active columns, a > 0): counted per
// column, then scattered with slot -(spill rank + 1).  Grid: (F / 2048
// chunks) x (S_max ranks); eight columns per thread.
__global__ void __launch_bounds__(256) csc_count_spill_kernel(BwdHybrid hv, int* col_count) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int r = blockIdx.y;
  if (r >= min(*hv.n_spill, hv.s_max)) return;
  const int j0 = (blockIdx.x * 256 + threadIdx.x) * 8;
  if (j0 >= hv.f) return;
  const uint4 av = *reinterpret_cast<const uint4*>(hv.spill_a + static_cast<int64_t>(r) * hv.f + j0);
  const uint32_t w[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (__uint_as_float(w[i] << 16) > 0.0f) atomicAdd(&col_count[j0 + 2 * i], 1);
    if (__uint_as_float(w[i] & 0xFFFF0000u) > 0.0f) atomicAdd(&col_count[j0 + 2 * i + 1], 1);
  }
}

__global__ void __launch_bounds__(256) csc_scatter_spill_kernel(BwdHybrid hv, int* col_cursor, int2* csc) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int r = blockIdx.y;
  if (r >= min(*hv.n_spill, hv.s_max)) return;
  const int j0 = (blockIdx.x * 256 + threadIdx.x) * 8;
  if (j0 >= hv.f) return;
  const int t = hv.spill_rows[r];
  const uint4 av = *reinterpret_cast<const uint4*>(hv.spill_a + static_cast<int64_t>(r) * hv.f + j0);
  const uint32_t w[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (__uint_as_float(h ? (w[i] & 0xFFFF0000u) : (w[i] << 16)) > 0.0f) {
        const int pos = atomicAdd(&col_cursor[j0 + 2 * i + h], 1);
        csc[pos] = make_int2(t, -(r + 1));
      }
}

// Per column (one warp): order the bucket by token.  Tokens are unique in a
// column, so an entry's position is the number of smaller tokens.
__global__ void __launch_bounds__(256) csc_sort_kernel(const int* col_start, int f, const int2* csc,
                                                       int2* sorted) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int c = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= f) return;
  const int s0 = col_start[c], n = col_start[c + 1] - s0;
  for (int i = lane; i < n; i += 32) {
    const int2 me = csc[s0 + i];
    int rank = 0;
    for (int m = 0; m < n; ++m) rank += csc[s0 + m].x < me.x;
    sorted[s0 + rank] = me;
  }
}

// Per column j (one CTA): weight-gradient rows from the column's entries (ELL
// and spill rows), summed in ascending token order, written (overwriting) in
// fp32.
struct DwParams {
  const uint16_t* x;
  const uint16_t* dy;
  BwdHybrid hv;
  BwdWs ws;
  float* dwg_t;
  float* dwu_t;
  float* dwd;
  int d;
};

constexpr int kDwStage = 256;  // entries of a column whose metadata is staged at once

template <int NV>
__global__ void __launch_bounds__(kBwdThreads) dw_ell_kernel(DwParams p) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  constexpr int VEC = 8;
  // the entries' tokens and (h, du, dg), loaded for a whole round of the
  // column's bucket by all threads at once; the rows of x and dy then
  // stream two entries at a time
  __shared__ int s_t[kDwStage];
  __shared__ float s_h[kDwStage], s_du[kDwStage], s_dg[kDwStage];
  const int j = blockIdx.x;
  const int tid = threadIdx.x;
  const int nvec = p.d / VEC;
  float ad[NV][VEC], au[NV][VEC], ag[NV][VEC];
#pragma unroll
  for (int k = 0; k < NV; ++k)
#pragma unroll
    for (int q = 0; q < VEC; ++q) ad[k][q] = au[k][q] = ag[k][q] = 0.0f;
  const int s0 = p.ws.col_start[j], s1 = p.ws.col_start[j + 1];
  for (int r0 = s0; r0 < s1; r0 += kDwStage) {
    const int rn = min(kDwStage, s1 - r0);
    __syncthreads();  // the previous round's metadata has been used
    for (int i = tid; i < rn; i += kBwdThreads) {
      int2 te = p.ws.csc_sorted[r0 + i];
      te.x = static_cast<int>(checked_index(te.x, p.hv.n));
      if (te.y >= 0) te.y = static_cast<int>(checked_index(te.y, p.hv.k));
      else te.y = -1 - static_cast<int>(checked_index(-te.y - 1, p.hv.s_max));
      float a, u, du, dg;
      if (te.y >= 0) {  // an ELL entry: slot te.y of row te.x
        const int64_t rk = static_cast<int64_t>(te.x) * p.hv.k + te.y;
        a = __uint_as_float(static_cast<uint32_t>(p.hv.ell_a[rk]) << 16);
        u = __uint_as_float(static_cast<uint32_t>(p.hv.ell_u[rk]) << 16);
        du = p.ws.du[rk];
        dg = p.ws.dg[rk];
      } else {  // an active column of spill rank -te.y - 1
        const int64_t r = -te.y - 1;
        a = __uint_as_float(static_cast<uint32_t>(p.hv.spill_a[r * p.hv.f + j]) << 16);
        u = __uint_as_float(static_cast<uint32_t>(p.hv.spill_u[r * p.hv.f + j]) << 16);
        du = __uint_as_float(static_cast<uint32_t>(p.ws.acat[r * 2 * p.hv.f + j]) << 16);
        dg = __uint_as_float(static_cast<uint32_t>(p.ws.acat[r * 2 * p.hv.f + p.hv.f + j]) << 16);
      }
      s_t[i] = te.x;
      s_h[i] = a * u;
      s_du[i] = du;
      s_dg[i] = dg;
    }
    __syncthreads();
    for (int i = 0; i < rn; i += 2) {
      const bool two = i + 1 < rn;
      const uint4* dyr0 = reinterpret_cast<const uint4*>(p.dy + static_cast<int64_t>(s_t[i]) * p.d);
      const uint4* xr0 = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(s_t[i]) * p.d);
      const uint4* dyr1 = reinterpret_cast<const uint4*>(p.dy + static_cast<int64_t>(s_t[two ? i + 1 : i]) * p.d);
      const uint4* xr1 = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(s_t[two ? i + 1 : i]) * p.d);
      uint4 y0[NV], x0[NV], y1[NV], x1[NV];
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int v = tid + k * kBwdThreads;
        const bool in = v < nvec;
        y0[k] = in ? __ldg(dyr0 + v) : make_uint4(0, 0, 0, 0);
        x0[k] = in ? __ldg(xr0 + v) : make_uint4(0, 0, 0, 0);
        y1[k] = in && two ? __ldg(dyr1 + v) : make_uint4(0, 0, 0, 0);
        x1[k] = in && two ? __ldg(xr1 + v) : make_uint4(0, 0, 0, 0);
      }
      // entry i, then entry i + 1: the sums keep ascending token order
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (e == 1 && !two) break;
        const float h = s_h[i + e], du = s_du[i + e], dg = s_dg[i + e];
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const uint4 yv = e ? y1[k] : y0[k], xv = e ? x1[k] : x0[k];
          const uint32_t ys[4] = {yv.x, yv.y, yv.z, yv.w}, xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float ya = __uint_as_float(ys[q] << 16), yb = __uint_as_float(ys[q] & 0xFFFF0000u);
            const float xa = __uint_as_float(xs[q] << 16), xb = __uint_as_float(xs[q] & 0xFFFF0000u);
            ad[k][2 * q] = fmaf(h, ya, ad[k][2 * q]);
            ad[k][2 * q + 1] = fmaf(h, yb, ad[k][2 * q + 1]);
            au[k][2 * q] = fmaf(du, xa, au[k][2 * q]);
            au[k][2 * q + 1] = fmaf(du, xb, au[k][2 * q + 1]);
            ag[k][2 * q] = fmaf(dg, xa, ag[k][2 * q]);
            ag[k][2 * q + 1] = fmaf(dg, xb, ag[k][2 * q + 1]);
          }
        }
      }
    }
  }
  const int64_t base = static_cast<int64_t>(j) * p.d;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = tid + k * kBwdThreads;
    if (v >= nvec) continue;
    float4* od = reinterpret_cast<float4*>(p.dwd + base) + 2 * v;
    float4* ou = reinterpret_cast<float4*>(p.dwu_t + base) + 2 * v;
    float4* og = reinterpret_cast<float4*>(p.dwg_t + base) + 2 * v;
    od[0] = make_float4(ad[k][0], ad[k][1], ad[k][2], ad[k][3]);
    od[1] = make_float4(ad[k][4], ad[k][5], ad[k][6], ad[k][7]);
    ou[0] = make_float4(au[k][0], au[k][1], au[k][2], au[k][3]);
    ou[1] = make_float4(au[k][4], au[k][5], au[k][6], au[k][7]);
    og[0] = make_float4(ag[k][0], ag[k][1], ag[k][2], ag[k][3]);
    og[1] = make_float4(ag[k][4], ag[k][5], ag[k][6], ag[k][7]);
  }
}

// -------------------------------------------------------- spill rows

// dst[c][col_off + r] = src[r][c] for r < rows, c < cols (bf16, 32x32 tiles).
__global__ void __launch_bounds__(256) transpose_kernel(const uint16_t* __restrict__ src, int rows,
                                                        int cols, int64_t src_pitch, uint16_t* dst,
                                                        int64_t dst_pitch, int col_off,
                                                        const int32_t* rows_dev, int rows_cap) {
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  // 64 x 64 tiles moved with 16-byte loads and stores (rows, cols, pitches,
  // col_off and the row limit are multiples of 8); the shared tile's row
  // pitch of 66 elements keeps the column reads off one bank
  __shared__ uint16_t tile[64][66];
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
  // with rows_dev, only the first min(*rows_dev, rows_cap) rows rounded up to
  // 64 are transposed (the K that the later GEMMs read)
  if (rows_dev) rows = min(rows, (min(*rows_dev, rows_cap) + 63) / 64 * 64);
  if (r0 >= rows) return;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int id = threadIdx.x + 256 * h;
    const int r = id >> 3, c8 = (id & 7) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r0 + r < rows && c0 + c8 < cols)
      v = *reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r0 + r) * src_pitch + c0 + c8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      tile[r][c8 + 2 * k] = static_cast<uint16_t>(w[k] & 0xFFFFu);
      tile[r][c8 + 2 * k + 1] = static_cast<uint16_t>(w[k] >> 16);
    }
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int id = threadIdx.x + 256 * h;
    const int c = id >> 3, r8 = (id & 7) * 8;  // destination row c0 + c, columns r0 + r8 ..
    if (c0 + c >= cols || r0 + r8 >= rows) continue;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[k] = static_cast<uint32_t>(tile[r8 + 2 * k][c]) | (static_cast<uint32_t>(tile[r8 + 2 * k + 1][c]) << 16);
    *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(c0 + c) * dst_pitch + col_off + r0 + r8) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Epilogue of dH = dY_s W_down^T: dU = dH a, dG = dH u [a > 0] -> acat
// (dU in columns [0, F), dG in [F, 2F)); zero rows past the kept spill rows.
struct EpiBwdSpill {
  const uint16_t* spill_a;
  const uint16_t* spill_u;
  uint16_t* acat;
  const int32_t* n_spill;
  int s_max;
  int f;
  int64_t m_rows;  // rows of the padded spill buffers
  float* part = nullptr;  // split-K parts (split_bwd_spill_kernel finishes them)
  int n_tiles_n = 1;
  int tile_n = 256;

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

  // rows up to the kept spill rows rounded up to 64 (the K the later GEMMs
  // read): the zero rows past the kept ones matter only that far
  __device__ __forceinline__ int m_limit(int m) const {
    const int c = min(*n_spill, s_max);
    return min(m, (c + 63) / 64 * 64);
  }

  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int64_t row, int n_blk, int lane) const {
    const int kept = min(*n_spill, s_max);
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
      uint32_t r[32];
      tmem_ld32(taddr + ch * 32, r);
      tmem_ld_wait();
      if (row >= m_rows) continue;
      const int col0 = n_blk * BN + ch * 32;
      const int64_t off = row * f + col0;
      const int64_t offc = row * 2 * f + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col0 + q * 8 + 8 > f) break;
        uint32_t du[4] = {0, 0, 0, 0}, dg[4] = {0, 0, 0, 0};
        if (row < kept) {
          const uint4 av = *reinterpret_cast<const uint4*>(spill_a + off + q * 8);
          const uint4 uv = *reinterpret_cast<const uint4*>(spill_u + off + q * 8);
          const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float o[2][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float dh = __uint_as_float(r[q * 8 + 2 * i + h]);
              const float a = __uint_as_float(h ? (aw[i] & 0xFFFF0000u) : (aw[i] << 16));
              const float u = __uint_as_float(h ? (uw[i] & 0xFFFF0000u) : (uw[i] << 16));
              o[h][0] = dh * a;
              o[h][1] = a > 0.0f ? dh * u : 0.0f;
            }
            du[i] = static_cast<uint32_t>(f32_to_bf16_bits(o[0][0])) | (static_cast<uint32_t>(f32_to_bf16_bits(o[1][0])) << 16);
            dg[i] = static_cast<uint32_t>(f32_to_bf16_bits(o[0][1])) | (static_cast<uint32_t>(f32_to_bf16_bits(o[1][1])) << 16);
          }
        }
        *reinterpret_cast<uint4*>(acat + offc + q * 8) = make_uint4(du[0], du[1], du[2], du[3]);
        *reinterpret_cast<uint4*>(acat + offc + f + q * 8) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
      }
    }
  }
};

// Finishes a split dH = dY_s W_down: dh = the parts summed in part order,
// dU = bf16(dh a), dG = bf16(dh u) where a > 0 (else 0), for the kept rows,
// and zero rows up to the kept rows rounded up to 64 (the K the later GEMMs
// read); nothing when the GEMM did not split.  A thread per 8 columns.
static __global__ void __launch_bounds__(256) split_bwd_spill_kernel(const float* __restrict__ part,
                                                                     const uint16_t* __restrict__ spill_a,
                                                                     const uint16_t* __restrict__ spill_u,
                                                                     uint16_t* __restrict__ acat,
                                                                     const int32_t* __restrict__ n_spill,
                                                                     int s_max, int f, int ncp) {
  grid_dep_wait();  // the parts come from the GEMM before
  grid_dep_launch();
  const int nsplit = split_word_read(part);
  const int kept = min(*n_spill, s_max);
  if (nsplit <= 1 || kept <= 0) return;
  const int64_t rows_pad = static_cast<int64_t>((kept + 255) / 256) * 256;
  const int64_t rows = (kept + 63) / 64 * 64;
  const int per_row = f / 8;
  const int64_t total = rows * per_row;
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t r = i / per_row;
    const int c = static_cast<int>(i % per_row) * 8;
    uint32_t du[4] = {0, 0, 0, 0}, dg[4] = {0, 0, 0, 0};
    if (r < kept) {
      float dh[8];
      sum_parts8(part, nsplit, rows_pad, ncp, r, c, dh);
      const uint4 av = *reinterpret_cast<const uint4*>(spill_a + r * f + c);
      const uint4 uv = *reinterpret_cast<const uint4*>(spill_u + r * f + c);
      const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float o[2][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float a = __uint_as_float(h ? (aw[k] & 0xFFFF0000u) : (aw[k] << 16));
          const float u = __uint_as_float(h ? (uw[k] & 0xFFFF0000u) : (uw[k] << 16));
          o[h][0] = dh[2 * k + h] * a;
          o[h][1] = a > 0.0f ? dh[2 * k + h] * u : 0.0f;
        }
        du[k] = static_cast<uint32_t>(f32_to_bf16_bits(o[0][0])) | (static_cast<uint32_t>(f32_to_bf16_bits(o[1][0])) << 16);
        dg[k] = static_cast<uint32_t>(f32_to_bf16_bits(o[0][1])) | (static_cast<uint32_t>(f32_to_bf16_bits(o[1][1])) << 16);
      }
    }
    *reinterpret_cast<uint4*>(acat + r * 2 * f + c) = make_uint4(du[0], du[1], du[2], du[3]);
    *reinterpret_cast<uint4*>(acat + r * 2 * f + f + c) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
  }
}

static int launch_transpose(const uint16_t* src, int rows, int cols, int64_t src_pitch,
                            uint16_t* dst, int64_t dst_pitch, int col_off, cudaStream_t st,
                            const int32_t* rows_dev = nullptr, int rows_cap = 0) {
  dim3 grid((cols + 63) / 64, (rows + 63) / 64);
  return launch_pdl(transpose_kernel, grid, dim3(256), 0, st, "hybrid_ffn_bwd (transpose)", src, rows, cols,
                    src_pitch, dst, dst_pitch, col_off, rows_dev, rows_cap);
}

template <int NV>
static int launch_ell_bwd(const EllBwdParams& p, int64_t n, cudaStream_t st) {
  return launch_pdl(ell_bwd_kernel<NV>, dim3(static_cast<unsigned>(n)), dim3(kBwdThreads), 0, st,
                    "hybrid_ffn_bwd (ELL rows)", p);
}

template <int NV>
static int launch_dw(const DwParams& q, int f, cudaStream_t st) {
  return launch_pdl(dw_ell_kernel<NV>, dim3(f), dim3(kBwdThreads), 0, st, "hybrid_ffn_bwd (weight gradients)", q);
}

}  // namespace sge

using namespace sge;

extern "C" size_t hybrid_ffn_bwd_workspace_bytes(int64_t n_tokens, int64_t d_model, int64_t d_ff,
                                                 int ell_cap, int s_max) {
  if (n_tokens < 0 || d_model < 0 || d_ff < 0 || ell_cap < 0 || s_max < 0) return 0;
  return carve(nullptr, n_tokens, d_model, d_ff, ell_cap, s_max).bytes;
}

// [W_up | W_gate] as the dX GEMM's K-major B operand: w_ug[i][j] =
// W_up[i][j] = wu_t[j][i], w_ug[i][F + j] = W_gate[i][j] = wg_t[j][i].
static int build_up_gate(const void* wu_t, const void* wg_t, uint16_t* w_ug, int64_t f, int64_t d,
                         cudaStream_t st) {
  int rc = launch_transpose(static_cast<const uint16_t*>(wu_t), static_cast<int>(f), static_cast<int>(d), d,
                            w_ug, 2 * f, 0, st);
  if (rc) return rc;
  return launch_transpose(static_cast<const uint16_t*>(wg_t), static_cast<int>(f), static_cast<int>(d), d,
                          w_ug, 2 * f, static_cast<int>(f), st);
}

extern "C" int sge_transpose_up_gate(const void* wu_t, const void* wg_t, void* w_ug, int64_t d_ff,
                                     int64_t d_model, void* stream) {
  NvtxRange nvtx_range("sge_transpose_up_gate");
  clear_error();
  if (d_ff < 8 || d_ff % 8 || d_model < 8 || d_model % 8 || d_ff > (1 << 30) || d_model > (1 << 30))
    return fail(SGE_ERR_ARG, "sge_transpose_up_gate: d_ff and d_model must be multiples of 8");
  if (!wu_t || !wg_t || !w_ug) return fail(SGE_ERR_ARG, "sge_transpose_up_gate: null pointer");
  if (!aligned16(wu_t) || !aligned16(wg_t) || !aligned16(w_ug))
    return fail(SGE_ERR_ARG, "sge_transpose_up_gate: pointer not 16-byte aligned");
  return build_up_gate(wu_t, wg_t, static_cast<uint16_t*>(w_ug), d_ff, d_model,
                       static_cast<cudaStream_t>(stream));
}

extern "C" int hybrid_ffn_bwd(const void* x, const void* dy, const sge_hybrid* hy,
                              const void* wg_t, const void* wu_t, const void* wd, const void* w_ug,
                              void* dx, float* dwg_t, float* dwu_t, float* dwd, int64_t d_model,
                              void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("hybrid_ffn_bwd");
  clear_error();
  if (!hy) return fail(SGE_ERR_ARG, "hybrid_ffn_bwd: null hybrid descriptor");
  if (hy->dtype != SGE_BF16) return fail(SGE_ERR_UNSUPPORTED, "hybrid_ffn_bwd: bf16 only");
  if (hy->n_tokens < 0 || hy->d_ff < 8 || hy->d_ff > 65535 || hy->d_ff % 8 || hy->ell_cap < 0 ||
      hy->ell_cap > kBwdMaxK || hy->s_max < 0)
    return fail(SGE_ERR_ARG, "hybrid_ffn_bwd: bad hybrid sizes");
  if (d_model < 8 || d_model % 8) return fail(SGE_ERR_ARG, "hybrid_ffn_bwd: d_model %% 8 != 0");
  if (d_model > 4 * kBwdThreads * 8)
    return fail(SGE_ERR_UNSUPPORTED, "hybrid_ffn_bwd: d_model %lld > 4096", (long long)d_model);
  const int64_t n = hy->n_tokens, f = hy->d_ff, d = d_model;
  const int k = hy->ell_cap, s_max = hy->s_max;
  if (!x || !dy || !wg_t || !wu_t || !wd || !dx || !dwg_t || !dwu_t || !dwd)
    return fail(SGE_ERR_ARG, "hybrid_ffn_bwd: null pointer");
  if (!aligned16(x) || !aligned16(dy) || !aligned16(wg_t) || !aligned16(wu_t) || !aligned16(wd) ||
      !aligned16(dx) || !aligned16(dwg_t) || !aligned16(dwu_t) || !aligned16(dwd) || (w_ug && !aligned16(w_ug)))
    return fail(SGE_ERR_ARG, "hybrid_ffn_bwd: pointer not 16-byte aligned");
  const BwdWs need = carve(nullptr, n, d, f, k, s_max);
  if (!workspace || workspace_bytes < need.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(SGE_ERR_ARG, "hybrid_ffn_bwd: workspace of %zu bytes, %zu needed (256-byte aligned)",
                workspace_bytes, need.bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n == 0) {
    cudaMemsetAsync(dwg_t, 0, sizeof(float) * f * d, st);
    cudaMemsetAsync(dwu_t, 0, sizeof(float) * f * d, st);
    cudaMemsetAsync(dwd, 0, sizeof(float) * f * d, st);
    return check_launch("hybrid_ffn_bwd (zero gradients)");
  }
  const BwdWs ws = carve(workspace, n, d, f, k, s_max);
  BwdHybrid hv{n, static_cast<int>(f), k, s_max, hy->row_nnz, hy->spill_slot, hy->spill_rows,
               hy->n_spill, hy->ell_idx, static_cast<const uint16_t*>(hy->ell_a),
               static_cast<const uint16_t*>(hy->ell_u), static_cast<const uint16_t*>(hy->spill_a),
               static_cast<const uint16_t*>(hy->spill_u)};
  const auto* xb = static_cast<const uint16_t*>(x);
  const auto* dyb = static_cast<const uint16_t*>(dy);
  const int64_t nvec = d / 8;
  const int sp = (s_max + 63) / 64 * 64;
  int rc;
  // ---- ELL rows: dh, du, dg, dx
  EllBwdParams p{xb, dyb, static_cast<const uint16_t*>(wg_t), static_cast<const uint16_t*>(wu_t),
                 static_cast<const uint16_t*>(wd), static_cast<uint16_t*>(dx), hv, ws, static_cast<int>(d)};
  if (nvec <= kBwdThreads) rc = launch_ell_bwd<1>(p, n, st);
  else if (nvec <= 2 * kBwdThreads) rc = launch_ell_bwd<2>(p, n, st);
  else if (nvec <= 3 * kBwdThreads) rc = launch_ell_bwd<3>(p, n, st);
  else rc = launch_ell_bwd<4>(p, n, st);
  if (rc) return rc;
  // ---- spill rows: dH = dY_s W_down^T on tensor cores, epilogue dU | dG
  using Sh = TcPairShape<256, 1, 2>;  // N = F: with few spill rows K is split over the CTA pairs
  using Sx = TcPairShape<256, 1, 2>;  // N = d: few tiles, K = 2F split over the CTA pairs
  if (s_max > 0) {
    if ((rc = launch_pdl(gather_rows_kernel, dim3(sp), dim3(256), 0, st, "hybrid_ffn_bwd (gather)", dyb,
                         hy->spill_rows, hy->n_spill, s_max, static_cast<int>(d), ws.dys)))
      return rc;
    CUtensorMap m1a, m1b;
    if ((rc = make_tmap_bf16(&m1a, ws.dys, sp, d, d, kBM))) return rc;
    if ((rc = make_tmap_bf16(&m1b, wd, f, d, d, Sh::BN / 2))) return rc;
    // few spill rows: K (= d) split over the CTA pairs, the parts finished by
    // split_bwd_spill_kernel (the part area is the dX GEMM's, used later)
    const int tiles_h = static_cast<int>((f + Sh::BN - 1) / Sh::BN);
    EpiBwdSpill e1{hv.spill_a, hv.spill_u, ws.acat, hy->n_spill, s_max, static_cast<int>(f), sp,
                   ws.part, tiles_h, Sh::BN};
    if ((rc = launch_tc_gemm_pair<Sh>(m1a, m1b, m1b, sp, f, d, e1, nullptr, st, "hybrid_ffn_bwd (dH)",
                                      kSplitMax)))
      return rc;
    if ((rc = launch_pdl(split_bwd_spill_kernel, dim3(split_grid(sp, static_cast<int>(f))), dim3(256), 0, st,
                         "hybrid_ffn_bwd (dH part sums)", static_cast<const float*>(ws.part), hv.spill_a,
                         hv.spill_u, ws.acat, static_cast<const int32_t*>(hy->n_spill), s_max,
                         static_cast<int>(f), tiles_h * Sh::BN)))
      return rc;
  }
  // ---- every stored entry (ELL and spill rows) bucketed by hidden unit,
  // ordered by token
  cudaError_t e = cudaMemsetAsync(ws.col_count, 0, sizeof(int) * f, st);
  if (e != cudaSuccess) return fail(SGE_ERR_CUDA, "hybrid_ffn_bwd: %s", cudaGetErrorString(e));
  const unsigned rb = static_cast<unsigned>((n + 7) / 8);
  const dim3 sgrid(static_cast<unsigned>((f + 2047) / 2048), static_cast<unsigned>(s_max > 0 ? s_max : 1));
  const char* what = "hybrid_ffn_bwd (column buckets)";
  if ((rc = launch_pdl(csc_count_kernel, dim3(rb), dim3(256), 0, st, what, hv, ws.col_count))) return rc;
  if (s_max > 0 && (rc = launch_pdl(csc_count_spill_kernel, sgrid, dim3(256), 0, st, what, hv, ws.col_count)))
    return rc;
  if ((rc = launch_pdl(csc_scan_kernel, dim3(1), dim3(1024), 0, st, what, ws.col_count, static_cast<int>(f),
                       ws.col_start, ws.col_cursor)))
    return rc;
  if ((rc = launch_pdl(csc_scatter_kernel, dim3(rb), dim3(256), 0, st, what, hv, ws.col_cursor, ws.csc))) return rc;
  if (s_max > 0 && (rc = launch_pdl(csc_scatter_spill_kernel, sgrid, dim3(256), 0, st, what, hv, ws.col_cursor,
                                    ws.csc)))
    return rc;
  if ((rc = launch_pdl(csc_sort_kernel, dim3(static_cast<unsigned>((f + 7) / 8)), dim3(256), 0, st, what,
                       ws.col_start, static_cast<int>(f), ws.csc, ws.csc_sorted)))
    return rc;
  // ---- weight gradients, each row written once
  DwParams q{xb, dyb, hv, ws, dwg_t, dwu_t, dwd, static_cast<int>(d)};
  if (nvec <= kBwdThreads) rc = launch_dw<1>(q, static_cast<int>(f), st);
  else if (nvec <= 2 * kBwdThreads) rc = launch_dw<2>(q, static_cast<int>(f), st);
  else if (nvec <= 3 * kBwdThreads) rc = launch_dw<3>(q, static_cast<int>(f), st);
  else rc = launch_dw<4>(q, static_cast<int>(f), st);
  if (rc || s_max == 0) return rc;
  // ---- dX_s = [dU | dG] [W_up ; W_gate]^T -> dx rows of the spill tokens
  const uint16_t* bcat = static_cast<const uint16_t*>(w_ug);
  if (!bcat) {
    if ((rc = build_up_gate(wu_t, wg_t, ws.bcat, f, d, st))) return rc;
    bcat = ws.bcat;
  }
  CUtensorMap m2a, m2b;
  if ((rc = make_tmap_bf16(&m2a, ws.acat, sp, 2 * f, 2 * f, kBM))) return rc;
  if ((rc = make_tmap_bf16(&m2b, bcat, d, 2 * f, 2 * f, Sx::BN / 2))) return rc;
  const int tiles_n = static_cast<int>((d + Sx::BN - 1) / Sx::BN);
  EpiScatterRows e2{static_cast<uint16_t*>(dx), hy->spill_rows, hy->n_spill, s_max, static_cast<int>(d),
                    ws.part, tiles_n, Sx::BN};
  if ((rc = launch_tc_gemm_pair<Sx>(m2a, m2b, m2b, sp, d, 2 * f, e2, nullptr, st, "hybrid_ffn_bwd (dX)",
                                    kSplitMax)))
    return rc;
  return launch_split_scatter(ws.part, hy->spill_rows, hy->n_spill, s_max, static_cast<int>(d),
                              tiles_n * Sx::BN, static_cast<uint16_t*>(dx), st, "hybrid_ffn_bwd (split sum)");
}
