// Persistent tcgen05 GEMM engine for sm_100a:  D[M][N] = A[M][K] . B[N][K]^T
// (both operands K-major bf16, fp32 accumulation in tensor memory), with a
// pluggable epilogue that reads the accumulator tile straight out of TMEM.
//
// One CTA per SM (6 or 10 warps), looping over output tiles:
//   warp 0      TMA producer: A and B tiles (128-byte swizzle) into a ring of
//               STAGES shared-memory stages, completion on `full` mbarriers.
//   warp 1      TMEM allocator and MMA issuer: one elected thread issues
//               tcgen05.mma (M = 128, N = BN, K = 16 per instruction) and
//               releases each stage with tcgen05.commit -> `empty`.
//   warps 2..    epilogue: tcgen05.ld of the tile (thread i of warp w holds
//               accumulator row 32*(w%4) + i), then the Epilogue functor;
//               4 warps, or 8 with the tile's columns in two halves.
// The accumulator is double-buffered in TMEM so the epilogue of one tile
// overlaps the main loop of the next.  With NB = 2 the engine multiplies A
// by two B matrices at once into two accumulators (gate and up projections
// of the dense gated FFN share the A tile).
//
// No TMA multicast loads anywhere: every CTA loads its own tiles.  The
// single-CTA engine runs without clusters; the CTA-pair engine below runs in
// 2-CTA clusters (cta_group::2), each CTA loading its half of the operands
// into its own shared memory.
// Every wait is bounded (sge::mbar_wait); a timeout sets SGE_FLAG_TIMEOUT in
// diag, raises a CTA-wide abort flag, and the CTA drains its in-flight TMA
// loads and MMAs (bounded) before freeing TMEM and returning.
#pragma once

#include "sge_common.cuh"

namespace sge {

constexpr int kBM = 128;  // UMMA M: rows of A per tile = TMEM lanes
constexpr int kBK = 64;   // K per stage: one 128-byte swizzle row of bf16

// Epilogue warps: 4 x HALVES.  With HALVES = 2 two warps share each TMEM
// lane quarter and each takes half the tile's columns (the epilogue is then
// called with BN / 2 columns); two-accumulator tiles (NB = 2) keep HALVES = 1.
template <int BN_, int NB_, int HALVES_ = 1>
struct TcShape {
  static constexpr int BN = BN_;
  static constexpr int NB = NB_;
  static constexpr int HALVES = HALVES_;
  static constexpr int THREADS = 64 + 128 * HALVES;
  static_assert(HALVES == 1 || (HALVES == 2 && NB == 1), "column halves need one accumulator");
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + NB * B_BYTES;
  static constexpr int STAGES = (196 * 1024) / STAGE_BYTES > 8 ? 8 : (196 * 1024) / STAGE_BYTES;
  static constexpr int ACC_COLS = BN * NB;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align slack*/ + 256 /*barriers*/;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM columns");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1024-byte aligned sub-tiles");
};

struct TileCoord {
  int m_blk, n_blk;
};

// Rows of A the single-CTA engine loads per tile (the row count of its A
// tensor map's box): a batch of at most 64 rows loads only its rows, rounded
// up to 8, instead of 128 rows that are mostly zero-filled past the end (the
// fill costs TMA time: 1 token took 24.9 us against 20.5 us for 64).  The
// MMA still multiplies 128 rows; the rows past the box read stale shared
// memory and their results are never stored (the epilogue stops at the
// batch's rows).
__host__ __device__ constexpr int a_box_rows(int64_t m) {
  return m <= 8 ? 8 : m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : kBM;
}

// Rows of A an epilogue needs: an epilogue may bound M by a count that only
// the device knows (Epi::m_limit); tiles past it are skipped.
template <class E>
__device__ __forceinline__ auto epi_m_limit_impl(const E& e, int m, int) -> decltype(e.m_limit(m)) {
  return e.m_limit(m);
}
template <class E>
__device__ __forceinline__ int epi_m_limit_impl(const E&, int m, long) {
  return m;
}
template <class E>
__device__ __forceinline__ int epi_m_limit(const E& e, int m) {
  return epi_m_limit_impl(e, m, 0);
}

// K an epilogue needs: an epilogue may bound K by a device-side count
// (Epi::k_limit, returning a multiple of kBK or K itself); K-blocks past it
// are skipped, and with no K-block left every tile is skipped (its product
// is zero: only epilogues that add D to their output may bound K).
template <class E>
__device__ __forceinline__ auto epi_k_limit_impl(const E& e, int k, int) -> decltype(e.k_limit(k)) {
  return e.k_limit(k);
}
template <class E>
__device__ __forceinline__ int epi_k_limit_impl(const E&, int k, long) {
  return k;
}
template <class E>
__device__ __forceinline__ int epi_k_limit(const E& e, int k) {
  return epi_k_limit_impl(e, k, 0);
}

// Split-K (CTA-pair engine): an epilogue may ask for its K range to be cut
// into Epi::splits() parts, each an output tile of its own whose partial
// product the epilogue combines (Epi::run_split); default 1.
template <class E>
__device__ __forceinline__ auto epi_splits_impl(const E& e, int) -> decltype(e.splits()) {
  return e.splits();
}
template <class E>
__device__ __forceinline__ int epi_splits_impl(const E&, long) {
  return 1;
}
template <class E>
__device__ __forceinline__ int epi_splits(const E& e) {
  return epi_splits_impl(e, 0);
}

// The epilogue call of one output tile: run_split (given the split and the
// number of splits) for epilogues that have it, run otherwise.
template <int BN, class E>
__device__ __forceinline__ auto epi_run_impl(const E& e, uint32_t taddr, int64_t row, int n_blk, int split,
                                             int nsplit, int lane, int)
    -> decltype(e.template run_split<BN>(taddr, row, n_blk, split, nsplit, lane)) {
  return e.template run_split<BN>(taddr, row, n_blk, split, nsplit, lane);
}
template <int BN, class E>
__device__ __forceinline__ void epi_run_impl(const E& e, uint32_t taddr, int64_t row, int n_blk, int, int,
                                             int lane, long) {
  e.template run<BN>(taddr, row, n_blk, lane);
}

__device__ __forceinline__ TileCoord tile_coord(int tile, int m_blocks) {
  return TileCoord{tile % m_blocks, tile / m_blocks};
}

// Bounded wait that also gives up when another role of the CTA aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int32_t* diag) {
  uint64_t t0 = 0;  // the clock is read only once a wait has lasted kWaitSpins tries
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if ((i & (kWaitSpins - 1)) == 0) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > kWaitNs) break;
    }
  }
  if (diag) atomicOr(reinterpret_cast<int*>(diag + SGE_DIAG_FLAGS), SGE_FLAG_TIMEOUT);
  *abort_flag = 1;
  return false;
}

template <class Shape, class Epilogue>
__global__ void __launch_bounds__(Shape::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_b0,
                   const __grid_constant__ CUtensorMap map_b1, int M, int N, int K,
                   Epilogue epi, int32_t* diag) {
  constexpr int BN = Shape::BN, NB = Shape::NB, STAGES = Shape::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Shape::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tmem_full[a], 1);
      mbar_init(&tmem_empty[a], 4 * Shape::HALVES);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b0);
    if (NB == 2) tma_prefetch_desc(&map_b1);
  }
  if (warp == 1) tmem_alloc(tmem_holder, Shape::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  grid_dep_wait();  // a no-op unless launched with programmatic dependent launch
  grid_dep_launch();
  const int m_blocks = (epi_m_limit(epi, M) + kBM - 1) / kBM;
  const int n_blocks = (N + BN - 1) / BN;
  const int k_blocks = (epi_k_limit(epi, K) + kBK - 1) / kBK;
  const int num_tiles = k_blocks > 0 ? m_blocks * n_blocks : 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t armed = 0;  // bit s: stage s has a load whose completion is unobserved
      uint32_t armed_par = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, m_blocks);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, diag)) break;
          uint8_t* sa = smem + s * Shape::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], a_box_rows(M) * kBK * 2 + NB * Shape::B_BYTES);
          tma_load_2d(sa, &map_a, &full[s], kb * kBK, tc.m_blk * kBM);
          tma_load_2d(sa + Shape::A_BYTES, &map_b0, &full[s], kb * kBK, tc.n_blk * BN);
          if (NB == 2)
            tma_load_2d(sa + Shape::A_BYTES + Shape::B_BYTES, &map_b1, &full[s], kb * kBK,
                        tc.n_blk * BN);
          armed |= 1u << s;
          armed_par = (armed_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // Drain: every stage's most recent load has landed before we leave
      // (immediate in the normal path, where the MMA already consumed it).
      for (int t = 0; t < STAGES; ++t)
        if (armed & (1u << t)) mbar_wait(&full[t], (armed_par >> t) & 1, diag);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, BN);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool issued = false;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!wait_or_abort(&tmem_empty[acc], ((it >> 1) & 1) ^ 1, abort_flag, diag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * Shape::ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!wait_or_abort(&full[s], ph, abort_flag, diag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Shape::STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t adesc = umma_desc_sw128(sa + k * 32);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              const uint64_t bdesc = umma_desc_sw128(sa + Shape::A_BYTES + b * Shape::B_BYTES + k * 32);
              umma_bf16(d_tmem + b * BN, adesc, bdesc, idesc, (kb | k) != 0);
            }
          }
          issued = true;
          umma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tmem_full[acc]);
      }
      // Drain: all issued MMAs complete before TMEM is released.
      if (issued) {
        umma_commit(drain);
        mbar_wait(drain, 0, diag);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;  // column half (HALVES = 2)
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const bool ok = wait_or_abort(&tmem_full[acc], (it >> 1) & 1, abort_flag, diag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const TileCoord tc = tile_coord(tile, m_blocks);
      const uint32_t taddr = tmem_base + acc * Shape::ACC_COLS + half * (BN / Shape::HALVES) +
                             (static_cast<uint32_t>(quarter * 32) << 16);
      const int64_t row = static_cast<int64_t>(tc.m_blk) * kBM + quarter * 32 + lane;
      epi.template run<BN / Shape::HALVES>(taddr, row, tc.n_blk * Shape::HALVES + half, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Shape::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): a cluster of two CTAs on two SMs computes a
// 256 x BN tile.  CTA r loads rows [128 r, 128 r + 128) of the A tile and
// half of each B tile (BN/2 rows) into its own shared memory; both CTAs'
// TMA bytes complete on the leader's (rank 0) `full` barrier.  The leader's
// MMA thread issues M = 256 tcgen05.mma instructions that read A and B from
// both CTAs and write each CTA's 128 accumulator rows into that CTA's TMEM;
// its commits arrive on both CTAs' barriers (multicast commit).  Each CTA's
// epilogue drains its own TMEM and releases the accumulator on the leader's
// `tmem_empty` barrier (count 8: four warps in each CTA).  Per SM this moves
// half the B bytes of the single-CTA engine for the same work.
template <int BN_, int NB_, int HALVES_ = 1>
struct TcPairShape {
  static constexpr int BN = BN_;  // N of one MMA (both CTAs together)
  static constexpr int NB = NB_;
  static constexpr int HALVES = HALVES_;
  static constexpr int THREADS = 64 + 128 * HALVES;
  static_assert(HALVES == 1 || (HALVES == 2 && NB == 1), "column halves need one accumulator");
  static constexpr int BM = 2 * kBM;
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = (BN / 2) * kBK * 2;  // this CTA's half
  static constexpr int STAGE_BYTES = A_BYTES + NB * B_BYTES;
  static constexpr int STAGES = (196 * 1024) / STAGE_BYTES > 8 ? 8 : (196 * 1024) / STAGE_BYTES;
  static constexpr int ACC_COLS = BN * NB;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=256");
  static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM columns");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1024-byte aligned sub-tiles");
};

template <class Shape, class Epilogue>
__global__ void __launch_bounds__(Shape::THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_b0,
                        const __grid_constant__ CUtensorMap map_b1, int M, int N, int K,
                        Epilogue epi, int32_t* diag) {
  constexpr int BN = Shape::BN, NB = Shape::NB, STAGES = Shape::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Shape::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(cluster_id_x());
  const int n_pairs = static_cast<int>(cluster_count_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tmem_full[a], 1);
      mbar_init(&tmem_empty[a], 8 * Shape::HALVES);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b0);
    if (NB == 2) tma_prefetch_desc(&map_b1);
  }
  if (warp == 1) tmem_alloc_pair(tmem_holder, Shape::TMEM_COLS);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive / TMA
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // with programmatic dependent launch the set-up above overlaps the previous
  // kernel; everything below may read what it wrote.  The successor may
  // launch only after this wait: a successor that skips its own wait can
  // then rely on every kernel before this one having completed.
  grid_dep_wait();
  grid_dep_launch();
  const int m_blocks = (epi_m_limit(epi, M) + Shape::BM - 1) / Shape::BM;
  const int n_blocks = (N + BN - 1) / BN;
  const int k_blocks = (epi_k_limit(epi, K) + kBK - 1) / kBK;
  // split-K: K-blocks per split, and the number of non-empty splits
  const int want_splits = max(1, min(epi_splits(epi), k_blocks));
  const int kb_per = k_blocks > 0 ? (k_blocks + want_splits - 1) / want_splits : 0;
  const int nsplit = kb_per > 0 ? (k_blocks + kb_per - 1) / kb_per : 1;
  const int num_tiles = k_blocks > 0 ? m_blocks * n_blocks * nsplit : 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t armed = 0, armed_par = 0;
      for (int tile = pair; tile < num_tiles && !*abort_flag; tile += n_pairs) {
        const int split = tile % nsplit;
        const TileCoord tc = tile_coord(tile / nsplit, m_blocks);
        const int a_row = tc.m_blk * Shape::BM + static_cast<int>(rank) * kBM;
        const int b_row = tc.n_blk * BN + static_cast<int>(rank) * (BN / 2);
        const int kb_end = min(k_blocks, (split + 1) * kb_per);
        for (int kb = split * kb_per; kb < kb_end; ++kb) {
          if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, diag)) break;
          uint8_t* sa = smem + s * Shape::STAGE_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * Shape::STAGE_BYTES);
          tma_load_2d_pair(sa, &map_a, &full[s], kb * kBK, a_row);
          tma_load_2d_pair(sa + Shape::A_BYTES, &map_b0, &full[s], kb * kBK, b_row);
          if (NB == 2)
            tma_load_2d_pair(sa + Shape::A_BYTES + Shape::B_BYTES, &map_b1, &full[s], kb * kBK, b_row);
          armed |= 1u << s;
          armed_par = (armed_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // Drain: the leader's barrier counts both CTAs' bytes, so once the
      // leader has seen every armed stage land, no load of either CTA is in
      // flight (the closing cluster barrier holds the other CTA until then).
      if (leader)
        for (int t = 0; t < STAGES; ++t)
          if (armed & (1u << t)) mbar_wait(&full[t], (armed_par >> t) & 1, diag);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(Shape::BM, BN);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int tile = pair; tile < num_tiles && !*abort_flag; tile += n_pairs, ++it) {
        const int acc = it & 1;
        if (!wait_or_abort(&tmem_empty[acc], ((it >> 1) & 1) ^ 1, abort_flag, diag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * Shape::ACC_COLS;
        bool ok = true;
        const int split = tile % nsplit;
        const int kb0 = split * kb_per, kb_end = min(k_blocks, kb0 + kb_per);
        for (int kb = kb0; kb < kb_end; ++kb) {
          if (!wait_or_abort(&full[s], ph, abort_flag, diag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Shape::STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t adesc = umma_desc_sw128(sa + k * 32);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              const uint64_t bdesc = umma_desc_sw128(sa + Shape::A_BYTES + b * Shape::B_BYTES + k * 32);
              umma2_bf16(d_tmem + b * BN, adesc, bdesc, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
            }
          }
          umma2_commit_mc(&empty[s], 0x3);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma2_commit_mc(&tmem_full[acc], 0x3);
      }
      // Drain: both CTAs learn that every issued MMA has completed.
      umma2_commit_mc(drain, 0x3);
    }
    if (lane == 0) mbar_wait(drain, 0, diag);
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // column half (HALVES = 2)
    const uint32_t leader_tmem_empty0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += n_pairs, ++it) {
      const int acc = it & 1;
      const bool ok = wait_or_abort(&tmem_full[acc], (it >> 1) & 1, abort_flag, diag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const TileCoord tc = tile_coord(tile / nsplit, m_blocks);
      const uint32_t taddr = tmem_base + acc * Shape::ACC_COLS + half * (BN / Shape::HALVES) +
                             (static_cast<uint32_t>(quarter * 32) << 16);
      const int64_t row = static_cast<int64_t>(tc.m_blk) * Shape::BM + rank * kBM + quarter * 32 + lane;
      epi_run_impl<BN / Shape::HALVES>(epi, taddr, row, tc.n_blk * Shape::HALVES + half, tile % nsplit,
                                       nsplit, lane, 0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tmem_empty0 + acc * 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still touch its barriers or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Shape::TMEM_COLS);
  }
}

}  // namespace sge
