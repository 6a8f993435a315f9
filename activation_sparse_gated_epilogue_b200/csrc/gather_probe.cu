// Measurement helper: how fast whole rows picked at random from a table
// stream from L2 into shared memory on this GPU.
//
// The fused up/down kernel moves one W_up row and one W_down row per stored
// entry from L2 to the SMs; its arithmetic hides behind that traffic.  This
// kernel measures the traffic's ceiling with the same mechanism and nothing
// else: every SM runs kProbeWarps warps, each streaming its share of the rows
// through a two-slot ring with cp.async.bulk (one mbarrier per slot) and
// reading every row back from shared memory.  The bench divides the fused
// kernel's row bytes per second by this rate.
//
// The slot count is a kernel argument on purpose: measured on B200, the same
// loop with the count fixed at compile time streams at less than half the
// rate (8.3 against 18 TB/s at 24 warps and 4 KB rows).
#include "sge_host.h"
#include "sge_common.cuh"

namespace sge {

constexpr int kProbeWarps = 24;
constexpr int kProbeSlots = 2;
constexpr int kProbeSmem = 200 * 1024;

__global__ void gather_probe_kernel(const uint8_t* __restrict__ table, int64_t table_rows,
                                    const int32_t* __restrict__ ids, int64_t n_ids64, int row_bytes,
                                    int S, uint32_t* sink, int32_t* diag) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int n_ids = static_cast<int>(n_ids64);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  uint8_t* ring = smem + (size_t)warp * S * row_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)nwarps * S * row_bytes) + warp * S;
  if (lane == 0)
    for (int s = 0; s < S; ++s) mbar_init(full + s, 1);
  fence_mbar_init();
  __syncwarp();
  const int gw = blockIdx.x * nwarps + warp, ngw = gridDim.x * nwarps;
  const int n_mine = gw < n_ids ? (n_ids - gw + ngw - 1) / ngw : 0;
  auto ld_id = [&](int k) { return k < n_mine ? ids[gw + (size_t)k * ngw] : 0; };
  int id_cur = ld_id(lane), id_nxt = ld_id(32 + lane);
  auto id_of = [&](int k, int kb) {
    const int a = __shfl_sync(0xffffffffu, id_cur, k & 31), b = __shfl_sync(0xffffffffu, id_nxt, k & 31);
    return (k >> 5) == kb ? a : b;
  };
  auto issue = [&](int k, int id) {
    const int s = k % S;
    id = id < 0 ? 0 : (id >= table_rows ? static_cast<int>(table_rows - 1) : id);
    const uint8_t* src = table + (size_t)id * row_bytes;
    mbar_arrive_expect_tx(full + s, static_cast<uint32_t>(row_bytes));
    bulk_load(ring + (size_t)s * row_bytes, src, static_cast<uint32_t>(row_bytes), full + s);
  };
  for (int k = 0; k < S && k < n_mine; ++k) {
    const int id = id_of(k, 0);
    if (lane == 0) issue(k, id);
  }
  unsigned acc = 0;
  const int nv = row_bytes / 16;
  int k = 0;
  for (; k < n_mine; ++k) {
    const int s = k % S;
    if (k > 0 && (k & 31) == 0) { id_cur = id_nxt; id_nxt = ld_id(k + 32 + lane); }
    const int idn = id_of(k + S, k >> 5);
    if (!mbar_wait(full + s, (k / S) & 1, diag)) break;
    const uint32_t base = smem_u32(ring + (size_t)s * row_bytes);
    for (int v = lane; v < nv; v += 32) {
      uint32_t a, b, c, d;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(base + v * 16));
      acc ^= a ^ b ^ c ^ d;
    }
    __syncwarp();
    if (lane == 0 && k + S < n_mine) issue(k + S, idn);
  }
  for (int r = k; r < n_mine && r < k + S; ++r) mbar_wait(full + r % S, (r / S) & 1, nullptr);
  if (acc == 0x12345678u) sink[0] = acc;
}

}  // namespace sge

using namespace sge;

extern "C" int sge_l2_gather_probe(const void* table, int64_t table_rows, int row_bytes,
                                   const int32_t* ids, int64_t n_ids, uint32_t* sink,
                                   int32_t* diag, void* stream) {
  clear_error();
  if (table_rows < 1 || n_ids < 0 || row_bytes < 16 || row_bytes % 16)
    return fail(SGE_ERR_ARG, "sge_l2_gather_probe: bad sizes");
  if (!table || !ids || !sink) return fail(SGE_ERR_ARG, "sge_l2_gather_probe: null pointer");
  if (!aligned16(table)) return fail(SGE_ERR_ARG, "sge_l2_gather_probe: table not 16-byte aligned");
  int warps = kProbeSmem / (kProbeSlots * row_bytes + 8 * kProbeSlots);
  if (warps > kProbeWarps) warps = kProbeWarps;
  if (warps < 1) return fail(SGE_ERR_UNSUPPORTED, "sge_l2_gather_probe: rows of %d bytes", row_bytes);
  if (n_ids == 0) return SGE_OK;
  if (n_ids >= (1LL << 31)) return fail(SGE_ERR_UNSUPPORTED, "sge_l2_gather_probe: too many ids");
  const int smem = warps * kProbeSlots * (row_bytes + 8);
  int rc = set_smem_limit(reinterpret_cast<const void*>(gather_probe_kernel), smem);
  if (rc) return rc;
  gather_probe_kernel<<<sm_count(), warps * 32, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(table), table_rows, ids, n_ids, row_bytes, kProbeSlots, sink, diag);
  return check_launch("sge_l2_gather_probe");
}
