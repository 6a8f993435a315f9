/*
 * sge.h -- C ABI of the activation-sparse gated-epilogue FFN library for
 * NVIDIA B200 (sm_100a).
 *
 * The method: "Sparser, Faster, Lighter Transformer Language Models" (Cetin,
 * Peluchetti, Castillo, Naruse, Murakami, Jones; ICML 2026).  The feed-forward
 * block is the gated FFN
 *
 *     y = (ReLU(x W_gate) (.) (x W_up)) W_down
 *
 * (pwwt.cn summary, section 01 and figure "Gated FFN up, gate and down
 * projection"; the printed formula is lost, this is its plain reading with
 * no bias terms).  ReLU makes most hidden activations exact zeros; the gate
 * activations are packed into TwELL (tile-wise ELLPACK) directly in the gate
 * GEMM's epilogue (section 02, figures "TwELL cuts the column direction into
 * tiles" and "gate projection with TwELL storage generation"), and one fused
 * kernel does the up and down projections over the nonzeros only, without
 * writing the hidden activation h to memory (section 02, last paragraph).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, row-major and contiguous (the
 *    fused call's two weight matrices take a row stride, ldw), owned by the
 *    caller; the library never allocates or frees device memory and keeps no
 *    pointer after the call returns.
 *  - Every pointer must be 16-byte aligned; d_model must be a multiple of 8.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    are asynchronous on that stream; outputs are overwritten (beta = 0).
 *  - The return value is SGE_OK or an error code, decided on the host before
 *    anything is launched (bad argument, unsupported shape, launch failure);
 *    sge_last_error() then holds a message (thread-local).
 *  - Data-dependent conditions found on the device are reported in the
 *    caller's optional `diag` word (int32[4], device memory), which kernels
 *    ADD to (atomically), so the caller zeroes it when it wants fresh counts:
 *      diag[SGE_DIAG_OVERFLOW_TILES]  TwELL tiles whose count exceeded C
 *      diag[SGE_DIAG_SPILL_ROWS]      hybrid rows with nnz > K
 *      diag[SGE_DIAG_DROPPED_ROWS]    spill rows beyond S_max (not computed)
 *      diag[SGE_DIAG_FLAGS]           OR of SGE_FLAG_* bits
 *    SGE_FLAG_TIMEOUT means a bounded pipeline wait gave up (a bug or a
 *    stuck device); the outputs of that call are then undefined.
 *
 * Weights are stored neuron-major (row j is the j-th hidden unit):
 *    wg_t[F][d] = W_gate^T,  wu_t[F][d] = W_up^T,  wd[F][d] = W_down.
 *
 * TwELL layout (per row t, per column tile b of width T, capacity C slots):
 *    count[N][F/T]     uint8   true number of active columns (may exceed C)
 *    idx  [N][F/T][C]  uint8   local column (0..T-1) of the stored entries,
 *                              ascending
 *    val  [N][F/T][C]  dtype   ReLU(g) of the stored entries, rounded to
 *                              nearest even
 * A column is active iff its fp32 gate pre-activation g > 0.  Only the first
 * min(count, C) slots of a tile are written and read.
 */
#ifndef SGE_H
#define SGE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define SGE_OK 0
#define SGE_ERR_ARG 1         /* null / misaligned pointer, bad size */
#define SGE_ERR_UNSUPPORTED 2 /* valid but not implemented shape or dtype */
#define SGE_ERR_CUDA 3        /* CUDA runtime / driver error at launch */

/* element types */
#define SGE_F32 0
#define SGE_BF16 1

/* diag word slots and flags */
#define SGE_DIAG_OVERFLOW_TILES 0
#define SGE_DIAG_SPILL_ROWS 1
#define SGE_DIAG_DROPPED_ROWS 2
#define SGE_DIAG_FLAGS 3
#define SGE_FLAG_TIMEOUT 1
#define SGE_FLAG_BOUNDS 2  /* debug builds: an index outside its range */

/* Library version (major * 10000 + minor * 100 + patch). */
int sge_version(void);

/*
 * sge_debug_flags -- the debug build's index checks.  libsge_debug.so is the
 * same library compiled with SGE_DEBUG: every computed index a kernel uses
 * to address memory that comes from data (stored TwELL columns, token and
 * spill lists, ELL columns, weight-gradient buckets) is checked against its
 * range; one outside it sets SGE_FLAG_BOUNDS in a device word and is
 * replaced by an index inside the range, so the kernel finishes without
 * touching memory it does not own (no trap).  Returns the OR of the flags
 * raised since the last clear (synchronising the device), clearing them if
 * `clear` is nonzero; -1 in the release build (no checks compiled); -2 on a
 * CUDA error (message in sge_last_error).
 */
int sge_debug_flags(int clear);

/* Message of the last failed call on this host thread ("" if none). */
const char* sge_last_error(void);

/*
 * twell_gate_pack -- gate projection with TwELL produced in the epilogue.
 * (pwwt.cn summary, section 02: TwELL generated directly in the epilogue of
 * the gate projection, no separate conversion kernel, no dense gate
 * activation in global memory.)
 *
 *   G = x W_gate  (fp32 accumulation), then per row t and tile b:
 *   count[t][b] = #{j in tile b : G[t][j] > 0}; the first min(count, C) active
 *   columns (ascending) are stored as idx = j - bT, val = ReLU(G[t][j]).
 *
 *   x      [N][d]   dtype     input activations
 *   wg_t   [F][d]   dtype     W_gate transposed (neuron-major)
 *   dtype  SGE_BF16: tcgen05 tensor-core GEMM (bf16 x bf16 -> fp32);
 *          SGE_F32:  CUDA-core fp32 FMA GEMM.
 *   tile   T: 16, 32, 64 or 128, dividing F
 *   cap    C: 1 <= C <= T
 *   count, idx, val: TwELL output as laid out above (val in `dtype`)
 *   diag   nullable int32[4]; adds the number of tiles with count > C
 * Errors: SGE_ERR_ARG for null/misaligned pointers, N, d or F < 1, d % 8 != 0,
 * F % T != 0, C outside [1, T]; SGE_ERR_UNSUPPORTED for other T or dtype.
 */
int twell_gate_pack(const void* x, const void* wg_t, int64_t n_tokens, int64_t d_model,
                    int64_t d_ff, int dtype, int tile, int cap, uint8_t* count, uint8_t* idx,
                    void* val, int32_t* diag, void* stream);

/*
 * twell_fused_up_down -- up and down projections over the TwELL nonzeros in
 * one pass.  (pwwt.cn summary, section 02, last paragraph: one custom kernel
 * does the up and down projections in a single traversal, fusing the two
 * products so that the intermediate h never goes to global memory.)
 *
 *   y[t] = sum over stored entries (j, a) of row t of
 *          h * wd[j],  h = a * (x[t] . wu_t[j])
 *   with fp32 accumulation of both products; for bf16, h is rounded to bf16
 *   before the down projection (the precision the dense bf16 FFN gives h).
 *   y is written in `dtype`.
 *
 *   x [N][d], y [N][d] in dtype; count/idx/val the TwELL produced by
 *   twell_gate_pack with the same T and C.
 *   wu_t, wd   F rows of d elements each (row j of wu_t is column j of W_up),
 *              rows ldw elements apart in both (ldw >= d, a multiple of 8).
 *              ldw = d: two separate [F][d] matrices.  The fastest layout
 *              interleaves them: one [F][2d] matrix whose row j holds
 *              W_up[:, j] then W_down[j, :], passed as wu_t = its start,
 *              wd = wu_t + d elements and ldw = 2d (sge_interleave_up_down
 *              builds it).  When d * element size is a multiple of 512 bytes,
 *              one copy then brings both rows of an entry.
 *   workspace  device scratch of at least
 *              twell_fused_up_down_workspace_bytes(N, d) bytes (N-proportional
 *              lists plus a pool of about 64 MiB), 256-byte aligned, owned by
 *              the caller; it holds per-token entry counts, the job lists,
 *              the fp32 partial outputs of the units that heavy tokens are
 *              split into, and counters; it must not be shared by calls that
 *              may run concurrently.  Empty tokens get y = 0.
 *   tile       T, with F / T <= 256 TwELL tiles per row.
 *   diag       nullable int32[4]; diag[SGE_DIAG_FLAGS] gets SGE_FLAG_TIMEOUT
 *              if a pipeline wait gave up (y is then invalid).
 * Results are deterministic: repeated calls on the same inputs give the same
 * bits, whatever the scheduling.  Batches of at most 64 tokens (with rows of
 * at most 4 KB) run a small-batch kernel whose fp32 sums are ordered
 * differently from the larger batches' kernel: a token's y can differ between
 * the two in the last bits.
 * Errors: as twell_gate_pack; SGE_ERR_ARG for a missing, short or misaligned
 * workspace or a bad ldw; SGE_ERR_UNSUPPORTED for d > 4096 or
 * F / T > 256.
 */
size_t twell_fused_up_down_workspace_bytes(int64_t n_tokens, int64_t d_model);

int twell_fused_up_down(const void* x, const uint8_t* count, const uint8_t* idx, const void* val,
                        const void* wu_t, const void* wd, int64_t ldw, void* y, int64_t n_tokens,
                        int64_t d_model, int64_t d_ff, int dtype, int tile, int cap,
                        void* workspace, size_t workspace_bytes, int32_t* diag, void* stream);

/*
 * twell_fused_up_down_noalloc -- twell_fused_up_down for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a
 * deployment convenience of this library.
 *
 * Some callers have no way to obtain a workspace: runtimes that forbid
 * cudaMalloc once they are serving, servers that have given all device memory
 * to their own pools, plugins that only receive the tensors they operate on.
 * This entry point takes the same arguments as twell_fused_up_down minus the
 * workspace and allocates nothing (no cudaMalloc, no cudaFree, no allocating
 * library routine).  Its scratch is a fixed device array built into the
 * library, sized for at most twell_fused_up_down_noalloc_max_tokens()
 * tokens (65536; about 6.6 MB, held on every GPU that loads the library
 * until the process exits).  Larger N is rejected with SGE_ERR_UNSUPPORTED.
 *
 * The first call in a device's context looks up the array's device address
 * there (cudaGetSymbolAddress) and, under CUDA's lazy module loading (the
 * default), that lookup loads the library's device code, which commits
 * device memory for the array.  A caller that may not allocate once it is
 * serving therefore makes one call during start-up, before any stream
 * capture: a call with n_tokens = 0 does only this set-up (its pointers may
 * be NULL).  After a device reset, or in a new context, the next call looks
 * the address up again.  Every call shares the one array, so calls that may overlap on
 * the GPU (different streams, or different host threads on the same device)
 * race and must be serialised by the caller.  Results agree with those of
 * twell_fused_up_down up to fp32 rounding order: the array's smaller pool for
 * partial outputs splits the heaviest tokens into fewer, longer units, which
 * also makes heavy-tailed batches slower than with a workspace.
 */
int64_t twell_fused_up_down_noalloc_max_tokens(void);

int twell_fused_up_down_noalloc(const void* x, const uint8_t* count, const uint8_t* idx,
                                const void* val, const void* wu_t, const void* wd, int64_t ldw,
                                void* y, int64_t n_tokens, int64_t d_model, int64_t d_ff,
                                int dtype, int tile, int cap, int32_t* diag, void* stream);

/*
 * twell_hybrid_up_down -- the up and down projections from TwELL with the
 * heavy tokens routed to tensor cores (inference).  ("Sparser, Faster,
 * Lighter Transformer Language Models", pwwt.cn summary, section 03 and
 * figure "routing of the hybrid-format sparse operator": tokens with few
 * active gates take the sparse path, the rare highly active tokens a dense
 * backup path on tensor cores; kongchang.com page, "core idea": a fast path
 * with a dense fallback.)  Computes the same y as twell_fused_up_down:
 *   y[t] = sum over stored entries (j, a) of row t of bf16(a u) wd[j],
 *   u = x[t] . wu_t[j], fp32 accumulation, y in bf16,
 * up to the order of the fp32 sums (which differs from
 * twell_fused_up_down's, so the last bits of y may differ).
 *
 * Routing: a token with more than K = ell_cap stored entries (the sum of
 * min(count, C) over its tiles) is heavy; heavy tokens are ranked in
 * ascending token order and the first S_max = s_max of them run as two
 * tcgen05 GEMMs over all F hidden units (U = X_s W_up with an epilogue
 * forming h = bf16(a u), zero where the TwELL stores no entry; then
 * Y_s = H_s W_down scattered into y).  Every other token (light, or heavy
 * past S_max) runs on CUDA cores first, one warp per token streaming its
 * entries' W_up and W_down rows through shared memory; no token is dropped
 * (heavy tokens past S_max are slow on that path: size S_max for the heavy
 * tokens expected).  Batches of at most 64 tokens,
 * and s_max = 0, run the per-entry path for every token (a spill GEMM would
 * stream all of W_up and W_down for a few rows).  No ELL repack and nothing
 * saved for a backward pass (hybrid_pack / hybrid_ffn_fwd do that).
 *
 *   x [N][d], y [N][d]   bf16
 *   count/idx/val        the TwELL of twell_gate_pack (bf16 values), tile T,
 *                        capacity C
 *   wu_t, wd, ldw        as for twell_fused_up_down (the interleaved layout
 *                        of sge_interleave_up_down is the fastest); the
 *                        spill GEMM reads wu_t with row stride ldw
 *   wd_t [d][F]          bf16  W_down transposed (row i = column i of
 *                        W_down), the K-major operand of the down GEMM; a
 *                        weight layout built once; may be NULL if s_max = 0
 *   ell_cap              K >= 0.  A spill row costs the two GEMMs over all
 *                        F hidden units, a light entry one copy of its
 *                        weight rows, so the break-even grows with F: K =
 *                        F/512 measured within 2% of the best K at 1%
 *                        density for F = 8192 and F = 10240
 *   s_max                spill capacity in tokens, >= 0
 *   workspace            >= twell_hybrid_up_down_workspace_bytes(N, d, F,
 *                        s_max) bytes, 256-byte aligned, caller-owned, not
 *                        shared by calls that may run concurrently (the
 *                        per-entry kernel's lists and pool, the spill list,
 *                        the spill operands X_s [S_max][d], A_s and H_s
 *                        [S_max][F] in bf16, and 21 MB for the down GEMM's
 *                        split-K parts, used when the heavy tokens make
 *                        fewer output tiles than there are CTA pairs)
 *   diag                 nullable; [SGE_DIAG_SPILL_ROWS] gains the number of
 *                        heavy tokens (those past S_max included),
 *                        [SGE_DIAG_FLAGS] SGE_FLAG_TIMEOUT if a wait gave up
 * Deterministic: repeated calls give the same bits.  Rows with a tile whose
 * count exceeds C use their stored entries only, as in twell_fused_up_down.
 * Errors: as twell_fused_up_down; SGE_ERR_ARG for negative K or S_max,
 * F % 8 != 0, a short or misaligned workspace, a missing wd_t.
 */
size_t twell_hybrid_up_down_workspace_bytes(int64_t n_tokens, int64_t d_model, int64_t d_ff,
                                            int s_max);

int twell_hybrid_up_down(const void* x, const uint8_t* count, const uint8_t* idx, const void* val,
                         const void* wu_t, const void* wd, int64_t ldw, const void* wd_t, void* y,
                         int64_t n_tokens, int64_t d_model, int64_t d_ff, int tile, int cap,
                         int ell_cap, int s_max, void* workspace, size_t workspace_bytes,
                         int32_t* diag, void* stream);

/*
 * sge_interleave_up_down -- builds the interleaved weight layout that
 * twell_fused_up_down streams fastest: w_ud [F][2d], row j = wu_t[j] (d
 * elements) then wd[j] (d elements).  A layout step for loading weights, done
 * once; it is not part of the forward pass.
 *   wu_t [F][d], wd [F][d] contiguous; w_ud [F][2d] caller-allocated, not
 *   overlapping them; dtype SGE_BF16 or SGE_F32.  Stream-ordered copies.
 * Errors: SGE_ERR_ARG for null pointers or bad sizes; SGE_ERR_CUDA.
 */
int sge_interleave_up_down(const void* wu_t, const void* wd, void* w_ud, int64_t d_ff,
                           int64_t d_model, int dtype, void* stream);

/*
 * dense_ffn_fwd -- the dense gated FFN the method is compared against
 * (pwwt.cn summary, lead and section 04: speed-ups are quoted against the
 * dense model).  bf16 only, on tcgen05 tensor cores:
 *   h = bf16(ReLU(x W_gate) (.) (x W_up))   (one GEMM, two accumulators)
 *   y = bf16(h W_down)
 *
 *   x [N][d], wg_t [F][d], wu_t [F][d]   bf16
 *   wd_t [d][F]  bf16  W_down TRANSPOSED (row i = column i of W_down), the
 *                      K-major layout of the second GEMM's B operand
 *   h  [N][F]  bf16  caller-provided workspace for the hidden activation
 *   y  [N][d]  bf16
 * Errors: SGE_ERR_ARG as above and for F % 8 != 0.
 */
int dense_ffn_fwd(const void* x, const void* wg_t, const void* wu_t, const void* wd_t, void* h,
                  void* y, int64_t n_tokens, int64_t d_model, int64_t d_ff, int32_t* diag,
                  void* stream);

/*
 * Hybrid format for training ("Sparser, Faster, Lighter Transformer Language
 * Models", pwwt.cn summary, section 03 and figure "routing of the
 * hybrid-format sparse operator": tokens with few active gates go to a
 * compressed ELL matrix, rare highly active tokens to a dense backup path on
 * tensor cores; kongchang.com page, "custom CUDA kernels: fusion and
 * compression": TwELL is compressed into this hybrid form).  bf16 only.
 *
 * All buffers are caller-owned device memory described by this struct:
 *   row_nnz    int32 [N]          stored entries of row t (sum of min(count, C));
 *                                 a row with a tile whose count exceeds C
 *                                 (entries lost to the capacity) and at most
 *                                 K stored entries gets K + 1 instead, so that
 *                                 it goes to the spill (where hybrid_ffn_fwd
 *                                 can recompute it exactly)
 *   spill_slot int32 [N]          rank of row t among the spill rows if
 *                                 row_nnz > K and that rank < S_max, else -1
 *   spill_rows int32 [S_max]      token of each kept spill row (ascending)
 *   n_spill    int32 [1]          number of rows with row_nnz > K (may
 *                                 exceed S_max; rows ranked >= S_max are
 *                                 dropped: their y, dx and dW contributions
 *                                 are zero and diag reports them)
 *   ell_idx    uint16 [N][K]      columns of an ELL row's entries, ascending,
 *                                 0xFFFF after row_nnz (requires F <= 65535)
 *   ell_a      bf16 [N][K]        a = ReLU(g) of those entries, 0 after row_nnz
 *   ell_u      bf16 [N][K]        u = x . W_up[:, j], written by hybrid_ffn_fwd
 *   spill_a    bf16 [S_max][F]    dense a of each kept spill row
 *   spill_u    bf16 [S_max][F]    dense u of each kept spill row, written by
 *                                 hybrid_ffn_fwd
 * ELL rows are rows with row_nnz <= K (ties go to ELL).
 */
typedef struct sge_hybrid {
  int64_t n_tokens;
  int64_t d_ff;
  int32_t ell_cap; /* K, 0 <= K <= 512 */
  int32_t s_max;   /* spill capacity in rows, >= 0 */
  int32_t dtype;   /* SGE_BF16 */
  int32_t reserved;
  int32_t* row_nnz;
  int32_t* spill_slot;
  int32_t* spill_rows;
  int32_t* n_spill;
  uint16_t* ell_idx;
  void* ell_a;
  void* ell_u;
  void* spill_a;
  void* spill_u;
} sge_hybrid;

/*
 * hybrid_pack -- compress a TwELL (count/idx/val with tile T and capacity C,
 * as written by twell_gate_pack) into the hybrid form described by `hy`
 * (which names N, F, K, S_max and the output buffers).  Deterministic:
 * spill ranks follow ascending token order.  diag (nullable) gains the
 * number of spill rows in [SGE_DIAG_SPILL_ROWS] and of dropped rows in
 * [SGE_DIAG_DROPPED_ROWS].
 */
int hybrid_pack(const uint8_t* count, const uint8_t* idx, const void* val, int tile, int cap,
                sge_hybrid* hy, int32_t* diag, void* stream);

/*
 * hybrid_ffn_fwd -- the gated FFN forward from the hybrid form, saving u.
 *   ELL rows: y[t] = sum_e bf16(a_e u_e) W_down[j_e], u_e = x[t] . W_up[:, j_e]
 *             (fp32 accumulation; u_e saved to ell_u in bf16)
 *   spill rows: U = X_s W_up (all F columns, tcgen05), saved to spill_u;
 *             H = bf16(A (.) U); Y_s = H W_down (tcgen05), scattered to y.
 *             When the spill rows make fewer output tiles of Y_s than
 *             there are CTA pairs, its K (= F) is split over the pairs and
 *             the fp32 parts are added in a fixed order (deterministic).
 *             With wg_t given, A is first recomputed from the gate,
 *             A = bf16(ReLU(X_s W_gate)) (one tcgen05 GEMM with two B
 *             operands, W_gate and W_up) and written to spill_a: the rows
 *             that went to the spill because a TwELL tile overflowed its
 *             capacity C then come out as if C = T (the safety valve of a
 *             capacity below the tile width).  With wg_t NULL the spill rows
 *             use spill_a as packed.
 *   dropped rows: y = 0.
 *   x [N][d], y [N][d], wu_t [F][d], wd [F][d], wd_t [d][F] (W_down
 *   transposed, the K-major operand of the spill GEMM; may be NULL when
 *   S_max == 0), wg_t [F][d] or NULL; workspace >=
 *   hybrid_ffn_fwd_workspace_bytes(d, F, S_max), 16-byte aligned: X_s and
 *   H_s [S_max][d + F] bf16, then (S_max > 0) 21 MB of split-K parts.
 */
size_t hybrid_ffn_fwd_workspace_bytes(int64_t d_model, int64_t d_ff, int s_max);

int hybrid_ffn_fwd(const void* x, const sge_hybrid* hy, const void* wu_t, const void* wd,
                   const void* wd_t, const void* wg_t, void* y, int64_t d_model, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * hybrid_ffn_bwd -- gradients of the gated FFN from the hybrid form (after
 * hybrid_ffn_fwd filled ell_u / spill_u).  The pages print no backward
 * formulas; these are the derivatives of y = sum_j a_j u_j W_down[j] over the
 * stored entries (a_j > 0, so dReLU = 1 there; other entries contribute 0):
 *   dh = dy . W_down[j], du = dh a, dg = dh u,
 *   dx = sum_j du W_up[:, j] + dg W_gate[:, j],
 *   dW_down[j] = sum_t a u dy_t, dW_up[:, j] = sum_t du x_t,
 *   dW_gate[:, j] = sum_t dg x_t.
 * ELL rows run on CUDA cores; spill rows' dh and dx run as tcgen05 GEMMs
 * (the dx GEMM's K = 2F split over the CTA pairs when its output has fewer
 * tiles than there are pairs; parts added in a fixed order).
 * The weight gradients sum every stored entry (ELL entries and the spill
 * rows' active columns) per hidden unit in ascending token order, one fp32
 * row written once per unit.  Deterministic.
 *   x, dy, dx [N][d] bf16; wg_t, wu_t, wd [F][d] bf16;
 *   w_ug [d][2F] bf16 or NULL: [W_up | W_gate] (row i = W_up[i, :] then
 *   W_gate[i, :]), the dX GEMM's operand, built once per weight update by
 *   sge_transpose_up_gate; NULL builds it in the workspace on every call;
 *   dwg_t, dwu_t [F][d] fp32 (neuron-major like the weights), dwd [F][d] fp32,
 *   all overwritten; dropped rows get dx = 0 and add nothing.
 *   workspace >= hybrid_ffn_bwd_workspace_bytes(N, d, F, K, S_max) bytes,
 *   256-byte aligned.
 */
size_t hybrid_ffn_bwd_workspace_bytes(int64_t n_tokens, int64_t d_model, int64_t d_ff, int ell_cap,
                                      int s_max);

int hybrid_ffn_bwd(const void* x, const void* dy, const sge_hybrid* hy, const void* wg_t,
                   const void* wu_t, const void* wd, const void* w_ug, void* dx, float* dwg_t,
                   float* dwu_t, float* dwd, int64_t d_model, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * sge_transpose_up_gate -- builds w_ug [d][2F] = [W_up | W_gate] (row i:
 * W_up[i, :] = column i of wu_t, then W_gate[i, :]) for hybrid_ffn_bwd, a
 * layout step for loading (or updating) the weights, not part of a step.
 *   wu_t, wg_t [F][d] bf16; w_ug [d][2F] bf16, caller-allocated.
 * Errors: SGE_ERR_ARG for null or misaligned pointers, F or d not a multiple
 * of 8.  Stream-ordered.
 */
int sge_transpose_up_gate(const void* wu_t, const void* wg_t, void* w_ug, int64_t d_ff,
                          int64_t d_model, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SGE_H */
