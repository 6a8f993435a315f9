/*
 * sge_selftest.h -- the test-only self-test library libsge_selftest.so (not
 * part of libsge.so and not for production use): failure handling of the
 * tcgen05 GEMM engines.  The paper has no counterpart: this is a test of the
 * library's own bounded waits.
 *
 * sge_selftest_wait_timeout -- runs the GEMM engine (pair != 0: the CTA-pair
 * engine, else the single-CTA engine) on an m x n x k bf16 problem whose
 * tile pipeline can never fill: the B operand's tensor map covers fewer rows
 * per load than the stage expects, so no stage barrier completes.  Built
 * with a 20 ms wait deadline (libsge.so uses 4 s), the kernel's MMA issuer
 * gives up, sets SGE_FLAG_TIMEOUT in diag[SGE_DIAG_FLAGS], raises the CTA's
 * abort flag; the producer and epilogue leave, the CTA waits (bounded) for
 * its loads in flight, frees its tensor memory and returns.  No tile reaches
 * the epilogue: tiles_done (device int32, caller-zeroed) stays 0.  The call
 * takes well under a second and leaves the context usable.
 *   a [m][k], b [n][k]  bf16 device buffers (contents unused), 16-byte aligned
 *   diag  int32[4] device, caller-zeroed; tiles_done int32[1] device
 * Returns SGE_OK once launched; SGE_ERR_ARG for bad sizes or pointers.
 */
#ifndef SGE_SELFTEST_H
#define SGE_SELFTEST_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int sge_selftest_wait_timeout(int pair, const void* a, const void* b, int64_t m, int64_t n, int64_t k,
                              int32_t* diag, int32_t* tiles_done, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SGE_SELFTEST_H */
