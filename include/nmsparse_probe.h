/*
 * nmsparse_probe.h -- measurement probes, ablation GEMMs and test controls
 * of libnmsparse (not part of the hot path; the papers have no counterpart).
 * The probes calibrate the roofline denominators on the chip the library
 * runs on.
 */
#ifndef NMSPARSE_PROBE_H
#define NMSPARSE_PROBE_H

#include <stddef.h>
#include <stdint.h>

#include "nmsparse.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Tensor-pipe probe: `ctas` CTAs (one per SM when ctas <= SM count) each issue
 * 4*iters back-to-back tcgen05.mma (sparse = 0: kind::f16 M=128 K=16) or
 * tcgen05.mma.sp (sparse = 1: M=128, K=32 logical) instructions with N = n
 * (128, 192 or 256) on operands resident in shared memory, accumulating in
 * tensor memory.  cycles[i] / nanos[i] (device arrays of `ctas` entries,
 * caller-owned) receive CTA i's SM clock cycles and global-timer nanoseconds
 * from the first issue to the completion of the last MMA.                   */
nm_status nm_probe_mma(int sparse, int n, int ctas, int iters, unsigned long long *cycles,
                       unsigned long long *nanos, void *stream);

/* HBM probe: dst[i] = src[i] for `bytes` bytes (16-byte aligned, multiple of
 * 16), grid of `blocks` CTAs of 256 threads with 16-byte streaming accesses. */
nm_status nm_probe_copy(const void *src, void *dst, size_t bytes, int blocks, void *stream);

/* Ablation baseline: the single-CTA, one-tile-per-CTA tcgen05 GEMM (128 x 128
 * tiles, M = 128 instructions) that nm_sparse_gemm / nm_dense_gemm replace with
 * the persistent CTA-pair kernel.  sparse = 1: W_or_packed is the output of
 * nm_sparse_prepare(..., R, K, m = 4, ...) (ldw unused); sparse = 0: W_or_packed
 * is a dense bf16 [R x K] matrix with leading dimension ldw.  Same arguments,
 * alignment rules and output as the library GEMMs.                          */
nm_status nm_gemm_1cta(int sparse, const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                       const void *W_or_packed, int64_t R, int64_t ldw, uint16_t *Y, int64_t ldy,
                       void *stream);

/* Ablation: the same product as nm_sparse_gemm with the whole activation lift
 * done inside the GEMM (no workspace): for 6:8, lift warps copy columns 2..5
 * of every group from the two raw X tiles in shared memory into the third
 * stage; for 4:6 / 8:10 they copy every window's columns from X with cp.async.
 * Same arguments and output as nm_sparse_gemm (without ws).                */
nm_status nm_sparse_gemm_fused(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                               const void *packed, int64_t R, int m, uint16_t *Y, int64_t ldy,
                               void *stream);

/* Ablation: nm_sparse_gemm with the 256-row x 256-token CTA-pair tile (one
 * M = 256 sparse MMA per step) instead of the library's 512-row x (<= 240)-
 * token tile (two MMAs per step sharing B).  Same arguments, workspace and
 * output as nm_sparse_gemm.                                                */
nm_status nm_sparse_gemm_tile256(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                 const void *packed, int64_t R, int m, uint16_t *Y, int64_t ldy,
                                 void *ws, size_t ws_bytes, void *stream);

/* Test controls for the bounded device waits (failure detection without a
 * GPU fault).  Every barrier and stream-K flag wait gives up after a limit,
 * records NM_ERR_TIMEOUT in the device error word and lets its kernel finish;
 * these two calls make such a wait run out on purpose, from the host.
 *   nm_test_set_wait_limit_ns: the limit for kernels launched afterwards on
 *     the current device, 1 ns .. 1 s; 0 restores the default of one second
 *     (larger -> NM_ERR_SHAPE).
 *   nm_test_withhold_stream_k_flag: the stream-K CTA pair with this index
 *     (-1: none, the default) still writes its partial sums but never
 *     publishes their flags, so the pair that owns the tile waits in vain.
 * Both are synchronous copies to device variables; set them back before
 * normal use.  Not for production calls.                                   */
nm_status nm_test_set_wait_limit_ns(unsigned long long ns);
nm_status nm_test_withhold_stream_k_flag(int cluster);

/* Path control for the H reduction.  With several token ranges per column
 * strip, nm_hessian_diag combines a strip's ranges inside one thread-block
 * cluster (distributed shared memory) when every cluster fits on the device
 * at once, and otherwise through the workspace pairs and a second kernel.
 * on = 0 forces the second path (to test it on a device where clusters fit),
 * on = 1 restores the automatic choice.  A host setting, not thread-safe
 * against concurrent calls; not for production use.                        */
nm_status nm_test_hessian_clusters(int on);

/* How many kernels nm_hessian_diag(X of T x K) launches on the current device
 * with the current path setting: 1 (one token range, or the ranges combined
 * inside clusters) or 2 (the workspace path's second kernel); 0 for T or
 * K < 1.  A query for launch accounting; launches nothing.                  */
int nm_hessian_launch_count(int64_t T, int64_t K);

#ifdef __cplusplus
}
#endif

#endif /* NMSPARSE_PROBE_H */
