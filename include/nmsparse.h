/*
 * nmsparse.h -- C ABI of the B200 (sm_100a) N:M-pruned linear layer.
 *
 * The hot path these calls implement, with the passage that defines each step
 * (page title, section):
 *   nm_hessian_diag   H_j = mean_t x_{t,j}^2, the diagonal Gauss-Newton proxy of
 *                     the input activations. Sparsity Induction for Accurate
 *                     Post-Training Pruning of LLMs (arXiv 2602.21652), sec. 2C
 *                     "Efficientie: Snelle Hessian Update".
 *   nm_hessian_rescale  H / s^2 under equivalent scaling: the O(d_in) score
 *                     refresh of Sparsity Induction sec. 2C.
 *   nm_hutchinson_diag  Rademacher estimate of diag(X^T X / T), SparseForge,
 *                     "Estimativa de Importancia Consciente do Hessiano".
 *   nm_score          s = (H + eps) * W^2. SparseForge (arXiv 2605.06402),
 *                     "Estimativa de Importancia Consciente do Hessiano".
 *                     With X == NULL: s = |W_latent|, Sparse-BitNet (arXiv
 *                     2603.05168) sec. 2 "Geracao de Mascara Baseada em Magnitude".
 *   nm_prune_compress keep the top-n scores of every group of m consecutive
 *                     weights along the input dimension (ties -> lower index),
 *                     compress the kept values, emit 2:4 metadata.
 *                     SparseForge "Mistura Progressiva" (hard top-N target);
 *                     Sparse-BitNet sec. 1 (N:M definition) and sec. 2
 *                     ("Quantizar e depois Mascarar": the values compressed are
 *                     whatever V the caller passes, e.g. ternary W_q).
 *   nm_score_prune_compress  the two steps above in one pass: the scores are
 *                     formed in registers and never written.
 *   slide_pack        (2N-2):2N -> N-1 overlapping width-4 windows at stride 2,
 *                     each 2:4. SlideSparse (arXiv 2603.05232) sec. 2A.
 *   lift_activations  X'[t, g*4(N-1) + 4w + i] = X[t, g*2N + 2w + i].
 *                     SlideSparse sec. 2B "Elevacao de Ativacao".
 *   nm_sparse_prepare canonical values + window metadata -> the GEMM's operand
 *                     layout. SlideSparse sec. 2C item 2 (initialisation phase).
 *   nm_sparse_prepare_from_mask  slide_pack and nm_sparse_prepare in one pass.
 *   nm_sparse_gemm    Y = X * W_sparse^T on the sparse tensor cores, over the
 *                     lifted activations for (2N-2):2N. SlideSparse sec. 2C
 *                     item 3 (online phase).
 *   nm_dense_gemm     Y = X * W^T, dense tcgen05 GEMM (the comparison point).
 *   nm_ternary_quantize  gamma = mean|W|, W_q = clip(rint(W/gamma),-1,1)*gamma.
 *                     Sparse-BitNet sec. 1 item 1 (BitNet b1.58 ternary weights).
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing; its only state is one device error word, the static
 *     scratch array of nm_hessian_diag_noalloc and the GEMM schedule setting
 *     of nm_gemm_set_schedule.
 *   - bf16 tensors are passed as uint16_t bit patterns.  Matrices are row-major
 *     with a leading dimension (elements) ld >= the row length.
 *   - X is [T x K] (tokens x in-features), W is [R x K] (out x in features),
 *     Y is [T x R].  Groups of m run along K.  G = ceil(K/m), the tail group is
 *     zero-padded (score 0, value 0).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and returns an nm_status.  Argument errors are detected on
 *     the host before anything is launched; in that case nothing is launched and
 *     no output is touched.  The library never aborts, exits or traps.
 *   - Pointers given to TMA-fed calls (the GEMMs and nm_sparse_prepare's
 *     output) must be 16-byte aligned and their leading dimensions multiples of
 *     8 elements; other calls need 16-byte aligned X/W/S and ld % 8 == 0 too.
 *     Violations return NM_ERR_ALIGN.
 *   - Outputs are fully overwritten, padding included.
 *   - Kernels that wait on barriers give up after about one second, record
 *     NM_ERR_TIMEOUT in the device error word and return; read it with
 *     nm_check_device_error.
 */
#ifndef NMSPARSE_H
#define NMSPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NM_OK = 0,
    NM_ERR_NULL = 1,         /* a required pointer is NULL */
    NM_ERR_SHAPE = 2,        /* a size is < 1, an ld is too small, or a size is too large */
    NM_ERR_ALIGN = 3,        /* pointer not 16-byte aligned or ld not a multiple of 8 */
    NM_ERR_UNSUPPORTED = 4,  /* n:m pattern not supported by this call */
    NM_ERR_WORKSPACE = 5,    /* workspace or packed buffer smaller than required */
    NM_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed */
    NM_ERR_TIMEOUT = 7,      /* a device-side barrier wait gave up (device error word) */
    NM_ERR_DEVICE = 8,       /* a device-side consistency check failed (device error word) */
    NM_ERR_TOO_LARGE = 9     /* reserved: no call returns it */
} nm_status;

/* Human-readable name of a status code.  Never NULL. */
const char *nm_status_string(int status);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns NM_OK, NM_ERR_TIMEOUT, NM_ERR_DEVICE or NM_ERR_CUDA. */
nm_status nm_check_device_error(void *stream);

/* Library version, (major << 16) | minor. */
int nm_version(void);

/* ------------------------------------------------------------------------ */
/* a1: diagonal Gauss-Newton proxy (Sparsity Induction, sec. 2C).
 *   H[j] = fl( fl(sum_t X[t,j]^2) / T ): the exact sum of the squares (each a
 *   dyadic rational) rounded once to fp64, to nearest with ties to even, then
 *   one correctly rounded division by T.  No summation order enters the
 *   result: it equals math.fsum of the squares divided by T, bit for bit, on
 *   any implementation.  A column holding a NaN gives NaN; otherwise one
 *   holding an infinity gives +inf.
 *   X  : [T x K] bf16, ldx >= K, 1 <= T <= NM_HESSIAN_MAX_TOKENS.
 *   H  : [K] fp64 (output), 8-byte aligned.
 *   ws : scratch of nm_hessian_workspace_bytes(T, K) bytes, 16-byte aligned
 *        (may be NULL when that is 0: T <= 128 or K of about 56,000 and
 *        more); at most a few MB whatever T.  Contents on return unspecified.
 *        Unused where the token ranges of a column strip are combined inside
 *        a thread-block cluster (when every cluster fits on the device).
 *   Errors: NULL X or H -> NM_ERR_NULL; T, K < 1, ldx < K, T too large ->
 *   NM_ERR_SHAPE; alignment -> NM_ERR_ALIGN; short ws -> NM_ERR_WORKSPACE.  */
#define NM_HESSIAN_MAX_TOKENS 2147483647ll
size_t nm_hessian_workspace_bytes(int64_t T, int64_t K);
nm_status nm_hessian_diag(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, double *H,
                          void *ws, size_t ws_bytes, void *stream);

/* Allocation-free variant of nm_hessian_diag.  The papers have no counterpart:
 * this is a convenience of this library for callers that cannot allocate
 * device memory -- for example a plugin running inside a host framework that
 * owns all device memory and hands its plugins no allocator, or a
 * latency-critical loop where a cudaMalloc/cudaFree (which may synchronise the
 * device) is not acceptable.  It returns exactly what nm_hessian_diag returns
 * (the same kernels; H is the correctly rounded sum divided by T, so it is
 * bit-identical) but keeps the blocks' partial sums in a fixed scratch array
 * inside the library instead of a caller-provided workspace.  The caller
 * still passes X and H.
 *   Limit: the array holds NM_HESSIAN_NOALLOC_MAX_PAIRS partial pairs (2 MiB).
 *   A call never needs more: the number of token ranges is capped at
 *   NM_HESSIAN_NOALLOC_MAX_PAIRS / K (each block then takes more tokens), and
 *   a single range, which K above NM_HESSIAN_NOALLOC_MAX_PAIRS / 2 gets,
 *   needs no scratch.  So every size nm_hessian_diag accepts is accepted;
 *   sizes beyond that (T > NM_HESSIAN_MAX_TOKENS) return NM_ERR_SHAPE and
 *   launch nothing.
 *   Memory: the scratch is a static device array; every GPU that loads the
 *   library holds those 2 MiB until the process exits.
 *   Set-up: the first call on each device that needs the array looks up its
 *   device address (with that device current) and caches it; make that first
 *   call before any stream capture.  The cached address belongs to the
 *   device's current context: after cudaDeviceReset the library must be
 *   unloaded and loaded again before this entry point is used.  It calls no
 *   cudaMalloc, cudaFree or other allocating routine.
 *   Where a column strip's token ranges fit on the device as one
 *   thread-block cluster each (so on a B200), their partial sums are
 *   combined in the clusters' shared memory and the array is not used; it
 *   serves devices where they do not fit.
 *   Sharing: all calls on a device share the one array and it keeps the last
 *   call's contents (every pair is written before it is read, so nothing
 *   needs clearing).  Calls whose kernels may overlap on the GPU -- on
 *   different streams, or from different host threads -- race on the array
 *   and must be serialised by the caller.                                   */
#define NM_HESSIAN_NOALLOC_MAX_PAIRS 131072
nm_status nm_hessian_diag_noalloc(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, double *H,
                                  void *stream);

/* a1 + a2: importance score (SparseForge, Hessian-aware importance).
 *   X != NULL: H = nm_hessian_diag(X) (written to H, which must be non-NULL),
 *              S[i,j] = fp32( (H[j] + eps) * W[i,j]^2 ), fp64 add and multiply,
 *              one round-to-nearest-even to fp32.
 *   X == NULL: S[i,j] = |W[i,j]| (latent-magnitude score; H, ws unused).
 *   W : [R x K] bf16, ldw >= K.  S : [R x K] fp32, row stride K (output).
 *   ws: as for nm_hessian_diag.                                             */
nm_status nm_score(const uint16_t *X, int64_t T, int64_t ldx, const uint16_t *W, int64_t R,
                   int64_t K, int64_t ldw, double eps, double *H, float *S, void *ws,
                   size_t ws_bytes, void *stream);

/* a2 only, from a given H: S[i,j] = fp32((H[j] + eps) * W[i,j]^2). */
nm_status nm_score_from_hessian(const double *H, double eps, const uint16_t *W, int64_t R,
                                int64_t K, int64_t ldw, float *S, void *stream);

/* a3: group top-n selection, compression and 2:4 metadata.
 *   S     : [R x K] fp32 scores (>= 0, finite), row stride lds >= K.
 *   V     : [R x K] bf16 values to compress (W, or ternary W_q), ldv >= K.
 *   n, m  : 1 <= n < m <= 16.
 *   mask  : [R x ceil(G*m/32)] uint32 (output): bit (c%32) of word c/32 of a
 *           row is set iff column c is kept (padding columns included; bits
 *           past G*m are zero).
 *   vals  : [R x G*n] bf16 (output): the kept values of each group in
 *           ascending column order (a kept padding column stores 0).
 *   meta24: [R x ceil(G/2)] bytes (output, only when m == 4, else may be NULL):
 *           one nibble per group, idx0 | idx1 << 2 (idx0 < idx1), the even
 *           group in the low nibble.
 * Ties go to the lower column index; -0 and +0 tie.                         */
nm_status nm_prune_compress(const float *S, int64_t lds, const uint16_t *V, int64_t ldv,
                            int64_t R, int64_t K, int n, int m, uint32_t *mask, uint16_t *vals,
                            uint8_t *meta24, void *stream);

/* O(d_in) score refresh (Sparsity Induction sec. 2C "Snelle Hessian Update"):
 * under the equivalent per-channel scaling W' = W diag(s), X' = X diag(1/s)
 * the proxy of X' is H'_j = H_j / (s_j * s_j) (fp64: one multiply, one
 * division), so the scores of W' follow from nm_score_from_hessian(H', ...)
 * without re-reading X.  H, s, H_out: [K] fp64, 8-byte aligned; H_out may be
 * H itself.                                                                 */
nm_status nm_hessian_rescale(const double *H, const double *s, int64_t K, double *H_out, void *stream);

/* Hutchinson's stochastic estimate of diag(A), A = X^T X / T, from S
 * Rademacher vectors z_s (SparseForge, arXiv 2605.06402, "Estimativa de
 * Importancia Consciente do Hessiano"; the vectors are inputs, drawn by the
 * caller):   D_k = (1/S) sum_s z_s[k] (X^T (X z_s))[k] / T.
 * Its expectation is H_k of nm_hessian_diag; the error falls as 1/sqrt(S).
 *   X     : bf16 [T x ldx] row-major, 16-byte aligned, ldx % 8 == 0, ldx >= K.
 *   zbits : uint32 [S x ceil(K/32)], 4-byte aligned; bit k % 32 of word k / 32
 *           of row s set = z_s[k] = -1, clear = +1.  1 <= S <= 256.
 *   D     : fp64 [K] (written), 8-byte aligned.
 *   ws    : nm_hutchinson_workspace_bytes(T, K, S) bytes, 16-byte aligned,
 *           owned by the caller; contents on return unspecified.  It holds,
 *           each region padded to 1 KiB: Z as bf16 [S16 x ldz] (S16 = S
 *           rounded up to 16, ldz = K rounded up to 8), [Z^T Z^T Z^T] as bf16
 *           [K x C3] (C3 = 3S rounded up to 64), the fp32 partials of U = X Z^T
 *           [nsplit x T x S16], U split into bf16 pieces [T x C3] and fp64
 *           partials of D [ceil(T/128) x K]; nsplit = min(8, ceil(K/64),
 *           ceil(148 / ceil(T/128))).

 * Arithmetic (tensor cores, bf16 operands, fp32 accumulation): U = X Z^T
 * over K split into nsplit ranges, the partials added in ascending order;
 * each u split exactly into three bf16 pieces; P = Z^T U^T from the pieces;
 * x * P summed in fp32 over 32 tokens, in fp64 over 128-token tiles, the tiles
 * in ascending order, then one multiply by 1/(S T).  Deterministic run to run.
 * Errors: NULL -> NM_ERR_NULL; S outside [1, 256], T or K < 1 or above
 * 2^31 - 128, ldx < K -> NM_ERR_SHAPE; alignment -> NM_ERR_ALIGN; short
 * workspace -> NM_ERR_WORKSPACE.                                            */
size_t nm_hutchinson_workspace_bytes(int64_t T, int64_t K, int64_t S);
nm_status nm_hutchinson_diag(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, const uint32_t *zbits,
                             int64_t S, double *D, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* FP8 path (SlideSparse, arXiv 2603.05232, sec. 2B: the activation lift is
 * fused into the per-token INT8/FP8/FP4 quantisation kernel; sec. 2C: online,
 * the fused quantise-and-lift kernel, then the sparse GEMM).  Format E4M3
 * (largest finite 448); codes are fp32(x * inv), inv = fp32(1 / scale),
 * rounded to nearest even, saturating; scale = amax / 448 in fp32 (1 when
 * amax is 0), per token for
 * the activations and per weight row (over its kept values) for the weights.
 * m in {4, 6, 8, 10} (2:4 and the (2N-2):2N patterns); the lifted columns are
 * in natural window order (window w of group g = columns g m + 2w .. + 3),
 * padded with zero codes to KLf = nm_lifted_cols_f8(K, m), a multiple of 256.
 *
 * nm_quant_lift_f8: X bf16 [T x ldx] (16-byte aligned, ldx % 8 == 0) ->
 *   Xq E4M3 codes [T x ldq] (16-byte aligned, ldq % 16 == 0, ldq >= KLf; all
 *   ldq columns are written, zero past the lifted width) and xscale fp32 [T].
 * nm_sparse_prepare_f8: vals [R x G n] bf16 and window metadata wmeta
 *   (meta24 for m = 4; nm_slide_pack's for m > 4, one nibble per window, row
 *   stride ceil(windows / 2) bytes) -> packed: codes [Rpad x KLf/2] (Rpad = R
 *   rounded up to 128; the kept order is the window order), then metadata
 *   blocks of 4096 bytes per (128-row tile, 256-column K' block) = two atoms
 *   of [128 rows x 16 bytes] (row-major; byte i of atom a of block kb holds the
 *   nibbles of windows 64 kb + 32 a + 2i (low) and + 1 (high)), then the row
 *   scales fp32 [Rpad].  Size: nm_sparse_prepare_f8_bytes(R, K, m).
 * nm_sparse_gemm_f8: Y[t, r] = bf16(xscale[t] ws[r] sum E4M3 products), the
 *   products accumulated in fp32 by tcgen05.mma.sp kind::f8f6f4; Y bf16
 *   [T x ldy], ldy % 8 == 0, ldy >= R.
 * Errors: NULL -> NM_ERR_NULL; other m -> NM_ERR_UNSUPPORTED; sizes, ld too
 * small -> NM_ERR_SHAPE; alignment -> NM_ERR_ALIGN; short packed buffer ->
 * NM_ERR_WORKSPACE.                                                         */
int64_t nm_lifted_cols_f8(int64_t K, int m);
size_t nm_sparse_prepare_f8_bytes(int64_t R, int64_t K, int m);
nm_status nm_quant_lift_f8(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, int m, uint8_t *Xq, int64_t ldq,
                           float *xscale, void *stream);
nm_status nm_sparse_prepare_f8(const uint16_t *vals, const uint8_t *wmeta, int64_t R, int64_t K, int m,
                               void *packed, size_t packed_bytes, void *stream);
nm_status nm_sparse_gemm_f8(const uint8_t *Xq, int64_t T, int64_t K, int64_t ldq, const float *xscale,
                            const void *packed, int64_t R, int m, uint16_t *Y, int64_t ldy, void *stream);

/* a2 + a3 fused: exactly nm_score_from_hessian followed by nm_prune_compress
 * (bit-identical mask, vals and meta24), with each score formed in registers
 * from W -- fp32((H_j + eps) * W_ij^2), fp64 add and multiplies, rounded once;
 * or |W_ij| when H == NULL -- and never written: HBM traffic per weight drops
 * from 2 + 4 (score) + 4 + 2 (prune) bytes read/written to the 2 (+ 2 for a
 * separate V) read by the selection.
 *   H : [K] fp64 (8-byte aligned) or NULL.  W : [R x K] bf16, ldw >= K,
 *   ldw % 8 == 0.  V, mask, vals, meta24 and all rules as nm_prune_compress;
 *   V may be W itself (then W is read once).                                */
nm_status nm_score_prune_compress(const double *H, double eps, const uint16_t *W, int64_t ldw,
                                  const uint16_t *V, int64_t ldv, int64_t R, int64_t K, int n, int m,
                                  uint32_t *mask, uint16_t *vals, uint8_t *meta24, void *stream);

/* a4: sliding-window pack (SlideSparse, sec. 2A), m = 2N in {4, 6, 8, 10},
 * n = m - 2.  Survivor k (0-based, ascending) of a group goes to window k/2,
 * in-window index q_k - 2*(k/2) in [0, 3].  The window values are exactly
 * nm_prune_compress's `vals`; only the metadata is new.
 *   mask  : as written by nm_prune_compress with n = m - 2.
 *   wmeta : [R x ceil(G*(N-1)/2)] bytes (output), one nibble idx0 | idx1 << 2
 *           per window in (group, window) order, even window in the low nibble.
 * A group that does not hold exactly m-2 survivors sets NM_ERR_DEVICE in the
 * device error word (its nibbles are written as 0).                        */
nm_status slide_pack(const uint32_t *mask, int64_t R, int64_t K, int m, uint8_t *wmeta,
                     void *stream);

/* a5 (standalone form): activation lifting (SlideSparse, sec. 2B).
 *   XL[t, g*4(N-1) + 4w + i] = X[t, g*m + 2w + i], 0 where g*m+2w+i >= K.
 *   X : [T x K] bf16, ldx >= K.  XL : [T x G*(N-1)*4] bf16, ldxl >= that.
 * nm_sparse_gemm runs this step itself for 4:6 and 8:10 (into its workspace)
 * before a 2:4 GEMM of width K'; the standalone call exists for tests and for
 * callers that keep X' for several layers.                                  */
nm_status lift_activations(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, int m,
                           uint16_t *XL, int64_t ldxl, void *stream);

/* a6: operand preparation (SlideSparse sec. 2C item 2, initialisation).
 * Lays the window values and window metadata of a layer out in the order and
 * tiling nm_sparse_gemm reads (padded rows and windows hold zero values and
 * the index pair (0,1)).  For m == 4 the metadata is meta24 (identical to the
 * window metadata of a 2:4 pattern).  The packed buffer is opaque; its size
 * is nm_sparse_prepare_bytes(R, K, m).                                      */
size_t nm_sparse_prepare_bytes(int64_t R, int64_t K, int m);
nm_status nm_sparse_prepare(const uint16_t *vals, const uint8_t *wmeta, int64_t R, int64_t K,
                            int m, void *packed, size_t packed_bytes, void *stream);

/* a4 + a6 in one pass: the same packed operand as slide_pack followed by
 * nm_sparse_prepare, with each window's index pair formed from the mask bits
 * as the metadata is written (the sliding-window pack of SlideSparse sec. 2A:
 * survivor k of a group at window k/2, index q_k - 2*(k/2)), so the window
 * metadata is never stored.  m in {4, 6, 8, 10}, n = m - 2 (for 2:4 the pairs
 * are meta24's).
 *   vals  : [R x G n] bf16 from nm_prune_compress, 4-byte aligned.
 *   mask  : [R x ceil(G m / 32)] u32 from nm_prune_compress, 4-byte aligned.
 * A group that does not hold exactly m - 2 survivors sets NM_ERR_DEVICE in
 * the device error word (its pairs are written as padding).  Errors as for
 * nm_sparse_prepare.                                                        */
nm_status nm_sparse_prepare_from_mask(const uint16_t *vals, const uint32_t *mask, int64_t R, int64_t K,
                                      int m, void *packed, size_t packed_bytes, void *stream);

/* a7: sparse GEMM (SlideSparse sec. 2C item 3; 2:4 sparse tensor cores).
 *   Y[t, r] = sum_k X[t,k] * (mask (.) V)[r,k], fp32 accumulation in tensor
 *   memory, bf16 output (round to nearest even).
 *   X : [T x K] bf16, ldx >= K, ldx % 8 == 0.   Y : [T x R] bf16, ldy >= R.
 *   packed: from nm_sparse_prepare(..., R, K, m, ...).  m in {4, 6, 8, 10}.
 *   Activation lifting (SlideSparse sec. 2B), by pattern:
 *     2:4  none;
 *     6:8  two thirds of the lifted operand are tiles of X itself (windows 0
 *          and 2 of every group are X's own columns), loaded straight into the
 *          GEMM's shared-memory staging; the middle windows (columns 2..5 of
 *          every group) are first gathered into `ws` (T x K/2) and loaded the
 *          same way;
 *     4:6, 8:10  the lifted activations X' are written to `ws` (T x K') and the
 *          product runs as a 2:4 GEMM over K'.
 *   ws : device scratch, 16-byte aligned; nm_sparse_gemm_workspace_bytes(T,
 *        K, m) bytes give the fastest schedule.  Its first part holds the
 *        staged activations above (T x K/2 bf16 for 6:8, T x K' for 4:6 and
 *        8:10, nothing for 2:4; too small -> NM_ERR_WORKSPACE); the rest, at
 *        the next 256-byte boundary, holds stream-K partial sums (below).  A
 *        workspace without that part (NULL for 2:4) still works, always with
 *        whole-tile scheduling.
 *   Scheduling: a persistent grid of CTA pairs (one per two SMs) walks the
 *   output tiles of 512 weight rows x up to 240 tokens.  When the tiles leave part of the last wave idle
 *   (decode-sized T, few tiles) the K' blocks of all tiles are split evenly
 *   over the pairs instead (stream-K); the pair that starts a split tile adds
 *   the fp32 partial sums of the pairs after it in ascending order, so results
 *   are deterministic for a given device and schedule.  The workspace must
 *   not be shared by calls that may run at the same time (other streams).
 *   Waits between pairs are bounded: after one second the call gives up and
 *   sets NM_ERR_TIMEOUT in the device error word.                          */
size_t nm_sparse_gemm_workspace_bytes(int64_t T, int64_t K, int m);
nm_status nm_sparse_gemm(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                         const void *packed, int64_t R, int m, uint16_t *Y, int64_t ldy,
                         void *ws, size_t ws_bytes, void *stream);

/* a8: dense reference GEMM on the tensor cores, Y = X * W^T (W = mask (.) V
 * densified by the caller), fp32 accumulation, bf16 output.  Same tiling and
 * scheduling as nm_sparse_gemm; ws (16-byte aligned, may be NULL: whole-tile
 * scheduling) of nm_dense_gemm_workspace_bytes(T, K, R) bytes enables
 * stream-K.                                                                 */
size_t nm_dense_gemm_workspace_bytes(int64_t T, int64_t K, int64_t R);
nm_status nm_dense_gemm(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, const uint16_t *W,
                        int64_t R, int64_t ldw, uint16_t *Y, int64_t ldy, void *ws,
                        size_t ws_bytes, void *stream);

/* Upper bound on the CTA pairs a stream-K launch uses (its partial-sum
 * region is sized for this many: 2*8 slots of 32 x 240 fp32 plus 2*8 64-bit
 * flags per pair).                                                          */
#define NM_GEMM_STREAMK_MAX_CLUSTERS 96

/* Process-wide GEMM schedule, for tests and measurements (not thread-safe
 * against GEMM calls being issued concurrently on other host threads).
 *   policy   : 0 automatic (default), 1 whole tiles only, 2 stream-K whenever
 *              the workspace allows it.
 *   clusters : 0 = as many CTA pairs as fit on the device at once, else at
 *              most this many.
 * Returns NM_ERR_SHAPE for a policy outside 0..2 or clusters < 0.          */
nm_status nm_gemm_set_schedule(int policy, int clusters);

/* Ternary absmean quantisation (Sparse-BitNet sec. 1 item 1), input
 * preparation of the ternary 6:8 layer.
 *   gamma = fl( fl(sum of |W|) / (R*K) ): the exact sum of the magnitudes
 *           rounded once to fp64 (nearest, ties to even), one division -- no
 *           summation order enters it;
 *   q     = clip(rint(W / gamma), -1, 1) (fp64 division, ties to even);
 *   W_q   = q * bf16(gamma), bf16(gamma) rounded to nearest even from fp64,
 *           zeros stored as +0.
 *   W : [R x K] bf16, ldw >= K.  Wq : [R x K] bf16 (output, row stride K).
 *   gamma : one fp64 on the device (output).  ws : nm_ternary_workspace_bytes(R).
 * If bf16(gamma) falls outside the normal bf16 range (W holding an infinity
 * or a NaN included) the device error word gets NM_ERR_DEVICE and Wq is all
 * zero.  ws: R * 16 + 16 bytes, 16-byte aligned.                           */
size_t nm_ternary_workspace_bytes(int64_t R);
nm_status nm_ternary_quantize(const uint16_t *W, int64_t R, int64_t K, int64_t ldw, uint16_t *Wq,
                              double *gamma, void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NMSPARSE_H */
