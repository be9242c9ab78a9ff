// nm_hutch.cu -- Hutchinson's stochastic estimate of diag(X^T X / T) on the
// 5th-generation tensor cores.
//
// SparseForge (arXiv 2605.06402), "Estimativa de Importancia Consciente do
// Hessiano": the Hessian diagonal is estimated with Rademacher vectors z_s,
//     D_k = (1/S) sum_s z_s[k] (A z_s)[k],   A = X^T X / T,
// whose expectation is H_k = (1/T) sum_t x_{t,k}^2.  With u_s = X z_s this is
//     D_k = (1/(S T)) sum_t x_{t,k} p_{t,k},   p_{t,k} = sum_s z_s[k] u_{t,s},
// two dense contractions with a short inner dimension (S <= 256):
//
//   1. U = X Z^T     [T x S]: tcgen05 GEMM, M = 128 tokens, N = S rounded up to
//                    16, K = the layer width split over up to 8 CTAs per token
//                    tile; fp32 partials in the workspace.
//   2. combine       the K-split partials added in ascending order (fp32) and
//                    each u split exactly into three bf16 pieces hi + mid + lo
//                    (8 significant bits each cover fp32's 24), laid out as
//                    U3 = [hi | mid | lo | 0-pad] with 3S columns padded to 64.
//   3. P = Z3 U3^T   tcgen05 GEMM, M = 128 columns k, N = 128 tokens, inner
//                    dimension 3S (Z3 = [Z^T | Z^T | Z^T]), so P = Z^T U^T in
//                    fp32 with bf16 operands and no loss from rounding U.  The
//                    epilogue multiplies each accumulator row (a column k of X)
//                    by the X tile staged in shared memory and sums over the
//                    tile's tokens: fp32 over 32 tokens, fp64 over the tile.
//   4. finish        the token-tile partials in ascending order, times 1/(S T)
//                    (a programmatic dependent of step 3).
//
// Every summation order is fixed by the shapes alone, so the estimate is the
// same run to run.  The sign vectors are inputs (one bit per entry).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nm_common.cuh"
#include "nm_host.cuh"

namespace nm {

constexpr int HQ_M = 128;           // accumulator rows per CTA (tokens in 1, columns in 3)
constexpr int HQ_N2 = 128;          // tokens per tile in step 3
constexpr int HQ_THREADS = 256;     // warp 0 TMA, warp 1 MMA + tensor memory, warps 4-7 epilogue
constexpr int HQ_MAX_S = 256;
constexpr int HQ_MAX_SPLIT = 8;     // K-split of step 1
constexpr int HQ_TARGET_CTAS = 148; // one wave of CTAs on a B200 for step 1's split
constexpr int HQ_STAGE_LIMIT = 200 * 1024;
constexpr int HQ2_STAGES = 4;
constexpr int HQ2_NB = 3;                             // X tiles / accumulators in flight
constexpr int HQ2_AB_BYTES = 2 * HQ_M * 128;          // A and B tiles of one 64-wide block: 32 KB
constexpr int HQ2_X_BYTES = HQ_N2 * HQ_M * 2;         // X tile [128 tokens x 128 columns]: 32 KB
constexpr int HQ2_SMEM_BYTES = HQ2_STAGES * HQ2_AB_BYTES + HQ2_NB * HQ2_X_BYTES + 256 + 1024;

constexpr uint16_t BF16_ONE = 0x3F80u, BF16_MINUS_ONE = 0xBF80u;

__device__ __forceinline__ uint16_t sign_bf16(const uint32_t *__restrict__ zbits, int64_t words, int64_t s,
                                              int64_t k) {
    return ((__ldg(zbits + s * words + (k >> 5)) >> (k & 31)) & 1u) ? BF16_MINUS_ONE : BF16_ONE;
}

// Z [S16 x ldz] (rows past S zero), eight values (16 bytes) per thread
__global__ void __launch_bounds__(256) k_hq_signs_z(const uint32_t *__restrict__ zbits, int S, int64_t K,
                                                    int S16, int64_t ldz, uint16_t *__restrict__ Zb) {
    const int64_t words = (K + 31) / 32;
    const int64_t zrow = ldz / 8, nz = S16 * zrow;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nz; i += stride) {
        const int64_t srow = i / zrow, k0 = (i - srow * zrow) * 8;
        uint32_t o[4] = {0u, 0u, 0u, 0u};
        if (srow < S && k0 < K) {
            const uint32_t bits = __ldg(zbits + srow * words + (k0 >> 5)) >> (k0 & 31);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t v = (k0 + j < K) ? (((bits >> j) & 1u) ? BF16_MINUS_ONE : BF16_ONE) : 0u;
                o[j >> 1] |= v << (16 * (j & 1));
            }
        }
        *reinterpret_cast<uint4 *>(Zb + i * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Z3 [K x C3]: row k = z_0..z_{S-1} at [k], three times, then zeros.  A block
// holds 256 / S16 rows, one thread per (row, sample); sample slots past S
// write the zero padding.
__global__ void __launch_bounds__(256) k_hq_signs_z3(const uint32_t *__restrict__ zbits, int S, int64_t K,
                                                     int S16, int C3, uint16_t *__restrict__ Z3) {
    const int64_t words = (K + 31) / 32;
    const int rpb = 256 / S16;
    const int rl = threadIdx.x / S16, sidx = threadIdx.x - rl * S16;
    if (rl >= rpb) return;
    for (int64_t k = static_cast<int64_t>(blockIdx.x) * rpb + rl; k < K; k += static_cast<int64_t>(gridDim.x) * rpb) {
        uint16_t *row = Z3 + k * C3;
        if (sidx < S) {
            const uint16_t v = ((__ldg(zbits + sidx * words + (k >> 5)) >> (k & 31)) & 1u) ? BF16_MINUS_ONE : BF16_ONE;
            row[sidx] = v;
            row[S + sidx] = v;
            row[2 * S + sidx] = v;
        }
        for (int c = 3 * S + sidx; c < C3; c += S16) row[c] = 0;
    }
}

// ---------------------------------------------------------------------------
// Step 1: U partial [split][T][S16] = X[tile, k-range] * Z[:, k-range]^T.
// Stage s: A = X tile [128 x 64] (16 KB), B = Z tile [S16 x 64]; both TMA,
// 128-byte swizzle, K-major.  Stage count and size are set at launch.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(HQ_THREADS, 1)
    k_hq_u(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmZ, int64_t T,
           int64_t nkb, int nsplit, int S16, int stages, int stage_bytes, uint32_t tmem_cols,
           float *__restrict__ Up) {
    extern __shared__ uint8_t hq_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(hq_smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + stages * stage_bytes);
    uint64_t *full = bars, *empty = bars + stages, *accum = bars + 2 * stages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tt = blockIdx.x, sp = blockIdx.y;
    const int64_t kb0 = sp * nkb / nsplit, kb1 = (sp + 1) * nkb / nsplit;
    const uint32_t tx = static_cast<uint32_t>(HQ_M * 128 + S16 * 128);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmZ);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int64_t i = 0;
            for (int64_t kb = kb0; kb < kb1; ++kb, ++i) {
                const int s = static_cast<int>(i % stages);
                if (i >= stages && !mbar_wait(&empty[s], static_cast<uint32_t>(((i / stages) & 1) ^ 1))) {
                    *abort_flag = 1;
                    break;
                }
                uint8_t *st = smem + s * stage_bytes;
                mbar_arrive_expect_tx(&full[s], tx);
                tma_load_2d(st, &tmX, &full[s], static_cast<int32_t>(kb * 64), static_cast<int32_t>(tt * HQ_M));
                tma_load_2d(st + HQ_M * 128, &tmZ, &full[s], static_cast<int32_t>(kb * 64), 0);
            }
            if (*abort_flag)  // let the copies already issued land
                for (int64_t j = (i > stages ? i - stages : 0); j < i; ++j)
                    mbar_wait(&full[j % stages], static_cast<uint32_t>((j / stages) & 1));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(HQ_M, static_cast<uint32_t>(S16), false, 0);
            bool ok = true;
            int64_t i = 0;
            for (int64_t kb = kb0; kb < kb1; ++kb, ++i) {
                const int s = static_cast<int>(i % stages);
                if (!mbar_wait(&full[s], static_cast<uint32_t>((i / stages) & 1))) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * stage_bytes), b0 = a0 + HQ_M * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16(tmem, make_sdesc(a0 + j * 32, 16, 1024, 2), make_sdesc(b0 + j * 32, 16, 1024, 2),
                             idesc, (i > 0 || j > 0) ? 1u : 0u);
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(accum);
            else *abort_flag = 1;
        }
    } else if (warp >= 4) {
        const int ew = warp - 4;
        // an empty K range (more splits than blocks never happens: nsplit <= nkb)
        bool ok = __all_sync(0xffffffffu, mbar_wait(accum, 0));
        if (ok) {
            tc_fence_after();
            const int64_t t = tt * HQ_M + ew * 32 + lane;
            float *row = Up + (sp * T + t) * S16;
            for (int c0 = 0; c0 < S16; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(ew * 32) << 16) + c0, v);
                tmem_ld_wait();
                if (t < T) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4 *>(row + c0 + 4 * q) =
                            make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                        __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// Step 2: u = sum of the K-split partials (ascending), split into three bf16
// pieces hi, mid, lo (u - hi and the next remainder are exact in fp32) stored
// at columns s, S + s, 2S + s of U3; the columns from 3S to C3 are zero.  A
// block holds 256 / S16 tokens, one thread per (token, sample).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_hq_combine(const float *__restrict__ Up, int64_t T, int S, int S16,
                                                    int nsplit, int C3, uint16_t *__restrict__ U3) {
    const int tpb = 256 / S16;
    const int tl = threadIdx.x / S16, sidx = threadIdx.x - tl * S16;
    if (tl >= tpb) return;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * tpb + tl; t < T; t += static_cast<int64_t>(gridDim.x) * tpb) {
        uint16_t *row = U3 + t * C3;
        if (sidx < S) {
            float u = Up[t * S16 + sidx];
            for (int q = 1; q < nsplit; ++q) u = __fadd_rn(u, Up[(q * T + t) * S16 + sidx]);
            const __nv_bfloat16 hi = __float2bfloat16_rn(u);
            const float r1 = __fsub_rn(u, __bfloat162float(hi));
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const float r2 = __fsub_rn(r1, __bfloat162float(mid));
            const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
            row[sidx] = *reinterpret_cast<const uint16_t *>(&hi);
            row[S + sidx] = *reinterpret_cast<const uint16_t *>(&mid);
            row[2 * S + sidx] = *reinterpret_cast<const uint16_t *>(&lo);
        }
        for (int c = 3 * S + sidx; c < C3; c += S16) row[c] = 0;
    }
}

// ---------------------------------------------------------------------------
// Step 3: persistent CTAs over the (column tile, token tile) units, token
// tiles fastest.  Per unit: the X tile [128 tokens x 128 columns] (one TMA
// box, no swizzle) into one of three buffers, the A = Z3 and B = U3 tiles of
// each 64-wide block of the inner dimension through a four-stage ring, the
// accumulator P [128 columns x 128 tokens] into one of three tensor-memory
// buffers, so that up to three units are in flight.  Epilogue thread =
// accumulator row = column k: sum_j x[j][k] * P[k][j].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(HQ_THREADS, 1)
    k_hq_p(const __grid_constant__ CUtensorMap tmZ3, const __grid_constant__ CUtensorMap tmU3,
           const __grid_constant__ CUtensorMap tmXt, int64_t K, int64_t ktiles, int64_t ttiles, int ncb,
           double *__restrict__ Dpart) {
    extern __shared__ uint8_t hq_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(hq_smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *xbuf = smem + HQ2_STAGES * HQ2_AB_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(xbuf + HQ2_NB * HQ2_X_BYTES);
    uint64_t *ab_full = bars, *ab_empty = bars + HQ2_STAGES;
    uint64_t *x_full = bars + 2 * HQ2_STAGES, *x_empty = x_full + HQ2_NB;
    uint64_t *acc_full = x_empty + HQ2_NB, *acc_empty = acc_full + HQ2_NB;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + HQ2_NB);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    grid_dep_launch();  // step 4 may be scheduled; it waits for this grid to finish
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t units = ktiles * ttiles;
    const int64_t mine = units > blockIdx.x ? (units - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    auto unit_of = [&](int64_t i) { return static_cast<int64_t>(blockIdx.x) + i * gridDim.x; };
    // use i of buffer i % NB is that buffer's (i / NB)-th phase
    auto use_parity = [](int64_t i) { return static_cast<uint32_t>((i / HQ2_NB) & 1); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < HQ2_STAGES; ++s) {
            mbar_init(&ab_full[s], 1);
            mbar_init(&ab_empty[s], 1);
        }
        for (int b = 0; b < HQ2_NB; ++b) {
            mbar_init(&x_full[b], 1);
            mbar_init(&x_empty[b], 4);
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmZ3);
        prefetch_tmap(&tmU3);
        prefetch_tmap(&tmXt);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int64_t g = 0;   // stage counter over all units
            int64_t xi = 0;  // X tiles issued
            bool ok = true;
            for (int64_t i = 0; i < mine && ok; ++i) {
                const int64_t q = unit_of(i), kt = q / ttiles, tt = q - kt * ttiles;
                const int b = static_cast<int>(i % HQ2_NB);
                if (i >= HQ2_NB && !mbar_wait(&x_empty[b], use_parity(i) ^ 1u)) { ok = false; break; }
                mbar_arrive_expect_tx(&x_full[b], HQ2_X_BYTES);
                tma_load_2d(xbuf + b * HQ2_X_BYTES, &tmXt, &x_full[b], static_cast<int32_t>(kt * HQ_M),
                            static_cast<int32_t>(tt * HQ_N2));
                ++xi;
                for (int cb = 0; cb < ncb; ++cb, ++g) {
                    const int s = static_cast<int>(g % HQ2_STAGES);
                    if (g >= HQ2_STAGES &&
                        !mbar_wait(&ab_empty[s], static_cast<uint32_t>(((g / HQ2_STAGES) & 1) ^ 1))) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * HQ2_AB_BYTES;
                    mbar_arrive_expect_tx(&ab_full[s], HQ2_AB_BYTES);
                    tma_load_2d(st, &tmZ3, &ab_full[s], cb * 64, static_cast<int32_t>(kt * HQ_M));
                    tma_load_2d(st + HQ_M * 128, &tmU3, &ab_full[s], cb * 64, static_cast<int32_t>(tt * HQ_N2));
                }
            }
            if (!ok) {  // let the copies already issued land
                *abort_flag = 1;
                for (int64_t j = (g > HQ2_STAGES ? g - HQ2_STAGES : 0); j < g; ++j)
                    mbar_wait(&ab_full[j % HQ2_STAGES], static_cast<uint32_t>((j / HQ2_STAGES) & 1));
                for (int64_t j = (xi > HQ2_NB ? xi - HQ2_NB : 0); j < xi; ++j)
                    mbar_wait(&x_full[j % HQ2_NB], use_parity(j));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(HQ_M, HQ_N2, false, 0);
            int64_t g = 0;
            bool ok = true;
            for (int64_t i = 0; i < mine && ok; ++i) {
                const int b = static_cast<int>(i % HQ2_NB);
                if (i >= HQ2_NB && !mbar_wait(&acc_empty[b], use_parity(i) ^ 1u)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(b * HQ_N2);
                for (int cb = 0; cb < ncb; ++cb, ++g) {
                    const int s = static_cast<int>(g % HQ2_STAGES);
                    if (!mbar_wait(&ab_full[s], static_cast<uint32_t>((g / HQ2_STAGES) & 1)) || *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * HQ2_AB_BYTES), b0 = a0 + HQ_M * 128;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16(d, make_sdesc(a0 + j * 32, 16, 1024, 2), make_sdesc(b0 + j * 32, 16, 1024, 2),
                                 idesc, (cb > 0 || j > 0) ? 1u : 0u);
                    mma_commit(&ab_empty[s]);
                }
                if (ok) mma_commit(&acc_full[b]);
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp >= 4) {
        const int ew = warp - 4;
        const int kl = ew * 32 + lane;  // accumulator row = column within the tile
        for (int64_t i = 0; i < mine; ++i) {
            const int64_t q = unit_of(i), kt = q / ttiles, tt = q - kt * ttiles;
            const int b = static_cast<int>(i % HQ2_NB);
            const uint32_t ph = use_parity(i);
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], ph) && mbar_wait(&x_full[b], ph));
            if (!ok || *abort_flag) break;
            tc_fence_after();
            const uint16_t *xs = reinterpret_cast<const uint16_t *>(xbuf + b * HQ2_X_BYTES) + kl;
            double d = 0.0;
#pragma unroll 1
            for (int cc = 0; cc < HQ_N2 / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + static_cast<uint32_t>(b * HQ_N2 + cc * 32) +
                                       (static_cast<uint32_t>(ew * 32) << 16),
                                   v);
                tmem_ld_wait();
                float r = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float x = __uint_as_float(static_cast<uint32_t>(xs[(cc * 32 + j) * HQ_M]) << 16);
                    r = __fmaf_rn(x, __uint_as_float(v[j]), r);
                }
                d = __dadd_rn(d, static_cast<double>(r));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&acc_empty[b]);
                mbar_arrive(&x_empty[b]);
            }
            const int64_t k = kt * HQ_M + kl;
            if (k < K) Dpart[tt * K + k] = d;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Step 4: D_k = (sum over token tiles, ascending) / (S T); launched as a
// programmatic dependent of step 3, loads issued 16 partials ahead of the adds
__global__ void __launch_bounds__(64) k_hq_finish(const double *__restrict__ Dpart, int64_t ttiles, int64_t K,
                                                  double scale, double *__restrict__ D) {
    grid_dep_wait();
    const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (k >= K) return;
    double total = 0.0;
    int64_t c = 0;
    for (; c + 16 <= ttiles; c += 16) {
        double v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = Dpart[(c + u) * K + k];
#pragma unroll
        for (int u = 0; u < 16; ++u) total = __dadd_rn(total, v[u]);
    }
    for (; c < ttiles; ++c) total = __dadd_rn(total, Dpart[c * K + k]);
    D[k] = __dmul_rn(total, scale);
}

}  // namespace nm

// ===========================================================================
// C ABI
// ===========================================================================
using namespace nm;

namespace {

struct HqGeom {
    int64_t S16, C3, ldz, nkb, ttiles, ktiles, nsplit;
    size_t off_z3, off_up, off_u3, off_dp, total;
};

size_t align1k(size_t b) { return (b + 1023) / 1024 * 1024; }

// every size and offset follows from T, K and S alone
HqGeom hq_geometry(int64_t T, int64_t K, int64_t S) {
    HqGeom g{};
    g.S16 = (S + 15) / 16 * 16;
    g.C3 = (3 * S + 63) / 64 * 64;
    g.ldz = (K + 7) / 8 * 8;
    g.nkb = (K + 63) / 64;
    g.ttiles = (T + HQ_M - 1) / HQ_M;
    g.ktiles = (K + HQ_M - 1) / HQ_M;
    // K-split of step 1: enough CTAs to cover 148 SMs, at most 8 and at most
    // one per 64-column block
    int64_t ns = (HQ_TARGET_CTAS + g.ttiles - 1) / g.ttiles;
    ns = ns > HQ_MAX_SPLIT ? HQ_MAX_SPLIT : ns;
    ns = ns > g.nkb ? g.nkb : ns;
    g.nsplit = ns < 1 ? 1 : ns;
    size_t off = align1k(static_cast<size_t>(g.S16 * g.ldz) * 2);
    g.off_z3 = off;
    off += align1k(static_cast<size_t>(K * g.C3) * 2);
    g.off_up = off;
    off += align1k(static_cast<size_t>(g.nsplit * T * g.S16) * 4);
    g.off_u3 = off;
    off += align1k(static_cast<size_t>(T * g.C3) * 2);
    g.off_dp = off;
    off += align1k(static_cast<size_t>(g.ttiles * K) * 8);
    g.total = off;
    return g;
}

int hq_sm_count() {
    static int n[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HQ_TARGET_CTAS;
    if (n[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : HQ_TARGET_CTAS;
    }
    return n[dev];
}

}  // namespace

extern "C" size_t nm_hutchinson_workspace_bytes(int64_t T, int64_t K, int64_t S) {
    if (T < 1 || K < 1 || S < 1 || S > HQ_MAX_S) return 0;
    return hq_geometry(T, K, S).total;
}

extern "C" nm_status nm_hutchinson_diag(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                        const uint32_t *zbits, int64_t S, double *D, void *ws,
                                        size_t ws_bytes, void *stream) {
    if (!X || !zbits || !D || !ws) return NM_ERR_NULL;
    if (T < 1 || K < 1 || ldx < K || S < 1 || S > HQ_MAX_S) return NM_ERR_SHAPE;
    if (T > (int64_t(1) << 31) - HQ_N2 || K > (int64_t(1) << 31) - HQ_M) return NM_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(X) & 15u) || (reinterpret_cast<uintptr_t>(ws) & 15u) || (ldx % 8) != 0 ||
        (reinterpret_cast<uintptr_t>(zbits) & 3u) || (reinterpret_cast<uintptr_t>(D) & 7u))
        return NM_ERR_ALIGN;
    const HqGeom g = hq_geometry(T, K, S);
    if (ws_bytes < g.total) return NM_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint16_t *Zb = reinterpret_cast<uint16_t *>(w);
    uint16_t *Z3 = reinterpret_cast<uint16_t *>(w + g.off_z3);
    float *Up = reinterpret_cast<float *>(w + g.off_up);
    uint16_t *U3 = reinterpret_cast<uint16_t *>(w + g.off_u3);
    double *Dp = reinterpret_cast<double *>(w + g.off_dp);

    // step 1 shared memory: as many stages (at most 6) as fit
    const int stage_bytes = static_cast<int>(HQ_M * 128 + (g.S16 * 128 + 1023) / 1024 * 1024);
    int stages = HQ_STAGE_LIMIT / stage_bytes;
    stages = stages > 6 ? 6 : stages;
    const int smem1 = stages * stage_bytes + 256 + 1024;  // stages, barriers, alignment slack
    uint32_t tcols = 32;
    while (tcols < static_cast<uint32_t>(g.S16)) tcols <<= 1;

    CUtensorMap tmX1, tmZ, tmZ3, tmU3, tmX3;
    if (!make_tmap_bf16(&tmX1, X, T, K, ldx, 64, HQ_M, true) ||
        !make_tmap_bf16(&tmZ, Zb, g.S16, K, g.ldz, 64, static_cast<uint32_t>(g.S16), true) ||
        !make_tmap_bf16(&tmZ3, Z3, K, g.C3, g.C3, 64, HQ_M, true) ||
        !make_tmap_bf16(&tmU3, U3, T, g.C3, g.C3, 64, HQ_N2, true) ||
        !make_tmap_bf16(&tmX3, X, T, K, ldx, HQ_M, HQ_N2, false))
        return NM_ERR_CUDA;
    if (!set_smem_attr<k_hq_u>(HQ_STAGE_LIMIT + 256 + 1024) ||
        !set_smem_attr<k_hq_p>(HQ2_SMEM_BYTES))
        return NM_ERR_CUDA;

    const int64_t nz = g.S16 * g.ldz / 8;
    k_hq_signs_z<<<static_cast<unsigned>((nz + 255) / 256 < 1024 ? (nz + 255) / 256 : 1024), 256, 0, st>>>(
        zbits, static_cast<int>(S), K, static_cast<int>(g.S16), g.ldz, Zb);
    const int64_t rpb = 256 / g.S16;
    const int64_t zblocks = (K + rpb - 1) / rpb;
    k_hq_signs_z3<<<static_cast<unsigned>(zblocks < 4096 ? zblocks : 4096), 256, 0, st>>>(
        zbits, static_cast<int>(S), K, static_cast<int>(g.S16), static_cast<int>(g.C3), Z3);
    k_hq_u<<<dim3(static_cast<unsigned>(g.ttiles), static_cast<unsigned>(g.nsplit)), HQ_THREADS, smem1, st>>>(
        tmX1, tmZ, T, g.nkb, static_cast<int>(g.nsplit), static_cast<int>(g.S16), stages, stage_bytes, tcols, Up);
    const int64_t cblocks = (T + rpb - 1) / rpb;
    k_hq_combine<<<static_cast<unsigned>(cblocks < 8192 ? cblocks : 8192), 256, 0, st>>>(
        Up, T, static_cast<int>(S), static_cast<int>(g.S16), static_cast<int>(g.nsplit), static_cast<int>(g.C3),
        U3);
    const int64_t units = g.ktiles * g.ttiles;
    const int64_t grid3 = units < hq_sm_count() ? units : hq_sm_count();
    k_hq_p<<<static_cast<unsigned>(grid3), HQ_THREADS, HQ2_SMEM_BYTES, st>>>(
        tmZ3, tmU3, tmX3, K, g.ktiles, g.ttiles, static_cast<int>(g.C3 / 64), Dp);
    if (cudaGetLastError() != cudaSuccess) return NM_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((K + 63) / 64), 1, 1);
    cfg.blockDim = dim3(64, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_hq_finish, static_cast<const double *>(Dp), g.ttiles, K,
                           1.0 / (static_cast<double>(S) * static_cast<double>(T)), D) != cudaSuccess)
        return NM_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}
