// nm_f8.cu -- the FP8 (E4M3) form of the sparse layer.
//
// SlideSparse (arXiv 2603.05232) sec. 2B: the activation lift is only an index
// remap, so it is fused into the per-token INT8/FP8/FP4 quantisation kernel;
// sec. 2C: online, one fused quantise-and-lift kernel, then the sparse GEMM.
//
//   k_quant_lift_f8  one block per token: the row into shared memory with
//                    16-byte loads while taking its amax (warp and block max),
//                    scale = amax / 448 (1 when amax is 0), then the lifted row
//                    (natural window order, zero past the lifted width) read
//                    back from shared memory as E4M3 codes of fp32(x * inv),
//                    inv = fp32(1 / scale), round to nearest even, saturating;
//                    16 codes per 16-byte store.  Rows above 48 K columns skip
//                    the staging and gather from global memory instead.
//   k_prepare_f8     one block per weight row: the same per-row scale over the
//                    kept values, their codes (of fp32(w * inv)) in the packed
//                    order (the kept order is the window order), the metadata
//                    rearranged into the kind::f8f6f4 layout: per 128-row tile
//                    and 256-column K' block two 2 KB atoms of [128 rows x 16
//                    bytes], row-major, a nibble idx0 | idx1 << 2 per window.
//   k_gemm_f8        tcgen05.mma.sp kind::f8f6f4, one CTA per 128 weight rows
//                    x 128 tokens: per 256-column K' block A = codes [128 x
//                    128 bytes], B = lifted codes [128 x 256 bytes] (two TMA
//                    boxes, 128-byte swizzle), the metadata copied into tensor
//                    memory (each MMA, K = 64, reads two columns), four MMAs;
//                    the epilogue scales by ws[row] * xs[token] and stores bf16.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nm_common.cuh"
#include "nm_host.cuh"

namespace nm {

constexpr int F8_BM = 128, F8_BN = 128, F8_THREADS = 256, F8_STAGES = 4;
constexpr int F8_KB = 256;                                  // lifted columns per stage
constexpr int F8_A_BYTES = F8_BM * 128;                     // 16 KB
constexpr int F8_B_BYTES = F8_BN * 256;                     // 32 KB
constexpr int F8_E_BYTES = 4096;                            // two 2 KB atoms
constexpr int F8_STAGE_BYTES = F8_A_BYTES + F8_B_BYTES + F8_E_BYTES;
constexpr int F8_SMEM_BYTES = F8_STAGES * F8_STAGE_BYTES + 1024 + 256;
constexpr int F8_TMEM_COLS = 512;                           // two accumulators of 128 + metadata 8
constexpr int F8_TMEM_E = 2 * F8_BN;                        // metadata columns
static_assert(F8_STAGE_BYTES % 1024 == 0, "stage alignment");

// two fp32 values -> two E4M3 codes (round to nearest even, saturating); the
// first argument lands in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float f8_scale(float amax) { return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f; }

constexpr int64_t F8_STAGE_ROW_MAX = 48 * 1024;  // columns of a row staged in shared memory

__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    __syncthreads();  // red is reused by the next call
    return r;
}

constexpr int F8Q_THREADS = 128;  // per token; 12 tokens in flight per SM

__global__ void __launch_bounds__(F8Q_THREADS, 12) k_quant_lift_f8(const uint16_t *__restrict__ X, int64_t T, int64_t K,
                                                       int64_t ldx, int m, int64_t KL, uint8_t *__restrict__ Q,
                                                       int64_t ldq, float *__restrict__ scale, int staged) {
    __shared__ float red[F8Q_THREADS / 32];
    extern __shared__ __align__(16) uint16_t xrow[];  // the row, when staged
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const uint16_t *row = X + t * ldx;
        float amax = 0.0f;
        const int64_t K8 = K / 8;
        for (int64_t i = threadIdx.x; i < K8; i += blockDim.x) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(row) + i);
            if (staged) reinterpret_cast<uint4 *>(xrow)[i] = v;
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)),
                                         fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
        }
        for (int64_t k = K8 * 8 + threadIdx.x; k < K; k += blockDim.x) {
            const uint16_t b = row[k];
            if (staged) xrow[k] = b;
            amax = fmaxf(amax, fabsf(__uint_as_float(static_cast<uint32_t>(b) << 16)));
        }
        amax = block_max(amax, red);  // also orders the staging stores before the reads below
        const float s = f8_scale(amax), inv = __frcp_rn(s);
        if (threadIdx.x == 0) scale[t] = s;
        const uint16_t *src_row = staged ? xrow : row;
        uint8_t *qrow = Q + t * ldq;
        if (staged && m != 4) {
            // (2N-2):2N from the staged row, a group per thread: window w of a
            // group is its inputs 2w .. 2w + 3, so with the codes of input
            // pairs c16[i] = e4m3x2(x[2i], x[2i + 1]) window w is the word
            // c16[w] | c16[w + 1] << 16 -- every input converted once
            const int G = static_cast<int>((K + m - 1) / m), nwin = m / 2 - 1;
            const uint32_t *xw = reinterpret_cast<const uint32_t *>(xrow);
            uint32_t *qw = reinterpret_cast<uint32_t *>(qrow);
            for (int g = threadIdx.x; g < G; g += blockDim.x) {
                uint32_t c16[5];
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    if (i >= m / 2) break;
                    const int64_t col = static_cast<int64_t>(g) * m + 2 * i;  // even: a word of the row
                    uint32_t w2 = 0u;
                    if (col < K) {
                        w2 = xw[col / 2];
                        if (col + 1 >= K) w2 &= 0xFFFFu;  // the last input is the row's last
                    }
                    c16[i] = e4m3x2(__fmul_rn(__uint_as_float(w2 << 16), inv),
                                    __fmul_rn(__uint_as_float(w2 & 0xFFFF0000u), inv));
                }
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (w >= nwin) break;
                    qw[static_cast<int64_t>(g) * nwin + w] = c16[w] | (c16[w + 1] << 16);
                }
            }
            // lifted columns past the real ones (the row pitch's padding): zero
            for (int64_t c = KL + 4 * static_cast<int64_t>(threadIdx.x); c < ldq; c += 4 * blockDim.x)
                *reinterpret_cast<uint32_t *>(qrow + c) = 0u;
            __syncthreads();  // the staged row is read before the next token overwrites it
            continue;
        }
        const int per = 2 * m - 4;  // lifted columns per group
        for (int64_t c0 = 8 * static_cast<int64_t>(threadIdx.x); c0 < ldq; c0 += 8 * blockDim.x) {
            if (m == 4 && c0 + 8 <= K) {
                // 2:4: the lift is the identity; the chunk's 8 columns in one
                // 16-byte load (rows and chunks start on 16 bytes)
                const uint4 u = *reinterpret_cast<const uint4 *>(src_row + c0);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                float v[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[2 * j] = __fmul_rn(__uint_as_float(w[j] << 16), inv);
                    v[2 * j + 1] = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), inv);
                }
                *reinterpret_cast<uint2 *>(qrow + c0) =
                    make_uint2(e4m3x2(v[0], v[1]) | (e4m3x2(v[2], v[3]) << 16),
                               e4m3x2(v[4], v[5]) | (e4m3x2(v[6], v[7]) << 16));
                continue;
            }
            // group and offset of the chunk's first column once, then stepped
            int g = static_cast<int>(c0) / per, rem = static_cast<int>(c0) - g * per;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = static_cast<int>(c0) + j;
                float x = 0.0f;
                if (c < KL) {
                    const int src = g * m + 2 * (rem >> 2) + (rem & 3);
                    if (src < K) x = __uint_as_float(static_cast<uint32_t>(src_row[src]) << 16);
                }
                v[j] = __fmul_rn(x, inv);
                if (++rem == per) { rem = 0; ++g; }
            }
            *reinterpret_cast<uint2 *>(qrow + c0) =
                make_uint2(e4m3x2(v[0], v[1]) | (e4m3x2(v[2], v[3]) << 16),
                           e4m3x2(v[4], v[5]) | (e4m3x2(v[6], v[7]) << 16));
        }
        __syncthreads();  // the staged row is read before the next token overwrites it
    }
}

// one block per padded weight row: codes [Rpad x KLf / 2], metadata blocks,
// scales [Rpad]; rows past R get zero codes, 0x44 metadata and scale 1
__global__ void __launch_bounds__(256) k_prepare_f8(const uint16_t *__restrict__ vals, const uint8_t *__restrict__ wmeta,
                                                    int64_t R, int64_t L, int64_t nwin, int64_t wbytes,
                                                    int64_t Rpad, int64_t KLf, uint8_t *__restrict__ qv,
                                                    uint8_t *__restrict__ qmeta, float *__restrict__ qscale) {
    __shared__ float red[8];
    const int64_t nkb = KLf / F8_KB, half = KLf / 2;
    for (int64_t r = blockIdx.x; r < Rpad; r += gridDim.x) {
        const bool real = r < R;
        const uint16_t *vrow = vals + r * L;
        float amax = 0.0f;
        if (real)
            for (int64_t j = threadIdx.x; j < L; j += blockDim.x)
                amax = fmaxf(amax, fabsf(__uint_as_float(static_cast<uint32_t>(vrow[j]) << 16)));
        amax = block_max(amax, red);
        const float s = f8_scale(amax), inv = __frcp_rn(s);
        if (threadIdx.x == 0) qscale[r] = s;
        uint8_t *out = qv + r * half;
        for (int64_t j0 = 4 * static_cast<int64_t>(threadIdx.x); j0 < half; j0 += 4 * blockDim.x) {
            float v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t j = j0 + q;
                const float x = (real && j < L) ? __uint_as_float(static_cast<uint32_t>(vrow[j]) << 16) : 0.0f;
                v[q] = __fmul_rn(x, inv);
            }
            *reinterpret_cast<uint32_t *>(out + j0) = e4m3x2(v[0], v[1]) | (e4m3x2(v[2], v[3]) << 16);
        }
        // metadata: byte i of atom a of K' block kb = windows 64kb + 32a + 2i, +1
        const int64_t mt = r / F8_BM, lane = r - mt * F8_BM;
        for (int64_t b = threadIdx.x; b < nkb * 32; b += blockDim.x) {
            const int64_t kb = b >> 5, a = (b >> 4) & 1, i = b & 15;
            const int64_t w0 = 64 * kb + 32 * a + 2 * i;
            uint32_t lo = 0x4u, hi = 0x4u;  // padding window: indices 0 and 1 over zero values
            if (real) {
                const uint32_t byte = (w0 / 2 < wbytes) ? wmeta[r * wbytes + w0 / 2] : 0x44u;
                if (w0 < nwin) lo = byte & 0xFu;
                if (w0 + 1 < nwin) hi = byte >> 4;
            }
            qmeta[((mt * nkb + kb) * 2 + a) * 2048 + lane * 16 + i] = static_cast<uint8_t>(lo | (hi << 4));
        }
    }
}

__device__ __forceinline__ void mma_sp_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t e_tmem,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::f8f6f4 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
}

// kind::f8f6f4 instruction descriptor: E4M3 A and B (format 0), fp32 D,
// both K-major, sparse
__host__ __device__ constexpr uint32_t make_idesc_f8_sp(uint32_t M, uint32_t N) {
    return (1u << 2) | (1u << 4) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Persistent: one CTA per SM walks the (128-row, 128-token) tiles, weight-row
// tiles fastest (consecutive CTAs share a token tile in L2).  Warp roles: 0 =
// TMA producer (its stage ring runs on across tiles), 1 = MMA issuer +
// tensor-memory owner, 4..7 = epilogue.  Two accumulators of 128 columns
// alternate between tiles, so the epilogue of one tile (tensor memory ->
// scaled bf16, stored from registers: 32 consecutive weight rows of one token
// per warp instruction) overlaps the next tile's main loop.
__global__ void __launch_bounds__(F8_THREADS, 1)
    k_gemm_f8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const uint8_t *__restrict__ meta, int64_t nkb, const float *__restrict__ xs,
              const float *__restrict__ ws, int64_t T, int64_t R, int64_t n_m, int64_t ntiles,
              uint16_t *__restrict__ Y, int64_t ldy) {
    constexpr int S = F8_STAGES;
    extern __shared__ __align__(1024) uint8_t f8_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(f8_smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * F8_STAGE_BYTES);
    uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S, *acc_empty = bars + 2 * S + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 4);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto stA = [&](int s) { return smem + s * F8_STAGE_BYTES; };
    auto stB = [&](int s) { return smem + s * F8_STAGE_BYTES + F8_A_BYTES; };
    auto stE = [&](int s) { return smem + s * F8_STAGE_BYTES + F8_A_BYTES + F8_B_BYTES; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);  // the four epilogue warps
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, F8_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_e = tmem_base + F8_TMEM_E;

    if (warp == 0) {
        if (lane == 0) {
            int64_t it = 0;
            for (int64_t tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                const int64_t mt = tile % n_m, nt = tile / n_m;
                for (int64_t kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                    if (it >= S && !mbar_wait(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
                    mbar_arrive_expect_tx(&full[s], F8_STAGE_BYTES);
                    tma_load_2d(stA(s), &tmA, &full[s], static_cast<int32_t>(kb * 128), static_cast<int32_t>(mt * F8_BM));
                    tma_load_2d(stB(s), &tmB, &full[s], static_cast<int32_t>(kb * F8_KB), static_cast<int32_t>(nt * F8_BN));
                    tma_load_2d(stB(s) + F8_BN * 128, &tmB, &full[s], static_cast<int32_t>(kb * F8_KB + 128),
                                static_cast<int32_t>(nt * F8_BN));
                    bulk_load(stE(s), meta + (mt * nkb + kb) * F8_E_BYTES, F8_E_BYTES, &full[s]);
                }
            }
            if (*abort_flag)  // let the copies already issued land
                for (int64_t j = (it > S ? it - S : 0); j < it; ++j)
                    mbar_wait(&full[j % S], static_cast<uint32_t>((j / S) & 1));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_f8_sp(F8_BM, F8_BN);
            bool ok = true;
            int64_t it = 0, ti = 0;
            for (int64_t tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++ti) {
                const int buf = static_cast<int>(ti & 1);
                if (ti >= 2 && !mbar_wait(&acc_empty[buf], static_cast<uint32_t>(((ti >> 1) - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * F8_BN);
                for (int64_t kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    if (!mbar_wait(&full[s], static_cast<uint32_t>((it / S) & 1))) { ok = false; break; }
                    tc_fence_after();
                    tmem_cp_128x128b(tmem_e, make_sdesc(smem_u32(stE(s)), 2048, 128, 0));
                    tmem_cp_128x128b(tmem_e + 4, make_sdesc(smem_u32(stE(s) + 2048), 2048, 128, 0));
                    const uint32_t a0 = smem_u32(stA(s)), b0 = smem_u32(stB(s));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t ad = make_sdesc(a0 + j * 32, 16, 1024, 2);
                        const uint64_t bd = make_sdesc(b0 + (j >> 1) * (F8_BN * 128) + (j & 1) * 64, 16, 1024, 2);
                        mma_sp_f8(d, ad, bd, tmem_e + 2 * j, idesc, (kb > 0 || j > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[s]);
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp >= 4) {
        const int ew = warp - 4;
        int64_t ti = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++ti) {
            const int buf = static_cast<int>(ti & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], static_cast<uint32_t>((ti >> 1) & 1)))) break;
            tc_fence_after();
            const int64_t mt = tile % n_m, nt = tile / n_m;
            const int64_t r = mt * F8_BM + ew * 32 + lane;  // this lane's weight row
            const float wsr = ws[r];                          // ws holds Rpad entries
            const uint32_t src = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + static_cast<uint32_t>(buf * F8_BN);
#pragma unroll 1
            for (int cc = 0; cc < F8_BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(src + cc * 32, v);
                tmem_ld_wait();
                if (cc == F8_BN / 32 - 1) {  // the accumulator is in registers: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[buf]);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int64_t t = nt * F8_BN + cc * 32 + j;
                    if (t < T) {
                        const float y = __fmul_rn(__uint_as_float(v[j]), __fmul_rn(wsr, __ldg(xs + t)));
                        if (r < R) Y[t * ldy + r] = static_cast<uint16_t>(pack_bf16x2(y, 0.0f) & 0xFFFFu);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, F8_TMEM_COLS);
    }
}

}  // namespace nm

// ===========================================================================
// C ABI
// ===========================================================================
using namespace nm;

namespace {

struct F8Geom {
    int64_t G, nwin, KL, KLf, nkb, Rpad, wbytes;
    size_t vals_bytes, meta_bytes, total;
};

F8Geom f8_geometry(int64_t R, int64_t K, int m) {
    F8Geom g{};
    g.G = (K + m - 1) / m;
    g.nwin = g.G * (m / 2 - 1);
    g.KL = g.nwin * 4;
    g.KLf = (g.KL + F8_KB - 1) / F8_KB * F8_KB;
    g.nkb = g.KLf / F8_KB;
    g.Rpad = (R + F8_BM - 1) / F8_BM * F8_BM;
    g.wbytes = (g.nwin + 1) / 2;
    g.vals_bytes = static_cast<size_t>(g.Rpad) * static_cast<size_t>(g.KLf / 2);
    g.meta_bytes = static_cast<size_t>(g.Rpad / F8_BM) * static_cast<size_t>(g.nkb) * F8_E_BYTES;
    g.total = g.vals_bytes + g.meta_bytes + static_cast<size_t>(g.Rpad) * 4;
    return g;
}

bool f8_pattern_ok(int m) { return m >= 4 && m <= 10 && (m % 2) == 0; }

}  // namespace

extern "C" int64_t nm_lifted_cols_f8(int64_t K, int m) {
    if (K < 1 || !f8_pattern_ok(m)) return 0;
    return f8_geometry(1, K, m).KLf;
}

extern "C" size_t nm_sparse_prepare_f8_bytes(int64_t R, int64_t K, int m) {
    if (R < 1 || K < 1 || !f8_pattern_ok(m)) return 0;
    return f8_geometry(R, K, m).total;
}

extern "C" nm_status nm_quant_lift_f8(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, int m, uint8_t *Xq,
                                      int64_t ldq, float *xscale, void *stream) {
    if (!X || !Xq || !xscale) return NM_ERR_NULL;
    if (!f8_pattern_ok(m)) return NM_ERR_UNSUPPORTED;
    if (T < 1 || K < 1 || ldx < K) return NM_ERR_SHAPE;
    const F8Geom g = f8_geometry(1, K, m);
    if (ldq < g.KLf || ldq > (int64_t(1) << 31) - 8) return NM_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(X) & 15u) || (reinterpret_cast<uintptr_t>(Xq) & 15u) || (ldx % 8) != 0 ||
        (ldq % 16) != 0 || (reinterpret_cast<uintptr_t>(xscale) & 3u))
        return NM_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int staged = K <= F8_STAGE_ROW_MAX ? 1 : 0;
    const int smem = staged ? static_cast<int>((K + 7) / 8 * 16) : 0;
    if (staged && !set_smem_attr<k_quant_lift_f8>(static_cast<int>(F8_STAGE_ROW_MAX * 2))) return NM_ERR_CUDA;
    k_quant_lift_f8<<<static_cast<unsigned>(T < 65535 * 4 ? T : 65535 * 4), F8Q_THREADS, smem, st>>>(
        X, T, K, ldx, m, g.KL, Xq, ldq, xscale, staged);
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

extern "C" nm_status nm_sparse_prepare_f8(const uint16_t *vals, const uint8_t *wmeta, int64_t R, int64_t K, int m,
                                          void *packed, size_t packed_bytes, void *stream) {
    if (!vals || !wmeta || !packed) return NM_ERR_NULL;
    if (!f8_pattern_ok(m)) return NM_ERR_UNSUPPORTED;
    if (R < 1 || K < 1) return NM_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(packed) & 15u) return NM_ERR_ALIGN;
    const F8Geom g = f8_geometry(R, K, m);
    if (packed_bytes < g.total) return NM_ERR_WORKSPACE;
    uint8_t *p = static_cast<uint8_t *>(packed);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    k_prepare_f8<<<static_cast<unsigned>(g.Rpad < 65535 * 4 ? g.Rpad : 65535 * 4), 256, 0, st>>>(
        vals, wmeta, R, g.G * (m - 2), g.nwin, g.wbytes, g.Rpad, g.KLf, p, p + g.vals_bytes,
        reinterpret_cast<float *>(p + g.vals_bytes + g.meta_bytes));
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

// SMs of the current device (148 if the query fails)
static int f8_sm_count() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        return 148;
    return v;
}

extern "C" nm_status nm_sparse_gemm_f8(const uint8_t *Xq, int64_t T, int64_t K, int64_t ldq, const float *xscale,
                                       const void *packed, int64_t R, int m, uint16_t *Y, int64_t ldy,
                                       void *stream) {
    if (!Xq || !xscale || !packed || !Y) return NM_ERR_NULL;
    if (!f8_pattern_ok(m)) return NM_ERR_UNSUPPORTED;
    if (T < 1 || K < 1 || R < 1 || ldy < R) return NM_ERR_SHAPE;
    const F8Geom g = f8_geometry(R, K, m);
    if (ldq < g.KLf || (T + F8_BN - 1) / F8_BN > 65535) return NM_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(Xq) & 15u) || (reinterpret_cast<uintptr_t>(packed) & 15u) ||
        (reinterpret_cast<uintptr_t>(Y) & 15u) || (ldq % 16) != 0 || (ldy % 8) != 0 ||
        (reinterpret_cast<uintptr_t>(xscale) & 3u))
        return NM_ERR_ALIGN;
    const uint8_t *p = static_cast<const uint8_t *>(packed);
    CUtensorMap ta, tb;
    if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p, g.Rpad, g.KLf / 2, g.KLf / 2, 128, F8_BM, true) ||
        !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Xq, T, g.KLf, ldq, 128, F8_BN, true))
        return NM_ERR_CUDA;
    if (!set_smem_attr<k_gemm_f8>(F8_SMEM_BYTES)) return NM_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t n_m = g.Rpad / F8_BM, ntiles = n_m * ((T + F8_BN - 1) / F8_BN);
    const int64_t nsm = f8_sm_count();
    const unsigned grid = static_cast<unsigned>(ntiles < nsm ? ntiles : nsm);
    k_gemm_f8<<<grid, F8_THREADS, F8_SMEM_BYTES, st>>>(
        ta, tb, p + g.vals_bytes, g.nkb, xscale, reinterpret_cast<const float *>(p + g.vals_bytes + g.meta_bytes),
        T, R, n_m, ntiles, Y, ldy);
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}
