// nm_prune.cu -- score, prune/compress, slide pack, lift and ternary kernels.
//
// All of these are HBM-streaming kernels: each reads its operand once with
// coalesced vector loads and writes its outputs once.  Bit-exact by
// construction with any implementation of the same definitions:
//   * H (and the ternary gamma) is the exact sum rounded once, then divided
//     once, so no summation order enters it (see "Exact sums" below);
//   * S uses fp64 add/multiply with explicit round-to-nearest intrinsics (no
//     FMA contraction) and one fp64 -> fp32 rounding;
//   * selection is integer logic on fp32 comparisons.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "nm_common.cuh"
#include "nm_host.cuh"

namespace nm {

__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
    return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------------------
// Exact sums (H and the ternary gamma).  Both are means of terms that are
// integer multiples of a power of two: a bf16 value with exponent field e and
// significand m (m = 128 + fraction for e >= 1, the fraction for e = 0) is
// m 2^(max(e,1) - 134), its square m^2 2^(2 max(e,1) - 268).  The library
// returns the exact sum rounded once to fp64 (nearest, ties to even), divided
// once by the count, so that no summation order enters the result.  Three
// facts let the kernels sum in any order and still be exact:
//  (1) fp64 additions of non-negative terms, all integer multiples of a unit
//      u, are exact while the sum stays below 2^53 u: every partial sum is
//      then a multiple of u below 2^53 u, hence representable, and once an
//      addition rounds the running sum is >= 2^53 u for good.  A run whose
//      result is below that bound was therefore summed exactly; u is the
//      unit of the run's smallest nonzero term.
//  (1') The same chain done twice, rounding every step up and then down,
//      brackets the exact sum (up >= exact >= down, whatever the signs);
//      equal results are the exact sum.
//  (2) Knuth's TwoSum splits a + b into s + e exactly (round to nearest), so a
//      chain of exact partial sums carried as a pair (s, c), the e's summed
//      into c up and down as in (1'), is the exact total when c's two results
//      agree; fl(s + c) is then its correct rounding.
//  (3) Anything that fails a check (a subnormal, an infinity, a NaN, or a
//      range of magnitudes wider than the checks allow) is summed again in
//      parts or with integer arithmetic (BigAcc).
// ---------------------------------------------------------------------------

// fp64 whose high word is hw and low word zero
__device__ __forceinline__ double hw_double(uint32_t hw) {
    return __hiloint2double(static_cast<int>(hw), 0);
}
__device__ __forceinline__ uint32_t vmin_s16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// TwoSum into (s, c) with c carried both up and down (fact 2)
__device__ __forceinline__ void two_sum_acc2(double &s, double &cu, double &cd, double a) {
    const double t = __dadd_rn(s, a);
    const double bb = __dsub_rn(t, s);
    const double err = __dadd_rn(__dsub_rn(s, __dsub_rn(t, bb)), __dsub_rn(a, bb));
    s = t;
    cu = __dadd_ru(cu, err);
    cd = __dadd_rd(cd, err);
}

// Integer accumulator: sum of d[i] 2^(32 i - BIAS), 32-bit digits carried in
// signed 64-bit limbs (carries resolved once, in round_rn), so up to 2^31 adds.
template <int NDIG, int BIAS>
struct BigAcc {
    long long d[NDIG];
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int i = 0; i < NDIG; ++i) d[i] = 0;
    }
    // += v * 2^(pos - BIAS) (v < 2^53, 0 <= pos), negative when neg
    __device__ void add_bits(unsigned long long v, int pos, bool neg) {
        const int q = pos >> 5, b = pos & 31;
        const unsigned long long lo = (v << b) & 0xFFFFFFFFull;
        const unsigned long long mid = b ? ((v >> (32 - b)) & 0xFFFFFFFFull) : ((v >> 32) & 0xFFFFFFFFull);
        const unsigned long long hi = b ? (v >> (64 - b)) : 0ull;
        const long long sg = neg ? -1 : 1;
        d[q] += sg * static_cast<long long>(lo);
        if (q + 1 < NDIG) d[q + 1] += sg * static_cast<long long>(mid);
        if (q + 2 < NDIG) d[q + 2] += sg * static_cast<long long>(hi);
    }
    // += v, v finite and an integer multiple of 2^-BIAS
    __device__ void add_double(double v) {
        const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(v));
        const int ef = static_cast<int>((u >> 52) & 0x7FF);
        unsigned long long mant = u & 0xFFFFFFFFFFFFFull;
        if (ef == 0 && mant == 0) return;
        if (ef) mant |= 1ull << 52;
        int pos = (ef ? ef : 1) - 1075 + BIAS;  // position of mant's bit 0
        if (pos < 0) {                          // only zero bits drop here
            mant >>= -pos;
            pos = 0;
        }
        add_bits(mant, pos, (u >> 63) != 0);
    }
    // the value rounded to the nearest double (ties to even); must be >= 0
    __device__ double round_rn() const {
        long long n[NDIG];
        long long carry = 0;
#pragma unroll
        for (int i = 0; i < NDIG; ++i) {
            const long long v = d[i] + carry;
            carry = v >> 32;  // arithmetic shift: floor division
            n[i] = v & 0xFFFFFFFFll;
        }
        int top = NDIG - 1;
        while (top >= 0 && n[top] == 0) --top;
        if (top < 0) return 0.0;
        const unsigned long long d2 = static_cast<unsigned long long>(n[top]);
        const unsigned long long d1 = top >= 1 ? static_cast<unsigned long long>(n[top - 1]) : 0ull;
        const unsigned long long d0 = top >= 2 ? static_cast<unsigned long long>(n[top - 2]) : 0ull;
        bool sticky_low = false;
        for (int i = 0; i < top - 2; ++i) sticky_low |= n[i] != 0;
        const unsigned __int128 w = (static_cast<unsigned __int128>(d2) << 64) |
                                    (static_cast<unsigned __int128>(d1) << 32) | d0;
        const int tb = 64 + 31 - __clz(static_cast<unsigned>(d2));  // top bit of w
        const int sh = tb - 52;                                       // >= 12
        unsigned long long sig = static_cast<unsigned long long>(w >> sh);
        const unsigned __int128 rem = w & ((static_cast<unsigned __int128>(1) << sh) - 1);
        const bool rbit = ((rem >> (sh - 1)) & 1) != 0;
        const bool sticky = (rem & ((static_cast<unsigned __int128>(1) << (sh - 1)) - 1)) != 0 || sticky_low;
        if (rbit && (sticky || (sig & 1ull))) ++sig;  // 2^53 is still exact
        return scalbn(static_cast<double>(sig), sh + 32 * (top - 2) - BIAS);
    }
};

// sums of squares: units of 2^-266 (the square of the smallest subnormal),
// room for T < 2^31 squares below 2^256
constexpr int HB_NDIG = 19;
constexpr int HB_BIAS = 266;
using SqAcc = BigAcc<HB_NDIG, HB_BIAS>;

// sum of x^2 over one column of X, exactly, rounded once; NaN if the column
// holds a NaN, else +inf if it holds an infinity.  One thread, plain loads:
// the path for columns whose fast sums failed a check.
__device__ __noinline__ double exact_sq_column(const uint16_t *__restrict__ X, int64_t ldx, int64_t T, int64_t col) {
    SqAcc a;
    a.clear();
    bool nan = false, inf = false;
    for (int64_t t = 0; t < T; ++t) {
        const uint32_t b = X[t * ldx + col] & 0x7FFFu;
        const int e = static_cast<int>(b >> 7);
        const uint32_t f = b & 0x7Fu;
        if (e == 255) {
            nan |= f != 0;
            inf |= f == 0;
            continue;
        }
        if (b == 0) continue;
        const unsigned long long m = e ? 128u + f : f;
        a.add_bits(m * m, 2 * (e ? e : 1) - 268 + HB_BIAS, false);
    }
    if (nan) return __longlong_as_double(0x7FF8000000000000ll);
    if (inf) return __longlong_as_double(0x7FF0000000000000ll);
    return a.round_rn();
}

// ---------------------------------------------------------------------------
// a1: H_j = fl(fl(sum_t x_{t,j}^2) / T).
//
// Block: 256 threads = 8 warps over one 128-column strip of X and a range of
// 128-token chunks (blockIdx.y).  Each chunk tile [128 tokens x 128 columns]
// bf16 (32 KB) comes into shared memory by TMA, three in flight (two blocks
// per SM); rows past T and columns past K arrive as zeros.  In a tile, warp w
// owns tokens 16w .. 16w+15 (a run) and lane l columns 4l .. 4l+3 (one 8-byte
// shared-memory load per token, a warp reads one 256-byte row).  Per run a
// thread sums x^2 per column twice, rounding up and rounding down (fact 1);
// equal results are the exact run sum, which goes into the column's TwoSum
// pair (fact 2).  A run whose two sums differ is summed again from the tile,
// split into the values within 12 binades of the run's largest and the rest,
// each part checked the same way; what still fails (an infinity, a NaN, a
// range wider than that) marks the column for the integer path.  The eight
// warps' pairs are added in shared memory, again checking c up against down.
// A block that saw every token divides and writes H; otherwise it writes its
// exact pair (s, c) -- or NaN in s for a marked column -- and k_hsq_finish
// adds the pairs of a column.
//
// x comes from its bits without a conversion: d = x 2^-896 is the fp64 with
// high word (bits & 0x7FFF) << 13 (exact for every finite bf16, zeros and
// subnormals included), |x| = d * 2^896 exactly, and fma(x, x, acc) rounds
// like acc + x^2 (x^2 exact in fp64, below 2^256).  An infinity or a NaN reads
// as 2^128 (1 + f/128).  The check of fact (1) needs the run's smallest
// nonzero magnitude, kept two columns at a time as a signed 16-bit minimum of
// t + 0x7FFF over the magnitude bits t (0x7FFF for a zero, the largest;
// 0x8000 + t - 1, negative and increasing in t, otherwise); a run holding an
// infinity, a NaN or a subnormal (exponent field 255 or 0) fails it and is
// looked at bit by bit.
// ---------------------------------------------------------------------------
constexpr int HX_THREADS = 256;
constexpr int HX_WARPS = HX_THREADS / 32;
constexpr int HX_VEC = 4;                 // columns per thread
constexpr int HX_COLS = 32 * HX_VEC;      // columns per block (one TMA box row: 256 bytes)
constexpr int HX_RUN = 16;                // tokens per checked run (one warp per run)
constexpr int HX_CHUNK = HX_RUN * HX_WARPS;   // tokens per tile: 128
constexpr int HX_STAGES = 3;
constexpr int HX_TILE_BYTES = HX_CHUNK * HX_COLS * 2;                   // 32 KB
constexpr int HX_SMEM_BYTES = HX_STAGES * HX_TILE_BYTES + 64 + 1024;    // + barriers, alignment
constexpr int64_t HX_SLOTS = 2 * 148;     // resident blocks at 2 per SM on 148 SMs: the grid's target

struct HPair {
    double s, c;
};

// x^2 of the two bf16 halves of a word (low half: w << 13; high half: w >> 3)
// into the sums of columns k, k + 1, and their smallest magnitudes into key
__device__ __forceinline__ void sq_word(uint32_t w, double (&a)[HX_VEC], uint32_t &key, int k) {
    const double x0 = __dmul_rn(hw_double((w << 13) & 0x0FFFE000u), 0x1p896);
    const double x1 = __dmul_rn(hw_double((w >> 3) & 0x0FFFE000u), 0x1p896);
    a[k] = __fma_rn(x0, x0, a[k]);
    a[k + 1] = __fma_rn(x1, x1, a[k + 1]);
    key = vmin_s16x2(key, (w & 0x7FFF7FFFu) + 0x7FFF7FFFu);
}

// fact (1) for a run: no nonzero value (key 0x7FFF), or a normal smallest
// value (exponent field e >= 1) and a sum below 2^53 units of its square,
// 2^(2e - 268 + 53), whose fp64 exponent field is 2e + 808, and below 2^256
// (an infinity or a NaN, read as 2^128 (1 + f/128), squares to at least that;
// finite squares are smaller)
__device__ __forceinline__ bool sq_run_exact(double a, uint32_t key16) {
    if (key16 == 0x7FFFu) return true;
    const int e = static_cast<int>((key16 - 0x7FFFu) >> 7);
    return e >= 1 && a < hw_double(static_cast<uint32_t>(2 * e + 808) << 20) && a < 0x1p256;
}

// A run that failed its check, summed again from the tile in two parts: the
// values within 12 binades of the run's largest (16 squares below
// 2^(2 emax - 252) on a grid of 2^(2 emax - 292): exact) and the smaller ones,
// each summed up and down (fact 1').  x = d * 2^896 is exact for subnormals
// too.  ok = false for an infinity, a NaN, or a run too wide for that split.
// `col` points at the column's first element of the run in the tile (row
// pitch HX_COLS elements).
struct RunSplit {
    double big, small;
    bool ok;
};
__device__ __noinline__ RunSplit sq_run_split(const uint16_t *col) {
    RunSplit r{0.0, 0.0, false};
    uint32_t b[HX_RUN];
    int emax = 0;
#pragma unroll
    for (int u = 0; u < HX_RUN; ++u) {
        b[u] = col[u * HX_COLS] & 0x7FFFu;
        if (b[u] >= 0x7F80u) return r;
        emax = max(emax, static_cast<int>(b[u] >> 7));
    }
    const int thr = emax - 12;
    double bu = 0.0, bd = 0.0, su = 0.0, sd = 0.0;
#pragma unroll
    for (int u = 0; u < HX_RUN; ++u) {
        const double x = __dmul_rn(hw_double(b[u] << 13), 0x1p896);
        if (static_cast<int>(b[u] >> 7) >= thr) {
            bu = __fma_ru(x, x, bu);
            bd = __fma_rd(x, x, bd);
        } else {
            su = __fma_ru(x, x, su);
            sd = __fma_rd(x, x, sd);
        }
    }
    r.big = bu;
    r.small = su;
    r.ok = bu == bd && su == sd;
    return r;
}

__global__ void __launch_bounds__(HX_THREADS, 2)
    k_hsq(const __grid_constant__ CUtensorMap tmX, const uint16_t *__restrict__ X, int64_t T, int64_t K,
          int64_t ldx, HPair *__restrict__ part, double *__restrict__ H, int ccomb) {
    extern __shared__ uint8_t hx_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(hx_smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + HX_STAGES * HX_TILE_BYTES);
    grid_dep_launch();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int32_t xcol = static_cast<int32_t>(blockIdx.x) * HX_COLS;
    // token range blockIdx.y of gridDim.y: chunks [y n / split, (y + 1) n / split)
    const int64_t nchunks = (T + HX_CHUNK - 1) / HX_CHUNK;
    const int64_t cbeg = static_cast<int64_t>(blockIdx.y) * nchunks / gridDim.y;
    const int64_t mine = (static_cast<int64_t>(blockIdx.y) + 1) * nchunks / gridDim.y - cbeg;
    if (threadIdx.x == 0) {
        for (int st = 0; st < HX_STAGES; ++st) mbar_init(&full[st], 1);
        fence_barrier_init();
        prefetch_tmap(&tmX);
        for (int64_t i = 0; i < mine && i < HX_STAGES; ++i) {
            mbar_arrive_expect_tx(&full[i], HX_TILE_BYTES);
            tma_load_2d(smem + i * HX_TILE_BYTES, &tmX, &full[i], xcol, static_cast<int32_t>((cbeg + i) * HX_CHUNK));
        }
    }
    __syncthreads();
    double s[HX_VEC], cu[HX_VEC], cd[HX_VEC];
#pragma unroll
    for (int k = 0; k < HX_VEC; ++k) s[k] = cu[k] = cd[k] = 0.0;
    uint32_t bad = 0;
    int64_t issued = mine < HX_STAGES ? mine : HX_STAGES;
    bool ok = true;
    int64_t i = 0;
    for (; i < mine; ++i) {
        const int st = static_cast<int>(i % HX_STAGES);
        ok = __syncthreads_and(mbar_wait(&full[st], static_cast<uint32_t>((i / HX_STAGES) & 1)));
        if (!ok) break;  // timed out (error word set)
        const uint16_t *tile = reinterpret_cast<const uint16_t *>(smem + st * HX_TILE_BYTES) +
                               (warp * HX_RUN) * HX_COLS + HX_VEC * lane;
        double a[HX_VEC] = {0.0, 0.0, 0.0, 0.0};
        uint32_t key0 = 0x7FFF7FFFu, key1 = 0x7FFF7FFFu;
#pragma unroll
        for (int u = 0; u < HX_RUN; ++u) {
            const uint2 v = *reinterpret_cast<const uint2 *>(tile + u * HX_COLS);
            sq_word(v.x, a, key0, 0);
            sq_word(v.y, a, key1, 2);
        }
        const uint32_t keys[HX_VEC] = {key0 & 0xFFFFu, key0 >> 16, key1 & 0xFFFFu, key1 >> 16};
#pragma unroll
        for (int k = 0; k < HX_VEC; ++k) {
            if (sq_run_exact(a[k], keys[k])) {
                two_sum_acc2(s[k], cu[k], cd[k], a[k]);
            } else {
                const RunSplit r = sq_run_split(tile + k);
                if (r.ok) {
                    two_sum_acc2(s[k], cu[k], cd[k], r.big);
                    two_sum_acc2(s[k], cu[k], cd[k], r.small);
                } else {
                    bad |= 1u << k;
                }
            }
        }
        __syncthreads();  // stage st consumed by every warp
        if (threadIdx.x == 0 && issued < mine) {
            mbar_arrive_expect_tx(&full[st], HX_TILE_BYTES);
            tma_load_2d(smem + st * HX_TILE_BYTES, &tmX, &full[st], xcol,
                        static_cast<int32_t>((cbeg + issued) * HX_CHUNK));
            ++issued;
        }
    }
    if (!ok) {  // let the copies in flight (chunks i .. issued - 1) land, then leave
        if (threadIdx.x == 0)
            for (int64_t j = i; j < issued; ++j)
                mbar_wait(&full[j % HX_STAGES], static_cast<uint32_t>((j / HX_STAGES) & 1));
        if (!ccomb) return;  // a cluster member still meets its peers at the barriers
        __syncthreads();
    }
    const int j = threadIdx.x;
    const int64_t col = static_cast<int64_t>(xcol) + j;
    const bool owner = j < HX_COLS && col < K;  // thread j finishes column col
    // cluster combine: this block's exact pair per column, for rank 0 to read
    double *res_s = reinterpret_cast<double *>(smem + HX_TILE_BYTES);
    double *res_c = res_s + HX_COLS;
    if (ok) {
        // the pipeline is drained: stage memory holds the warps' pairs
        double(*sh_s)[HX_COLS] = reinterpret_cast<double(*)[HX_COLS]>(smem);
        double(*sh_cu)[HX_COLS] = reinterpret_cast<double(*)[HX_COLS]>(smem + HX_WARPS * HX_COLS * 8);
        double(*sh_cd)[HX_COLS] = reinterpret_cast<double(*)[HX_COLS]>(smem + 2 * HX_WARPS * HX_COLS * 8);
        uint8_t(*sh_bad)[HX_COLS] = reinterpret_cast<uint8_t(*)[HX_COLS]>(smem + 3 * HX_WARPS * HX_COLS * 8);
#pragma unroll
        for (int k = 0; k < HX_VEC; ++k) {
            sh_s[warp][HX_VEC * lane + k] = s[k];
            sh_cu[warp][HX_VEC * lane + k] = cu[k];
            sh_cd[warp][HX_VEC * lane + k] = cd[k];
            sh_bad[warp][HX_VEC * lane + k] = static_cast<uint8_t>((bad >> k) & 1u);
        }
        __syncthreads();
        if (owner) {
            double S = 0.0, CU = 0.0, CD = 0.0;
            bool marked = false;
#pragma unroll
            for (int w = 0; w < HX_WARPS; ++w) {
                two_sum_acc2(S, CU, CD, sh_s[w][j]);
                CU = __dadd_ru(CU, sh_cu[w][j]);
                CD = __dadd_rd(CD, sh_cd[w][j]);
                marked |= sh_bad[w][j] != 0;
            }
            marked |= CU != CD;  // c not exact: its up and down sums differ (fact 2)
            if (ccomb) {
                res_s[j] = marked ? __longlong_as_double(0x7FF8000000000000ll) : S;
                res_c[j] = marked ? 0.0 : CU;
            } else if (part == nullptr) {  // the block saw every token
                const double sum = marked ? exact_sq_column(X, ldx, T, col) : __dadd_rn(S, CU);
                H[col] = __ddiv_rn(sum, static_cast<double>(T));
            } else {
                HPair p;
                p.s = marked ? __longlong_as_double(0x7FF8000000000000ll) : S;
                p.c = marked ? 0.0 : CU;
                part[static_cast<int64_t>(blockIdx.y) * K + col] = p;
            }
        }
    }
    if (!ccomb) return;
    __syncwarp();  // the cluster barrier wants converged warps
    // the token ranges of the strip are one cluster: rank 0 adds the members'
    // pairs from their shared memory as k_hsq_finish adds them from global
    // memory; the second barrier keeps every member resident until then
    cluster_sync_all();
    if (ok && owner && cluster_ctarank() == 0) {
        const int nr = static_cast<int>(gridDim.y);
        double S = 0.0, CU = 0.0, CD = 0.0;
        bool marked = false;
        for (int r = 0; r < nr; ++r) {
            const double ps = ld_dsmem_f64(mapa_shared(res_s + j, static_cast<uint32_t>(r)));
            const double pc = ld_dsmem_f64(mapa_shared(res_c + j, static_cast<uint32_t>(r)));
            marked |= isnan(ps);
            two_sum_acc2(S, CU, CD, ps);
            CU = __dadd_ru(CU, pc);
            CD = __dadd_rd(CD, pc);
        }
        double sum;
        if (marked) {
            sum = exact_sq_column(X, ldx, T, col);
        } else if (CU == CD) {
            sum = __dadd_rn(S, CU);
        } else {
            SqAcc acc;
            acc.clear();
            for (int r = 0; r < nr; ++r) {
                acc.add_double(ld_dsmem_f64(mapa_shared(res_s + j, static_cast<uint32_t>(r))));
                acc.add_double(ld_dsmem_f64(mapa_shared(res_c + j, static_cast<uint32_t>(r))));
            }
            sum = acc.round_rn();
        }
        H[col] = __ddiv_rn(sum, static_cast<double>(T));
    }
    __syncwarp();
    cluster_sync_all();
}

// adds the blocks' exact pairs of a column -- with TwoSum, c up and down as
// in fact 2, or where those differ with integer arithmetic -- and rounds once
// (a marked pair: the column again, on the integer path); launched as a
// programmatic dependent of k_hsq
__global__ void __launch_bounds__(128) k_hsq_finish(const HPair *__restrict__ part, int64_t nparts,
                                                    const uint16_t *__restrict__ X, int64_t T, int64_t K,
                                                    int64_t ldx, double *__restrict__ H) {
    grid_dep_wait();
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= K) return;
    double S = 0.0, CU = 0.0, CD = 0.0;
    bool marked = false;
    // the pairs eight at a time: their loads go out together
    for (int64_t y0 = 0; y0 < nparts; y0 += 8) {
        HPair p[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) p[q] = y0 + q < nparts ? part[(y0 + q) * K + j] : HPair{0.0, 0.0};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            marked |= isnan(p[q].s);
            two_sum_acc2(S, CU, CD, p[q].s);
            CU = __dadd_ru(CU, p[q].c);
            CD = __dadd_rd(CD, p[q].c);
        }
    }
    double sum;
    if (marked) {
        sum = exact_sq_column(X, ldx, T, j);
    } else if (CU == CD) {
        sum = __dadd_rn(S, CU);
    } else {
        SqAcc a;
        a.clear();
        for (int64_t y = 0; y < nparts; ++y) {
            const HPair p = part[y * K + j];
            a.add_double(p.s);
            a.add_double(p.c);
        }
        sum = a.round_rn();
    }
    H[j] = __ddiv_rn(sum, static_cast<double>(T));
}

// grid of the H reduction: (column strips, token ranges); the 128-token
// chunks are spread evenly over the ranges
struct HGrid {
    int64_t cblocks, split;
};
inline HGrid h_grid(int64_t T, int64_t K, int64_t max_split) {
    HGrid g;
    g.cblocks = (K + HX_COLS - 1) / HX_COLS;
    const int64_t nchunks = (T + HX_CHUNK - 1) / HX_CHUNK;
    int64_t split = HX_SLOTS / g.cblocks;  // one wave of resident blocks, no partial second one
    split = split > nchunks ? nchunks : split;
    split = split > max_split ? max_split : split;
    g.split = split < 1 ? 1 : split;
    return g;
}

// ---------------------------------------------------------------------------
// a2: S = fp32((H + eps) * W^2) (or |W| when H == nullptr), 8 elements/thread.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float score_one(const double *__restrict__ H, double eps, int64_t j,
                                           uint16_t wb) {
    if (H == nullptr) return fabsf(bf16_to_f32(wb));
    const double w = bf16_to_f64(wb);
    const double h = __dadd_rn(__ldg(H + j), eps);
    return __double2float_rn(__dmul_rn(h, __dmul_rn(w, w)));
}

// O(d_in) refresh of H under per-channel equivalent scaling (Sparsity
// Induction sec. 2C): H'_j = H_j / (s_j * s_j), fp64 multiply then division.
__global__ void __launch_bounds__(256) k_hessian_rescale(const double *__restrict__ H,
                                                         const double *__restrict__ sc, int64_t K,
                                                         double *__restrict__ out) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j < K) out[j] = __ddiv_rn(H[j], __dmul_rn(sc[j], sc[j]));
}

// Where a3 takes its selection scores from: the stored S, or -- a2 fused into
// a3, S never written -- computed in registers from W exactly as k_score
// does: fp32((H_j + eps) * w^2) with fp64 add and multiplies, or |w| when H is
// null.
struct ScoreSrc {
    const float *S;      // stored scores (used when not fused)
    int64_t lds;
    const uint16_t *W;   // fused: the weights the scores come from
    int64_t ldw;
    const double *H;     // fused: null -> magnitude score
    double eps;
};

__device__ __forceinline__ float fused_score(const double *__restrict__ H, double eps, int64_t c,
                                             uint16_t wb) {
    if (H == nullptr) return fabsf(bf16_to_f32(wb));
    const double w = bf16_to_f64(wb);
    return __double2float_rn(__dmul_rn(__dadd_rn(__ldg(H + c), eps), __dmul_rn(w, w)));
}

// grid: x = 4096-column slice of a row (256 threads x 2 chunks x 8 elements),
// y (+65535 z) = row.  Both chunks' loads are issued before any arithmetic.
// Each block: SCORE_ROWS rows x 4096 columns; a thread owns two 8-column
// chunks of each of its rows.  All W loads of a thread are issued before any
// arithmetic (SCORE_ROWS x 2 x 16 bytes in flight), and H + eps is formed
// once per column and reused for every row.
constexpr int SCORE_ROWS = 4;

__global__ void __launch_bounds__(256, 4) k_score(const double *__restrict__ H, double eps,
                                               const uint16_t *__restrict__ W, int64_t R,
                                               int64_t K, int64_t ldw, float *__restrict__ S) {
    const int64_t i0 = (blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535) * SCORE_ROWS;
    if (i0 >= R) return;
    int64_t j0[2];
    bool full[2];
    uint4 wv[2][SCORE_ROWS];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        j0[c] = (static_cast<int64_t>(blockIdx.x) * 512 + c * 256 + threadIdx.x) * 8;
        full[c] = j0[c] + 8 <= K;
#pragma unroll
        for (int r = 0; r < SCORE_ROWS; ++r)
            if (full[c] && i0 + r < R)
                wv[c][r] = __ldg(reinterpret_cast<const uint4 *>(W + (i0 + r) * ldw + j0[c]));
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        if (j0[c] >= K) continue;
        if (!full[c]) {
            for (int r = 0; r < SCORE_ROWS && i0 + r < R; ++r)
                for (int64_t j = j0[c]; j < K; ++j)
                    S[(i0 + r) * K + j] = score_one(H, eps, j, W[(i0 + r) * ldw + j]);
            continue;
        }
        double hp[8];
        if (H != nullptr) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const double2 hv = __ldg(reinterpret_cast<const double2 *>(H + j0[c]) + u);
                hp[2 * u] = __dadd_rn(hv.x, eps);
                hp[2 * u + 1] = __dadd_rn(hv.y, eps);
            }
        }
#pragma unroll
        for (int r = 0; r < SCORE_ROWS; ++r) {
            if (i0 + r >= R) break;
            const uint32_t wr[4] = {wv[c][r].x, wv[c][r].y, wv[c][r].z, wv[c][r].w};
            float sv[8];
            if (H != nullptr) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const double w = bf16_to_f64(static_cast<uint16_t>(wr[u >> 1] >> (16 * (u & 1))));
                    sv[u] = __double2float_rn(__dmul_rn(hp[u], __dmul_rn(w, w)));
                }
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    sv[u] = fabsf(bf16_to_f32(static_cast<uint16_t>(wr[u >> 1] >> (16 * (u & 1)))));
            }
            float *srow = S + (i0 + r) * K;
            if ((K & 3) == 0) {
                float4 *d = reinterpret_cast<float4 *>(srow + j0[c]);
                d[0] = make_float4(sv[0], sv[1], sv[2], sv[3]);
                d[1] = make_float4(sv[4], sv[5], sv[6], sv[7]);
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) srow[j0[c] + u] = sv[u];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// a3: group top-n + compression + 2:4 metadata.  One thread per group, one
// block per (row, 256-group slice).  Mask words of a warp's 32 groups are
// assembled in shared memory (32*m bits = m whole words, word-aligned).
// ---------------------------------------------------------------------------
constexpr int PRUNE_THREADS = 256;

// V values of one group [c0, c0 + m), zero past K (vector loads when whole)
template <int M>
__device__ __forceinline__ void load_values(const uint16_t *__restrict__ vrow, int64_t c0, int64_t K,
                                            int m_rt, uint16_t *v) {
    constexpr int MM = M > 0 ? M : 16;
    const int m = M > 0 ? M : m_rt;
    if (M > 0 && c0 + M <= K) {
        if constexpr (M % 8 == 0) {
#pragma unroll
            for (int q = 0; q < M; q += 8) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(vrow + c0 + q));
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[q + 2 * e] = static_cast<uint16_t>(w[e] & 0xFFFFu);
                    v[q + 2 * e + 1] = static_cast<uint16_t>(w[e] >> 16);
                }
            }
        } else if constexpr (M % 4 == 0) {
#pragma unroll
            for (int q = 0; q < M; q += 4) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(vrow + c0 + q));
                v[q] = u.x & 0xFFFFu; v[q + 1] = u.x >> 16; v[q + 2] = u.y & 0xFFFFu; v[q + 3] = u.y >> 16;
            }
        } else {
#pragma unroll
            for (int q = 0; q < M; q += 2) {
                const uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(vrow + c0 + q));
                v[q] = u & 0xFFFFu; v[q + 1] = u >> 16;
            }
        }
    } else {
#pragma unroll
        for (int q = 0; q < MM; ++q) {
            const int64_t c = c0 + q;
            v[q] = (q < m && c < K) ? __ldg(vrow + c) : static_cast<uint16_t>(0);
        }
    }
}

// fused a2: the group's scores from its weights (zero past K); the values are
// the weights themselves when V is W
template <int M>
__device__ __forceinline__ void load_group_fused(const ScoreSrc &src, int64_t row,
                                                 const uint16_t *__restrict__ vrow, int64_t c0,
                                                 int64_t K, int m_rt, float *s, uint16_t *v) {
    constexpr int MM = M > 0 ? M : 16;
    const int m = M > 0 ? M : m_rt;
    const uint16_t *wrow = src.W + row * src.ldw;
    uint16_t w[MM];
    load_values<M>(wrow, c0, K, m, w);
    if (M > 0 && M % 2 == 0 && src.H != nullptr && c0 + M <= K &&
        (reinterpret_cast<uintptr_t>(src.H + c0) & 15u) == 0) {
        // whole group: H in 16-byte pairs
#pragma unroll
        for (int q = 0; q < MM; q += 2) {
            const double2 h = __ldg(reinterpret_cast<const double2 *>(src.H + c0 + q));
            const double wa = bf16_to_f64(w[q]), wb = bf16_to_f64(w[q + 1]);
            s[q] = __double2float_rn(__dmul_rn(__dadd_rn(h.x, src.eps), __dmul_rn(wa, wa)));
            s[q + 1] = __double2float_rn(__dmul_rn(__dadd_rn(h.y, src.eps), __dmul_rn(wb, wb)));
        }
    } else {
#pragma unroll
        for (int q = 0; q < MM; ++q)
            s[q] = (q < m && c0 + q < K) ? fused_score(src.H, src.eps, c0 + q, w[q]) : 0.0f;
    }
    if (vrow == wrow) {
#pragma unroll
        for (int q = 0; q < MM; ++q) v[q] = w[q];
    } else {
        load_values<M>(vrow, c0, K, m, v);
    }
}

template <int M>
__device__ __forceinline__ void load_group(const float *__restrict__ srow,
                                           const uint16_t *__restrict__ vrow, int64_t c0,
                                           int64_t K, int m_rt, float *s, uint16_t *v) {
    constexpr int MM = M > 0 ? M : 16;
    const int m = M > 0 ? M : m_rt;
    if (M > 0 && c0 + M <= K) {
        if constexpr (M % 4 == 0) {
#pragma unroll
            for (int q = 0; q < M; q += 4) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(srow + c0 + q));
                s[q] = f.x; s[q + 1] = f.y; s[q + 2] = f.z; s[q + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < M; q += 2) {
                const float2 f = __ldg(reinterpret_cast<const float2 *>(srow + c0 + q));
                s[q] = f.x; s[q + 1] = f.y;
            }
        }
        if constexpr (M % 8 == 0) {
#pragma unroll
            for (int q = 0; q < M; q += 8) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(vrow + c0 + q));
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[q + 2 * e] = static_cast<uint16_t>(w[e] & 0xFFFFu);
                    v[q + 2 * e + 1] = static_cast<uint16_t>(w[e] >> 16);
                }
            }
        } else if constexpr (M % 4 == 0) {
#pragma unroll
            for (int q = 0; q < M; q += 4) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(vrow + c0 + q));
                v[q] = u.x & 0xFFFFu; v[q + 1] = u.x >> 16; v[q + 2] = u.y & 0xFFFFu; v[q + 3] = u.y >> 16;
            }
        } else {
#pragma unroll
            for (int q = 0; q < M; q += 2) {
                const uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(vrow + c0 + q));
                v[q] = u & 0xFFFFu; v[q + 1] = u >> 16;
            }
        }
    } else {
#pragma unroll
        for (int q = 0; q < MM; ++q) {
            const int64_t c = c0 + q;
            if (q < m && c < K) { s[q] = __ldg(srow + c); v[q] = __ldg(vrow + c); }
            else { s[q] = 0.0f; v[q] = 0; }
        }
    }
}

// one group: keep bits, the 2:4 index pair (i0 | i1 << 2; m == 4), and the
// compressed values written to dst
template <int M>
__device__ __forceinline__ void select_group(const float (&s)[M > 0 ? M : 16],
                                             const uint16_t (&v)[M > 0 ? M : 16], int n, int m,
                                             uint16_t *__restrict__ dst, uint32_t &keepbits,
                                             uint32_t &nib) {
    constexpr int MM = M > 0 ? M : 16;  // static trip count (runtime m <= MM)
    int i0 = 0, i1 = 0;
    if (M > 0 && n == m - 2) {
        // (m-2):m keeps all but the two lowest positions of the order (score
        // descending, index ascending): find them with two linear scans.  A
        // later position with an equal score ranks below an earlier one, so
        // "<=" picks the highest index among equal minima.
        int d0 = 0;
        float s0 = s[0];
#pragma unroll
        for (int q = 1; q < MM; ++q)
            if (s[q] <= s0) { s0 = s[q]; d0 = q; }
        int d1 = -1;
        float s1 = 0.0f;
#pragma unroll
        for (int q = 0; q < MM; ++q)
            if (q != d0 && (d1 < 0 || s[q] <= s1)) { s1 = s[q]; d1 = q; }
        const int dlo = d0 < d1 ? d0 : d1, dhi = d0 < d1 ? d1 : d0;
        keepbits = ((1u << MM) - 1u) & ~(1u << d0) & ~(1u << d1);
        // output k = v[k], v[k+1] or v[k+2] depending on the dropped positions;
        // pairs of outputs are packed and stored right here (n = MM - 2 is even)
#pragma unroll
        for (int k2 = 0; k2 < (MM - 2) / 2; ++k2) {
            uint32_t word = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int k = 2 * k2 + h;
                const int q = k + (k >= dlo ? 1 : 0) + (k + 1 >= dhi ? 1 : 0);
                const uint32_t val =
                    q == k ? v[k] : (q == k + 1 ? v[k + 1] : v[(k + 2 < MM) ? k + 2 : k]);
                word |= val << (16 * h);
            }
            reinterpret_cast<uint32_t *>(dst)[k2] = word;
        }
        i0 = (dlo == 0) ? (dhi == 1 ? 2 : 1) : 0;  // first kept position (m == 4 metadata)
        i1 = 0;
#pragma unroll
        for (int q = MM - 1; q >= 0; --q)
            if (q != dlo && q != dhi && q != i0) i1 = (i1 == 0 || q < i1) ? q : i1;
    } else {
        // general n:m: keep position q iff fewer than n positions beat it
        uint32_t outw[(MM + 1) / 2];
#pragma unroll
        for (int k = 0; k < (MM + 1) / 2; ++k) outw[k] = 0u;
#pragma unroll
        for (int q = 0; q < MM; ++q) {
            int rank = 0;
#pragma unroll
            for (int p = 0; p < MM; ++p)
                rank += (p < m && (s[p] > s[q] || (s[p] == s[q] && p < q))) ? 1 : 0;
            if (q < m && rank < n) keepbits |= 1u << q;
        }
        // compress: output k takes the k-th kept position (ascending); values
        // are selected with static indices so everything stays in registers
        uint32_t rem = keepbits;
#pragma unroll
        for (int k = 0; k < MM - 1; ++k) {
            if (k < n) {
                const int q = __ffs(rem) - 1;
                rem &= rem - 1u;
                if (k == 0) i0 = q;
                if (k == 1) i1 = q;
                uint32_t val = 0;
#pragma unroll
                for (int i = 0; i < MM; ++i) val = (i == q) ? static_cast<uint32_t>(v[i]) : val;
                outw[k >> 1] |= val << (16 * (k & 1));
            }
        }
                if (n % 8 == 0) {
#pragma unroll
            for (int k = 0; k < (MM - 1) / 8; ++k)
                if (8 * k < n)
                    *reinterpret_cast<uint4 *>(dst + 8 * k) =
                        make_uint4(outw[4 * k], outw[4 * k + 1], outw[4 * k + 2], outw[4 * k + 3]);
        } else if (n % 4 == 0) {
#pragma unroll
            for (int k = 0; k < (MM - 1) / 4; ++k)
                if (4 * k < n)
                    *reinterpret_cast<uint2 *>(dst + 4 * k) = make_uint2(outw[2 * k], outw[2 * k + 1]);
        } else if (n % 2 == 0) {
#pragma unroll
            for (int k = 0; k < (MM - 1) / 2; ++k)
                if (2 * k < n) *reinterpret_cast<uint32_t *>(dst + 2 * k) = outw[k];
        } else {
#pragma unroll
            for (int k = 0; k < MM - 1; ++k)
                if (k < n) dst[k] = static_cast<uint16_t>(outw[k >> 1] >> (16 * (k & 1)));
        }
    }
    nib = static_cast<uint32_t>(i0 | (i1 << 2));
}

// groups per thread (all loads issued before any selection).  Measured on
// B200: four groups help 2:4, whose single group is only 24 bytes of loads;
// for m >= 6 one group per thread is faster (higher occupancy).
template <int M>
struct PruneGPT {
    static constexpr int value = M == 4 ? 4 : 1;
};

// grid: x over slices of PRUNE_THREADS * GPT groups of a row, y (+65535 z) =
// row.  Warp w of block b owns groups [32 GPT (8b + w), + 32 GPT); in step i
// lane l takes group 32 i + l of that range, so every load instruction of a
// warp reads 32 consecutive groups and every step yields m whole mask words.
template <int M, bool FUSED>
__global__ void __launch_bounds__(PRUNE_THREADS)
    k_prune(const ScoreSrc src, const uint16_t *__restrict__ V, int64_t ldv,
            int64_t K, int64_t G, int n, int m_rt, uint32_t *__restrict__ mask,
            uint16_t *__restrict__ vals, uint8_t *__restrict__ meta24) {
    constexpr int MM = M > 0 ? M : 16;
    constexpr int GPT = PruneGPT<M>::value;
    const int m = M > 0 ? M : m_rt;
    __shared__ uint32_t words[PRUNE_THREADS / 32][16];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535;
    const int64_t wg0 = (static_cast<int64_t>(blockIdx.x) * (PRUNE_THREADS / 32) + warp) * 32 * GPT;
    if (wg0 >= G) return;  // warp-uniform
    const int64_t mwords = (G * m + 31) / 32;
    const uint16_t *vrow = V + row * ldv;
    uint16_t *vout = vals + row * (G * n);

    float s[GPT][MM];
    uint16_t v[GPT][MM];
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
        const int64_t g = wg0 + i * 32 + lane;
        if (g < G) {
            if constexpr (FUSED) load_group_fused<M>(src, row, vrow, g * m, K, m, s[i], v[i]);
            else load_group<M>(src.S + row * src.lds, vrow, g * m, K, m, s[i], v[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
        const int64_t gw = wg0 + i * 32;  // first group of this step
        if (gw >= G) break;                // warp-uniform
        const int64_t g = gw + lane;
        const bool valid = g < G;
        uint32_t keepbits = 0, nib = 0;
        if (valid) select_group<M>(s[i], v[i], n, m, vout + g * n, keepbits, nib);
        const int64_t w0 = gw * m / 32;  // first mask word of this step
        if constexpr (M == 4 || M == 8) {
            // 32 / M groups per mask word: OR the lanes' bits together with
            // shuffles; the first lane of each word stores it
            constexpr int GPW = 32 / (M > 0 ? M : 32);
            uint32_t wbits = keepbits << (M * (lane % GPW));
#pragma unroll
            for (int o = 1; o < GPW; o <<= 1) wbits |= __shfl_xor_sync(0xffffffffu, wbits, o);
            const int64_t wi = w0 + lane / GPW;
            if ((lane % GPW) == 0 && wi < mwords) mask[row * mwords + wi] = wbits;
        } else {
            // groups straddle words: assemble the step's m words in shared memory
            if (lane < 16) words[warp][lane] = 0u;
            __syncwarp();
            if (valid) {
                const uint32_t off = static_cast<uint32_t>(lane) * m;
                atomicOr(&words[warp][off >> 5], keepbits << (off & 31));
                if ((off & 31) + m > 32) atomicOr(&words[warp][(off >> 5) + 1], keepbits >> (32 - (off & 31)));
            }
            __syncwarp();
            if (lane < m && w0 + lane < mwords) mask[row * mwords + w0 + lane] = words[warp][lane];
            __syncwarp();
        }
        if (M == 4 && meta24 != nullptr && n == 2) {
            // 8 nibbles (groups gw + 8j .. gw + 8j + 7) per 32-bit word
            uint32_t mb = nib << (4 * (lane & 7));
            mb |= __shfl_xor_sync(0xffffffffu, mb, 1);
            mb |= __shfl_xor_sync(0xffffffffu, mb, 2);
            mb |= __shfl_xor_sync(0xffffffffu, mb, 4);
            const int64_t mbytes = (G + 1) / 2;
            if ((lane & 7) == 0 && valid) {
                const int64_t b0 = g / 2;  // first byte of this word
                uint8_t *dst = meta24 + row * mbytes + b0;
                if (b0 + 4 <= mbytes && (reinterpret_cast<uintptr_t>(dst) & 3u) == 0) {
                    *reinterpret_cast<uint32_t *>(dst) = mb;
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (b0 + j < mbytes) dst[j] = static_cast<uint8_t>(mb >> (8 * j));
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// a3 for 2:4: one thread per run of 8 groups = 32 columns = one mask word.
// Loads 128 bytes of S and 64 bytes of V, keeps everything in registers, and
// writes 32 bytes of values, one mask word and one 32-bit word of metadata (8
// nibbles) -- no shuffles, no shared memory, four stores per 32 columns.
// grid: x over runs of a row (128 threads per block), y (+65535 z) = row.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void drop_two_of_4(const float (&s)[4], int &dlo, int &dhi) {
    // the two positions ranked last (score descending, index ascending):
    // "<=" picks the highest index among equal minima
    int d0 = 0;
    float s0 = s[0];
#pragma unroll
    for (int q = 1; q < 4; ++q)
        if (s[q] <= s0) { s0 = s[q]; d0 = q; }
    int d1 = -1;
    float s1 = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        if (q != d0 && (d1 < 0 || s[q] <= s1)) { s1 = s[q]; d1 = q; }
    dlo = d0 < d1 ? d0 : d1;
    dhi = d0 < d1 ? d1 : d0;
}

// 32 bf16 of a row from column c0 as 16 packed words, zero past K
__device__ __forceinline__ void load_run32(const uint16_t *__restrict__ p, int64_t c0, int64_t K,
                                           uint32_t (&w)[16]) {
    if (c0 + 32 <= K) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p) + j);
            w[4 * j] = u.x; w[4 * j + 1] = u.y; w[4 * j + 2] = u.z; w[4 * j + 3] = u.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t lo = c0 + 2 * j < K ? __ldg(p + 2 * j) : 0u;
            const uint32_t hi = c0 + 2 * j + 1 < K ? __ldg(p + 2 * j + 1) : 0u;
            w[j] = lo | (hi << 16);
        }
    }
}

// select + compress + store one 32-column run (8 groups) of a row
__device__ __forceinline__ void prune24_run(const float (&sc)[32], const uint32_t (&vw)[16], int64_t row,
                                            int64_t run, int64_t G, uint32_t *__restrict__ mask,
                                            uint16_t *__restrict__ vals, uint8_t *__restrict__ meta24) {
    const int64_t mwords = (G * 4 + 31) / 32, mbytes = (G + 1) / 2;
    uint32_t mword = 0, nibs = 0, out[8];
#pragma unroll
    for (int gi = 0; gi < 8; ++gi) {
        const float s4[4] = {sc[4 * gi], sc[4 * gi + 1], sc[4 * gi + 2], sc[4 * gi + 3]};
        int dlo, dhi;
        drop_two_of_4(s4, dlo, dhi);
        // kept positions i0 < i1 = the two of {0,1,2,3} other than dlo, dhi
        const int i0 = dlo == 0 ? (dhi == 1 ? 2 : 1) : 0;
        const int i1 = dhi == 3 ? (dlo == 2 ? 1 : 2) : 3;
        const uint32_t v4[4] = {vw[2 * gi] & 0xFFFFu, vw[2 * gi] >> 16, vw[2 * gi + 1] & 0xFFFFu,
                                vw[2 * gi + 1] >> 16};
        const uint32_t a = i0 == 0 ? v4[0] : (i0 == 1 ? v4[1] : v4[2]);
        const uint32_t b = i1 == 3 ? v4[3] : (i1 == 2 ? v4[2] : v4[1]);
        out[gi] = a | (b << 16);
        mword |= ((1u << i0) | (1u << i1)) << (4 * gi);
        nibs |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * gi);
    }
    const int64_t g0 = run * 8;  // first group of the run
    const int ng = G - g0 < 8 ? static_cast<int>(G - g0) : 8;
    uint16_t *vdst = vals + row * (G * 2) + g0 * 2;
    if (ng == 8 && ((reinterpret_cast<uintptr_t>(vdst) & 15u) == 0)) {
        reinterpret_cast<uint4 *>(vdst)[0] = make_uint4(out[0], out[1], out[2], out[3]);
        reinterpret_cast<uint4 *>(vdst)[1] = make_uint4(out[4], out[5], out[6], out[7]);
    } else {
#pragma unroll
        for (int gi = 0; gi < 8; ++gi)
            if (gi < ng) reinterpret_cast<uint32_t *>(vdst)[gi] = out[gi];
    }
    if (run < mwords) mask[row * mwords + run] = mword & (ng == 8 ? 0xFFFFFFFFu : ((1u << (4 * ng)) - 1u));
    uint8_t *mdst = meta24 + row * mbytes + g0 / 2;
    const int nb = (ng + 1) / 2;
    if (nb == 4 && ((reinterpret_cast<uintptr_t>(mdst) & 3u) == 0)) {
        *reinterpret_cast<uint32_t *>(mdst) = nibs;
    } else {
        nibs &= ng == 8 ? 0xFFFFFFFFu : ((1u << (4 * ng)) - 1u);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < nb) mdst[j] = static_cast<uint8_t>(nibs >> (8 * j));
    }
}

__global__ void __launch_bounds__(128, 8)
    k_prune24(const ScoreSrc src, const uint16_t *__restrict__ V, int64_t ldv,
              int64_t K, int64_t G, uint32_t *__restrict__ mask, uint16_t *__restrict__ vals,
              uint8_t *__restrict__ meta24) {
    const int64_t row = blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535;
    const int64_t run = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t c0 = run * 32;
    if (c0 >= K) return;
    const uint16_t *vrow = V + row * ldv + c0;
    const float *srow = src.S + row * src.lds + c0;
    float sc[32];
    uint32_t vw[16];
    if (c0 + 32 <= K) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(srow) + j);
            sc[4 * j] = f.x; sc[4 * j + 1] = f.y; sc[4 * j + 2] = f.z; sc[4 * j + 3] = f.w;
        }
    } else {
        // ragged end of the row: zero padding (score 0, value 0)
#pragma unroll
        for (int j = 0; j < 32; ++j) sc[j] = c0 + j < K ? __ldg(srow + j) : 0.0f;
    }
    load_run32(vrow, c0, K, vw);
    prune24_run(sc, vw, row, run, G, mask, vals, meta24);
}

// 2:4 with a2 fused: the block's 4096 columns of H + eps are staged once in
// shared memory, transposed so that lane t reading its j-th column hits
// consecutive words ([j][t], 129-double pitch), and reused for P24F_ROWS rows;
// each thread scores its 32-column run of W in registers.
// grid: x = 4096-column slices (128 threads), y (+65535 z) = row blocks.
constexpr int P24F_ROWS = 4;

__global__ void __launch_bounds__(128, 5)  // 96 registers: five blocks (33 KB of H each) per SM
    k_prune24_fused(const ScoreSrc src, const uint16_t *__restrict__ V, int64_t ldv, int64_t R,
                    int64_t K, int64_t G, uint32_t *__restrict__ mask, uint16_t *__restrict__ vals,
                    uint8_t *__restrict__ meta24) {
    __shared__ double hs[32 * 129];
    const int t = threadIdx.x;
    const int64_t cbase = static_cast<int64_t>(blockIdx.x) * 4096;
    const int64_t r0 = (blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535) * P24F_ROWS;
    const bool hess = src.H != nullptr;
    if (hess) {
        for (int i = t; i < 4096; i += 128) {
            const int64_t c = cbase + i;
            hs[(i & 31) * 129 + (i >> 5)] = c < K ? __dadd_rn(__ldg(src.H + c), src.eps) : 0.0;
        }
        __syncthreads();
    }
    const int64_t run = cbase / 32 + t;
    const int64_t c0 = run * 32;
    if (c0 >= K) return;
    // the next row's weights are loaded while this row is scored
    uint32_t wnext[16];
    load_run32(src.W + r0 * src.ldw + c0, c0, K, wnext);
#pragma unroll 1
    for (int rr = 0; rr < P24F_ROWS; ++rr) {
        const int64_t row = r0 + rr;
        if (row >= R) break;
        const uint16_t *wrow = src.W + row * src.ldw + c0;
        const uint16_t *vrow = V + row * ldv + c0;
        uint32_t ww[16], vw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) ww[j] = wnext[j];
        if (rr + 1 < P24F_ROWS && row + 1 < R) load_run32(wrow + src.ldw, c0, K, wnext);
        float sc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const uint16_t wb = static_cast<uint16_t>(ww[j >> 1] >> (16 * (j & 1)));
            if (c0 + j >= K) {
                sc[j] = 0.0f;
            } else if (hess) {
                const double w = bf16_to_f64(wb);
                sc[j] = __double2float_rn(__dmul_rn(hs[j * 129 + t], __dmul_rn(w, w)));
            } else {
                sc[j] = fabsf(bf16_to_f32(wb));
            }
        }
        if (vrow == wrow) {
#pragma unroll
            for (int j = 0; j < 16; ++j) vw[j] = ww[j];
        } else {
            load_run32(vrow, c0, K, vw);
        }
        prune24_run(sc, vw, row, run, G, mask, vals, meta24);
    }
}

// ---------------------------------------------------------------------------
// a4: sliding-window pack.  Each thread handles GT consecutive groups whose
// mask bits start on a 32-bit word boundary (GT*m a multiple of 32) and whose
// window nibbles fill whole bytes (GT*(m/2-1) even): it reads GT*m/32 words and
// writes GT*(m/2-1)/2 bytes.  A grid-stride loop over (row, run) pairs.
// ---------------------------------------------------------------------------
template <int M>
struct SlideRun {
    static constexpr int NWIN = M / 2 - 1;
    static constexpr int GT = M == 4 ? 8 : (M == 6 ? 16 : (M == 8 ? 8 : 16));
    static constexpr int WORDS = GT * M / 32;       // mask words in
    static constexpr int BYTES = GT * NWIN / 2;     // window bytes out
};

template <int M>
__global__ void __launch_bounds__(256)
    k_slide_pack(const uint32_t *__restrict__ mask, int64_t R, int64_t G, int64_t mwords,
                 int64_t wbytes, uint8_t *__restrict__ wmeta) {
    using RC = SlideRun<M>;
    // (2N-2):2N: a group's window nibbles come from one lookup in the
    // compile-time window table (entry 0xFFFF: not exactly m - 2 survivors)
    __shared__ uint16_t tab[M == 4 ? 1 : (1 << M)];
    if (M != 4) {
        for (int i = threadIdx.x; i < (1 << M); i += blockDim.x) tab[i] = g_wintab.v[wt_offset(M) + i];
        __syncthreads();
    }
    const uint64_t rpr = static_cast<uint64_t>((G + RC::GT - 1) / RC::GT);  // runs per row
    const uint64_t total = rpr * static_cast<uint64_t>(R);
    const bool narrow = total <= 0xFFFFFFFFull;
    bool bad = false;
    for (uint64_t idx = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const uint64_t row = narrow ? static_cast<uint32_t>(idx) / static_cast<uint32_t>(rpr) : idx / rpr;
        const uint64_t run = idx - row * rpr;
        const int64_t g0 = static_cast<int64_t>(run) * RC::GT;
        const uint32_t *mrow = mask + row * mwords + run * RC::WORDS;
        uint32_t w[RC::WORDS];
#pragma unroll
        for (int i = 0; i < RC::WORDS; ++i)
            w[i] = (static_cast<int64_t>(run) * RC::WORDS + i < mwords) ? __ldg(mrow + i) : 0u;
        uint32_t ow[(RC::BYTES + 3) / 4];
#pragma unroll
        for (int i = 0; i < (RC::BYTES + 3) / 4; ++i) ow[i] = 0u;
#pragma unroll
        for (int gi = 0; gi < RC::GT; ++gi) {
            if (g0 + gi >= G) break;
            const int b0 = gi * M;  // bit offset of this group in the run
            uint32_t bits = w[b0 >> 5] >> (b0 & 31);
            if ((b0 & 31) + M > 32) bits |= w[(b0 >> 5) + 1] << (32 - (b0 & 31));
            bits &= (1u << M) - 1u;
            uint32_t nibs;  // window w's nibble at bits 4w
            if (M == 4) {
                // 2:4: the two survivors, ascending, are the set bits
                if (__popc(bits) != 2) { bad = true; continue; }
                nibs = static_cast<uint32_t>(__ffs(bits) - 1) | (static_cast<uint32_t>(__ffs(bits & (bits - 1u)) - 1) << 2);
            } else {
                nibs = tab[bits];
                if (nibs == 0xFFFFu) { bad = true; continue; }
            }
            const int wi = gi * RC::NWIN;  // first nibble of the group in the run
            const int sh = 4 * (wi & 7);
            ow[wi >> 3] |= nibs << sh;
            if ((wi & 7) + RC::NWIN > 8) ow[(wi >> 3) + 1] |= nibs >> (32 - sh);
        }
        const int64_t byte0 = g0 * RC::NWIN / 2;
        uint8_t *dst = wmeta + row * wbytes + byte0;
        if (byte0 + RC::BYTES <= wbytes && (reinterpret_cast<uintptr_t>(dst) & 3u) == 0) {
#pragma unroll
            for (int i = 0; i < RC::BYTES / 4; ++i) reinterpret_cast<uint32_t *>(dst)[i] = ow[i];
        } else {
#pragma unroll
            for (int i = 0; i < RC::BYTES; ++i)
                if (byte0 + i < wbytes) dst[i] = static_cast<uint8_t>(ow[i >> 2] >> (8 * (i & 3)));
        }
    }
    if (bad) raise_error(ERRBIT_DEVICE);
}

// ---------------------------------------------------------------------------
// a5 (standalone): activation lift.  One thread per (token, group); window w
// of a group is the column pairs (w, w+1) of that group, as 32-bit words.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    k_lift(const uint16_t *__restrict__ X, int64_t T, int64_t K, int64_t ldx, int m, int64_t G,
           uint16_t *__restrict__ XL, int64_t ldxl) {
    const int Ns = m / 2, nwin = Ns - 1;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t t = blockIdx.y;
    if (g >= G || t >= T) return;
    const uint16_t *src = X + t * ldx + g * m;
    uint16_t *dst = XL + t * ldxl + g * nwin * 4;
    uint32_t x[8];  // m/2 column pairs
    if (g * m + m <= K) {
        for (int p = 0; p < Ns; ++p) x[p] = __ldg(reinterpret_cast<const uint32_t *>(src) + p);
    } else {
        for (int p = 0; p < Ns; ++p) {
            const int64_t c = g * m + 2 * p;
            const uint32_t a = c < K ? __ldg(src + 2 * p) : 0u;
            const uint32_t b = c + 1 < K ? __ldg(src + 2 * p + 1) : 0u;
            x[p] = a | (b << 16);
        }
    }
    uint32_t *d32 = reinterpret_cast<uint32_t *>(dst);
    for (int w = 0; w < nwin; ++w) {
        d32[2 * w] = x[w];
        d32[2 * w + 1] = x[w + 1];
    }
}

// ---------------------------------------------------------------------------
// ternary absmean quantisation: gamma = fl(fl(sum |w|) / (R K)).
//
// k_row_abs_sum: one warp per row; lane l sums |w| of the 8-column chunks
// l, l + 32, ... in fp64 as d = |w| 2^-896 (high word (bits & 0x7FFF) << 13:
// exact for zeros and subnormals too), once rounding up and once down (fact
// 1), and keeps the largest magnitude bits (an infinity or a NaN fails the
// row).  The 32 lanes' sums are added with TwoSum (fact 2).  The row's exact
// pair is written scaled back by 2^896 (exact), or NaN in s for a row that
// failed a check.  k_gamma adds the pairs with integer arithmetic in one
// block (a marked row summed again on the integer path) and divides once.
// ---------------------------------------------------------------------------
constexpr int GB_NDIG = 12;   // |w| sums: units of 2^-160, below 2^190
constexpr int GB_BIAS = 160;
using AbsAcc = BigAcc<GB_NDIG, GB_BIAS>;

__device__ __forceinline__ void abs_word(uint32_t w, double &up, double &dn, uint32_t &kmax) {
    const double d0 = hw_double((w << 13) & 0x0FFFE000u), d1 = hw_double((w >> 3) & 0x0FFFE000u);
    up = __dadd_ru(__dadd_ru(up, d0), d1);
    dn = __dadd_rd(__dadd_rd(dn, d0), d1);
    kmax = vmax_u16x2(kmax, w & 0x7FFF7FFFu);
}

__global__ void __launch_bounds__(256)
    k_row_abs_sum(const uint16_t *__restrict__ W, int64_t R, int64_t K, int64_t ldw, HPair *__restrict__ rec) {
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= R) return;  // warp-uniform
    const uint16_t *w = W + row * ldw;
    const int64_t nchunks = (K + 7) / 8;
    double up = 0.0, dn = 0.0;
    uint32_t kmax = 0u;
    int64_t c = lane;
    for (; c + 96 < nchunks && 8 * (c + 96) + 8 <= K; c += 128) {  // four chunks in flight
        uint4 u[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) u[k] = __ldg(reinterpret_cast<const uint4 *>(w + 8 * (c + 32 * k)));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            abs_word(u[k].x, up, dn, kmax);
            abs_word(u[k].y, up, dn, kmax);
            abs_word(u[k].z, up, dn, kmax);
            abs_word(u[k].w, up, dn, kmax);
        }
    }
    for (; c < nchunks; c += 32) {
        const int64_t j0 = 8 * c;
        if (j0 + 8 <= K) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(w + j0));
            abs_word(u.x, up, dn, kmax);
            abs_word(u.y, up, dn, kmax);
            abs_word(u.z, up, dn, kmax);
            abs_word(u.w, up, dn, kmax);
        } else {
            for (int64_t j = j0; j < K; ++j) abs_word(w[j], up, dn, kmax);  // high half zero
        }
    }
    const uint32_t mx = max(kmax & 0xFFFFu, kmax >> 16);
    bool bad = __any_sync(0xffffffffu, mx >= 0x7F80u || up != dn);
    double S = 0.0, CU = 0.0, CD = 0.0;
    for (int l = 0; l < 32; ++l) two_sum_acc2(S, CU, CD, __shfl_sync(0xffffffffu, up, l));
    if (lane != 0) return;
    bad |= CU != CD;
    HPair p;
    p.s = bad ? __longlong_as_double(0x7FF8000000000000ll) : __dmul_rn(S, 0x1p896);
    p.c = bad ? 0.0 : __dmul_rn(CU, 0x1p896);
    rec[row] = p;
}

// fp64 -> bf16 bits, round to nearest even, normal range only (0xFFFF if not
// representable as a normal bf16 or zero).  From the IEEE-754 definition.
__device__ uint32_t f64_to_bf16_bits(double v) {
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(v));
    const uint32_t sign = static_cast<uint32_t>(u >> 63) << 15;
    const int biased = static_cast<int>((u >> 52) & 0x7FFull);
    const unsigned long long frac = u & 0xFFFFFFFFFFFFFull;
    if (biased == 0 && frac == 0) return sign;
    int e = biased - 1023;
    if (e < -126 || e > 127) return 0xFFFFu;
    // significand with the implicit bit: 53 bits; bf16 keeps the top 8
    const unsigned long long sig = frac | (1ull << 52);
    unsigned long long top = sig >> 45;
    const unsigned long long tail = sig & ((1ull << 45) - 1ull);
    const bool up = tail > (1ull << 44) || (tail == (1ull << 44) && (top & 1ull));
    top += up ? 1ull : 0ull;
    if (top >> 8) { top >>= 1; ++e; }
    if (e > 127) return 0xFFFFu;
    return sign | (static_cast<uint32_t>(e + 127) << 7) | static_cast<uint32_t>(top & 0x7Full);
}

// clip(rint(fl(w / gamma)), -1, 1) without the division.  fl(|w| / gamma) > 0.5
// exactly when |w| / gamma > 0.5 + 2^-54 (the half-way point to the next
// double, which rounds to even = 0.5), i.e. |w| > h + 2^-54 gamma with
// h = gamma / 2.  For h < |w| <= 2h the difference |w| - h is exact (Sterbenz);
// above 2h the condition holds outright.  rint(x) for |x| > 0.5 is at least 1
// and clips to 1; |x| <= 0.5 gives 0 (0.5 ties to even).  gamma is a normal
// double (bf16(gamma) was representable), so gamma / 2 and 2^-54 gamma are
// exact.  The predicate grows with |w|, and non-negative bf16 values grow
// with their bit patterns, so it holds exactly for the magnitudes
// (bits & 0x7FFF) at or above one threshold: the smallest pattern for which
// it holds, found once by bisection over [0, 0x7F80] (0x7F80, +inf, always
// holds).  W itself is finite whenever bf16(gamma) is representable (an
// infinity or NaN in W makes gamma infinite or NaN, which zeroes the output).
__device__ __forceinline__ bool ternary_is_one(uint32_t mag_bits, double h, double tiny) {
    const double a = bf16_to_f64(static_cast<uint16_t>(mag_bits));
    return a > 2.0 * h || (a > h && __dsub_rn(a, h) > tiny);
}

__device__ uint32_t ternary_threshold(double gamma) {
    const double h = 0.5 * gamma, tiny = gamma * 0x1p-54;
    uint32_t lo = 0u, hi = 0x7F80u;  // the answer lies in [lo, hi]; hi holds
    while (lo < hi) {
        const uint32_t mid = (lo + hi) >> 1;
        if (ternary_is_one(mid, h, tiny))
            hi = mid;
        else
            lo = mid + 1u;
    }
    return lo;
}

// gamma from the rows' exact pairs.  First with TwoSum (fact 2): every
// thread adds its rows' pairs, the warps and then the block combine their
// (s, c up, c down) triples; when no row was marked and c up equals c down
// the total s + c is exact and is rounded once.  Otherwise every thread adds
// its rows into an integer accumulator (a marked row summed again from W),
// the block adds the accumulators digit by digit and rounds once.  Then one
// division by R*K.  One block of 1024 threads.
__device__ __forceinline__ void triple_shfl_add(double &S, double &CU, double &CD, int off) {
    const double s2 = __shfl_down_sync(0xffffffffu, S, off);
    const double u2 = __shfl_down_sync(0xffffffffu, CU, off);
    const double d2 = __shfl_down_sync(0xffffffffu, CD, off);
    two_sum_acc2(S, CU, CD, s2);
    CU = __dadd_ru(CU, u2);
    CD = __dadd_rd(CD, d2);
}

__global__ void __launch_bounds__(1024) k_gamma(const HPair *__restrict__ rec, const uint16_t *__restrict__ W,
                                                int64_t R, int64_t K, int64_t ldw,
                                                double *__restrict__ gamma_out, uint32_t *__restrict__ gb_out) {
    __shared__ long long part[32][GB_NDIG];
    __shared__ double tri[3][32];
    __shared__ double fast_total;
    __shared__ int fast_ok;
    grid_dep_wait();    // the rows' pairs
    grid_dep_launch();  // the apply grid may start loading W
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double S = 0.0, CU = 0.0, CD = 0.0;
    bool marked = false;
    for (int64_t i0 = threadIdx.x; i0 < R; i0 += 4 * static_cast<int64_t>(blockDim.x)) {
        HPair p[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t i = i0 + q * static_cast<int64_t>(blockDim.x);
            p[q] = i < R ? rec[i] : HPair{0.0, 0.0};
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            marked |= isnan(p[q].s);
            two_sum_acc2(S, CU, CD, p[q].s);
            CU = __dadd_ru(CU, p[q].c);
            CD = __dadd_rd(CD, p[q].c);
        }
    }
    for (int off = 16; off >= 1; off >>= 1) triple_shfl_add(S, CU, CD, off);
    if (lane == 0) {
        tri[0][warp] = S;
        tri[1][warp] = CU;
        tri[2][warp] = CD;
    }
    marked = __syncthreads_or(marked) != 0;
    if (warp == 0) {
        const int nw = static_cast<int>(blockDim.x / 32);
        S = lane < nw ? tri[0][lane] : 0.0;
        CU = lane < nw ? tri[1][lane] : 0.0;
        CD = lane < nw ? tri[2][lane] : 0.0;
        for (int off = 16; off >= 1; off >>= 1) triple_shfl_add(S, CU, CD, off);
        if (lane == 0) {
            // a NaN pair (marked row) makes S NaN: then the integer path decides
            fast_ok = !marked && CU == CD;
            fast_total = __dadd_rn(S, CU);
        }
    }
    __syncthreads();
    double total;
    bool nan = false, inf = false;
    if (fast_ok) {
        if (threadIdx.x != 0) return;
        total = fast_total;
    } else {
        AbsAcc a;
        a.clear();
        for (int64_t i = threadIdx.x; i < R; i += blockDim.x) {
            const HPair p = rec[i];
            if (!isnan(p.s)) {
                a.add_double(p.s);
                a.add_double(p.c);
                continue;
            }
            for (int64_t j = 0; j < K; ++j) {  // the integer path for a marked row
                const uint32_t b = W[i * ldw + j] & 0x7FFFu;
                const int e = static_cast<int>(b >> 7);
                if (e == 255) {
                    nan |= (b & 0x7Fu) != 0;
                    inf |= (b & 0x7Fu) == 0;
                } else if (b) {
                    a.add_bits(e ? 128u + (b & 0x7Fu) : b, (e ? e : 1) - 134 + GB_BIAS, false);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < GB_NDIG; ++i) {
            long long v = a.d[i];
            for (int off = 16; off >= 1; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
            if (lane == 0) part[warp][i] = v;
        }
        nan = __syncthreads_or(nan) != 0;
        inf = __syncthreads_or(inf) != 0;
        if (threadIdx.x != 0) return;
        AbsAcc tot;
        tot.clear();
        for (int wv = 0; wv < static_cast<int>(blockDim.x / 32); ++wv)
#pragma unroll
            for (int i = 0; i < GB_NDIG; ++i) tot.d[i] += part[wv][i];
        total = tot.round_rn();
    }
    if (nan) total = __longlong_as_double(0x7FF8000000000000ll);
    else if (inf) total = __longlong_as_double(0x7FF0000000000000ll);
    const double gamma = __ddiv_rn(total, __dmul_rn(static_cast<double>(R), static_cast<double>(K)));
    uint32_t gb = f64_to_bf16_bits(gamma);
    if (gamma == 0.0 || gb == 0xFFFFu) {
        raise_error(ERRBIT_DEVICE);
        gb = 0xFFFFu;
    }
    *gamma_out = gamma;
    gb_out[0] = gb;
    gb_out[1] = gb == 0xFFFFu ? 0x7F80u : ternary_threshold(gamma);
}

// W_q = clip(rint(W / gamma), -1, 1) * bf16(gamma): +-bf16(gamma) where
// |w|'s bits reach the threshold, else 0.  grid: x over 8-column chunks of a
// row (16-byte load, 16-byte store), y (+65535 z) = row.  Launched as a
// programmatic dependent of k_gamma: W is loaded before the wait for gamma.
__device__ __forceinline__ uint32_t ternary_pair(uint32_t w2, uint32_t thr, uint32_t gb) {
    const uint32_t lo = (w2 & 0x7FFFu) >= thr ? ((w2 & 0x8000u) | gb) : 0u;
    const uint32_t hi = ((w2 >> 16) & 0x7FFFu) >= thr ? (((w2 >> 16) & 0x8000u) | gb) : 0u;
    return lo | (hi << 16);
}

__global__ void __launch_bounds__(256)
    k_ternary_apply(const uint16_t *__restrict__ W, int64_t R, int64_t K, int64_t ldw,
                    const uint32_t *__restrict__ gb_p, uint16_t *__restrict__ Wq) {
    const int64_t i = blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535;
    const int64_t j0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
    const bool full = i < R && j0 + 8 <= K && (K & 7) == 0;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (full) u = __ldg(reinterpret_cast<const uint4 *>(W + i * ldw + j0));
    grid_dep_wait();  // gamma, its bf16 bits and the threshold
    if (i >= R || j0 >= K) return;
    const uint32_t gb = gb_p[0];
    const bool ok = gb != 0xFFFFu;
    const uint32_t thr = ok ? gb_p[1] : 0x10000u;  // nothing reaches 0x10000
    const uint32_t g = ok ? gb : 0u;
    uint16_t *dst = Wq + i * K + j0;
    if (full) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(ternary_pair(u.x, thr, g), ternary_pair(u.y, thr, g),
                                                     ternary_pair(u.z, thr, g), ternary_pair(u.w, thr, g));
    } else {
        for (int64_t j = j0; j < K && j < j0 + 8; ++j)
            dst[j - j0] = static_cast<uint16_t>(ternary_pair(W[i * ldw + j], thr, g));
    }
}

}  // namespace nm

// ===========================================================================
// C ABI
// ===========================================================================
using namespace nm;

namespace {

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline nm_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

inline int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

}  // namespace

namespace {

// the H reduction: one launch when a block sees every token; otherwise the
// partial pairs into `part`, then the finish as a programmatic dependent so
// that its launch overlaps the main kernel.  `max_split` caps the number of
// token ranges (the pairs `part` can hold are max_split * K).
// clusters of k_hsq with `split` blocks that the current device holds at
// once (0 on an error), cached per device and cluster size
std::atomic<int> g_hsq_clusters{1};  // 0: the workspace path only (test control)

int hsq_active_clusters(int64_t cblocks, int64_t split) {
    static int cache[64][9] = {};
    int dev = 0;
    if (split < 2 || split > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev][split] == 0) {
        // the kernel's shared-memory size must be allowed before the query
        // (else it reports that nothing fits); a failed query is not cached
        if (!set_smem_attr<k_hsq>(HX_SMEM_BYTES)) return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(cblocks), static_cast<unsigned>(split), 1);
        cfg.blockDim = dim3(HX_THREADS, 1, 1);
        cfg.dynamicSmemBytes = HX_SMEM_BYTES;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 1;
        at[0].val.clusterDim.y = static_cast<unsigned>(split);
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_hsq, &cfg) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cache[dev][split] = n > 0 ? n : -1;
    }
    return cache[dev][split] > 0 ? cache[dev][split] : 0;
}

nm_status launch_hsq(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, double *H, HPair *part,
                     int64_t max_split, cudaStream_t s) {
    using namespace nm;
    const HGrid g = h_grid(T, K, part ? max_split : 1);
    if (g.cblocks > 0x7FFFFFFF || g.split > 65535) return NM_ERR_SHAPE;
    CUtensorMap tm;
    if (!make_tmap_bf16(&tm, X, T, K, ldx, HX_COLS, HX_CHUNK, false)) return NM_ERR_CUDA;
    if (!set_smem_attr<k_hsq>(HX_SMEM_BYTES)) return NM_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(g.cblocks), static_cast<unsigned>(g.split));
    if (g.split == 1) {
        k_hsq<<<grid, HX_THREADS, HX_SMEM_BYTES, s>>>(tm, X, T, K, ldx, nullptr, H, 0);
        return launch_status();
    }
    // several token ranges: as one cluster per strip (at most 8 ranges),
    // combined in distributed shared memory, when every cluster is resident
    // at once; otherwise through the workspace pairs and k_hsq_finish
    const HGrid gc = h_grid(T, K, max_split < 8 ? max_split : 8);
    if (gc.split > 1 && g_hsq_clusters.load() != 0 && hsq_active_clusters(gc.cblocks, gc.split) >= gc.cblocks) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(gc.cblocks), static_cast<unsigned>(gc.split), 1);
        cfg.blockDim = dim3(HX_THREADS, 1, 1);
        cfg.dynamicSmemBytes = HX_SMEM_BYTES;
        cfg.stream = s;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 1;
        at[0].val.clusterDim.y = static_cast<unsigned>(gc.split);
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, k_hsq, tm, X, T, K, ldx, static_cast<HPair *>(nullptr), H, 1) != cudaSuccess)
            return NM_ERR_CUDA;
        return launch_status();
    }
    k_hsq<<<grid, HX_THREADS, HX_SMEM_BYTES, s>>>(tm, X, T, K, ldx, part, nullptr, 0);
    if (cudaGetLastError() != cudaSuccess) return NM_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((K + 127) / 128), 1, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_hsq_finish, static_cast<const HPair *>(part), g.split, X, T, K, ldx, H) !=
        cudaSuccess)
        return NM_ERR_CUDA;
    return launch_status();
}

// the checks shared by both H entry points (no launch, no output touched)
nm_status check_hessian_args(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, const double *H) {
    if (!X || !H) return NM_ERR_NULL;
    if (T < 1 || K < 1 || ldx < K) return NM_ERR_SHAPE;
    if (T > NM_HESSIAN_MAX_TOKENS || K > 0x3FFFFFFFll) return NM_ERR_SHAPE;
    if (!aligned16(X) || (ldx % 8) != 0 || (reinterpret_cast<uintptr_t>(H) & 7u)) return NM_ERR_ALIGN;
    return NM_OK;
}

}  // namespace

extern "C" nm_status nm_test_hessian_clusters(int on) {
    if (on != 0 && on != 1) return NM_ERR_SHAPE;
    g_hsq_clusters.store(on);
    return NM_OK;
}

extern "C" int nm_hessian_launch_count(int64_t T, int64_t K) {
    if (T <= 0 || K <= 0) return 0;
    if (h_grid(T, K, INT64_MAX).split <= 1) return 1;
    const HGrid gc = h_grid(T, K, 8);
    if (gc.split > 1 && g_hsq_clusters.load() != 0 && hsq_active_clusters(gc.cblocks, gc.split) >= gc.cblocks)
        return 1;
    return 2;
}

extern "C" size_t nm_hessian_workspace_bytes(int64_t T, int64_t K) {
    if (T <= 0 || K <= 0) return 0;
    const HGrid g = h_grid(T, K, INT64_MAX);
    return g.split > 1 ? static_cast<size_t>(g.split) * static_cast<size_t>(K) * sizeof(HPair) : 0;
}

extern "C" nm_status nm_hessian_diag(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                     double *H, void *ws, size_t ws_bytes, void *stream) {
    const nm_status st = check_hessian_args(X, T, K, ldx, H);
    if (st != NM_OK) return st;
    const size_t need = nm_hessian_workspace_bytes(T, K);
    if (need > 0 && (!ws || ws_bytes < need)) return NM_ERR_WORKSPACE;
    if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 15u)) return NM_ERR_ALIGN;
    return launch_hsq(X, T, K, ldx, H, static_cast<HPair *>(ws), INT64_MAX, as_stream(stream));
}

extern "C" nm_status nm_hessian_rescale(const double *H, const double *s, int64_t K, double *H_out,
                                        void *stream) {
    if (!H || !s || !H_out) return NM_ERR_NULL;
    if (K < 1 || (K + 255) / 256 > 0x7FFFFFFF) return NM_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(s) |
         reinterpret_cast<uintptr_t>(H_out)) & 7u)
        return NM_ERR_ALIGN;
    k_hessian_rescale<<<static_cast<unsigned>((K + 255) / 256), 256, 0, as_stream(stream)>>>(H, s, K, H_out);
    return launch_status();
}

extern "C" nm_status nm_score_from_hessian(const double *H, double eps, const uint16_t *W,
                                           int64_t R, int64_t K, int64_t ldw, float *S,
                                           void *stream) {
    if (!W || !S) return NM_ERR_NULL;
    if (R < 1 || K < 1 || ldw < K) return NM_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(S) || (ldw % 8) != 0) return NM_ERR_ALIGN;
    const int64_t rb = (R + SCORE_ROWS - 1) / SCORE_ROWS;  // row blocks
    dim3 grid(static_cast<unsigned>((K + 4095) / 4096), static_cast<unsigned>(rb < 65535 ? rb : 65535),
              static_cast<unsigned>((rb + 65534) / 65535));
    k_score<<<grid, 256, 0, as_stream(stream)>>>(H, eps, W, R, K, ldw, S);
    return launch_status();
}

extern "C" nm_status nm_score(const uint16_t *X, int64_t T, int64_t ldx, const uint16_t *W,
                              int64_t R, int64_t K, int64_t ldw, double eps, double *H, float *S,
                              void *ws, size_t ws_bytes, void *stream) {
    if (!W || !S) return NM_ERR_NULL;
    if (R < 1 || K < 1 || ldw < K) return NM_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(S) || (ldw % 8) != 0) return NM_ERR_ALIGN;
    if (X == nullptr) return nm_score_from_hessian(nullptr, 0.0, W, R, K, ldw, S, stream);
    if (!H) return NM_ERR_NULL;
    const nm_status st = nm_hessian_diag(X, T, K, ldx, H, ws, ws_bytes, stream);
    if (st != NM_OK) return st;
    return nm_score_from_hessian(H, eps, W, R, K, ldw, S, stream);
}

namespace {

// a3 launch (FUSED: with a2 in registers), arguments already validated
template <bool FUSED>
nm_status launch_prune(const ScoreSrc &src, const uint16_t *V, int64_t ldv, int64_t R, int64_t K, int n,
                       int m, uint32_t *mask, uint16_t *vals, uint8_t *meta24, cudaStream_t s) {
    const int64_t G = (K + m - 1) / m;
    uint8_t *meta = (m == 4 && n == 2) ? meta24 : nullptr;
    auto grid_for = [&](int gpt) {
        const int64_t per = static_cast<int64_t>(PRUNE_THREADS) * gpt;
        return dim3(static_cast<unsigned>((G + per - 1) / per), static_cast<unsigned>(R < 65535 ? R : 65535),
                    static_cast<unsigned>((R + 65534) / 65535));
    };
    switch (m) {
        case 4:
            if (n == 2 && !FUSED) {
                const int64_t runs = (K + 31) / 32;
                dim3 g24(static_cast<unsigned>((runs + 127) / 128), static_cast<unsigned>(R < 65535 ? R : 65535),
                         static_cast<unsigned>((R + 65534) / 65535));
                k_prune24<<<g24, 128, 0, s>>>(src, V, ldv, K, G, mask, vals, meta);
                break;
            }
            if (n == 2 && FUSED) {
                const int64_t rb = (R + P24F_ROWS - 1) / P24F_ROWS;
                dim3 g24(static_cast<unsigned>((K + 4095) / 4096), static_cast<unsigned>(rb < 65535 ? rb : 65535),
                         static_cast<unsigned>((rb + 65534) / 65535));
                k_prune24_fused<<<g24, 128, 0, s>>>(src, V, ldv, R, K, G, mask, vals, meta);
                break;
            }
            k_prune<4, FUSED><<<grid_for(PruneGPT<4>::value), PRUNE_THREADS, 0, s>>>(src, V, ldv, K, G, n, m, mask, vals, meta);
            break;
        case 6: k_prune<6, FUSED><<<grid_for(PruneGPT<6>::value), PRUNE_THREADS, 0, s>>>(src, V, ldv, K, G, n, m, mask, vals, meta); break;
        case 8: k_prune<8, FUSED><<<grid_for(PruneGPT<8>::value), PRUNE_THREADS, 0, s>>>(src, V, ldv, K, G, n, m, mask, vals, meta); break;
        case 10: k_prune<10, FUSED><<<grid_for(PruneGPT<10>::value), PRUNE_THREADS, 0, s>>>(src, V, ldv, K, G, n, m, mask, vals, meta); break;
        default: k_prune<0, FUSED><<<grid_for(PruneGPT<0>::value), PRUNE_THREADS, 0, s>>>(src, V, ldv, K, G, n, m, mask, vals, meta); break;
    }
    return launch_status();
}

}  // namespace

extern "C" nm_status nm_prune_compress(const float *S, int64_t lds, const uint16_t *V, int64_t ldv,
                                       int64_t R, int64_t K, int n, int m, uint32_t *mask,
                                       uint16_t *vals, uint8_t *meta24, void *stream) {
    if (!S || !V || !mask || !vals) return NM_ERR_NULL;
    if (m == 4 && n == 2 && !meta24) return NM_ERR_NULL;
    if (R < 1 || K < 1 || lds < K || ldv < K) return NM_ERR_SHAPE;
    if (m < 2 || m > 16 || n < 1 || n >= m) return NM_ERR_UNSUPPORTED;
    if (!aligned16(S) || !aligned16(V) || !aligned16(vals) || !aligned16(mask) ||
        (lds % 8) != 0 || (ldv % 8) != 0)
        return NM_ERR_ALIGN;
    if (R > 65535LL * 65535LL) return NM_ERR_SHAPE;
    const ScoreSrc src{S, lds, nullptr, 0, nullptr, 0.0};
    return launch_prune<false>(src, V, ldv, R, K, n, m, mask, vals, meta24, as_stream(stream));
}

extern "C" nm_status nm_score_prune_compress(const double *H, double eps, const uint16_t *W, int64_t ldw,
                                             const uint16_t *V, int64_t ldv, int64_t R, int64_t K, int n,
                                             int m, uint32_t *mask, uint16_t *vals, uint8_t *meta24,
                                             void *stream) {
    if (!W || !V || !mask || !vals) return NM_ERR_NULL;
    if (m == 4 && n == 2 && !meta24) return NM_ERR_NULL;
    if (R < 1 || K < 1 || ldw < K || ldv < K) return NM_ERR_SHAPE;
    if (m < 2 || m > 16 || n < 1 || n >= m) return NM_ERR_UNSUPPORTED;
    if (!aligned16(W) || !aligned16(V) || !aligned16(vals) || !aligned16(mask) || (ldw % 8) != 0 ||
        (ldv % 8) != 0 || (H && (reinterpret_cast<uintptr_t>(H) & 7u)))
        return NM_ERR_ALIGN;
    if (R > 65535LL * 65535LL) return NM_ERR_SHAPE;
    const ScoreSrc src{nullptr, 0, W, ldw, H, eps};
    return launch_prune<true>(src, V, ldv, R, K, n, m, mask, vals, meta24, as_stream(stream));
}

extern "C" nm_status slide_pack(const uint32_t *mask, int64_t R, int64_t K, int m, uint8_t *wmeta,
                                void *stream) {
    if (!mask || !wmeta) return NM_ERR_NULL;
    if (R < 1 || K < 1) return NM_ERR_SHAPE;
    if (m != 4 && m != 6 && m != 8 && m != 10) return NM_ERR_UNSUPPORTED;
    if (R > 65535LL * 65535LL) return NM_ERR_SHAPE;
    const int64_t G = (K + m - 1) / m;
    const int64_t mwords = (G * m + 31) / 32;
    const int64_t wbytes = (G * (m / 2 - 1) + 1) / 2;
    cudaStream_t s = as_stream(stream);
    auto grid_for = [&](int gt) {
        const int64_t runs = (G + gt - 1) / gt * R;
        int64_t blocks = (runs + 255) / 256;
        const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
        return static_cast<unsigned>(blocks < cap ? blocks : cap);
    };
    switch (m) {
        case 4: k_slide_pack<4><<<grid_for(SlideRun<4>::GT), 256, 0, s>>>(mask, R, G, mwords, wbytes, wmeta); break;
        case 6: k_slide_pack<6><<<grid_for(SlideRun<6>::GT), 256, 0, s>>>(mask, R, G, mwords, wbytes, wmeta); break;
        case 8: k_slide_pack<8><<<grid_for(SlideRun<8>::GT), 256, 0, s>>>(mask, R, G, mwords, wbytes, wmeta); break;
        default: k_slide_pack<10><<<grid_for(SlideRun<10>::GT), 256, 0, s>>>(mask, R, G, mwords, wbytes, wmeta); break;
    }
    return launch_status();
}

extern "C" nm_status lift_activations(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, int m,
                                      uint16_t *XL, int64_t ldxl, void *stream) {
    if (!X || !XL) return NM_ERR_NULL;
    if (m != 4 && m != 6 && m != 8 && m != 10) return NM_ERR_UNSUPPORTED;
    const int64_t G = (K + m - 1) / m;
    const int64_t KL = G * (m / 2 - 1) * 4;
    if (T < 1 || K < 1 || ldx < K || ldxl < KL) return NM_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(XL) || (ldx % 8) != 0 || (ldxl % 8) != 0) return NM_ERR_ALIGN;
    if (T > 65535) return NM_ERR_SHAPE;
    dim3 grid(static_cast<unsigned>((G + 255) / 256), static_cast<unsigned>(T));
    k_lift<<<grid, 256, 0, as_stream(stream)>>>(X, T, K, ldx, m, G, XL, ldxl);
    return launch_status();
}

extern "C" size_t nm_ternary_workspace_bytes(int64_t R) {
    return R > 0 ? static_cast<size_t>(R) * sizeof(HPair) + 16 : 0;
}

extern "C" nm_status nm_ternary_quantize(const uint16_t *W, int64_t R, int64_t K, int64_t ldw,
                                         uint16_t *Wq, double *gamma, void *ws, size_t ws_bytes,
                                         void *stream) {
    if (!W || !Wq || !gamma || !ws) return NM_ERR_NULL;
    if (R < 1 || K < 1 || ldw < K) return NM_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(ws) || (ldw % 8) != 0) return NM_ERR_ALIGN;
    if (ws_bytes < nm_ternary_workspace_bytes(R)) return NM_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    HPair *rec = static_cast<HPair *>(ws);
    uint32_t *gb = reinterpret_cast<uint32_t *>(rec + R);
    if ((R + 7) / 8 > 0x7FFFFFFF || R > 65535LL * 65535LL) return NM_ERR_SHAPE;
    k_row_abs_sum<<<static_cast<unsigned>((R + 7) / 8), 256, 0, s>>>(W, R, K, ldw, rec);
    // k_gamma and the apply grid are programmatic dependents: each may start
    // once its predecessor lets it and waits in-kernel for that one's results
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(1024, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_gamma, static_cast<const HPair *>(rec), W, R, K, ldw, gamma, gb) != cudaSuccess)
        return NM_ERR_CUDA;
    cfg.gridDim = dim3(static_cast<unsigned>((K + 2047) / 2048), static_cast<unsigned>(R < 65535 ? R : 65535),
                       static_cast<unsigned>((R + 65534) / 65535));
    cfg.blockDim = dim3(256, 1, 1);
    if (cudaLaunchKernelEx(&cfg, k_ternary_apply, W, R, K, ldw, static_cast<const uint32_t *>(gb), Wq) !=
        cudaSuccess)
        return NM_ERR_CUDA;
    return launch_status();
}

// ---------------------------------------------------------------------------
// Allocation-free H reduction: the partial pairs live in this file-scope
// device array instead of a caller workspace.  Host code must not pass the
// array's name to a kernel (on the host it is only a stand-in symbol): its
// device address is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) HPair g_hessian_noalloc_scratch[NM_HESSIAN_NOALLOC_MAX_PAIRS];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
HPair *g_noalloc_ptr[kMaxDevices] = {};

// device address of the scratch array for the current device (set-up on first use)
nm_status noalloc_scratch(HPair **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_hessian_noalloc_scratch) != cudaSuccess || p == nullptr)
            return NM_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<HPair *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return NM_OK;
}

}  // namespace

extern "C" nm_status nm_hessian_diag_noalloc(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                             double *H, void *stream) {
    const nm_status st = check_hessian_args(X, T, K, ldx, H);
    if (st != NM_OK) return st;
    // the token ranges are capped so that their pairs fit the array (a block
    // then takes more tokens); one range needs no scratch at all
    const int64_t max_split = NM_HESSIAN_NOALLOC_MAX_PAIRS / K;
    HPair *part = nullptr;
    if (max_split > 1 && h_grid(T, K, max_split).split > 1) {
        const nm_status s2 = noalloc_scratch(&part);
        if (s2 != NM_OK) return s2;
    }
    return launch_hsq(X, T, K, ldx, H, part, part ? max_split : 1, as_stream(stream));
}
