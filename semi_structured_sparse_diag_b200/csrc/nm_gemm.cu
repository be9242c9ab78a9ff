// nm_gemm.cu -- tcgen05 dense and 2:4-sparse GEMMs with TMA staging, the
// SlideSparse activation lift fused into the shared-memory staging, and the
// operand-preparation kernel.
//
// Problem: Y[T x R] = X[T x K] * W^T.  The tensor core computes D = A * B^T
// with A = weight tile (128 rows of W, K-major), B = activation tile (BN
// tokens, K-major) and D in tensor memory: lane = row of W, column = token.
//
// Sparse operand (SlideSparse, sec. 2A/2C): every width-4 window along the
// lifted dimension K' holds exactly two kept weights, so W' is 2:4 and runs on
// tcgen05.mma.sp: A holds 2 values per window (K'/2 per row), the 4-bit index
// pair of each window sits in tensor memory (copied from shared memory with
// tcgen05.cp).  For (2N-2):2N patterns the B tile is the lifted activation
// X', built by four warps from a raw X tile in shared memory (sec. 2B).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <chrono>
#include <mutex>

#include "nm_common.cuh"
#include "nm_host.cuh"

namespace nm {

constexpr int BM = 128;          // weight rows per tile (MMA M)
constexpr int GEMM_THREADS = 256;
constexpr int EBLK_BYTES = 2048; // metadata of 128 rows x 128 lifted columns

// ---------------------------------------------------------------------------
// packed operand layout (opaque to callers):
//   [0, Rpad*KLpad)                  values, row-major [Rpad x KLpad/2] bf16
//   [Rpad*KLpad, + Rpad*KLpad/8)     metadata blocks, (row tile of 128, K'
//                                    block of 128) order, 2048 bytes each
// Rpad = R rounded up to 256 (one CTA pair tile), KLpad = nkb * 128.
//
// K' order.  A K' block holds 32 windows ("slots") of 4 lifted columns.
//   m = 4, 6, 10: natural order: slot s of block kb is window wi = 32*kb + s,
//                 i.e. group wi / nwin, window wi % nwin (nwin = m/2 - 1).
//   m = 8       : blocks come in threes per 32 groups (256 columns of X):
//                 block 3j   : groups 32j .. 32j+15, windows 0 and 2 of each
//                              group = columns 8g .. 8g+7 of X, in X's order;
//                 block 3j+1 : groups 32j+16 .. 32j+31, likewise;
//                 block 3j+2 : window 1 (columns 8g+2 .. 8g+5) of groups
//                              32j .. 32j+31.
//                 Blocks 3j and 3j+1 are plain tiles of X (TMA loads them into
//                 the operand buffer); only block 3j+2 is built by the lift.
// Any consistent K' order gives the same product, because A (values and
// index pairs) and B (lifted activations) are permuted together.
// ---------------------------------------------------------------------------
struct PackedGeom {
    int64_t G, nwin, KL, KLpad, Rpad, nkb, vals_bytes, meta_bytes;
};

__host__ __device__ inline PackedGeom packed_geom(int64_t R, int64_t K, int m) {
    PackedGeom p;
    p.G = (K + m - 1) / m;
    p.nwin = p.G * (m / 2 - 1);
    p.KL = p.nwin * 4;
    p.nkb = m == 8 ? 3 * ((p.G + 31) / 32) : (p.KL + 127) / 128;
    p.KLpad = p.nkb * 128;
    p.Rpad = (R + 255) / 256 * 256;
    p.vals_bytes = p.Rpad * p.KLpad;       // Rpad x KLpad/2 bf16
    p.meta_bytes = p.Rpad * p.KLpad / 8;   // 4 bits per window of 4
    return p;
}

// (group, window) held by slot s of K' block kb
__host__ __device__ inline void slot_window(int m, int64_t kb, int s, int64_t &g, int &w) {
    if (m == 8) {
        const int64_t j = kb / 3;
        const int type = static_cast<int>(kb - 3 * j);
        if (type < 2) {
            g = 32 * j + 16 * type + s / 2;
            w = 2 * (s & 1);
        } else {
            g = 32 * j + s;
            w = 1;
        }
    } else {
        // nwin = m/2 - 1 is 1, 2 or 4 for m = 4, 6, 10
        const int sh = m == 4 ? 0 : (m == 6 ? 1 : 2);
        const int64_t wi = 32 * kb + s;
        g = wi >> sh;
        w = static_cast<int>(wi & ((1 << sh) - 1));
    }
}

// Metadata block byte b of a (128 row x 128 lifted column) tile holds the index
// pairs of two adjacent slots of one row.  The order is the one
// tcgen05.cp.128x128b + tcgen05.mma.sp expect for kind::f16 with 128 rows
// per CTA:
//   lane L = b/16 = m0 + 8*k1 + 16*m2, byte-in-lane = 4*k2 + 2*m1 + kh,
//   row = m0 + 8*m1 + 16*m2, first lifted column = 8*kh + 16*k1 + 32*k2.
// (k2 selects the tensor-memory column, i.e. the MMA k-step of 32 columns.)
__host__ __device__ inline void meta_byte_coords(int b, int &row, int &col) {
    const int L = b >> 4, within = b & 15;
    const int k2 = within >> 2, m1 = (within >> 1) & 1, kh = within & 1;
    const int m0 = L & 7, k1 = (L >> 3) & 1, m2 = L >> 4;
    row = m0 + 8 * m1 + 16 * m2;
    col = 8 * kh + 16 * k1 + 32 * k2;
}

// values, natural K' order (m = 4, 6, 10): the packed row is the row of vals
// (a window's pair of values = one 4-byte word, window wi at word wi) padded
// with zeros.  A thread moves the same 16-byte chunk of PV_ROWS consecutive
// rows, every load issued before the first store (64 bytes in flight per
// thread); 16-byte loads when every row of vals starts on 16 bytes (vec),
// else four 4-byte loads.  grid x = chunks of a row, y (+65535 z) = blocks
// of PV_ROWS rows.
constexpr int PV_ROWS = 4;
__global__ void __launch_bounds__(256)
    k_prepare_vals(const uint16_t *__restrict__ vals, int64_t R, int64_t words, int64_t Rpad, int64_t KLh,
                   bool vec, uint16_t *__restrict__ out) {
    grid_dep_launch();  // the metadata grid may run alongside
    const int64_t r0 = (blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535) * PV_ROWS;
    const int64_t c8 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // chunk
    if (r0 >= Rpad || c8 * 8 >= KLh) return;
    const int64_t w0 = 4 * c8;
    uint4 o[PV_ROWS];
#pragma unroll
    for (int i = 0; i < PV_ROWS; ++i) {
        const int64_t r = r0 + i;
        const uint32_t *vrow = reinterpret_cast<const uint32_t *>(vals) + r * words;
        o[i] = make_uint4(0u, 0u, 0u, 0u);
        if (r < R) {
            if (vec && w0 + 4 <= words) {
                o[i] = __ldg(reinterpret_cast<const uint4 *>(vrow + w0));
            } else {
                o[i].x = w0 < words ? __ldg(vrow + w0) : 0u;
                o[i].y = w0 + 1 < words ? __ldg(vrow + w0 + 1) : 0u;
                o[i].z = w0 + 2 < words ? __ldg(vrow + w0 + 2) : 0u;
                o[i].w = w0 + 3 < words ? __ldg(vrow + w0 + 3) : 0u;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < PV_ROWS; ++i)
        if (r0 + i < Rpad) *reinterpret_cast<uint4 *>(out + (r0 + i) * KLh + c8 * 8) = o[i];
}

// values, 6:8: a warp per row, PV68_JW blocks of 32 groups per warp.  A
// block's 96 words of vals (3 per group: windows 0, 1, 2) sit in the lanes'
// registers (word 32 c + lane in register c, all loads issued first); the 96
// output words of the block's three K' blocks -- windows 0 and 2 of groups
// 0-15, of groups 16-31, then window 1 of all 32 -- are gathered with
// shuffles: output word 32 c + lane takes source word s0 = 3 (lane / 2) +
// 2 (lane % 2), s0 + 48 or 3 lane + 1.  grid: x = PV68_JW blocks of 32 groups,
// y (+65535 z) = 8 rows.
constexpr int PV68_JW = 4;
__global__ void __launch_bounds__(256)
    k_prepare_vals68(const uint16_t *__restrict__ vals, int64_t R, int64_t G, int64_t Rpad, int64_t nj,
                     int64_t KLh, uint16_t *__restrict__ out) {
    grid_dep_launch();  // the metadata grid may run alongside
    const int lane = threadIdx.x & 31;
    const int64_t r = (blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535) * 8 + (threadIdx.x >> 5);
    if (r >= Rpad) return;  // warp-uniform
    const int64_t jb = static_cast<int64_t>(blockIdx.x) * PV68_JW;
    const int64_t words = 3 * G;
    const uint32_t *srow = reinterpret_cast<const uint32_t *>(vals) + (r < R ? r : 0) * words;
    uint32_t *drow = reinterpret_cast<uint32_t *>(out + r * KLh);
    const int64_t avail = r < R ? words - 96 * jb : 0;  // real words of the row from block jb on
    uint32_t v[PV68_JW][3];
#pragma unroll
    for (int k = 0; k < PV68_JW; ++k)
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const int w = 96 * k + 32 * c + lane;
            v[k][c] = w < avail ? __ldg(srow + 96 * jb + w) : 0u;
        }
    const int s0 = 3 * (lane >> 1) + 2 * (lane & 1), s1 = s0 + 48, s2 = 3 * lane + 1;
#pragma unroll
    for (int k = 0; k < PV68_JW; ++k) {
        if (jb + k >= nj) break;  // warp-uniform
        const uint32_t a0 = __shfl_sync(0xffffffffu, v[k][0], s0 & 31);
        const uint32_t a1 = __shfl_sync(0xffffffffu, v[k][1], s0 & 31);
        const uint32_t b1 = __shfl_sync(0xffffffffu, v[k][1], s1 & 31);
        const uint32_t b2 = __shfl_sync(0xffffffffu, v[k][2], s1 & 31);
        const uint32_t c0 = __shfl_sync(0xffffffffu, v[k][0], s2 & 31);
        const uint32_t c1 = __shfl_sync(0xffffffffu, v[k][1], s2 & 31);
        const uint32_t c2 = __shfl_sync(0xffffffffu, v[k][2], s2 & 31);
        uint32_t *d = drow + 96 * (jb + k);
        d[lane] = s0 < 32 ? a0 : a1;
        d[32 + lane] = s1 < 64 ? b1 : b2;
        d[64 + lane] = s2 < 32 ? c0 : (s2 < 64 ? c1 : c2);
    }
}


// groups of K' block kb: [g_lo, g_hi)
__device__ __forceinline__ void block_groups(int m, int64_t kb, int64_t &g_lo, int64_t &g_hi) {
    if (m == 8) {
        const int64_t j = kb / 3;
        const int type = static_cast<int>(kb - 3 * j);
        g_lo = type < 2 ? 32 * j + 16 * type : 32 * j;
        g_hi = g_lo + (type < 2 ? 16 : 32);
    } else {
        const int sh = m == 4 ? 0 : (m == 6 ? 1 : 2);
        g_lo = (32 * kb) >> sh;
        g_hi = (32 * kb + 32) >> sh;
    }
}

// 2:4 from the mask, eight groups of a mask word at once: nibble i of the
// result is s0 | s1 << 2 for the two set bits s0 < s1 of group i (bits 4i ..
// 4i + 3 of w); a group without exactly two set bits gets the padding pair
// (0, 1), and sets bad if it is one of the first c (real) groups.  Per group
// b0..b3: s0 = 0 if b0, else 1 if b1, else 2; s1 = 3 if b3, else 2 if b2,
// else 1.
__device__ __forceinline__ uint32_t nib24_word(uint32_t w, int c, bool &bad) {
    constexpr uint32_t K1 = 0x11111111u;
    const uint32_t b0 = w & K1, b1 = (w >> 1) & K1, b2 = (w >> 2) & K1, b3 = (w >> 3) & K1;
    const uint32_t s0lo = b1 & ~b0, s0hi = K1 & ~(b0 | b1);
    const uint32_t s1lo = b3 | (K1 & ~b2), s1hi = b3 | b2;
    const uint32_t nib = s0lo | (s0hi << 1) | (s1lo << 2) | (s1hi << 3);
    const uint32_t x = (b0 + b1 + b2 + b3) ^ 0x22222222u;  // per group: zero iff two bits set
    const uint32_t z = (x | (x >> 1) | (x >> 2)) & K1;      // bit 4i: group i invalid
    bad |= (z & (c >= 8 ? 0xFFFFFFFFu : (1u << (4 * c)) - 1u)) != 0u;
    const uint32_t keep = (K1 & ~z) * 0xFu;
    return (nib & keep) | (0x44444444u & ~keep);
}

// keeps the first c nibbles of w (0 <= c <= 8) and pads the rest with 4
__device__ __forceinline__ uint32_t keep_nibbles(uint32_t w, int c) {
    const uint32_t m = c >= 8 ? 0xFFFFFFFFu : (c <= 0 ? 0u : (1u << (4 * c)) - 1u);
    return (w & m) | (0x44444444u & ~m);
}

// little-endian 32-bit word of row bytes [off, off + 4), zero past `len`
// bytes; one aligned load when `aligned` (the row and off are 4-byte aligned
// and the row length a multiple of 4), else byte loads
__device__ __forceinline__ uint32_t row_word(const uint8_t *__restrict__ row, int64_t off, int64_t len,
                                             bool aligned) {
    if (aligned) return off + 4 <= len ? __ldg(reinterpret_cast<const uint32_t *>(row + off)) : 0u;
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b)
        if (off + b < len) v |= static_cast<uint32_t>(__ldg(row + off + b)) << (8 * b);
    return v;
}

// Where word k2 (slots 8 k2 .. 8 k2 + 7) of a row's 16 metadata bytes for K'
// block kb comes from: the groups [g_lo, g_lo + ng) of the block, c of them
// in this word (c <= 0: padding only).
struct MetaPos {
    int64_t kb, g_lo;
    int ng, c;
    bool mid;
};

template <int M>
__device__ __forceinline__ MetaPos meta_pos(int64_t kb, int64_t G, int k2) {
    MetaPos p;
    int64_t g_hi;
    block_groups(M, kb, p.g_lo, g_hi);
    p.kb = kb;
    p.ng = static_cast<int>((g_hi < G ? g_hi : G) - p.g_lo);
    p.mid = M == 8 && (kb % 3) == 2;
    const int gpw = M == 8 ? (p.mid ? 8 : 4) : 8 / (M / 2 - 1);  // groups per output word
    p.c = p.ng - gpw * k2;
    return p;
}

// the input words behind word k2 of row `row` (none for a padding row or word)
template <int M, bool FROM_MASK>
__device__ __forceinline__ void meta_fetch(const uint8_t *__restrict__ wmeta, const uint32_t *__restrict__ mask,
                                           int64_t row, int64_t R, int64_t wbytes, int64_t mwords, bool aligned,
                                           const MetaPos &p, int k2, uint32_t (&x)[4]) {
    constexpr int NWIN = M / 2 - 1;
    x[0] = x[1] = x[2] = x[3] = 0u;
    if (row >= R || p.c <= 0) return;
    const uint32_t *mrow = FROM_MASK ? mask + row * mwords : nullptr;
    const uint8_t *brow = FROM_MASK ? nullptr : wmeta + row * wbytes;
    auto mw = [&](int64_t q) -> uint32_t { return q < mwords ? __ldg(mrow + q) : 0u; };
    if (!FROM_MASK && M != 8) {  // natural order: the word itself
        x[0] = row_word(brow, ((p.g_lo * NWIN) >> 1) + 4 * k2, wbytes, aligned);
    } else if (!FROM_MASK) {  // 6:8 window bytes: the run of the word's groups
        const int64_t off = (p.g_lo * 3) / 2 + (p.mid ? 12 * k2 : 6 * k2);
        const int64_t a = off & ~static_cast<int64_t>(3);
        x[0] = row_word(brow, a, wbytes, aligned);
        x[1] = row_word(brow, a + 4, wbytes, aligned);
        if (p.mid) {  // 12 bytes from a 4-byte boundary or 2 past it
            x[2] = row_word(brow, a + 8, wbytes, aligned);
            x[3] = row_word(brow, a + 12, wbytes, aligned);
        }
    } else if (M == 4) {
        x[0] = mw(p.g_lo / 8 + k2);
    } else if (M == 8) {
        const int64_t q = p.g_lo / 4 + (p.mid ? 2 * k2 : k2);
        x[0] = mw(q);
        if (p.mid) x[1] = mw(q + 1);
    } else {
        const int64_t bit0 = p.g_lo * M + static_cast<int64_t>(8 / NWIN * M) * k2;
        x[0] = mw(bit0 >> 5);
        x[1] = mw((bit0 >> 5) + 1);
    }
}

// word k2 of the row from its input words x (meta_fetch): 8 slot nibbles,
// the padding pair 4 for a padding row (x unused: R_ok false) or group
template <int M, bool FROM_MASK>
__device__ __forceinline__ uint32_t meta_form(const uint32_t (&x)[4], bool row_ok, const MetaPos &p, int k2,
                                              const uint16_t *tab, bool &bad) {
    constexpr int NWIN = M / 2 - 1;
    if (!row_ok || p.c <= 0) return 0x44444444u;
    if (!FROM_MASK && M != 8) return keep_nibbles(x[0], p.c * NWIN);
    if (M == 4) return keep_nibbles(nib24_word(x[0], p.c, bad), p.c);
    if (M == 6 || M == 10) {  // groups of 6 or 10 mask bits through the table
        constexpr int GPW = 8 / NWIN;
        const int64_t bit0 = p.g_lo * M + static_cast<int64_t>(GPW * M) * k2;
        const uint32_t v = __funnelshift_r(x[0], x[1], static_cast<uint32_t>(bit0 & 31));
        constexpr uint32_t wm = (1u << (4 * NWIN)) - 1u;
        uint32_t W = 0x44444444u;
#pragma unroll
        for (int i = 0; i < GPW; ++i) {
            if (i >= p.c) break;
            uint32_t e = tab[(v >> (M * i)) & ((1u << M) - 1u)];
            if (e == 0xFFFFu) {
                bad = true;
                e = 0x4444u;
            }
            const int sh = 4 * NWIN * i;
            W = (W & ~(wm << sh)) | ((e & wm) << sh);
        }
        return W;
    }
    // 6:8: K' blocks 0 and 1 of a triple take windows 0 and 2 of 16 groups
    // (two slots per group), block 2 window 1 of 32 groups (one slot each)
    const int GPW = p.mid ? 8 : 4;
    uint32_t e[8];
    if (FROM_MASK) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i >= GPW) break;
            const uint32_t bits = ((i < 4 ? x[0] : x[1]) >> (8 * (i & 3))) & 0xFFu;
            e[i] = i < p.c ? tab[bits] : 0x444u;
            if (e[i] == 0xFFFFu) {
                bad = true;
                e[i] = 0x444u;
            }
        }
    } else {
        // window bytes: group g's windows are nibbles 3 (g - g_lo) + w of the
        // span from byte 3 g_lo / 2; the word's run of groups starts at byte
        // 3 GPW k2 / 2 of the span, 0 or 2 bytes into x[0]
        const int64_t off = (p.g_lo * 3) / 2 + (p.mid ? 12 * k2 : 6 * k2);
        const uint32_t sh = static_cast<uint32_t>(8 * (off & 3));
        const uint32_t y0 = __funnelshift_r(x[0], x[1], sh), y1 = __funnelshift_r(x[1], x[2], sh);
        const uint32_t y2 = __funnelshift_r(x[2], x[3], sh);
        auto nib = [&](int n) -> uint32_t {  // nibble n of the run
            const uint32_t y = n < 8 ? y0 : (n < 16 ? y1 : y2);
            return (y >> (4 * (n & 7))) & 0xFu;
        };
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i >= GPW) break;
            e[i] = i < p.c ? (nib(3 * i) | (nib(3 * i + 1) << 4) | (nib(3 * i + 2) << 8)) : 0x444u;
        }
    }
    uint32_t W = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i >= GPW) break;
        if (p.mid)
            W |= ((e[i] >> 4) & 0xFu) << (4 * i);
        else
            W |= ((e[i] & 0xFu) | (((e[i] >> 8) & 0xFu) << 4)) << (8 * i);
    }
    return W;
}

// metadata: 256 threads per run of PM_TILES consecutive (128-row tile, K'
// block) tiles, a grid-stride loop over the runs.  Thread t = k2 + 4 m0 +
// 32 m2 forms word k2 (slots 8 k2 .. 8 k2 + 7, slot 2p in the low nibble of
// byte p) of rows A = 16 m2 + m0 and B = A + 8 of each tile straight from
// global memory -- from the window metadata (natural orders: a masked copy),
// or, with FROM_MASK, from the mask bits (the sliding-window pack fused in:
// 2:4 bit-parallel, the other patterns through the window table); all the
// run's input words are loaded before the first is used.  It writes both in
// the tensor-memory order of meta_byte_coords: lanes A and A + 8 (k1 = 0, 1)
// hold in word k2 the low, respectively high, half-words of A's and B's word
// k2; a warp's two stores per tile cover 256 contiguous bytes.  Padding rows
// and slots get the pair (0, 1).
constexpr int PM_TILES = 4;
template <int M, bool FROM_MASK>
__global__ void __launch_bounds__(256)
    k_prepare_meta(const uint8_t *__restrict__ wmeta, const uint32_t *__restrict__ mask, int64_t R, int64_t G,
                   int64_t wbytes, int64_t mwords, int64_t nkb, int64_t ntiles, uint8_t *__restrict__ out) {
    __shared__ uint16_t tab[M == 4 ? 1 : (1 << M)];
    const int t = threadIdx.x;
    if (FROM_MASK && M != 4) {
        for (int i = t; i < (1 << M); i += blockDim.x) tab[i] = g_wintab.v[wt_offset(M) + i];
        __syncthreads();
    }
    const int k2 = t & 3, m0 = (t >> 2) & 7, m2 = t >> 5;
    const int la = m0 + 16 * m2;  // lane of k1 = 0 (and row A); k1 = 1 is la + 8 (row B)
    const bool aligned = (wbytes & 3) == 0 && (reinterpret_cast<uintptr_t>(wmeta) & 3u) == 0;
    const int64_t nruns = (ntiles + PM_TILES - 1) / PM_TILES;
    bool bad = false;
    for (int64_t run = blockIdx.x; run < nruns; run += gridDim.x) {
        const int64_t tile0 = run * PM_TILES;
        int64_t mt = tile0 / nkb, kb = tile0 - mt * nkb;
        MetaPos pos[PM_TILES];
        int64_t ra[PM_TILES];
        uint32_t xa[PM_TILES][4], xb[PM_TILES][4];
#pragma unroll
        for (int j = 0; j < PM_TILES; ++j) {
            pos[j] = meta_pos<M>(kb, G, k2);
            ra[j] = tile0 + j < ntiles ? mt * BM + la : R;  // past the last tile: nothing to load
            meta_fetch<M, FROM_MASK>(wmeta, mask, ra[j], R, wbytes, mwords, aligned, pos[j], k2, xa[j]);
            meta_fetch<M, FROM_MASK>(wmeta, mask, ra[j] + 8, R, wbytes, mwords, aligned, pos[j], k2, xb[j]);
            if (++kb == nkb) {
                kb = 0;
                ++mt;
            }
        }
#pragma unroll
        for (int j = 0; j < PM_TILES; ++j) {
            if (tile0 + j >= ntiles) break;
            const uint32_t wa = meta_form<M, FROM_MASK>(xa[j], ra[j] < R, pos[j], k2, tab, bad);
            const uint32_t wb = meta_form<M, FROM_MASK>(xb[j], ra[j] + 8 < R, pos[j], k2, tab, bad);
            uint32_t *o = reinterpret_cast<uint32_t *>(out + (tile0 + j) * EBLK_BYTES);
            o[la * 4 + k2] = __byte_perm(wa, wb, 0x5410);
            o[(la + 8) * 4 + k2] = __byte_perm(wa, wb, 0x7632);
        }
    }
    if (bad) raise_error(ERRBIT_DEVICE);
    grid_dep_wait();  // complete only after the values grid (see launch_prepare)
}

// 6:8 metadata from the mask, a K' block triple at a time: blocks 3j and
// 3j + 1 hold windows 0 and 2 of groups 32j .. 32j + 15 and 32j + 16 ..
// 32j + 31 (two slots per group), block 3j + 2 window 1 of all 32 (one slot
// each), and one window-table entry gives a group's three windows.  So 256
// threads per (128-row tile, triple), thread t = k2 + 4 m0 + 32 m2 looking up
// groups 32j + 8 k2 .. + 7 of rows A = 16 m2 + m0 and A + 8 once, form
// three words of each row: word k2 of block 3j + 2, and words 2 (k2 & 1) and
// 2 (k2 & 1) + 1 of block 3j + (k2 >> 1).  They are written in the
// tensor-memory order of meta_byte_coords as in k_prepare_meta.  A
// grid-stride loop over the (tile, triple) pairs.
__device__ __forceinline__ void meta68_row(uint32_t w0, uint32_t w1, int c, const uint16_t *tab, bool &bad,
                                           uint32_t &mid, uint32_t &lo, uint32_t &hi) {
    mid = 0u;
    lo = 0u;
    hi = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t e = 0x444u;  // a group past the last real one: padding pairs
        if (i < c) {
            e = tab[((i < 4 ? w0 : w1) >> (8 * (i & 3))) & 0xFFu];
            if (e == 0xFFFFu) {
                bad = true;
                e = 0x444u;
            }
        }
        mid |= ((e >> 4) & 0xFu) << (4 * i);
        const uint32_t pair = (e & 0xFu) | (((e >> 8) & 0xFu) << 4);  // windows 0 and 2
        if (i < 4)
            lo |= pair << (8 * i);
        else
            hi |= pair << (8 * (i - 4));
    }
}

__global__ void __launch_bounds__(256)
    k_prepare_meta68(const uint32_t *__restrict__ mask, int64_t R, int64_t G, int64_t mwords, int64_t nkb,
                     int64_t ntrip, uint8_t *__restrict__ out) {
    __shared__ uint16_t tab[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) tab[i] = g_wintab.v[wt_offset(8) + i];
    __syncthreads();
    const int t = threadIdx.x;
    const int k2 = t & 3, m0 = (t >> 2) & 7, m2 = t >> 5;
    const int la = m0 + 16 * m2;  // lane of k1 = 0 (row A); k1 = 1 is la + 8 (row B)
    const int64_t nj = nkb / 3;
    bool bad = false;
    for (int64_t it = blockIdx.x; it < ntrip; it += gridDim.x) {
        const int64_t mt = it / nj, j = it - mt * nj;
        const int64_t g0 = 32 * j + 8 * k2;  // this thread's first group
        const int c = static_cast<int>(G - g0 < 8 ? G - g0 : 8);  // its real groups (may be <= 0)
        const int64_t ra = mt * BM + la, rb = ra + 8;
        const int64_t q = g0 / 4;  // mask word of group g0 (8 bits per group)
        uint32_t a0 = 0u, a1 = 0u, b0 = 0u, b1 = 0u;
        if (c > 0) {
            if (ra < R) {
                a0 = __ldg(mask + ra * mwords + q);
                a1 = q + 1 < mwords ? __ldg(mask + ra * mwords + q + 1) : 0u;
            }
            if (rb < R) {
                b0 = __ldg(mask + rb * mwords + q);
                b1 = q + 1 < mwords ? __ldg(mask + rb * mwords + q + 1) : 0u;
            }
        }
        uint32_t ma, la0, la1, mb, lb0, lb1;
        meta68_row(a0, a1, ra < R ? c : 0, tab, bad, ma, la0, la1);
        meta68_row(b0, b1, rb < R ? c : 0, tab, bad, mb, lb0, lb1);
        uint32_t *om = reinterpret_cast<uint32_t *>(out + (mt * nkb + 3 * j + 2) * EBLK_BYTES);
        uint32_t *ot = reinterpret_cast<uint32_t *>(out + (mt * nkb + 3 * j + (k2 >> 1)) * EBLK_BYTES);
        const int w = 2 * (k2 & 1);
        om[la * 4 + k2] = __byte_perm(ma, mb, 0x5410);
        om[(la + 8) * 4 + k2] = __byte_perm(ma, mb, 0x7632);
        ot[la * 4 + w] = __byte_perm(la0, lb0, 0x5410);
        ot[(la + 8) * 4 + w] = __byte_perm(la0, lb0, 0x7632);
        ot[la * 4 + w + 1] = __byte_perm(la1, lb1, 0x5410);
        ot[(la + 8) * 4 + w + 1] = __byte_perm(la1, lb1, 0x7632);
    }
    if (bad) raise_error(ERRBIT_DEVICE);
    grid_dep_wait();  // complete only after the values grid (see launch_prepare)
}



// ---------------------------------------------------------------------------
// Single-CTA, one-tile-per-CTA GEMM (kept as the 1-CTA baseline of the
// ablation entry point; the library's GEMMs use the CTA-pair kernel below).
//   MODE_DENSE : A = W tile [128 x 64] per stage, 4 MMAs (K = 16 each).
//   MODE_SP24  : A = packed values [128 x 64] (= 128 lifted columns), B = X
//                tile [BN x 128] by TMA, E = 2 KB, 4 sparse MMAs (K = 32).
//   MODE_SPLIFT: as MODE_SP24 but B is built by four warps from a raw X tile
//                [BN x 128 columns] (natural window order).
// Warp roles: 0 = TMA producer, 1 = MMA issuer + tensor-memory owner,
// 4..7 = lift (MODE_SPLIFT) then epilogue (tensor memory -> bf16 -> TMA store).
// ---------------------------------------------------------------------------
enum { MODE_DENSE = 0, MODE_SP24 = 1, MODE_SPLIFT = 2 };

template <int MODE, int BN>
struct GemmCfg {
    static constexpr bool SPARSE = MODE != MODE_DENSE;
    static constexpr int A_BYTES = BM * 128;                              // 16 KB
    static constexpr int B_BYTES = SPARSE ? BN * 256 : BN * 128;         // 128 or 64 K cols
    static constexpr int X_BYTES = MODE == MODE_SPLIFT ? BN * 256 : 0;    // raw X, 128 cols
    static constexpr int E_BYTES = SPARSE ? EBLK_BYTES : 0;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + X_BYTES + E_BYTES;
    static constexpr int STAGES = MODE == MODE_DENSE ? 6 : (MODE == MODE_SP24 ? 4 : 2);
    static constexpr int OUT_BYTES = BN * BM * 2;
    static constexpr int TMEM_COLS = SPARSE ? (BN + 4 <= 256 ? 256 : 512) : (BN <= 128 ? 128 : 256);
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
    static constexpr uint32_t TX_BYTES = A_BYTES + (MODE == MODE_SPLIFT ? X_BYTES : B_BYTES) + E_BYTES;
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
    static_assert(OUT_BYTES <= STAGE_BYTES * STAGES, "epilogue staging");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int MODE, int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm_1cta(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmY, const uint8_t *__restrict__ meta, int64_t nkb,
           int m, int nwin) {
    using C = GemmCfg<MODE, BN>;
    constexpr int S = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES);
    uint64_t *full = bars, *empty = bars + S, *lifted = bars + 2 * S, *accum = bars + 3 * S;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * S + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, nt = blockIdx.y;

    auto stA = [&](int s) { return smem + s * C::STAGE_BYTES; };
    auto stB = [&](int s) { return smem + s * C::STAGE_BYTES + C::A_BYTES; };
    auto stX = [&](int s) { return smem + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES; };
    auto stE = [&](int s) {
        return smem + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES + C::X_BYTES;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&lifted[s], 4);
        }
        mbar_init(accum, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_e = tmem_base + BN;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int64_t kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = static_cast<int>(kb % S);
                const uint32_t ph = static_cast<uint32_t>((kb / S) & 1);
                if (kb >= S && !mbar_wait(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&full[s], C::TX_BYTES);
                if (MODE == MODE_DENSE) {
                    tma_load_2d(stA(s), &tmA, &full[s], static_cast<int32_t>(kb * 64), mt * BM);
                    tma_load_2d(stB(s), &tmB, &full[s], static_cast<int32_t>(kb * 64), nt * BN);
                } else {
                    tma_load_2d(stA(s), &tmA, &full[s], static_cast<int32_t>(kb * 64), mt * BM);
                    bulk_load(stE(s), meta + (static_cast<int64_t>(mt) * nkb + kb) * EBLK_BYTES,
                              EBLK_BYTES, &full[s]);
                    if (MODE == MODE_SP24) {
                        tma_load_2d(stB(s), &tmB, &full[s], static_cast<int32_t>(kb * 128), nt * BN);
                        tma_load_2d(stB(s) + BN * 128, &tmB, &full[s],
                                    static_cast<int32_t>(kb * 128 + 64), nt * BN);
                    } else {
                        const int64_t g_first = (kb * 32) / nwin;
                        const int32_t c0 = static_cast<int32_t>((g_first * m) & ~static_cast<int64_t>(7));
                        tma_load_2d(stX(s), &tmB, &full[s], c0, nt * BN);
                    }
                }
            }
            if (*abort_flag) {  // let copies already issued land before exiting
                const int64_t issued = kb;
                for (int64_t j = (issued > S ? issued - S : 0); j < issued; ++j)
                    mbar_wait(&full[j % S], static_cast<uint32_t>((j / S) & 1));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(BM, BN, C::SPARSE, 0);
            bool ok = true;
            for (int64_t kb = 0; kb < nkb && ok; ++kb) {
                const int s = static_cast<int>(kb % S);
                const uint32_t ph = static_cast<uint32_t>((kb / S) & 1);
                if (!mbar_wait(&full[s], ph)) { ok = false; break; }
                if (MODE == MODE_SPLIFT && !mbar_wait(&lifted[s], ph)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(stA(s)), b0 = smem_u32(stB(s));
                if (MODE == MODE_DENSE) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t ad = make_sdesc(a0 + j * 32, 16, 1024, 2);
                        const uint64_t bd = make_sdesc(b0 + j * 32, 16, 1024, 2);
                        mma_bf16(tmem_base, ad, bd, idesc, (kb > 0 || j > 0) ? 1u : 0u);
                    }
                } else {
                    tmem_cp_128x128b(tmem_e, make_sdesc(smem_u32(stE(s)), 2048, 128, 0));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t ad = make_sdesc(a0 + j * 32, 16, 1024, 2);
                        const uint64_t bd =
                            make_sdesc(b0 + (j >> 1) * (BN * 128) + (j & 1) * 64, 16, 1024, 2);
                        const uint32_t id = idesc | static_cast<uint32_t>(j & 1);
                        mma_sp_bf16(tmem_base, ad, bd, tmem_e + (j & ~1), id,
                                    (kb > 0 || j > 0) ? 1u : 0u);
                    }
                }
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(accum);
            else *abort_flag = 1;
        }
    } else if (warp >= 4) {
        const int ew = warp - 4;
        bool ok = true;
        if (MODE == MODE_SPLIFT) {
            // -------------------------------------------------------- lift
            for (int64_t kb = 0; kb < nkb; ++kb) {
                const int s = static_cast<int>(kb % S);
                const uint32_t ph = static_cast<uint32_t>((kb / S) & 1);
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph));
                if (!ok) break;
                const int64_t W0 = kb * 32;
                const int64_t g_first = W0 / nwin;
                const int64_t c0 = (g_first * m) & ~static_cast<int64_t>(7);
                const int64_t wi = W0 + lane;
                const int64_t g = wi / nwin;
                const int w = static_cast<int>(wi - g * nwin);
                const int src = static_cast<int>(g * m + 2 * w - c0);  // even, <= 124
                const uint8_t *xs = stX(s);
                uint8_t *bs = stB(s);
                const int chunk = lane >> 1;  // 16-byte chunk = 2 windows
                const int atom = chunk >> 3, cj = chunk & 7;
                for (int r = ew; r < BN; r += 4) {
                    const uint32_t *xrow = reinterpret_cast<const uint32_t *>(xs + r * 256);
                    const uint32_t lo = xrow[src >> 1], hi = xrow[(src >> 1) + 1];
                    uint8_t *dst = bs + atom * (BN * 128) + r * 128 + ((cj ^ (r & 7)) << 4) +
                                   ((lane & 1) << 3);
                    *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&lifted[s]);
            }
        }
        // ------------------------------------------------------------ epilogue
        // each warp owns 32 weight rows (its tensor-memory lane quarter) and
        // stores them with its own TMA store: no cross-warp barrier.
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(accum, 0));
        if (ok) {
            tc_fence_after();
            uint16_t *stage_out = reinterpret_cast<uint16_t *>(smem) + ew * (BN * 32);  // [BN][32]
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + cc * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t b = pack_bf16x2(__uint_as_float(v[j]), 0.0f) & 0xFFFFu;
                    stage_out[(cc * 32 + j) * 32 + lane] = static_cast<uint16_t>(b);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(&tmY, stage_out, mt * BM + ew * 32, nt * BN);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}


// ===========================================================================
// Persistent CTA-pair GEMM (tcgen05 cta_group::2).
//
// A cluster of two CTAs computes 256 weight rows x 256 tokens per tile: CTA r
// holds weight rows [128r, 128r+128) of the tile (its A) and tokens
// [128r, 128r+128) (its half of B).  The leader CTA (rank 0) issues every
// MMA; the tensor core reads A and B from both CTAs' shared memory, so each
// CTA feeds only half of B -- for the sparse instruction this halves the
// shared-memory reads per CTA and keeps the tensor pipe at its full rate
// (shared memory feeds the tensor core at 128 bytes/clock/SM).
//
// Warp roles (both CTAs):
//   warp 0      TMA producer: A (+ metadata E, + B where B is a plain tile of
//               X), completion bytes signalled on the leader's full[s];
//   warp 1      tensor-memory owner; in the leader also the MMA issuer;
//   warps 4-11  epilogue: tensor memory -> bf16 -> TMA store, 32 weight rows
//               x 128 tokens each;
//   warps 12-15 lift (SPLIFT / SP68 modes, SlideSparse sec. 2B): make this
//               CTA's lifted B half of each stage and tell the leader it is
//               ready (lifted[s]):
//               SPLIFT: copy each window's 4 columns of X from global memory
//               into the swizzled B buffer with cp.async, up to three stages
//               in flight (each warp arrives: 4 warps x 2 CTAs);
//               SP68:   raw blocks are TMA tiles of X counted on the leader's
//               full[s] like any other operand; warp 2 of the leader relays
//               their arrival to the peer CTA (xfull[s] there), and the lift
//               warps copy columns 2..5 of every group out of the two raw
//               stages into the third (odd) stage, then each signals it.
// Stages: a ring of S shared-memory stages per CTA; empty[s] and acc_full[b]
// are armed in both CTAs by multicast tcgen05.commit from the leader; in the
// lift modes empty[s] also waits for the 4 local lift warps (a raw stage is
// not refilled before the lift has read it).
// ===========================================================================
// PMODE_SP68T: 6:8 with every B block a TMA tile -- raw blocks from X, middle
// windows from X_mid (gathered by k_gather_mid before the GEMM).
enum { PMODE_DENSE = 0, PMODE_SP24 = 1, PMODE_SPLIFT = 2, PMODE_SP68 = 3, PMODE_SP68T = 4 };

template <int MODE>
struct PairCfg {
    static constexpr bool SPARSE = MODE != PMODE_DENSE;
    static constexpr bool LIFT = MODE == PMODE_SPLIFT || MODE == PMODE_SP68;
    static constexpr int BN = 256;                 // tokens per tile (both CTAs)
    static constexpr int BH = 128;                 // tokens per CTA
    static constexpr int A_BYTES = BM * 128;       // 128 rows x 128 bytes
    static constexpr int B_BYTES = SPARSE ? BH * 256 : BH * 128;
    static constexpr int E_BYTES = SPARSE ? EBLK_BYTES : 0;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + E_BYTES;
    static constexpr int STAGES = SPARSE ? 4 : 6;
    static constexpr int ACC_BUFS = SPARSE ? 1 : 2;     // accumulators of BN columns
    static constexpr int TMEM_COLS = 512;
    static constexpr int TMEM_E = 256;                  // metadata columns (sparse)
    static constexpr int EPI_WARPS = 8;
    static constexpr int EPI_BYTES = EPI_WARPS * 32 * 32 * 2;
    static constexpr int THREADS = LIFT ? 512 : 384;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(!SPARSE || TMEM_E >= ACC_BUFS * BN, "tensor memory");
};

__device__ __forceinline__ bool pair_needs_lift(int mode, int64_t kb) {
    return mode == PMODE_SPLIFT || (mode == PMODE_SP68 && (kb % 3) == 2);
}

// B by TMA: the stage's B half is a plain tile of X
__device__ __forceinline__ bool pair_b_by_tma(int mode, int64_t kb) {
    return mode == PMODE_DENSE || mode == PMODE_SP24 || mode == PMODE_SP68T ||
           (mode == PMODE_SP68 && (kb % 3) != 2);
}


// ---------------------------------------------------------------------------
// Work of one cluster.  Tile mode: whole tiles cluster, cluster + nclusters, ...
// Stream-K mode: the tiles' K' blocks laid end to end (tile-major) and cut into
// nclusters equal contiguous ranges; a range may start or end inside a tile.
// The cluster holding a split tile's first block owns it: it adds the fp32
// partial sums the later contributors (the next clusters) wrote to their slots,
// in ascending cluster order, and stores the result.  A contributor's part of a
// split tile is always the first segment of its range, the owner's part the
// last, so the owner only waits at the very end of its work.
// ---------------------------------------------------------------------------
// 6:8: the K' blocks in the order the library kernel's producer visits them --
// the blocks that are tiles of X itself first, the middle-window blocks (from
// the gathered X_mid) last -- so that the gather launched just before the GEMM
// overlaps the first two thirds of every tile's mainloop.  The packed layout
// is unchanged; only the order of the fp32 accumulation differs.
__device__ __forceinline__ int64_t visit68(int64_t v, int64_t nkb) {
    const int64_t nraw = 2 * (nkb / 3);
    return v < nraw ? 3 * (v >> 1) + (v & 1) : 3 * (v - nraw) + 2;
}

// Output tile order: bands of `gm` row tiles, each band walked token tile
// by token tile (the band's row tiles side by side).  Concurrent CTA pairs
// then share a few row tiles of weights and a few token tiles of X, which stay
// in L2 across the pairs and the waves of a band, instead of every wave
// streaming all of X again.  A bijection on [0, n_t * n_m); every role of a
// kernel uses it, so stream-K ranges over the same linear order.
__device__ __forceinline__ void tile_coords(int64_t tile, int64_t n_t, int64_t n_m, int64_t gm, int64_t &nt,
                                            int64_t &mt) {
    const int64_t band = tile / (gm * n_t);
    const int64_t rem = tile - band * gm * n_t;
    const int64_t rows = n_m - band * gm < gm ? n_m - band * gm : gm;  // row tiles of this band
    nt = rem / rows;
    mt = band * gm + (rem - nt * rows);
}
constexpr int64_t BAND_ROWS = 4096;   // weight rows per band of the tile order

struct SegIter {
    bool sk;
    int64_t nkb, pos, end, step;
    __device__ SegIter(bool sk_, int64_t cluster, int64_t nclusters, int64_t ntiles, int64_t nkb_)
        : sk(sk_), nkb(nkb_) {
        if (sk) {
            const int64_t total = ntiles * nkb;
            pos = cluster * total / nclusters;
            end = (cluster + 1) * total / nclusters;
            step = 0;
        } else {
            pos = cluster;
            end = ntiles;
            step = nclusters;
        }
    }
    __device__ bool more() const { return pos < end; }
    __device__ bool next(int64_t &tile, int64_t &kb0, int64_t &kb1) {
        if (pos >= end) return false;
        if (!sk) {
            tile = pos;
            kb0 = 0;
            kb1 = nkb;
            pos += step;
            return true;
        }
        tile = pos / nkb;
        kb0 = pos - tile * nkb;
        kb1 = kb0 + (end - pos) < nkb ? kb0 + (end - pos) : nkb;
        pos += kb1 - kb0;
        return true;
    }
};

// stream-K workspace: per (cluster, rank, epilogue warp) a slot of up to
// 32 rows x 240 columns fp32 ([column][row]; the 256-token pair tiles use the
// first 128 columns of their warp's slot) and a 64-bit flag that holds the
// launch's sequence number once the slot is written
constexpr int SK_SLOT_FLOATS = 32 * 240;
constexpr int64_t SK_MAX_CLUSTERS = NM_GEMM_STREAMK_MAX_CLUSTERS;

__host__ __device__ inline size_t sk_bytes(int64_t max_clusters) {
    return static_cast<size_t>(max_clusters) * 2 * 8 * (SK_SLOT_FLOATS * 4 + 8);
}

__device__ __forceinline__ void st_release_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// bounded wait for a stream-K flag (all lanes poll; one second limit)
__device__ __forceinline__ bool sk_wait_flag(const uint64_t *p, uint64_t seq) {
    if (ld_acquire_u64(p) == seq) return true;
    const uint64_t t0 = global_timer_ns(), limit = wait_limit_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire_u64(p) == seq) return true;
        if (global_timer_ns() - t0 > limit) {
            raise_error(ERRBIT_TIMEOUT);
            return false;
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(PairCfg<MODE>::THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmE,
                const __grid_constant__ CUtensorMap tmY,
                const uint16_t *__restrict__ X, int64_t T, int64_t K, int64_t ldx, int64_t R,
                int64_t nkb, int m, uint8_t *__restrict__ sk_ws, uint64_t seq, int stream_k) {
    using C = PairCfg<MODE>;
    const bool sk = stream_k != 0 && !C::LIFT;
    constexpr int S = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *epi_smem = smem + S * C::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(epi_smem + C::EPI_BYTES);
    uint64_t *full = bars, *empty = bars + S, *lifted = bars + 2 * S, *xfull = bars + 3 * S;
    uint64_t *acc_full = bars + 4 * S, *acc_empty = bars + 4 * S + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int64_t n_t = (T + C::BN - 1) / C::BN;
    const int64_t n_m = (R + 255) / 256;
    const int64_t ntiles = n_t * n_m;

    auto stA = [&](int s) { return smem + s * C::STAGE_BYTES; };
    auto stB = [&](int s) { return smem + s * C::STAGE_BYTES + C::A_BYTES; };
    auto stE = [&](int s) { return smem + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::LIFT ? 5 : 1);
            mbar_init(&lifted[s], 8);  // 4 lift warps (or the forwarder, x4) per CTA
            mbar_init(&xfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * C::EPI_WARPS);
        }
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmY);
        if (C::SPARSE) prefetch_tmap(&tmE);
        if (MODE == PMODE_SP68T) prefetch_tmap(&tmB2);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // everything above overlaps the previous kernel's tail (programmatic
    // dependent launch); global memory is touched only after this
    grid_dep_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int64_t it = 0;
            bool ok = true;
            SegIter seg(sk, cluster, nclusters, ntiles, nkb);
            int64_t tile, kb0, kb1;
            while (ok && seg.next(tile, kb0, kb1)) {
                int64_t nt, mt2;
                tile_coords(tile, n_t, n_m, BAND_ROWS / 256, nt, mt2);
                const int32_t arow = static_cast<int32_t>(mt2 * 256 + rank * 128);
                const int32_t brow = static_cast<int32_t>(nt * C::BN + rank * C::BH);
                for (int64_t kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                    if (it >= S && !mbar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
                    const bool btma = pair_b_by_tma(MODE, kb);
                    if (rank == 0) {
                        const uint32_t tx = 2u * static_cast<uint32_t>(
                            C::A_BYTES + C::E_BYTES + (btma ? C::B_BYTES : 0));
                        mbar_arrive_expect_tx(&full[s], tx);
                    }
                    const uint32_t bar = mapa_shared(&full[s], 0);
                    tma_load_2d_pair(stA(s), &tmA, bar, static_cast<int32_t>(kb * 64), arow);
                    if (C::SPARSE)
                        tma_load_2d_pair(stE(s), &tmE, bar, 0,
                                         static_cast<int32_t>(((mt2 * 2 + rank) * nkb + kb) * 8));
                    if (btma) {
                        if (MODE == PMODE_DENSE) {
                            tma_load_2d_pair(stB(s), &tmB, bar, static_cast<int32_t>(kb * 64), brow);
                        } else {
                            const bool mid = MODE == PMODE_SP68T && (kb % 3) == 2;
                            const int64_t x0 = MODE == PMODE_SP24 ? kb * 128
                                               : (mid ? (kb / 3) * 128 : (kb / 3) * 256 + (kb % 3) * 128);
                            const CUtensorMap *tb = mid ? &tmB2 : &tmB;
                            tma_load_2d_pair(stB(s), tb, bar, static_cast<int32_t>(x0), brow);
                            tma_load_2d_pair(stB(s) + C::BH * 128, tb, bar,
                                             static_cast<int32_t>(x0 + 64), brow);
                        }
                    }
                }
            }
            if (!ok && rank == 0) {  // let copies already issued land before exiting
                for (int64_t j = (it > S ? it - S : 0); j < it; ++j)
                    mbar_wait(&full[j % S], static_cast<uint32_t>((j / S) & 1));
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (rank == 0 && lane == 0) {
            const uint32_t idesc = make_idesc_bf16(256, C::BN, C::SPARSE, 0);
            int64_t it = 0, ti = 0;
            uint32_t lbits = 0;  // phase of lifted[s] (one phase per lifted use of stage s)
            bool ok = true;
            SegIter seg(sk, cluster, nclusters, ntiles, nkb);
            int64_t tile, kb0, kb1;
            for (; ok && seg.next(tile, kb0, kb1); ++ti) {
                const int buf = static_cast<int>(ti % C::ACC_BUFS);
                const uint32_t aph = static_cast<uint32_t>((ti / C::ACC_BUFS) & 1);
                if (ti >= C::ACC_BUFS && !mbar_wait_cluster(&acc_empty[buf], aph ^ 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem_base + static_cast<uint32_t>(buf * C::BN);
                for (int64_t kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                    if (!mbar_wait(&full[s], ph)) { ok = false; break; }
                    if (C::LIFT && pair_needs_lift(MODE, kb)) {
                        if (!mbar_wait_cluster(&lifted[s], (lbits >> s) & 1u)) { ok = false; break; }
                        lbits ^= 1u << s;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(stA(s)), b0 = smem_u32(stB(s));
                    if (!C::SPARSE) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16_pair(dcol, make_sdesc(a0 + j * 32, 16, 1024, 2),
                                          make_sdesc(b0 + j * 32, 16, 1024, 2), idesc,
                                          (kb > kb0 || j > 0) ? 1u : 0u);
                    } else {
                        const uint32_t te = tmem_base + C::TMEM_E;
                        tmem_cp_128x128b_pair(te, make_sdesc(smem_u32(stE(s)), 2048, 128, 0));
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_sp_bf16_pair(
                                dcol, make_sdesc(a0 + j * 32, 16, 1024, 2),
                                make_sdesc(b0 + (j >> 1) * (C::BH * 128) + (j & 1) * 64, 16, 1024, 2),
                                te + (j & ~1), idesc | static_cast<uint32_t>(j & 1),
                                (kb > kb0 || j > 0) ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[s]);
                }
                if (ok) mma_commit_pair(&acc_full[buf]);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;              // tensor-memory lane quarter
        const int h = (warp - 4) >> 2;       // token half of the tile
        uint16_t *stage_out = reinterpret_cast<uint16_t *>(epi_smem) + (warp - 4) * 1024;
        const uint32_t acc_empty_cl0 = mapa_shared(&acc_empty[0], 0);
        const uint32_t acc_empty_cl1 = mapa_shared(&acc_empty[1], 0);
        int64_t ti = 0;
        const int we = warp - 4;  // epilogue warp 0..7
        float *slots = reinterpret_cast<float *>(sk_ws);
        uint64_t *flags = reinterpret_cast<uint64_t *>(sk_ws + static_cast<size_t>(nclusters) * 2 * 8 *
                                                                   SK_SLOT_FLOATS * 4);
        const int64_t total = ntiles * nkb;
        SegIter seg(sk, cluster, nclusters, ntiles, nkb);
        int64_t tile, kb0, kb1;
        for (; seg.next(tile, kb0, kb1); ++ti) {
            int64_t nt, mt2;
            tile_coords(tile, n_t, n_m, BAND_ROWS / 256, nt, mt2);
            const int buf = static_cast<int>(ti % C::ACC_BUFS);
            const uint32_t aph = static_cast<uint32_t>((ti / C::ACC_BUFS) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], aph))) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * C::BN + h * 128);
            // 32-token chunks of this warp's half that hold real tokens
            const int64_t tok0 = nt * C::BN + h * 128;
            const int nvalid = tok0 >= T ? 0 : (T - tok0 >= 128 ? 4 : static_cast<int>((T - tok0 + 31) / 32));
            if (kb0 > 0) {
                // later part of a split tile: hand the fp32 partial to the owner
                // (the stores drain while the next segment's MMAs run)
                float *slot = slots + static_cast<size_t>((cluster * 2 + rank) * 8 + we) * SK_SLOT_FLOATS;
#pragma unroll 1
                for (int c = 0; c < nvalid; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) __stcg(slot + (c * 32 + j) * 32 + lane, __uint_as_float(v[j]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(buf == 0 ? acc_empty_cl0 : acc_empty_cl1);
                __threadfence();
                __syncwarp();
                if (lane == 0 && cluster != g_test_withhold_flag_cluster)
                    st_release_u64(flags + (cluster * 2 + rank) * 8 + we, seq);
                continue;
            }
            // owner: the clusters after this one that hold the rest of the tile
            int64_t last_contrib = cluster;
            if (sk && kb1 < nkb) {
                while (last_contrib + 1 < nclusters &&
                       (last_contrib + 1) * total / nclusters < (tile + 1) * nkb)
                    ++last_contrib;
                // clusters with an empty range (fewer blocks than clusters) write
                // nothing; after one wait times out the rest are not waited for
                bool got = true;
                for (int64_t cc = cluster + 1; cc <= last_contrib && got; ++cc)
                    if ((cc + 1) * total / nclusters > cc * total / nclusters)
                        got = sk_wait_flag(flags + (cc * 2 + rank) * 8 + we, seq);
            }
            uint32_t packed[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + c * 32, v);
                tmem_ld_wait();
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
                for (int64_t cc = cluster + 1; cc <= last_contrib && c < nvalid; ++cc) {
                    if ((cc + 1) * total / nclusters == cc * total / nclusters) continue;
                    const float *ps = slots + static_cast<size_t>((cc * 2 + rank) * 8 + we) * SK_SLOT_FLOATS +
                                      c * 32 * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j) f[j] += __ldcg(ps + j * 32 + lane);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) packed[c * 16 + i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf == 0 ? acc_empty_cl0 : acc_empty_cl1);
            const int32_t yr = static_cast<int32_t>(mt2 * 256 + rank * 128 + q * 32);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    stage_out[(2 * i) * 32 + lane] = static_cast<uint16_t>(packed[c * 16 + i] & 0xFFFFu);
                    stage_out[(2 * i + 1) * 32 + lane] = static_cast<uint16_t>(packed[c * 16 + i] >> 16);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, stage_out, yr,
                                 static_cast<int32_t>(nt * C::BN + h * 128 + c * 32));
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    } else if (MODE == PMODE_SP68 && warp == 2 && rank == 0) {
        // ---------------------------------------------------------- relay
        // raw blocks: once the leader's full[s] shows both CTAs' tiles have
        // landed, tell the peer CTA's lift warps (its xfull[s])
        const uint32_t xfull_peer0 = mapa_shared(&xfull[0], 1);
        int64_t it = 0;
        bool ok = true;
        for (int64_t tile = cluster; tile < ntiles && ok; tile += nclusters) {
            for (int64_t kb = 0; kb < nkb; ++kb, ++it) {
                if (kb % 3 == 2) continue;
                const int s = static_cast<int>(it % S);
                const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) {
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_cluster(xfull_peer0 + static_cast<uint32_t>(s) * 8u);
            }
        }
    } else if (C::LIFT && warp >= 12) {
        // ---------------------------------------------------------- lift
        const int lw = warp - 12;
        const uint32_t lifted_cl0 = mapa_shared(&lifted[0], 0);
        int64_t it = 0;
        uint32_t xbits = 0;  // phase of xfull[s] (one phase per raw use of stage s)
        bool ok = true;
        if (MODE == PMODE_SPLIFT) {
            // cp.async pipeline: stage of the block issued `d` steps ago, d = 1, 2
            int pend_s[2] = {-1, -1};
            for (int64_t tile = cluster; tile < ntiles && ok; tile += nclusters) {
                int64_t ntl, mtl;
                tile_coords(tile, n_t, n_m, BAND_ROWS / 256, ntl, mtl);
                const int64_t t0 = ntl * C::BN + rank * C::BH;
                for (int64_t kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                    if (it >= S && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u))) {
                        ok = false;
                        break;
                    }
                    int64_t g;
                    int w;
                    slot_window(m, kb, lane, g, w);
                    const int64_t col = g * m + 2 * w;  // first of the window's 4 columns
                    uint8_t *bs = stB(s);
                    const int chunk = (lane & 15) >> 1, atom = lane >> 4;
                    for (int row = lw; row < C::BH; row += 4) {
                        const int64_t t = t0 + row;
                        uint8_t *dst = bs + atom * (C::BH * 128) + row * 128 +
                                       ((chunk ^ (row & 7)) << 4) + ((lane & 1) << 3);
                        const bool tin = t < T;
                        const uint16_t *src = X + (tin ? t : 0) * ldx;
#pragma unroll
                        for (int hw = 0; hw < 2; ++hw) {
                            const int64_t c = col + 2 * hw;
                            if (tin && c + 2 <= K) {
                                cp_async4(dst + 4 * hw, src + c, 4u);
                            } else {  // past T or K: zeros (ragged last column keeps its value)
                                const uint32_t v = (tin && c < K) ? static_cast<uint32_t>(src[c]) : 0u;
                                *reinterpret_cast<uint32_t *>(dst + 4 * hw) = v;
                            }
                        }
                    }
                    cp_async_commit();
                    // the block issued two steps ago has landed: signal it
                    cp_async_wait_pending<2>();
                    if (pend_s[1] >= 0) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive_cluster(lifted_cl0 + static_cast<uint32_t>(pend_s[1]) * 8u);
                            mbar_arrive(&empty[pend_s[1]]);
                        }
                    }
                    pend_s[1] = pend_s[0];
                    pend_s[0] = s;
                }
            }
            // drain: signal the blocks still in flight, oldest first
            cp_async_wait_pending<0>();
            fence_proxy_async_smem();
            __syncwarp();
            for (int d = 1; d >= 0; --d) {
                if (pend_s[d] >= 0 && lane == 0) {
                    mbar_arrive_cluster(lifted_cl0 + static_cast<uint32_t>(pend_s[d]) * 8u);
                    mbar_arrive(&empty[pend_s[d]]);
                }
            }
        } else {  // PMODE_SP68
            for (int64_t tile = cluster; tile < ntiles && ok; tile += nclusters) {
                for (int64_t kb = 0; kb < nkb && ok; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    const int type = static_cast<int>(kb % 3);
                    if (type < 2) {
                        // raw block: its B half is a TMA tile of X in this CTA; the
                        // leader sees it land on full[s], the peer is told by the relay
                        bool landed;
                        if (rank == 0) {
                            landed = mbar_wait(&full[s], static_cast<uint32_t>((it / S) & 1));
                        } else {
                            landed = mbar_wait_cluster(&xfull[s], (xbits >> s) & 1u);
                            xbits ^= 1u << s;
                        }
                        if (!__all_sync(0xffffffffu, landed)) {
                            ok = false;
                            break;
                        }
                        // the odd stage of this super-block must be free
                        const int64_t it_odd = it + (2 - type);
                        const int so = static_cast<int>(it_odd % S);
                        if (type == 0 && it_odd >= S &&
                            !__all_sync(0xffffffffu,
                                        mbar_wait(&empty[so], static_cast<uint32_t>(((it_odd / S) & 1) ^ 1)))) {
                            ok = false;
                            break;
                        }
                        // columns 2..5 of a group = bytes 4..11 of its 16-byte chunk.
                        // Each quarter-warp reads one 128-byte row segment (one
                        // (row, atom) pair: 8 groups) with 16-byte loads, so every
                        // load and store instruction is free of bank conflicts.
                        const uint8_t *src = stB(s);
                        uint8_t *dst = stB(so);
                        const int c = lane & 7, k = lane >> 3;
                        uint32_t a[16], b[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int p = (lw * 16 + i) * 4 + k;  // (row, atom) pair
                            const int row = p >> 1, atom = p & 1;
                            const uint4 v = *reinterpret_cast<const uint4 *>(
                                src + atom * (C::BH * 128) + row * 128 + ((c ^ (row & 7)) << 4));
                            a[i] = v.y;
                            b[i] = v.z;
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int p = (lw * 16 + i) * 4 + k;
                            const int row = p >> 1, atom = p & 1;
                            const int gl = atom * 8 + c;          // group within the raw block
                            const int dchunk = gl >> 1;           // slot 16*type + gl
                            *reinterpret_cast<uint2 *>(dst + type * (C::BH * 128) + row * 128 +
                                                       ((dchunk ^ (row & 7)) << 4) + ((gl & 1) << 3)) =
                                make_uint2(a[i], b[i]);
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&empty[s]);  // done reading the raw stage
                    } else {
                        // odd block: its B half was filled by the two raw steps
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive_cluster(lifted_cl0 + static_cast<uint32_t>(s) * 8u);
                            mbar_arrive(&empty[s]);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ===========================================================================
// Wide sparse GEMM (library path for every pattern).
//
// Shared-memory bandwidth sets the rate of the sparse kernel above: a
// 2:4-sparse MMA step of the CTA pair (M = 256, N = 256, 32 lifted columns)
// keeps the tensor core busy for 128 clocks, but each CTA's shared memory must
// take in and hand out 12 KB of operands for it (4 KB of A, 8 KB of its B
// half: written by TMA, read by the tensor core), 192 clocks at 128 bytes per
// clock -- a ceiling of 2/3 of the sparse peak.  Here a pair computes 512
// weight rows x bn (<= 240) tokens with two MMAs per step that share the B
// tile: CTA r holds A rows [128r, 128r+128) and [256+128r, 256+128r+128) of
// the tile, each with its metadata, and bn/2 tokens of B.  Per step and CTA:
// 8 KB of A and 7.5 KB of B written, 8 KB of A and 2 x 7.5 KB of B read
// (each MMA reads B once), 308 clocks for 240 clocks of MMA: 78% of peak.
//
// Tensor memory (512 columns): accumulator 0 in [0, 240), its metadata at
// 240, accumulator 1's metadata at 248, accumulator 1 in [256, 496).  One
// accumulator pair per CTA, so the next tile's MMAs start once the epilogue
// warps have moved this tile's sums into registers (bf16).
// Warps: 0 producer, 1 tensor-memory owner and (leader) MMA issuer, 4-11
// epilogue (lane quarter warp % 4, accumulator (warp - 4) / 4): tcgen05.ld of
// the whole tile into registers as bf16, release of the accumulator, then
// plain global stores (a warp stores 32 consecutive weight rows of one token,
// 64 contiguous bytes, per instruction) -- no shared-memory staging, so the
// stores of one tile overlap the next tile's MMAs without waiting on TMA.
// Tiles where rows 256..511 lie past the padded R (a multiple of 256) skip
// accumulator 1's loads and MMAs.
// Schedules as k_gemm_pair: whole tiles, or stream-K (SegIter above).
// ===========================================================================
struct WideCfg {
    static constexpr int BN_MAX = 240;              // tokens per tile (both CTAs)
    static constexpr int BH_MAX = BN_MAX / 2;       // tokens per CTA
    static constexpr int A_BYTES = BM * 128;        // 128 rows x 64 values
    static constexpr int B_ATOM = BH_MAX * 128;     // 64 lifted columns x BH_MAX tokens
    static constexpr int OFF_A0 = 0, OFF_A1 = A_BYTES, OFF_B = 2 * A_BYTES;
    static constexpr int OFF_E0 = OFF_B + 2 * B_ATOM, OFF_E1 = OFF_E0 + EBLK_BYTES;
    static constexpr int STAGE_BYTES = OFF_E1 + EBLK_BYTES;
    static constexpr int STAGES = 3;
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 384;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    static constexpr int TMEM_COLS = 512;
    static constexpr int TMEM_D0 = 0, TMEM_E0 = 240, TMEM_E1 = 248, TMEM_D1 = 256;
    static_assert(STAGE_BYTES % 1024 == 0 && B_ATOM % 1024 == 0, "stage alignment");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(32 * BN_MAX <= SK_SLOT_FLOATS, "stream-K slot");
};

template <int MODE>
__global__ void __launch_bounds__(WideCfg::THREADS, 1)
    k_gemm_wide(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmE,
                const __grid_constant__ CUtensorMap tmY, uint16_t *__restrict__ Y, int64_t ldy, int64_t T,
                int64_t R, int64_t nkb, int bn, uint8_t *__restrict__ sk_ws, uint64_t seq, int stream_k) {
    using C = WideCfg;
    constexpr int S = C::STAGES;
    const bool sk = stream_k != 0;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES);
    uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S, *acc_empty = bars + 2 * S + 1;
    uint64_t *out_ready = bars + 2 * S + 2;  // [2]: an accumulator's output staged (4 warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int bh = bn >> 1;
    const int64_t n_t = (T + bn - 1) / bn;
    const int64_t Rpad = (R + 255) / 256 * 256;
    const int64_t n_m = (Rpad + 511) / 512;
    const int64_t ntiles = n_t * n_m;
    auto stage = [&](int s) { return smem + s * C::STAGE_BYTES; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * C::EPI_WARPS);
        mbar_init(&out_ready[0], 4);
        mbar_init(&out_ready[1], 4);
        fence_barrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmE);
        prefetch_tmap(&tmY);
        if (MODE == PMODE_SP68T) prefetch_tmap(&tmB2);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // everything above overlaps the previous kernel's tail (programmatic
    // dependent launch); global memory is touched only after this.  For 6:8
    // the producer reads only inputs older than that kernel (X, the packed
    // weights) until its first middle-window block and waits there; the MMA
    // warp touches no global memory.
    if (MODE != PMODE_SP68T || warp >= 2) grid_dep_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int64_t it = 0;
            bool ok = true;
            bool dep_done = MODE != PMODE_SP68T;
            SegIter seg(sk, cluster, nclusters, ntiles, nkb);
            int64_t tile, kb0, kb1;
            const uint32_t b_bytes = static_cast<uint32_t>(bh) * 256u;
            while (ok && seg.next(tile, kb0, kb1)) {
                int64_t nt, mt;
                tile_coords(tile, n_t, n_m, BAND_ROWS / 512, nt, mt);
                const bool has1 = mt * 512 + 256 < Rpad;
                const int32_t arow = static_cast<int32_t>(mt * 512 + rank * 128);
                const int32_t brow = static_cast<int32_t>(nt * bn + rank * bh);
                const int64_t e0 = (mt * 4 + rank) * nkb, e1 = (mt * 4 + 2 + rank) * nkb;
                const uint32_t tx = 2u * ((has1 ? 2u : 1u) * (C::A_BYTES + EBLK_BYTES) + b_bytes);
                for (int64_t v = kb0; v < kb1; ++v, ++it) {
                    const int64_t kb = MODE == PMODE_SP68T ? visit68(v, nkb) : v;
                    const bool mid = MODE == PMODE_SP68T && (kb % 3) == 2;
                    if (mid && !dep_done) {  // X_mid is the previous kernel's output
                        grid_dep_wait();
                        dep_done = true;
                    }
                    const int s = static_cast<int>(it % S);
                    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                    if (it >= S && !mbar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], tx);
                    const uint32_t bar = mapa_shared(&full[s], 0);
                    uint8_t *st = stage(s);
                    const int32_t ka = static_cast<int32_t>(kb * 64);
                    tma_load_2d_pair(st + C::OFF_A0, &tmA, bar, ka, arow);
                    tma_load_2d_pair(st + C::OFF_E0, &tmE, bar, 0, static_cast<int32_t>((e0 + kb) * 8));
                    if (has1) {
                        tma_load_2d_pair(st + C::OFF_A1, &tmA, bar, ka, arow + 256);
                        tma_load_2d_pair(st + C::OFF_E1, &tmE, bar, 0,
                                         static_cast<int32_t>((e1 + kb) * 8));
                    }
                    const int64_t x0 = MODE == PMODE_SP24 ? kb * 128
                                       : (mid ? (kb / 3) * 128 : (kb / 3) * 256 + (kb % 3) * 128);
                    const CUtensorMap *tb = mid ? &tmB2 : &tmB;
                    tma_load_2d_pair(st + C::OFF_B, tb, bar, static_cast<int32_t>(x0), brow);
                    tma_load_2d_pair(st + C::OFF_B + C::B_ATOM, tb, bar, static_cast<int32_t>(x0 + 64),
                                     brow);
                }
            }
            if (!ok && rank == 0) {  // let copies already issued land before exiting
                for (int64_t j = (it > S ? it - S : 0); j < it; ++j)
                    mbar_wait(&full[j % S], static_cast<uint32_t>((j / S) & 1));
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (rank == 0 && lane == 0) {
            const uint32_t idesc = make_idesc_bf16(256, bn, true, 0);
            int64_t it = 0, ti = 0;
            bool ok = true;
            SegIter seg(sk, cluster, nclusters, ntiles, nkb);
            int64_t tile, kb0, kb1;
            for (; ok && seg.next(tile, kb0, kb1); ++ti) {
                int64_t ntm, mtm;
                tile_coords(tile, n_t, n_m, BAND_ROWS / 512, ntm, mtm);
                const bool has1 = mtm * 512 + 256 < Rpad;
                if (ti >= 1 && !mbar_wait_cluster(acc_empty, static_cast<uint32_t>((ti - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + C::TMEM_D0, d1 = tmem_base + C::TMEM_D1;
                const uint32_t te0 = tmem_base + C::TMEM_E0, te1 = tmem_base + C::TMEM_E1;
                for (int64_t kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = static_cast<int>(it % S);
                    const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
                    if (!mbar_wait(&full[s], ph)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(stage(s));
                    tmem_cp_128x128b_pair(te0, make_sdesc(st + C::OFF_E0, 2048, 128, 0));
                    if (has1) tmem_cp_128x128b_pair(te1, make_sdesc(st + C::OFF_E1, 2048, 128, 0));
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t bd =
                            make_sdesc(st + C::OFF_B + (j >> 1) * C::B_ATOM + (j & 1) * 64, 16, 1024, 2);
                        const uint32_t acc = (kb > kb0 || j > 0) ? 1u : 0u;
                        const uint32_t id = idesc | static_cast<uint32_t>(j & 1);
                        mma_sp_bf16_pair(d0, make_sdesc(st + C::OFF_A0 + j * 32, 16, 1024, 2), bd,
                                         te0 + (j & ~1), id, acc);
                        if (has1)
                            mma_sp_bf16_pair(d1, make_sdesc(st + C::OFF_A1 + j * 32, 16, 1024, 2), bd,
                                             te1 + (j & ~1), id, acc);
                    }
                    mma_commit_pair(&empty[s]);
                }
                if (ok) mma_commit_pair(acc_full);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;         // tensor-memory lane quarter
        const int h = (warp - 4) >> 2;  // accumulator
        const int we = warp - 4;
        const uint32_t acc_empty_cl = mapa_shared(acc_empty, 0);
        float *slots = reinterpret_cast<float *>(sk_ws);
        uint64_t *flags = reinterpret_cast<uint64_t *>(sk_ws + static_cast<size_t>(nclusters) * 2 * 8 *
                                                                   SK_SLOT_FLOATS * 4);
        const int64_t total = ntiles * nkb;
        // a cluster whose range is empty (fewer K' blocks than clusters) writes nothing
        auto has_work = [&](int64_t cc) { return (cc + 1) * total / nclusters > cc * total / nclusters; };
        const bool all_work = total >= nclusters;
        SegIter seg(sk, cluster, nclusters, ntiles, nkb);
        int64_t tile, kb0, kb1, ti = 0;
        for (; seg.next(tile, kb0, kb1); ++ti) {
            int64_t nt, mt;
            tile_coords(tile, n_t, n_m, BAND_ROWS / 512, nt, mt);
            if (!__all_sync(0xffffffffu, mbar_wait(acc_full, static_cast<uint32_t>(ti & 1)))) break;
            tc_fence_after();
            const bool active = h == 0 || mt * 512 + 256 < Rpad;
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(h ? C::TMEM_D1 : C::TMEM_D0);
            const int64_t tok0 = nt * bn;
            const int64_t nv = T - tok0 < bn ? T - tok0 : bn;       // real tokens of the tile
            const int nch = active ? static_cast<int>((nv + 31) / 32) : 0;
            if (kb0 > 0) {
                // later part of a split tile: hand the fp32 partial (real tokens
                // only) to the owner; the stores drain while the next segment runs
                float *slot = slots + static_cast<size_t>((cluster * 2 + rank) * 8 + we) * SK_SLOT_FLOATS;
#pragma unroll 1
                for (int c = 0; c < nch; ++c) {
                    const int64_t wv = nv - c * 32;  // real tokens from this chunk on
                    uint32_t v[32];
                    if (c < 7) {
                        tmem_ld_32x32b_x32(tbase + c * 32, v);
                    } else {
                        uint32_t v16[16];
                        tmem_ld_32x32b_x16(tbase + c * 32, v16);
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = v16[j];
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < wv && (c < 7 || j < 16))
                            __stcg(slot + (c * 32 + j) * 32 + lane, __uint_as_float(v[j]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty_cl);
                __threadfence();
                __syncwarp();
                if (lane == 0 && cluster != g_test_withhold_flag_cluster)
                    st_release_u64(flags + (cluster * 2 + rank) * 8 + we, seq);
                continue;
            }
            // bf16 out.  The cluster's last segment: every pipeline stage is idle
            // (its loads landed and its MMAs completed), so the accumulator's
            // 128 rows x bn tokens are staged there ([token][row]) and leave as
            // one TMA store of 256-byte rows.  Earlier tiles: straight from
            // registers, lane = weight row, one store per token (32 consecutive
            // rows = 64 contiguous bytes), overlapping the next tile's MMAs.
            const bool last = !seg.more();
            const int64_t yrow = mt * 512 + h * 256 + rank * 128 + q * 32 + lane;
            const bool rok = yrow < R;
            uint16_t *ycol = Y + yrow;
            uint16_t *stg = reinterpret_cast<uint16_t *>(smem) + h * (128 * C::BN_MAX) + q * 32 + lane;
            auto store_chunk = [&](int c, const uint32_t (&w)[16]) {
                if (last) {
                    uint16_t *sp = stg + c * 32 * 128;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (c * 32 + 2 * i >= bn) break;
                        sp[(2 * i) * 128] = static_cast<uint16_t>(w[i] & 0xFFFFu);
                        sp[(2 * i + 1) * 128] = static_cast<uint16_t>(w[i] >> 16);
                    }
                    return;
                }
                const int64_t left = T - (tok0 + c * 32);
                const int cap = c * 32 + 16 >= bn ? 16 : 32;
                const int nvt = left < cap ? static_cast<int>(left) : cap;  // tokens to write
                if (!rok) return;
                uint16_t *yp = ycol + (tok0 + c * 32) * ldy;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (2 * i < nvt) yp[0] = static_cast<uint16_t>(w[i] & 0xFFFFu);
                    if (2 * i + 1 < nvt) yp[ldy] = static_cast<uint16_t>(w[i] >> 16);
                    yp += 2 * ldy;
                }
            };
            // after the staged chunks: one TMA store per accumulator, issued by
            // its lane-quarter-0 warp once the 4 warps have written their rows
            auto flush_staged = [&]() {
                if (!last || !active) return;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&out_ready[h]);
                if (q == 0 && lane == 0 && mbar_wait(&out_ready[h], 0)) {
                    tma_store_2d(&tmY, reinterpret_cast<uint16_t *>(smem) + h * (128 * C::BN_MAX),
                                 static_cast<int32_t>(mt * 512 + h * 256 + rank * 128),
                                 static_cast<int32_t>(tok0));
                    bulk_commit_group();
                    bulk_wait_group0();
                }
            };
            if (sk && kb1 < nkb) {
                // owner of a split tile (always this cluster's last segment, so
                // the accumulator may stay busy): wait for the clusters after this
                // one that hold the rest of the tile (each lane polls one flag),
                // then add their partial sums in ascending cluster order
                int64_t last_contrib = cluster;
                while (last_contrib + 1 < nclusters &&
                       (last_contrib + 1) * total / nclusters < (tile + 1) * nkb)
                    ++last_contrib;
                bool got = true;
                for (int64_t base = cluster + 1; base <= last_contrib && got; base += 32) {
                    const int64_t cc = base + lane;
                    bool mine = true;
                    if (cc <= last_contrib && (all_work || has_work(cc)))
                        mine = sk_wait_flag(flags + (cc * 2 + rank) * 8 + we, seq);
                    got = __all_sync(0xffffffffu, mine);
                }
#pragma unroll 1
                for (int c = 0; c < nch; ++c) {
                    uint32_t v[32];
                    if (c < 7) {
                        tmem_ld_32x32b_x32(tbase + c * 32, v);
                    } else {
                        uint32_t v16[16];
                        tmem_ld_32x32b_x16(tbase + c * 32, v16);
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = v16[j];
#pragma unroll
                        for (int j = 16; j < 32; ++j) v[j] = 0;
                    }
                    tmem_ld_wait();
                    float f[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
                    // 16 columns at a time, partials of two clusters in flight
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int64_t wv = nv - c * 32 - hh * 16;  // real tokens from here on
                        if (wv <= 0 || (c == 7 && hh == 1)) break;
                        for (int64_t base = cluster + 1; base <= last_contrib; base += 2) {
                            float pv[2][16];
                            bool use[2];
#pragma unroll
                            for (int k = 0; k < 2; ++k) {
                                const int64_t cc = base + k;
                                use[k] = cc <= last_contrib && (all_work || has_work(cc));
                                const float *ps = slots + (static_cast<size_t>((cc * 2 + rank) * 8 + we) *
                                                               SK_SLOT_FLOATS +
                                                           (c * 32 + hh * 16) * 32 + lane);
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    pv[k][j] = (use[k] && j < wv) ? __ldcg(ps + j * 32) : 0.0f;
                            }
#pragma unroll
                            for (int k = 0; k < 2; ++k)
                                if (use[k]) {
#pragma unroll
                                    for (int j = 0; j < 16; ++j) f[hh * 16 + j] += pv[k][j];
                                }
                        }
                    }
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
                    store_chunk(c, w);
                }
                flush_staged();  // last segment: the accumulator is not released
                continue;
            }
            if (last) {
                // last tile: 64 columns per tensor-memory load, straight into
                // the staging buffer; nothing waits for the accumulator
#pragma unroll 1
                for (int c2 = 0; 2 * c2 < nch; ++c2) {
                    uint32_t v[64];
                    tmem_ld_32x32b_x64(tbase + c2 * 64, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        if (2 * c2 + j >= nch) break;
                        uint32_t w[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            w[i] = pack_bf16x2(__uint_as_float(v[32 * j + 2 * i]),
                                               __uint_as_float(v[32 * j + 2 * i + 1]));
                        store_chunk(2 * c2 + j, w);
                    }
                }
                flush_staged();
                continue;
            }
            // whole tile, in two halves of four chunks: tensor memory -> bf16
            // registers -> stores; the accumulator is released once the second
            // half is in registers, before its stores
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[4][16];
#pragma unroll
                for (int cc4 = 0; cc4 < 4; ++cc4) {
                    const int c = half * 4 + cc4;
                    if (c < nch) {
                        if (c < 7) {
                            uint32_t v[32];
                            tmem_ld_32x32b_x32(tbase + c * 32, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                pk[cc4][i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        } else {
                            uint32_t v[16];
                            tmem_ld_32x32b_x16(tbase + c * 32, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                pk[cc4][i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
#pragma unroll
                            for (int i = 8; i < 16; ++i) pk[cc4][i] = 0;
                        }
                    }
                }
                if (half == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_cl);
                }
#pragma unroll
                for (int cc4 = 0; cc4 < 4; ++cc4)
                    if (half * 4 + cc4 < nch) store_chunk(half * 4 + cc4, pk[cc4]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}


// ---------------------------------------------------------------------------
// 6:8 middle windows: X_mid[t, 4g + i] = X[t, 8g + 2 + i] (i < 4), zero past K.
// One thread per two groups and GATHER_TOKENS consecutive tokens: all 16-byte
// loads first (2 per token), then one 16-byte store per token.
// grid: x over pairs of groups, y (+65535 z) over token runs.
// ---------------------------------------------------------------------------
constexpr int GATHER_TOKENS = 4;

__global__ void __launch_bounds__(256)
    k_gather_mid(const uint16_t *__restrict__ X, int64_t T, int64_t K, int64_t ldx, int64_t G,
                 uint16_t *__restrict__ Xmid, int64_t ldm) {
    grid_dep_launch();
    const int64_t t0 = (blockIdx.y + static_cast<int64_t>(blockIdx.z) * 65535) * GATHER_TOKENS;
    const int64_t h = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // group pair
    if (t0 >= T || 2 * h >= G) return;
    const bool full_k = 16 * h + 16 <= K;
    uint32_t o[GATHER_TOKENS][4];
#pragma unroll
    for (int u = 0; u < GATHER_TOKENS; ++u) {
        const int64_t t = t0 + u;
        if (t >= T) break;
        const uint16_t *src = X + t * ldx + 16 * h;
        if (full_k) {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(src));
            const uint4 b = __ldg(reinterpret_cast<const uint4 *>(src) + 1);
            o[u][0] = a.y; o[u][1] = a.z; o[u][2] = b.y; o[u][3] = b.z;
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t c = 16 * h + 8 * (j >> 1) + 2 + 2 * (j & 1);
                const uint32_t lo = c < K ? __ldg(src + (c - 16 * h)) : 0u;
                const uint32_t hi = c + 1 < K ? __ldg(src + (c + 1 - 16 * h)) : 0u;
                o[u][j] = lo | (hi << 16);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < GATHER_TOKENS; ++u) {
        const int64_t t = t0 + u;
        if (t >= T) break;
        uint16_t *dst = Xmid + t * ldm + 8 * h;
        if (2 * h + 2 <= G) {
            *reinterpret_cast<uint4 *>(dst) = make_uint4(o[u][0], o[u][1], o[u][2], o[u][3]);
        } else {  // last, odd group: four columns only
            *reinterpret_cast<uint2 *>(dst) = make_uint2(o[u][0], o[u][1]);
        }
    }
}

}  // namespace nm

// ===========================================================================
// host side: tensor maps and the C ABI
// ===========================================================================
using namespace nm;

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (n[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

// one flag per kernel instantiation and device (kernels of different modes
// share a signature, so the cache is keyed on the kernel itself)

// ---- single-CTA kernel (ablation baseline)
constexpr int GEMM_BN = 128;

template <int MODE, int BN>
nm_status launch_gemm_1cta(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &y,
                           const uint8_t *meta, int64_t nkb, int m, int nwin, int64_t R,
                           int64_t T, cudaStream_t s) {
    using Cfg = GemmCfg<MODE, BN>;
    if (!set_smem_attr<k_gemm_1cta<MODE, BN>>(Cfg::SMEM_BYTES)) return NM_ERR_CUDA;
    const int64_t mt = (R + BM - 1) / BM, ntl = (T + BN - 1) / BN;
    if (mt > 0x7FFFFFFF || ntl > 65535) return NM_ERR_SHAPE;
    dim3 grid(static_cast<unsigned>(mt), static_cast<unsigned>(ntl));
    k_gemm_1cta<MODE, BN><<<grid, GEMM_THREADS, Cfg::SMEM_BYTES, s>>>(a, b, y, meta, nkb, m, nwin);
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

// ---- persistent CTA-pair kernel

// schedule override (0 = automatic, 1 = whole tiles, 2 = stream-K) and
// cluster count override (0 = as many as fit on the device at once)
std::atomic<int> g_sched_policy{0};
std::atomic<int> g_sched_clusters{0};

// launch sequence numbers: unique per launch in this process and, being
// seeded from the clock, unlikely to equal a stale flag left by another one
uint64_t next_seq() {
    static std::atomic<uint64_t> ctr{
        static_cast<uint64_t>(std::chrono::steady_clock::now().time_since_epoch().count()) | 1u};
    return ctr.fetch_add(1);
}

// clusters of two that can be resident at once (per mode and device)
template <int MODE>
int64_t resident_clusters() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sm_count() / 2;
    if (cache[dev] == 0) {
        using Cfg = PairCfg<MODE>;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * static_cast<unsigned>(sm_count() / 2), 1, 1);
        cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
        cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_gemm_pair<MODE>, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = sm_count() / 2;
        }
        cache[dev] = n < sm_count() / 2 ? n : sm_count() / 2;
    }
    return cache[dev];
}

template <int MODE>
nm_status launch_pair(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &b2,
                      const CUtensorMap &e, const CUtensorMap &y, const uint16_t *X, int64_t T,
                      int64_t K, int64_t ldx, int64_t R, int64_t nkb, int m, void *sk_ws,
                      size_t sk_ws_bytes, cudaStream_t s) {
    using Cfg = PairCfg<MODE>;
    if (!set_smem_attr<k_gemm_pair<MODE>>(Cfg::SMEM_BYTES)) return NM_ERR_CUDA;
    const int64_t ntiles = ((T + Cfg::BN - 1) / Cfg::BN) * ((R + 255) / 256);
    int64_t res = resident_clusters<MODE>();
    const int forced = g_sched_clusters.load();
    if (forced > 0 && forced < res) res = forced;
    if (res > SK_MAX_CLUSTERS) res = SK_MAX_CLUSTERS;
    if (res < 1) res = 1;
    // stream-K when the tiles fill less than half the pairs (decode-sized T):
    // measured on B200, splitting tiles of a fuller grid (one to two waves)
    // loses more to the partial-sum traffic and to the clusters working on
    // unrelated K' blocks at the same time than it gains on the last wave
    const int policy = g_sched_policy.load();
    const bool sk_ok = !Cfg::LIFT && sk_ws != nullptr && sk_ws_bytes >= sk_bytes(res) &&
                       (reinterpret_cast<uintptr_t>(sk_ws) & 15u) == 0;
    const bool sk = sk_ok && (policy == 2 || (policy == 0 && 2 * ntiles <= res));
    int64_t clusters = sk ? res : (ntiles < res ? ntiles : res);
    if (clusters < 1) clusters = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    uint8_t *skp = sk ? static_cast<uint8_t *>(sk_ws) : nullptr;
    const uint64_t seq = sk ? next_seq() : 0;
    if (cudaLaunchKernelEx(&cfg, k_gemm_pair<MODE>, a, b, b2, e, y, X, T, K, ldx, R, nkb, m, skp, seq,
                           sk ? 1 : 0) != cudaSuccess)
        return NM_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

// tokens per wide tile.  Candidates: the fewest tiles of at most 240 tokens
// and, when that is already several, one or two more, each as even as
// multiples of 16 allow; the one with the least (waves of tiles over the
// resident CTA pairs) x (tokens per tile + 32), the N/2 + 32 clocks a sparse
// MMA of N tokens costs per K' step, so that a last, nearly empty wave is
// traded for slightly narrower tiles.  (One tile's worth of tokens stays one
// tile: more would only re-read the weights.)
int64_t wide_bn(int64_t T, int64_t R, int64_t pairs) {
    const int64_t n_m = ((R + 255) / 256 * 256 + 511) / 512;
    const int64_t nt0 = (T + WideCfg::BN_MAX - 1) / WideCfg::BN_MAX;
    const int64_t nt_last = nt0 >= 2 ? nt0 + 2 : nt0;
    int64_t best = 0, best_cost = 0;
    for (int64_t nt = nt0; nt <= nt_last; ++nt) {
        const int64_t per = (T + nt - 1) / nt;
        const int64_t bn = (per + 15) / 16 * 16;
        const int64_t tiles = ((T + bn - 1) / bn) * n_m;
        const int64_t cost = ((tiles + pairs - 1) / pairs) * (bn + 32);
        if (best == 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
        if (per <= 16) break;
    }
    return best;
}

// CTA pairs of k_gemm_wide<MODE> that can be resident at once on the current
// device (0 on a CUDA error), cached per device
template <int MODE>
int64_t wide_pairs() {
    using Cfg = WideCfg;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] == 0) {
        if (!set_smem_attr<k_gemm_wide<MODE>>(Cfg::SMEM_BYTES)) return 0;
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(2 * static_cast<unsigned>(sm_count() / 2), 1, 1);
        q.blockDim = dim3(Cfg::THREADS, 1, 1);
        q.dynamicSmemBytes = Cfg::SMEM_BYTES;
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = 2;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        q.attrs = qa;
        q.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_gemm_wide<MODE>, &q) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = sm_count() / 2;
        }
        cache[dev] = n < sm_count() / 2 ? n : sm_count() / 2;
    }
    int64_t res = cache[dev];
    const int forced = g_sched_clusters.load();
    if (forced > 0 && forced < res) res = forced;
    if (res > SK_MAX_CLUSTERS) res = SK_MAX_CLUSTERS;
    return res < 1 ? 1 : res;
}

template <int MODE>
nm_status launch_wide(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &b2,
                      const CUtensorMap &e, const CUtensorMap &y, uint16_t *Y, int64_t ldy, int64_t T,
                      int64_t R, int64_t nkb, int bn, void *sk_ws, size_t sk_ws_bytes, cudaStream_t s) {
    using Cfg = WideCfg;
    if (!set_smem_attr<k_gemm_wide<MODE>>(Cfg::SMEM_BYTES)) return NM_ERR_CUDA;
    const int64_t Rpad = (R + 255) / 256 * 256;
    const int64_t ntiles = ((T + bn - 1) / bn) * ((Rpad + 511) / 512);
    const int64_t res = wide_pairs<MODE>();  // with a forced pair count applied
    if (res == 0) return NM_ERR_CUDA;
    const int forced = g_sched_clusters.load();
    const int policy = g_sched_policy.load();
    const bool sk_ok = sk_ws != nullptr && sk_ws_bytes >= sk_bytes(res) &&
                       (reinterpret_cast<uintptr_t>(sk_ws) & 15u) == 0;
    const bool sk = sk_ok && (policy == 2 || (policy == 0 && 2 * ntiles <= res));
    // stream-K: at most ~4 pairs per tile unless the pair count is forced --
    // each extra contributor costs the tile's owner another round of partial
    // reads, more than the shorter K' range saves once HBM is the limit
    int64_t clusters = ntiles < res ? ntiles : res;
    if (sk) clusters = (forced > 0 || 4 * ntiles >= res) ? res : 4 * ntiles;
    if (clusters < 1) clusters = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    uint8_t *skp = sk ? static_cast<uint8_t *>(sk_ws) : nullptr;
    const uint64_t seq = sk ? next_seq() : 0;
    if (cudaLaunchKernelEx(&cfg, k_gemm_wide<MODE>, a, b, b2, e, y, Y, ldy, T, R, nkb, bn, skp, seq,
                           sk ? 1 : 0) != cudaSuccess)
        return NM_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

}  // namespace

extern "C" size_t nm_sparse_prepare_bytes(int64_t R, int64_t K, int m) {
    if (R < 1 || K < 1 || (m != 4 && m != 6 && m != 8 && m != 10)) return 0;
    const PackedGeom p = packed_geom(R, K, m);
    return static_cast<size_t>(p.vals_bytes + p.meta_bytes);
}

namespace {

// a6 (and, from the mask, a4): the packed values, then the metadata blocks
nm_status launch_prepare(const uint16_t *vals, const uint8_t *wmeta, const uint32_t *mask, int64_t R,
                         int64_t K, int m, void *packed, cudaStream_t s) {
    const PackedGeom p = packed_geom(R, K, m);
    const int n = m - 2;
    if (m == 8) {
        const int64_t nj = p.nkb / 3;
        const int64_t rb = (p.Rpad + 7) / 8;
        dim3 g68(static_cast<unsigned>((nj + PV68_JW - 1) / PV68_JW), static_cast<unsigned>(rb < 65535 ? rb : 65535),
                 static_cast<unsigned>((rb + 65534) / 65535));
        k_prepare_vals68<<<g68, 256, 0, s>>>(vals, R, p.G, p.Rpad, nj, p.KLpad / 2,
                                             static_cast<uint16_t *>(packed));
    } else {
        const int64_t chunks = p.KLpad / 16;  // 16-byte chunks of a packed row
        const int64_t words = p.G * n / 2;
        const bool vec = (words % 4) == 0 && (reinterpret_cast<uintptr_t>(vals) & 15u) == 0;
        const int64_t rb = (p.Rpad + PV_ROWS - 1) / PV_ROWS;
        dim3 vgrid(static_cast<unsigned>((chunks + 255) / 256), static_cast<unsigned>(rb < 65535 ? rb : 65535),
                   static_cast<unsigned>((rb + 65534) / 65535));
        k_prepare_vals<<<vgrid, 256, 0, s>>>(vals, R, words, p.Rpad, p.KLpad / 2, vec,
                                             static_cast<uint16_t *>(packed));
    }
    const int64_t nblocks = (p.Rpad / BM) * p.nkb;
    if (nblocks > 0x7FFFFFFF) return NM_ERR_SHAPE;
    uint8_t *meta = static_cast<uint8_t *>(packed) + p.vals_bytes;
    const int64_t mwords = (p.G * m + 31) / 32;
    const int64_t ntiles = (p.Rpad / BM) * p.nkb;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;  // 8 resident blocks of 256 threads per SM
    const int64_t nruns = (ntiles + PM_TILES - 1) / PM_TILES;
    const unsigned nb = static_cast<unsigned>(nruns < cap ? nruns : cap);
    const int64_t wb = (p.nwin + 1) / 2;
    // a programmatic dependent of the values kernel: the two grids write
    // disjoint parts of the operand from independent inputs and overlap; the
    // metadata kernel waits for the values grid before it completes, so the
    // stream's next kernel sees the whole operand
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nb, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint8_t *wm = mask ? nullptr : wmeta;
    const int64_t wbm = mask ? 0 : wb, mwm = mask ? mwords : 0;
    cudaError_t e;
    if (m == 8 && mask) {  // the main 6:8 path: a K' block triple per thread block
        const int64_t ntrip = (p.Rpad / BM) * (p.nkb / 3);
        cfg.gridDim = dim3(static_cast<unsigned>(ntrip < cap ? ntrip : cap), 1, 1);
        e = cudaLaunchKernelEx(&cfg, k_prepare_meta68, mask, R, p.G, mwords, p.nkb, ntrip, meta);
        return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
    }
#define NM_PREP_META(MM)                                                                                \
    e = mask ? cudaLaunchKernelEx(&cfg, k_prepare_meta<MM, true>, wm, mask, R, p.G, wbm, mwm, p.nkb, ntiles, meta) \
             : cudaLaunchKernelEx(&cfg, k_prepare_meta<MM, false>, wm, mask, R, p.G, wbm, mwm, p.nkb, ntiles, meta)
    switch (m) {
        case 4: NM_PREP_META(4); break;
        case 6: NM_PREP_META(6); break;
        case 8: NM_PREP_META(8); break;
        default: NM_PREP_META(10); break;
    }
#undef NM_PREP_META
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? NM_OK : NM_ERR_CUDA;
}

nm_status check_prepare(const uint16_t *vals, const void *meta_src, int64_t R, int64_t K, int m,
                        const void *packed, size_t packed_bytes) {
    if (!vals || !meta_src || !packed) return NM_ERR_NULL;
    if (R < 1 || K < 1) return NM_ERR_SHAPE;
    if (m != 4 && m != 6 && m != 8 && m != 10) return NM_ERR_UNSUPPORTED;
    if (!aligned16(packed) || (reinterpret_cast<uintptr_t>(vals) & 3u)) return NM_ERR_ALIGN;
    const PackedGeom p = packed_geom(R, K, m);
    if (packed_bytes < static_cast<size_t>(p.vals_bytes + p.meta_bytes)) return NM_ERR_WORKSPACE;
    if (p.Rpad > 65535LL * 65535LL) return NM_ERR_SHAPE;
    return NM_OK;
}

}  // namespace

extern "C" nm_status nm_sparse_prepare(const uint16_t *vals, const uint8_t *wmeta, int64_t R,
                                       int64_t K, int m, void *packed, size_t packed_bytes,
                                       void *stream) {
    const nm_status st = check_prepare(vals, wmeta, R, K, m, packed, packed_bytes);
    if (st != NM_OK) return st;
    return launch_prepare(vals, wmeta, nullptr, R, K, m, packed, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" nm_status nm_sparse_prepare_from_mask(const uint16_t *vals, const uint32_t *mask, int64_t R,
                                                 int64_t K, int m, void *packed, size_t packed_bytes,
                                                 void *stream) {
    const nm_status st = check_prepare(vals, mask, R, K, m, packed, packed_bytes);
    if (st != NM_OK) return st;
    if (reinterpret_cast<uintptr_t>(mask) & 3u) return NM_ERR_ALIGN;
    return launch_prepare(vals, nullptr, mask, R, K, m, packed, reinterpret_cast<cudaStream_t>(stream));
}

// extra device memory the online phase needs for (2N-2):2N patterns: the
// gathered middle windows (6:8) or the lifted activations (4:6, 8:10)
struct GemmWs {
    int64_t ld;      // leading dimension (elements) of the staged activations
    int64_t cols;    // their logical width
    size_t bytes;
};

static GemmWs gemm_ws(int64_t T, int64_t K, int m) {
    GemmWs w{0, 0, 0};
    if (T < 1 || K < 1 || m == 4) return w;
    const int64_t G = (K + m - 1) / m;
    w.cols = m == 8 ? G * 4 : G * (m / 2 - 1) * 4;
    w.ld = (w.cols + 7) / 8 * 8;
    w.bytes = static_cast<size_t>(T) * static_cast<size_t>(w.ld) * 2;
    return w;
}

// the stream-K region follows the staged activations, 256-byte aligned
static size_t sk_offset(const GemmWs &w) { return (w.bytes + 255) / 256 * 256; }

extern "C" size_t nm_sparse_gemm_workspace_bytes(int64_t T, int64_t K, int m) {
    if (T < 1 || K < 1 || (m != 4 && m != 6 && m != 8 && m != 10)) return 0;
    return sk_offset(gemm_ws(T, K, m)) + sk_bytes(SK_MAX_CLUSTERS);
}

extern "C" size_t nm_dense_gemm_workspace_bytes(int64_t T, int64_t K, int64_t R) {
    if (T < 1 || K < 1 || R < 1) return 0;
    return sk_bytes(SK_MAX_CLUSTERS);
}

extern "C" nm_status nm_gemm_set_schedule(int policy, int clusters) {
    if (policy < 0 || policy > 2 || clusters < 0) return NM_ERR_SHAPE;
    g_sched_policy.store(policy);
    g_sched_clusters.store(clusters);
    return NM_OK;
}

namespace {

struct SparseMaps {
    CUtensorMap a, e, y;
    bool ok;
};

SparseMaps sparse_maps(const void *packed, const PackedGeom &p, const uint16_t *Y, int64_t T,
                       int64_t R, int64_t ldy) {
    SparseMaps mp;
    const uint8_t *meta = static_cast<const uint8_t *>(packed) + p.vals_bytes;
    mp.ok = make_tmap_bf16(&mp.a, packed, p.Rpad, p.KLpad / 2, p.KLpad / 2, 64, BM, true) &&
            make_tmap_2d(&mp.e, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, meta, (p.Rpad / BM) * p.nkb * 8,
                         256, 256, 256, 8, false) &&
            make_tmap_bf16(&mp.y, Y, T, R, ldy, 32, 32, false);
    return mp;
}

nm_status check_sparse_args(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, const void *packed,
                            int64_t R, int m, const uint16_t *Y, int64_t ldy) {
    if (!X || !packed || !Y) return NM_ERR_NULL;
    if (T < 1 || K < 1 || R < 1 || ldx < K || ldy < R) return NM_ERR_SHAPE;
    if (m != 4 && m != 6 && m != 8 && m != 10) return NM_ERR_UNSUPPORTED;
    if (!aligned16(X) || !aligned16(Y) || !aligned16(packed) || (ldx % 8) != 0 || (ldy % 8) != 0)
        return NM_ERR_ALIGN;
    const PackedGeom p = packed_geom(R, K, m);
    if (p.nkb > 0x7FFFFFFF / 8 || (p.Rpad / BM) * p.nkb * 8 > 0x7FFFFFFF) return NM_ERR_SHAPE;
    return NM_OK;
}

}  // namespace

namespace {

// the online phase: stage the activations (6:8 middle windows, or the lifted
// X' for 4:6 and 8:10), then the GEMM with the wide tile (library) or the
// 256 x 256 pair tile (ablation)
nm_status sparse_gemm_impl(const uint16_t *X, int64_t T, int64_t K, int64_t ldx, const void *packed,
                           int64_t R, int m, uint16_t *Y, int64_t ldy, void *ws, size_t ws_bytes,
                           void *stream, bool wide) {
    nm_status st = check_sparse_args(X, T, K, ldx, packed, R, m, Y, ldy);
    if (st != NM_OK) return st;
    const GemmWs w = gemm_ws(T, K, m);
    if (w.bytes > 0 && (!ws || ws_bytes < w.bytes)) return NM_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return NM_ERR_ALIGN;
    const PackedGeom p = packed_geom(R, K, m);
    const SparseMaps mp = sparse_maps(packed, p, Y, T, R, ldy);
    if (!mp.ok) return NM_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // stream-K partial sums, when the caller's workspace has room for them
    const size_t sko = sk_offset(w);
    void *skw = ws && ws_bytes > sko ? static_cast<uint8_t *>(ws) + sko : nullptr;
    const size_t skb = skw ? ws_bytes - sko : 0;
    uint16_t *stage = static_cast<uint16_t *>(ws);
    // B operand(s): X itself (2:4, and the raw blocks of 6:8), X_mid (6:8), X' (4:6, 8:10)
    const uint16_t *b_src = X;
    int64_t b_cols = K, b_ld = ldx;
    if (m == 8) {
        const int64_t pairs = (p.G + 1) / 2;
        const int64_t runs = (T + GATHER_TOKENS - 1) / GATHER_TOKENS;
        dim3 grid(static_cast<unsigned>((pairs + 255) / 256), static_cast<unsigned>(runs < 65535 ? runs : 65535),
                  static_cast<unsigned>((runs + 65534) / 65535));
        k_gather_mid<<<grid, 256, 0, s>>>(X, T, K, ldx, p.G, stage, w.ld);
        if (cudaGetLastError() != cudaSuccess) return NM_ERR_CUDA;
    } else if (m != 4) {
        st = lift_activations(X, T, K, ldx, m, stage, w.ld, stream);
        if (st != NM_OK) return st;
        b_src = stage;
        b_cols = w.cols;
        b_ld = w.ld;
    }
    int bh = 128;
    if (wide) {
        const int64_t pairs = m == 8 ? wide_pairs<PMODE_SP68T>() : wide_pairs<PMODE_SP24>();
        if (pairs == 0) return NM_ERR_CUDA;
        bh = static_cast<int>(wide_bn(T, R, pairs) / 2);
    }
    CUtensorMap tb, tb2;
    if (!make_tmap_bf16(&tb, b_src, T, b_cols, b_ld, 64, static_cast<uint32_t>(bh), true)) return NM_ERR_CUDA;
    if (m == 8 && !make_tmap_bf16(&tb2, stage, T, w.cols, w.ld, 64, static_cast<uint32_t>(bh), true))
        return NM_ERR_CUDA;
    const CUtensorMap &b2 = m == 8 ? tb2 : tb;
    if (wide) {
        // output tile of one accumulator: 128 weight rows x bn tokens
        CUtensorMap ty;
        if (!make_tmap_bf16(&ty, Y, T, R, ldy, 128, static_cast<uint32_t>(2 * bh), false)) return NM_ERR_CUDA;
        if (m == 8)
            return launch_wide<PMODE_SP68T>(mp.a, tb, b2, mp.e, ty, Y, ldy, T, R, p.nkb, 2 * bh, skw, skb, s);
        return launch_wide<PMODE_SP24>(mp.a, tb, b2, mp.e, ty, Y, ldy, T, R, p.nkb, 2 * bh, skw, skb, s);
    }
    if (m == 8)
        return launch_pair<PMODE_SP68T>(mp.a, tb, b2, mp.e, mp.y, X, T, K, ldx, R, p.nkb, m, skw, skb, s);
    return launch_pair<PMODE_SP24>(mp.a, tb, b2, mp.e, mp.y, b_src, T, b_cols, b_ld, R, p.nkb, 4, skw,
                                   skb, s);
}

}  // namespace

extern "C" nm_status nm_sparse_gemm(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                    const void *packed, int64_t R, int m, uint16_t *Y, int64_t ldy,
                                    void *ws, size_t ws_bytes, void *stream) {
    return sparse_gemm_impl(X, T, K, ldx, packed, R, m, Y, ldy, ws, ws_bytes, stream, true);
}

extern "C" nm_status nm_sparse_gemm_tile256(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                            const void *packed, int64_t R, int m, uint16_t *Y,
                                            int64_t ldy, void *ws, size_t ws_bytes, void *stream) {
    return sparse_gemm_impl(X, T, K, ldx, packed, R, m, Y, ldy, ws, ws_bytes, stream, false);
}

extern "C" nm_status nm_sparse_gemm_fused(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                          const void *packed, int64_t R, int m, uint16_t *Y,
                                          int64_t ldy, void *stream) {
    nm_status st = check_sparse_args(X, T, K, ldx, packed, R, m, Y, ldy);
    if (st != NM_OK) return st;
    const PackedGeom p = packed_geom(R, K, m);
    const SparseMaps mp = sparse_maps(packed, p, Y, T, R, ldy);
    CUtensorMap tb;
    if (!mp.ok || !make_tmap_bf16(&tb, X, T, K, ldx, 64, 128, true)) return NM_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (m == 4)
        return launch_pair<PMODE_SP24>(mp.a, tb, tb, mp.e, mp.y, X, T, K, ldx, R, p.nkb, m, nullptr, 0, s);
    if (m == 8)
        return launch_pair<PMODE_SP68>(mp.a, tb, tb, mp.e, mp.y, X, T, K, ldx, R, p.nkb, m, nullptr, 0, s);
    return launch_pair<PMODE_SPLIFT>(mp.a, tb, tb, mp.e, mp.y, X, T, K, ldx, R, p.nkb, m, nullptr, 0, s);
}

extern "C" nm_status nm_dense_gemm(const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                   const uint16_t *W, int64_t R, int64_t ldw, uint16_t *Y,
                                   int64_t ldy, void *ws, size_t ws_bytes, void *stream) {
    if (!X || !W || !Y) return NM_ERR_NULL;
    if (T < 1 || K < 1 || R < 1 || ldx < K || ldw < K || ldy < R) return NM_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(W) || !aligned16(Y) || (ldx % 8) != 0 || (ldw % 8) != 0 ||
        (ldy % 8) != 0 || (ws && !aligned16(ws)))
        return NM_ERR_ALIGN;
    CUtensorMap ta, tb, ty;
    if (!make_tmap_bf16(&ta, W, R, K, ldw, 64, BM, true) ||
        !make_tmap_bf16(&tb, X, T, K, ldx, 64, 128, true) ||
        !make_tmap_bf16(&ty, Y, T, R, ldy, 32, 32, false))
        return NM_ERR_CUDA;
    const int64_t nkb = (K + 63) / 64;
    return launch_pair<PMODE_DENSE>(ta, tb, tb, ta, ty, X, T, K, ldx, R, nkb, 4, ws, ws ? ws_bytes : 0,
                                    reinterpret_cast<cudaStream_t>(stream));
}

extern "C" nm_status nm_gemm_1cta(int sparse, const uint16_t *X, int64_t T, int64_t K, int64_t ldx,
                                  const void *W_or_packed, int64_t R, int64_t ldw, uint16_t *Y,
                                  int64_t ldy, void *stream) {
    if (!X || !W_or_packed || !Y) return NM_ERR_NULL;
    if (T < 1 || K < 1 || R < 1 || ldx < K || ldy < R || (!sparse && ldw < K)) return NM_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(Y) || !aligned16(W_or_packed) || (ldx % 8) != 0 ||
        (ldy % 8) != 0 || (!sparse && (ldw % 8) != 0))
        return NM_ERR_ALIGN;
    CUtensorMap ta, tb, ty;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!make_tmap_bf16(&ty, Y, T, R, ldy, 32, GEMM_BN, false) ||
        !make_tmap_bf16(&tb, X, T, K, ldx, 64, GEMM_BN, true))
        return NM_ERR_CUDA;
    if (sparse) {
        const PackedGeom p = packed_geom(R, K, 4);
        if (!make_tmap_bf16(&ta, W_or_packed, p.Rpad, p.KLpad / 2, p.KLpad / 2, 64, BM, true))
            return NM_ERR_CUDA;
        const uint8_t *meta = static_cast<const uint8_t *>(W_or_packed) + p.vals_bytes;
        return launch_gemm_1cta<MODE_SP24, GEMM_BN>(ta, tb, ty, meta, p.nkb, 4, 1, R, T, s);
    }
    if (!make_tmap_bf16(&ta, W_or_packed, R, K, ldw, 64, BM, true)) return NM_ERR_CUDA;
    return launch_gemm_1cta<MODE_DENSE, GEMM_BN>(ta, tb, ty, nullptr, (K + 63) / 64, 4, 1, R, T, s);
}
