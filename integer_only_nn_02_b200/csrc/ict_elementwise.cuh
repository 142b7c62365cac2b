// ict_elementwise.cuh -- memory-bound kernels of the (C,e) training path:
//   requant (FIT of integer values into row-local groups),
//   ALIGN_MAX of an operand along its contracted index (optionally transposed),
//   the integer GELU stand-in (forward and backward),
//   the integer SGD-with-momentum update with per-group velocity.
// Source: "Memory-Efficient Integer-Only Training of Deep Neural Networks",
// Abstract (five integer building blocks), Figure 1b (integer SGD with momentum and
// per-group velocity), Table 6 (Product / Sum), Table 7 (pointwise activations keep
// the exponent).
#pragma once

#include "ict_device.cuh"

#include <type_traits>

namespace ict {

// ------------------------------------------------------------------ two-term sums

// a * 2^pa + b * 2^pb as one integer x at exponent r (the Sum primitive, Table 6).
// Exact while the exponents are at most 32 apart (|a|, |b| < 2^16, so x < 2^48).
// Beyond that the smaller term becomes a one-unit sticky below the larger one; the
// requantised result is unchanged because the group exponent is at least pa - 7 and
// both the true small term (< 2^(pa-16)) and the sticky (2^(pa-32)) sit strictly
// inside the same gap between consecutive multiples of 2^(pa-8) next to a * 2^pa.
struct TwoTerm {
    int64_t x;
    int r;
};
__device__ __forceinline__ TwoTerm two_term(int64_t a, int pa, int64_t b, int pb) {
    if (a == 0) return TwoTerm{b, pb};
    if (b == 0) return TwoTerm{a, pa};
    if (pa < pb) {
        int64_t t = a; a = b; b = t;
        int tp = pa; pa = pb; pb = tp;
    }
    const int d = pa - pb;
    if (d <= 32) return TwoTerm{a * (1ll << d) + b, pb};
    return TwoTerm{a * (1ll << 32) + (b > 0 ? 1 : -1), pa - 32};
}
__device__ __forceinline__ int need64(int64_t x, int r) {
    return x == 0 ? kNoExp : r + need_off64((uint64_t)(x < 0 ? -x : x));
}
// the same for B-bit mantissas (q_max = 2^(B-1) - 1)
__device__ __forceinline__ int need64q(int64_t x, int r, int bits) {
    return x == 0 ? kNoExp : r + need_off64q((uint64_t)(x < 0 ? -x : x), bits);
}

template <int L>
__device__ __forceinline__ int group_max(int v, unsigned mask) {
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(mask, v, o));
    return v;
}

// RNE(x * 2^-S) for a group-uniform S with |x| < 2^30 (S < 0: exact left shift).
struct Shift {
    int ls, rs, bias, om;
};
__device__ __forceinline__ Shift make_shift(int S) {
    Shift h;
    h.ls = S < 0 ? -S : 0;
    h.rs = S > 0 ? min(S, 31) : 0;
    h.bias = h.rs ? (1 << (h.rs - 1)) - 1 : 0;
    h.om = h.rs ? 1 : 0;
    return h;
}
__device__ __forceinline__ int apply_shift(int x, const Shift &h) {
    x <<= h.ls;
    return (x + h.bias + ((x >> h.rs) & h.om)) >> h.rs;
}

// Exact FIT of the group values a_mul * A_i * 2^pa + b_mul * B_i * 2^pb element by element
// in int64 (two_term: exact up to a 32-bit exponent gap, sticky beyond), for groups whose
// values do not fit the int32 fast path.  Kept out of line: it is rare and register-hungry.
// ------------------------------------------------------------------ requant (FIT)

// FIT of int32 (optionally the int64 sum of `nsplit` int32 slices) or int64 values
// into row-local groups (1, G).  One warp per group; element (i, j) has exponent
// base + row_exp[i] + col_exp[j].
struct RequantArgs {
    const int32_t *v32;
    const int64_t *v64;
    int nsplit;
    int64_t split_stride;
    int64_t rows, cols, ld;  // value (i, j) at v[i * ld + j * cs] (cs = 1 unless transposed)
    int64_t cs;
    int32_t base;
    const int8_t *row_exp;  // exponent of row i: row_exp[i / row_div] (NULL = 0)
    int row_div;
    const int8_t *col_exp;  // exponent of column j: col_exp[j / col_div] (NULL = 0)
    int col_div;
    int8_t *out;
    int64_t out_ld;
    int8_t *out_exp;
    int G;
    int64_t ngc;  // groups per row
    int qb;       // mantissa bits B of the FIT (|C| <= 2^(B-1) - 1)
};

__device__ __forceinline__ int64_t rq_value(const RequantArgs &a, int64_t i, int64_t j) {
    const int64_t at = i * a.ld + j * a.cs;
    if (a.v64) return a.v64[at];
    int64_t s = 0;
    for (int k = 0; k < a.nsplit; ++k) s += a.v32[k * a.split_stride + at];
    return s;
}

__global__ void __launch_bounds__(256) requant_rows_kernel(RequantArgs a) {
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw >= a.rows * a.ngc) return;
    const int64_t i = idiv(gw, a.ngc), g = gw - i * a.ngc;
    const int64_t j0 = g * a.G, j1 = min(a.cols, j0 + a.G);
    const int re = a.base + (a.row_exp ? a.row_exp[idiv(i, a.row_div)] : 0);
    int emax = kNoExp;
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const int64_t x = rq_value(a, i, j);
        if (x) emax = max(emax, need64q(x, re + (a.col_exp ? a.col_exp[idiv(j, a.col_div)] : 0), a.qb));
    }
    const int e = finalize_exp(warp_max(emax));
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const int64_t x = rq_value(a, i, j);
        a.out[i * a.out_ld + j] = (int8_t)requant64(x, re + (a.col_exp ? a.col_exp[idiv(j, a.col_div)] : 0), e);
    }
    if (lane == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// ------------------------------------------------------------------ ALIGN_MAX

struct AlignArgs {
    const int8_t *in;
    const int8_t *in_exp;
    int64_t rows, cols, ld;
    int g_rows, g_cols;
    int64_t ngc;
    int axis;  // 1: per-row e*, 0: per-column e*
    int8_t *out;
    int64_t out_ld;
    int8_t *e_star;           // [rows] (axis 1) or [cols] (axis 0)
    const int32_t *col_max;   // axis 0 with scratch: max per group column (<= kNoExp: none)
    int row_estar;            // axis 1: the alignment kernel computes and stores e* itself
    int col_scan;             // axis 0, transposed: each block finds its columns' e* itself
    int gv_shift1;            // log2(g_cols / 16) + 1 when that is a power of two, 32 for one
                              // group across the row, 0: the group of a vector is a division
};

__device__ __forceinline__ int estar_of(int m) { return m <= kNoExp ? kEZero : m; }

// e* per row: max over the row's group exponents, E_ZERO groups ignored.
__global__ void estar_rows_kernel(AlignArgs a) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.rows) return;
    const int8_t *e = a.in_exp + (i / a.g_rows) * a.ngc;
    int m = kNoExp;
    for (int64_t g = 0; g < a.ngc; ++g)
        if (e[g] != kEZero) m = max(m, (int)e[g]);
    a.e_star[i] = (int8_t)estar_of(m);
}

// e* per column without scratch: one block per group column, max over all group rows.
__global__ void __launch_bounds__(256) estar_cols_kernel(AlignArgs a) {
    const int64_t gj = blockIdx.x;
    const int64_t ngr = (a.rows + a.g_rows - 1) / a.g_rows;
    int m = kNoExp;
    for (int64_t gi = threadIdx.x; gi < ngr; gi += blockDim.x) {
        const int e = a.in_exp[gi * a.ngc + gj];
        if (e != kEZero) m = max(m, e);
    }
    m = warp_max(m);
    __shared__ int red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        int v = threadIdx.x < 8 ? red[threadIdx.x] : kNoExp;
        v = warp_max(v);
        const int8_t es = (int8_t)estar_of(v);
        const int64_t j1 = min(a.cols, (gj + 1) * a.g_cols);
        for (int64_t j = gj * a.g_cols + threadIdx.x; j < j1; j += 32) a.e_star[j] = es;
    }
}

// e* per column with an int32 scratch (pre-set to 0x80808080): each block reduces a band
// of group rows into a shared maximum per group column, then one atomicMax per group
// column in global memory.
// Up to two alignment jobs per launch (blockIdx.y or blockIdx.z selects the job), so that
// both operands of a contraction are prepared by one launch of each kernel.
struct AlignPair {
    AlignArgs a[2];
    int32_t *cm[2];
    int64_t used[2];
    int tiles0, tiles1;  // transposing kernels: 128 x 128 tiles of job 0 and of job 1
    int ntc[2];          // and tile columns of each job
};

__global__ void __launch_bounds__(256) estar_cols_scratch_kernel(const __grid_constant__ AlignPair P) {
    const AlignArgs &a = P.a[blockIdx.y];
    int32_t *const col_max = P.cm[blockIdx.y];
    extern __shared__ int sm[];  // [ngc]
    for (int64_t g = threadIdx.x; g < a.ngc; g += blockDim.x) sm[g] = kNoExp;
    __syncthreads();
    // a band of group rows per block
    const int64_t ngr = (a.rows + a.g_rows - 1) / a.g_rows, ngc = a.ngc;
    const int64_t band = (ngr + gridDim.x - 1) / gridDim.x, r0 = (int64_t)blockIdx.x * band;
    const int64_t r1 = min(ngr, r0 + band);
    const int W = (int)(ngc >> 2);
    if (r0 < r1 && (ngc & 3) == 0 && W <= 256 && (reinterpret_cast<uintptr_t>(a.in_exp) & 3) == 0) {
        // 4-byte words: thread (r, w) of the block takes word w of rows r0 + r, + per, ...
        // keeping four byte-wise signed maxima.  E_ZERO (-128) is the smallest byte, so it
        // only survives where every member is E_ZERO, and is dropped below.
        const int per = 256 / W, w = (int)threadIdx.x % W, rr = (int)threadIdx.x / W;
        if (rr < per) {
            const uint32_t *e = reinterpret_cast<const uint32_t *>(a.in_exp);
            uint32_t m = 0x80808080u;
            int64_t r = r0 + rr;
            for (; r + 3 * per < r1; r += 4 * per) {  // four loads in flight
                const uint32_t x0 = e[r * W + w], x1 = e[(r + per) * W + w];
                const uint32_t x2 = e[(r + 2 * per) * W + w], x3 = e[(r + 3 * per) * W + w];
                m = __vmaxs4(__vmaxs4(m, x0), __vmaxs4(x1, __vmaxs4(x2, x3)));
            }
            for (; r < r1; r += per) m = __vmaxs4(m, e[r * W + w]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int v = (int)(int8_t)(m >> (8 * q));
                if (v != kEZero) atomicMax(&sm[4 * w + q], v);
            }
        }
    } else if (r0 < r1) {
        for (int64_t idx = r0 * ngc + threadIdx.x; idx < r1 * ngc; idx += blockDim.x) {
            const int e = a.in_exp[idx];
            if (e != kEZero) atomicMax(&sm[idx % ngc], e);
        }
    }
    __syncthreads();
    for (int64_t g = threadIdx.x; g < a.ngc; g += blockDim.x)
        if (sm[g] > kNoExp) atomicMax(&col_max[g], sm[g]);
}

// RNE(C / 2^d) of 16 signed int8 mantissas (|C| <= 127), d >= 0; d >= 8 gives 0.  One
// half-precision FMA rounds two bytes at once:
//   h = 1024 + (C + 128)                     (fp16 bits 0x64uu, uu = C ^ 0x80)
//   h * 2^-d + (1536 - 2^(10-d) - 2^(7-d)) = 1536 + C * 2^-d
// The three operands are exact in fp16 and the fused multiply-add rounds once.  Its
// result lies in [1024, 2048), where fp16 integers are spaced by 1, so the rounding is
// to the nearest integer with ties to even, and the low byte of the result's bits
// (1536 is 0x6600) is RNE(C / 2^d) in two's complement; d = 0 is exact (1536 + C).  Per
// four bytes: one XOR, two byte permutes to build the halves, two f16x2 FMAs, one
// permute to pack, and no branches, so lanes with different shifts stay together.
__device__ __forceinline__ uint32_t fma_f16x2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}
// The FMA's two constants for a shift d in [0, 7], and for index 8 (a shift of 8 or
// more, or a zero group): multiplier 0 and addend 1536, which leaves every byte 0.
struct RneK {
    uint32_t sc, k;  // 2^-d and 1536 - 2^(10-d) - 2^(7-d) in both fp16 halves
};
__device__ __forceinline__ RneK rne_consts(int d) {
    if (d >= 8) return RneK{0u, 0x66006600u};
    const uint32_t kk = 1536u - (1024u >> d) - (128u >> d);  // an integer in [384, 1527]
    const uint32_t kb = kk >= 1024u ? kk + 0x6000u : (kk >= 512u ? 2u * kk + 0x5C00u : 4u * kk + 0x5800u);
    return RneK{(uint32_t)(15 - d) * 0x04000400u, kb * 0x10001u};
}
// Kernels that round many vectors keep the nine constant pairs in shared memory.
__device__ __forceinline__ void rne_table_init(RneK *t) {
    if (threadIdx.x < 9) t[threadIdx.x] = rne_consts(threadIdx.x);
}
// Table index of a vector with group exponent eg aligned to es: the shift, 8 for 8 or
// more and for a zero group.  A target below eg (never asked for) also maps to 8.
__device__ __forceinline__ int rne_index(int es, int eg) {
    return eg == kEZero ? 8 : (int)min((unsigned)(es - eg), 8u);
}
__device__ __forceinline__ uint4 rne_shift16_k(uint4 raw, RneK c) {
    const uint32_t src[4] = {raw.x ^ 0x80808080u, raw.y ^ 0x80808080u, raw.z ^ 0x80808080u, raw.w ^ 0x80808080u};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t lo = fma_f16x2(__byte_perm(src[q], 0x64646464u, 0x4140), c.sc, c.k);  // bytes 0, 1
        const uint32_t hi = fma_f16x2(__byte_perm(src[q], 0x64646464u, 0x4342), c.sc, c.k);  // bytes 2, 3
        o[q] = __byte_perm(lo, hi, 0x6420);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ uint4 rne_shift16(uint4 raw, int d) { return rne_shift16_k(raw, rne_consts(d)); }

// Target exponent of the 16-byte vector at column j of row i (axis 1: per row; axis 0:
// per column, from the column-max scratch or the e* vector).
__device__ __forceinline__ int align_target(const AlignArgs &a, int64_t i, int64_t j) {
    if (a.axis == 1) return i < a.rows ? a.e_star[i] : kEZero;
    if (a.col_max) return estar_of(a.col_max[idiv(j, a.g_cols)]);
    return a.e_star[j];
}

// Aligned mantissas in place of layout (cols a multiple of 16; g_cols a multiple of 16
// or spanning all columns; rows below 2^31).  Each row is taken by a segment of L lanes
// of a warp; lane lr holds the row's 16-byte vectors lr, lr + L, ..., NV of them, which
// covers the row.  The blocks are persistent: a segment walks rows i, i + S, ... (S
// segments in the grid) with two register buffers in turn, issuing every load of its
// next row before it rounds and stores the current one, so that each SM keeps a row per
// segment in flight.  With axis 1 and no given e*, the segment reduces the row's group
// exponents (at most 2 L of them) to e* and its lane 0 stores it.  An E_ZERO exponent
// (-128, the smallest byte) can take part in the max unchanged: it only wins when every
// group is zero, and then e* is E_ZERO as well.
template <int NV>
struct RowBatch {
    uint4 raw[NV];
    int eg[NV];
    int ep;  // axis 1: max of this lane's share of the row's group exponents, or the given e*
};

// EXACT: axis 1, one group row per row, g_cols / 16 a power of two and rows of exactly
// L NV vectors, which drops every per-vector guard and division.
template <int L, int NV, bool EXACT>
__device__ __forceinline__ void align_row_load(const AlignArgs &a, int i, int gsh, bool row_e, RowBatch<NV> &b) {
    const int lr = threadIdx.x % L;
    const int8_t *erow = a.in_exp + (EXACT ? (int64_t)i : idiv(i, a.g_rows)) * a.ngc;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.in + (int64_t)i * a.ld);
#pragma unroll
    for (int t = 0; t < NV; ++t) {
        const int v = lr + L * t;
        if (EXACT || v < (int)(a.cols >> 4)) {
            b.raw[t] = src[v];
            b.eg[t] = erow[EXACT || gsh >= 0 ? (v >> gsh) : (int)idiv(16 * (int64_t)v, a.g_cols)];
        }
    }
    if (row_e) {
        const int ngc = (int)a.ngc;
        b.ep = max(lr < ngc ? (int)erow[lr] : kEZero, lr + L < ngc ? (int)erow[lr + L] : kEZero);
    } else if (EXACT || a.axis == 1) {
        b.ep = a.e_star[i];
    }
}

template <int L, int NV, bool EXACT>
__device__ __forceinline__ void align_row_store(const AlignArgs &a, int i, unsigned seg, bool row_e,
                                                const RneK *tk, const RowBatch<NV> &b) {
    const int lr = threadIdx.x % L;
    int es = b.ep;
    if (row_e) {
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) es = max(es, __shfl_xor_sync(seg, es, o));
        if (lr == 0) a.e_star[i] = (int8_t)es;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(a.out + (int64_t)i * a.out_ld);
#pragma unroll
    for (int t = 0; t < NV; ++t) {
        const int v = lr + L * t;
        if (!EXACT && v >= (int)(a.cols >> 4)) break;
        int et = es;
        if (!EXACT && a.axis == 0) {
            et = align_target(a, i, 16 * (int64_t)v);
            if (a.col_max && i == 0)
                for (int q = 0; q < 16; ++q) a.e_star[16 * v + q] = (int8_t)et;
        }
        dst[v] = rne_shift16_k(b.raw[t], tk[rne_index(et, b.eg[t])]);
    }
}

template <int L, int NV, bool EXACT>
__global__ void __launch_bounds__(256, 2) align_rows_kernel(const __grid_constant__ AlignArgs a) {
    constexpr int kSegs = 256 / L;
    __shared__ RneK tk[9];
    rne_table_init(tk);
    __syncthreads();
    const int rows = (int)a.rows, S = (int)gridDim.x * kSegs;
    int i = (int)blockIdx.x * kSegs + (int)threadIdx.x / L;
    if (i >= rows) return;  // whole segments leave together
    const unsigned seg = (0xffffffffu >> (32 - L)) << ((threadIdx.x & 31) & ~(L - 1));
    const bool row_e = a.axis == 1 && a.row_estar;
    const int gsh = a.gv_shift1 - 1;
    RowBatch<NV> ba, bb;
    align_row_load<L, NV, EXACT>(a, i, gsh, row_e, ba);
    while (true) {  // two rows per trip, one buffer each: no register copies
        if (i + S < rows) align_row_load<L, NV, EXACT>(a, i + S, gsh, row_e, bb);
        align_row_store<L, NV, EXACT>(a, i, seg, row_e, tk, ba);
        if ((i += S) >= rows) break;
        if (i + S < rows) align_row_load<L, NV, EXACT>(a, i + S, gsh, row_e, ba);
        align_row_store<L, NV, EXACT>(a, i, seg, row_e, tk, bb);
        if ((i += S) >= rows) break;
    }
}

// Rows of at most four 16-byte vectors and (computing e*) at most four groups, such as the
// 64-channel pixel rows of a convolution, along the rows: one thread per row, every vector
// and group exponent of the row loaded at once (64 bytes in flight per thread); the row's
// e* is the largest of its group exponents (E_ZERO, the smallest byte, only when every
// group is zero).
__global__ void __launch_bounds__(256) align_rows_thin_kernel(const __grid_constant__ AlignArgs a) {
    __shared__ RneK tk[9];
    rne_table_init(tk);
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int nv = (int)(a.cols >> 4);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.rows; i += stride) {
        const int8_t *e = a.in_exp + idiv(i, a.g_rows) * a.ngc;
        uint4 raw[4];
        int eg[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            if (v < nv) {
                raw[v] = *reinterpret_cast<const uint4 *>(a.in + i * a.ld + 16 * v);
                eg[v] = e[idiv(16 * v, a.g_cols)];
            }
        }
        int es;
        if (a.row_estar) {
            es = kEZero;
            for (int g = 0; g < (int)a.ngc; ++g) es = max(es, (int)e[g]);
            a.e_star[i] = (int8_t)es;
        } else {
            es = a.e_star[i];
        }
#pragma unroll
        for (int v = 0; v < 4; ++v)
            if (v < nv)
                *reinterpret_cast<uint4 *>(a.out + i * a.out_ld + 16 * v) = rne_shift16_k(raw[v], tk[rne_index(es, eg[v])]);
    }
}

// The same for rows too wide for one batch per lane or with many groups: 64 x 256
// tiles, four threads per row with four 16-byte vectors each (columns j, j + 64,
// j + 128, j + 192), loaded before the row's target is known; with axis 1 and no given
// e*, the four threads of a row reduce a quarter of its group exponents each.
__global__ void __launch_bounds__(256) align_rows_wide_kernel(const __grid_constant__ AlignArgs a) {
    __shared__ RneK tk[9];
    rne_table_init(tk);
    __syncthreads();
    const int64_t i = (int64_t)blockIdx.y * 64 + (threadIdx.x >> 2);
    const int64_t j0 = (int64_t)blockIdx.x * 256 + (threadIdx.x & 3) * 16;
    if (i >= a.rows) return;  // whole 4-thread row groups leave together
    uint4 raw[4];
    int eg[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {  // the loads first
        const int64_t j = j0 + 64 * v;
        if (j < a.cols) {
            raw[v] = *reinterpret_cast<const uint4 *>(a.in + i * a.ld + j);
            eg[v] = a.in_exp[idiv(i, a.g_rows) * a.ngc + idiv(j, a.g_cols)];
        }
    }
    int es_row = 0;
    const bool row_e = a.axis == 1 && a.row_estar;
    if (row_e) {
        const int8_t *e = a.in_exp + idiv(i, a.g_rows) * a.ngc;
        int m = kEZero;
        for (int64_t g = threadIdx.x & 3; g < a.ngc; g += 4) m = max(m, (int)e[g]);
        const unsigned quad = 0xfu << (threadIdx.x & 28);
        m = max(m, __shfl_xor_sync(quad, m, 1));
        es_row = max(m, __shfl_xor_sync(quad, m, 2));
        if (blockIdx.x == 0 && (threadIdx.x & 3) == 0) a.e_star[i] = (int8_t)es_row;
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const int64_t j = j0 + 64 * v;
        if (j >= a.cols) continue;
        const int es = row_e ? es_row : align_target(a, i, j);
        if (a.axis == 0 && a.col_max && i == 0)
            for (int q = 0; q < 16; ++q) a.e_star[j + q] = (int8_t)es;
        *reinterpret_cast<uint4 *>(a.out + i * a.out_ld + j) = rne_shift16_k(raw[v], tk[rne_index(es, eg[v])]);
    }
}

// Aligned and transposed, 128 x 128 tiles (rows and cols are multiples of 16).  The
// grid is one-dimensional over the tiles of both jobs (job 0's first, P.tiles0 of
// them; P.ntc[z] tile columns per tile row).  Thread (warp w, lane l) aligns rows
// 16 w + 4 (l & 3) .. + 3 at columns 16 (l >> 2) .. + 15, transposes the 4 x 4 byte
// blocks in registers (8 byte permutes per 16 bytes) and stores 32-bit words into a
// shared tile whose 16-byte chunks are XOR-swizzled by the output row's 16-row band, so
// that both the word stores and the 16-byte reads that feed the coalesced global
// stores are free of bank conflicts.
__global__ void __launch_bounds__(256) align_transpose_kernel(const __grid_constant__ AlignPair P) {
    const int z = (int)blockIdx.x >= P.tiles0 ? 1 : 0;
    const AlignArgs &a = P.a[z];
    const int tile_id = (int)blockIdx.x - (z ? P.tiles0 : 0);
    const int tr = tile_id / P.ntc[z], tcol = tile_id - tr * P.ntc[z];
    __shared__ uint4 tile[128][8];  // [output row = input column][16-byte chunk, swizzled]
    __shared__ RneK tk[9];
    __shared__ int gmx[16];  // col_scan: e* of the column groups of this block's 128 columns
    rne_table_init(tk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r0 = (int64_t)tr * 128, c0 = (int64_t)tcol * 128;
    const int rq = 4 * warp + (lane & 3), cc = lane >> 2;  // row quad 0..31, column chunk 0..7
    const int64_t j = c0 + 16 * cc;
    // the tile's loads first (rows beyond the tensor read nothing): they do not depend on
    // the targets, so their latency overlaps the column scan
    uint4 raw[4];
    int eg[4];
    if (j < a.cols) {
        const int64_t gcol = idiv(j, a.g_cols);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t i = r0 + 4 * rq + t;
            const bool in = i < a.rows;
            raw[t] = in ? *reinterpret_cast<const uint4 *>(a.in + i * a.ld + j) : make_uint4(0, 0, 0, 0);
            eg[t] = in ? (int)a.in_exp[idiv(i, a.g_rows) * a.ngc + gcol] : kEZero;
        }
    }
    int64_t g_first = 0;
    if (a.col_scan) {
        // a strip of at most 128 columns spans at most 9 groups (groups are >= 16 wide)
        g_first = idiv(c0, a.g_cols);
        const int ng = (int)(idiv(min(c0 + 128, a.cols) - 1, a.g_cols) - g_first + 1);
        if (threadIdx.x < 16) gmx[threadIdx.x] = kNoExp;
        __syncthreads();
        const int64_t ngr = idiv(a.rows + a.g_rows - 1, a.g_rows);
        const int k = threadIdx.x % ng, per = 256 / ng;
        if (a.ngc == 1 && (reinterpret_cast<uintptr_t>(a.in_exp) & 3) == 0) {
            // one group column (one exponent per row group, consecutive bytes): four
            // exponents per load and every load issued before the first maximum
            const uint32_t *e4 = reinterpret_cast<const uint32_t *>(a.in_exp);
            const int64_t nw = ngr >> 2;
            uint32_t m4 = 0x80808080u;  // E_ZERO (-128) in every byte: the smallest
#pragma unroll 4
            for (int64_t w = threadIdx.x; w < nw; w += 256) m4 = __vmaxs4(m4, e4[w]);
            int m = max(max(sx8(m4, 0), sx8(m4, 1)), max(sx8(m4, 2), sx8(m4, 3)));
            for (int64_t r = 4 * nw + threadIdx.x; r < ngr; r += 256) m = max(m, (int)a.in_exp[r]);
            if (m != kEZero) atomicMax(&gmx[0], m);
        } else if (threadIdx.x < per * ng) {
            // E_ZERO (-128) is the smallest byte: it only wins where every member is zero
            int m0 = kEZero, m1 = kEZero, m2 = kEZero, m3 = kEZero;
            const int8_t *e = a.in_exp + g_first + k;
            int64_t r = threadIdx.x / ng;
            for (; r + 3 * per < ngr; r += 4 * per) {  // four loads in flight
                m0 = max(m0, (int)e[r * a.ngc]);
                m1 = max(m1, (int)e[(r + per) * a.ngc]);
                m2 = max(m2, (int)e[(r + 2 * per) * a.ngc]);
                m3 = max(m3, (int)e[(r + 3 * per) * a.ngc]);
            }
            for (; r < ngr; r += per) m0 = max(m0, (int)e[r * a.ngc]);
            const int m = max(max(m0, m1), max(m2, m3));
            if (m != kEZero) atomicMax(&gmx[k], m);
        }
    }
    __syncthreads();
    if (j < a.cols) {
        const int es_col = a.col_scan ? estar_of(gmx[idiv(j, a.g_cols) - g_first]) : 0;
        if (a.axis == 0 && (a.col_max || a.col_scan) && tr == 0 && rq == 0) {
            const int es = a.col_scan ? es_col : align_target(a, 0, j);
            for (int b = 0; b < 16; ++b) a.e_star[j + b] = (int8_t)es;
        }
        // axis 0: one target for the thread's 16 columns in all four rows
        const int es_c = a.axis == 0 ? (a.col_scan ? es_col : align_target(a, 0, j)) : 0;
        uint4 v[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int es = a.axis == 0 ? es_c : align_target(a, r0 + 4 * rq + t, j);
            v[t] = rne_shift16_k(raw[t], tk[rne_index(es, eg[t])]);
        }
        const uint32_t w[4][4] = {{v[0].x, v[0].y, v[0].z, v[0].w}, {v[1].x, v[1].y, v[1].z, v[1].w},
                                  {v[2].x, v[2].y, v[2].z, v[2].w}, {v[3].x, v[3].y, v[3].z, v[3].w}};
        uint32_t *tw = reinterpret_cast<uint32_t *>(tile);
        const int chunk = (rq >> 2) ^ cc;  // swizzled 16-byte chunk
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // columns 16 cc + 4 q .. + 3
            const uint32_t t0 = __byte_perm(w[0][q], w[1][q], 0x5140), t1 = __byte_perm(w[0][q], w[1][q], 0x7362);
            const uint32_t t2 = __byte_perm(w[2][q], w[3][q], 0x5140), t3 = __byte_perm(w[2][q], w[3][q], 0x7362);
            const uint32_t col[4] = {__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                                     __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632)};
#pragma unroll
            for (int k = 0; k < 4; ++k) tw[(16 * cc + 4 * q + k) * 32 + chunk * 4 + (rq & 3)] = col[k];
        }
    }
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int orow = pass * 32 + (threadIdx.x >> 3), m = threadIdx.x & 7;
        const int64_t oi = c0 + orow, oj = r0 + 16 * m;
        if (oi < a.cols && oj < a.rows)
            *reinterpret_cast<uint4 *>(a.out + oi * a.out_ld + oj) = tile[orow][m ^ (orow >> 4)];
    }
}

// The transposing alignment for jobs whose targets come from a column-max scratch or a
// given e* (no block scans its columns' exponents): the same tiles and thread layout,
// but persistent blocks that walk the tiles of both jobs with the grid's stride, issue
// the loads of their next tile before they round and transpose the current one, and
// alternate between two shared tiles, so that one barrier per tile suffices.
struct TrTile {
    uint4 raw[4];
    int eg[4];
    int es;  // axis 0: the target of the thread's 16 columns
};

__device__ __forceinline__ void tr_tile_decode(const AlignPair &P, int tile, int &z, int64_t &r0, int64_t &c0) {
    z = tile >= P.tiles0 ? 1 : 0;
    const int t = tile - (z ? P.tiles0 : 0);
    const int tr = t / P.ntc[z];
    r0 = (int64_t)tr * 128;
    c0 = (int64_t)(t - tr * P.ntc[z]) * 128;
}

// EXACT: every job aligns per column from a column-max scratch, with one group row per
// row and g_cols / 16 a power of two (or one group across the row): the group column
// is a shift and no division or target branch remains in the loop.
template <bool EXACT>
__device__ __forceinline__ void tr_tile_load(const AlignArgs &a, int64_t r0, int64_t j, int rq, TrTile &b) {
    if (j >= a.cols) return;
    const int64_t gcol = EXACT ? (j >> (a.gv_shift1 + 3)) : idiv(j, a.g_cols);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int64_t i = r0 + 4 * rq + t;
        const bool in = i < a.rows;
        b.raw[t] = in ? *reinterpret_cast<const uint4 *>(a.in + i * a.ld + j) : make_uint4(0, 0, 0, 0);
        b.eg[t] = in ? (int)a.in_exp[(EXACT ? i : idiv(i, a.g_rows)) * a.ngc + gcol] : kEZero;
    }
    if (EXACT) b.es = estar_of(a.col_max[gcol]);
    else b.es = a.axis == 0 ? align_target(a, 0, j) : 0;
}

template <bool EXACT>
__global__ void __launch_bounds__(256, 3) align_transpose_stream_kernel(const __grid_constant__ AlignPair P) {
    __shared__ uint4 tile[2][128][8];  // [buffer][output row = input column][16-byte chunk, swizzled]
    __shared__ RneK tk[9];
    rne_table_init(tk);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rq = 4 * warp + (lane & 3), cc = lane >> 2;  // row quad 0..31, column chunk 0..7
    const int total = P.tiles0 + P.tiles1;
    int tile_id = blockIdx.x;
    if (tile_id >= total) return;  // whole blocks
    TrTile cur, nxt;
    int z;
    int64_t r0, c0;
    tr_tile_decode(P, tile_id, z, r0, c0);
    tr_tile_load<EXACT>(P.a[z], r0, c0 + 16 * cc, rq, cur);
    for (int buf = 0; tile_id < total; tile_id += gridDim.x, buf ^= 1) {
        const int next = tile_id + gridDim.x;
        int zn = 0;
        int64_t rn = 0, cn = 0;
        if (next < total) {
            tr_tile_decode(P, next, zn, rn, cn);
            tr_tile_load<EXACT>(P.a[zn], rn, cn + 16 * cc, rq, nxt);
        }
        const AlignArgs &a = P.a[z];
        const int64_t j = c0 + 16 * cc;
        if (j < a.cols) {
            if ((EXACT || (a.axis == 0 && a.col_max)) && r0 == 0 && rq == 0)
                for (int q = 0; q < 16; ++q) a.e_star[j + q] = (int8_t)cur.es;
            uint4 v[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int es = EXACT || a.axis == 0 ? cur.es : align_target(a, r0 + 4 * rq + t, j);
                v[t] = rne_shift16_k(cur.raw[t], tk[rne_index(es, cur.eg[t])]);
            }
            const uint32_t w[4][4] = {{v[0].x, v[0].y, v[0].z, v[0].w}, {v[1].x, v[1].y, v[1].z, v[1].w},
                                      {v[2].x, v[2].y, v[2].z, v[2].w}, {v[3].x, v[3].y, v[3].z, v[3].w}};
            uint32_t *tw = reinterpret_cast<uint32_t *>(tile[buf]);
            const int chunk = (rq >> 2) ^ cc;  // swizzled 16-byte chunk
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // columns 16 cc + 4 q .. + 3
                const uint32_t t0 = __byte_perm(w[0][q], w[1][q], 0x5140), t1 = __byte_perm(w[0][q], w[1][q], 0x7362);
                const uint32_t t2 = __byte_perm(w[2][q], w[3][q], 0x5140), t3 = __byte_perm(w[2][q], w[3][q], 0x7362);
                const uint32_t col[4] = {__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                                         __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632)};
#pragma unroll
                for (int k = 0; k < 4; ++k) tw[(16 * cc + 4 * q + k) * 32 + chunk * 4 + (rq & 3)] = col[k];
            }
        }
        // one barrier per tile: the buffer written here was last read two tiles ago, and
        // every thread has passed the barrier of the tile in between since then
        __syncthreads();
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
            const int orow = pass * 32 + (threadIdx.x >> 3), m = threadIdx.x & 7;
            const int64_t oi = c0 + orow, oj = r0 + 16 * m;
            if (oi < a.cols && oj < a.rows)
                *reinterpret_cast<uint4 *>(a.out + oi * a.out_ld + oj) = tile[buf][orow][m ^ (orow >> 4)];
        }
        if (next < total) cur = nxt, z = zn, r0 = rn, c0 = cn;
    }
}

// ------------------------------------------------------------------ integer GELU

struct GeluArgs {
    const int8_t *h;
    const int8_t *h_exp;
    const int8_t *dg;
    const int8_t *dg_exp;
    int8_t *out;
    int8_t *out_exp;
    int64_t rows, cols, ld_h, ld_dg, ld_out;
    int g_rows, g_cols;
    int64_t ngc;
};

// h(x) = x * clip((x + 2) / 4, 0, 1) on one mantissa C at exponent e, result at e.
__device__ __forceinline__ int gelu_fwd_elem(int c, int e) {
    if (c == 0 || e == kEZero) return 0;
    if (e >= 2) return c > 0 ? c : 0;
    const int s = 2 - e;  // >= 1; T = 2^(1 - e) = 2^(s - 1)
    if (s - 1 <= 7) {
        const int t = 1 << (s - 1);
        if (c <= -t) return 0;
        if (c >= t) return c;
    }
    // interior: x (x + 2) / 4 at exponent e = RNE((C^2 + C * 2^(s-1)) / 2^s)
    if (s <= 24) return rne_shr32(c * c + c * (1 << (s - 1)), s);
    // C^2 / 2^s < 1/2: RNE(C / 2 + positive tiny) = floor((C + 1) / 2)
    return (c + 1) >> 1;
}

// One 16-byte vector per thread; the vector's group exponent fixes the curve's
// thresholds and the interior rounding shift for all 16 mantissas.
__global__ void __launch_bounds__(256) gelu_fwd_kernel(GeluArgs a) {
    const int64_t vecs_per_row = a.cols / 16;
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= a.rows * vecs_per_row) return;
    const int64_t i = idiv(v, vecs_per_row), j = (v - i * vecs_per_row) * 16;
    const int e = a.h_exp[idiv(i, a.g_rows) * a.ngc + idiv(j, a.g_cols)];
    const uint4 raw = *reinterpret_cast<const uint4 *>(a.h + i * a.ld_h + j);
    const uint32_t src[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[4] = {0, 0, 0, 0};
    if (e != kEZero) {
        if (e >= 2) {  // |x| >= 4 for every nonzero C: h(x) = max(x, 0)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o[q] = pack4(max(sx8(src[q], 0), 0), max(sx8(src[q], 1), 0), max(sx8(src[q], 2), 0),
                             max(sx8(src[q], 3), 0));
        } else {
            const int s = 2 - e;                           // interior: RNE(C (C + T) / 2^s)
            const int t = s - 1 >= 8 ? 256 : (1 << (s - 1));  // T = 2^(1-e); |C| < 256
            if (s <= 24) {
                const int T = 1 << (s - 1), bias = T - 1;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    int r[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int c = sx8(src[q], b);
                        const int x = c * (c + T);
                        const int in = (x + bias + ((x >> s) & 1)) >> s;
                        r[b] = c <= -t ? 0 : (c >= t ? c : in);
                    }
                    o[q] = pack4(r[0], r[1], r[2], r[3]);
                }
            } else {  // C^2 / 2^s < 1/2: RNE(C / 2 + a positive tiny term) = floor((C + 1) / 2)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    o[q] = pack4((sx8(src[q], 0) + 1) >> 1, (sx8(src[q], 1) + 1) >> 1,
                                 (sx8(src[q], 2) + 1) >> 1, (sx8(src[q], 3) + 1) >> 1);
            }
        }
    }
    *reinterpret_cast<uint4 *>(a.out + i * a.ld_out + j) = make_uint4(o[0], o[1], o[2], o[3]);
}

// dG * h'(x): h' = 0 for x <= -2, 1 for x >= 2, (x + 1) / 2 between; as a two-term
// value dG * C_h * 2^(e_d + e_h - 1) + dG * 2^(e_d - 1).
__device__ __forceinline__ TwoTerm gelu_bwd_elem(int ch, int eh, int cd, int ed) {
    if (cd == 0) return TwoTerm{0, 0};
    if (eh == kEZero) ch = 0;
    if (ch != 0) {
        if (eh >= 1) return ch > 0 ? TwoTerm{cd, ed} : TwoTerm{0, 0};  // |x| >= 2
        if (1 - eh <= 7) {
            const int t = 1 << (1 - eh);
            if (ch <= -t) return TwoTerm{0, 0};
            if (ch >= t) return TwoTerm{cd, ed};
        }
    }
    return two_term((int64_t)cd * ch, ed + eh - 1, cd, ed - 1);
}

__global__ void __launch_bounds__(256) gelu_bwd_kernel(GeluArgs a) {
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw >= a.rows * a.ngc) return;
    const int64_t i = idiv(gw, a.ngc), g = gw - i * a.ngc;
    const int64_t j0 = g * a.g_cols, j1 = min(a.cols, j0 + a.g_cols);
    const int eh = a.h_exp[i * a.ngc + g], ed = a.dg_exp[i * a.ngc + g];
    int emax = kNoExp;
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const TwoTerm t = gelu_bwd_elem(a.h[i * a.ld_h + j], eh, a.dg[i * a.ld_dg + j], ed);
        if (t.x) emax = max(emax, need64(t.x, t.r));
    }
    const int e = finalize_exp(warp_max(emax));
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const TwoTerm t = gelu_bwd_elem(a.h[i * a.ld_h + j], eh, a.dg[i * a.ld_dg + j], ed);
        a.out[i * a.ld_out + j] = (int8_t)requant64(t.x, t.r, e);
    }
    if (lane == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// Exact GELU backward of one group element by element (int64 two-term sums), for
// groups whose hidden exponent is so small that the int32 path would overflow.  Re-reads
// the inputs; lane li handles elements li, li + L, ...
template <int L>
__device__ __noinline__ void gelu_bwd_group_exact(const GeluArgs &a, int64_t i, int64_t g, int glen,
                                                  int li, unsigned gmask) {
    const int64_t j0 = g * a.g_cols;
    const int eh = a.h_exp[i * a.ngc + g], ed = a.dg_exp[i * a.ngc + g];
    int emax = kNoExp;
    for (int j = li; j < glen; j += L) {
        const TwoTerm t = gelu_bwd_elem(a.h[i * a.ld_h + j0 + j], eh, a.dg[i * a.ld_dg + j0 + j], ed);
        if (t.x) emax = max(emax, need64(t.x, t.r));
    }
    const int e = finalize_exp(group_max<L>(emax, gmask));
    for (int j = li; j < glen; j += L) {
        const TwoTerm t = gelu_bwd_elem(a.h[i * a.ld_h + j0 + j], eh, a.dg[i * a.ld_dg + j0 + j], ed);
        a.out[i * a.ld_out + j0 + j] = (int8_t)requant64(t.x, t.r, e);
    }
    if (li == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// GELU backward, L lanes per row-local group of 16 * L elements, one 16-byte chunk of H
// and dG per lane.  Per group: dG * h'(x) = hi * 2^(e_d - 1) + lo * 2^(e_d + e_h - 1) with
// hi in {0, C_d, 2 C_d} and lo = C_d * C_h inside (-2, 2); at the common exponent
// r0 = e_d - 1 - sh (sh = max(0, -e_h)) every value is hi * 2^sh + lo, exact in int32
// while sh <= 21.
template <int L>
__global__ void __launch_bounds__(256) gelu_bwd_vec_kernel(const __grid_constant__ GeluArgs a) {
    constexpr int GPW = 32 / L;
    const int lane = threadIdx.x & 31, sub = lane / L, li = lane % L;
    const unsigned gmask = L == 32 ? 0xffffffffu : (((1u << L) - 1u) << (sub * L));
    const int64_t total = a.rows * a.ngc;
    const int64_t nwarps = (int64_t)gridDim.x * 8;
    for (int64_t base = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * GPW; base < total;
         base += nwarps * GPW) {
        const int64_t gw = base + sub;
        if (gw >= total) continue;
        const int64_t i = idiv(gw, a.ngc), g = gw - i * a.ngc;
        const int64_t j0 = g * a.g_cols;
        const int glen = (int)min((int64_t)a.g_cols, a.cols - j0);
        // the group's mantissas and exponents are loaded together (no dependent round trip)
        const int off = li * 16;
        uint4 x = make_uint4(0, 0, 0, 0), y = make_uint4(0, 0, 0, 0);
        if (off < glen) {
            x = *reinterpret_cast<const uint4 *>(a.h + i * a.ld_h + j0 + off);
            y = *reinterpret_cast<const uint4 *>(a.dg + i * a.ld_dg + j0 + off);
        }
        const int eh = a.h_exp[gw], ed = a.dg_exp[gw];
        const int sh = (eh < 0 && eh != kEZero) ? -eh : 0;
        if (sh > 21) {
            gelu_bwd_group_exact<L>(a, i, g, glen, li, gmask);
            continue;
        }
        uint32_t hv[4] = {x.x, x.y, x.z, x.w}, dv[4] = {y.x, y.y, y.z, y.w};
        if (off < glen && glen - off < 16)
            for (int b = glen - off; b < 16; ++b) dv[b >> 2] &= ~(0xffu << (8 * (b & 3)));
        // |C_h| < T is the interior; e_h >= 1 (or E_ZERO) leaves only C_h = 0 inside
        const int T = (eh >= 1 || eh == kEZero) ? 1 : (1 - eh >= 8 ? 256 : (1 << (1 - eh)));
        int xv[16];
        int amax = 0;
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            const int ch = sx8(hv[b >> 2], b & 3), cd = sx8(dv[b >> 2], b & 3);
            const bool inside = ch > -T && ch < T;
            const int hi = ch <= -T ? 0 : (inside ? cd : 2 * cd);
            const int x = (hi << sh) + (inside ? cd * ch : 0);
            xv[b] = x;
            amax = max(amax, abs(x));
        }
        amax = group_max<L>(amax, gmask);
        const int r0 = ed - 1 - sh;
        const int e = finalize_exp(amax ? r0 + need_off32((uint32_t)amax) : kNoExp);
        const Shift h = make_shift(e == kEZero ? 0 : e - r0);
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = pack4(apply_shift(xv[4 * q], h), apply_shift(xv[4 * q + 1], h), apply_shift(xv[4 * q + 2], h),
                         apply_shift(xv[4 * q + 3], h));
        if (off < glen) {
            int8_t *dst = a.out + i * a.ld_out + j0 + off;
            if (glen - off >= 16) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
            } else {
                for (int b = 0; b < glen - off; ++b) dst[b] = (int8_t)(o[b >> 2] >> (8 * (b & 3)));
            }
        }
        if (li == 0) a.out_exp[gw] = (int8_t)e;
    }
}

// The same with one thread per group of V 16-byte vectors (G = 16 V columns, rows of
// whole vectors): the thread owns the group's H and dG mantissas, so the group's largest
// magnitude is a register reduction with no shuffles; groups run in row-major order over
// the grid's threads (consecutive threads, consecutive groups of a row), the next
// group's vectors and exponents are loaded before the current group is computed, and the
// row / group cursor advances without a division.  Rounding: on the fp32 pipe when the
// group's magnitudes are below 2^22 (rne_f32), else by the integer shift.
template <int V>
__global__ void __launch_bounds__(256) gelu_bwd_thread_kernel(const __grid_constant__ GeluArgs a) {
    constexpr int E = 16 * V;
    const int64_t total = a.rows * a.ngc;
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    int64_t gw = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gw >= total) return;
    int64_t i = gw / a.ngc, g = gw - i * a.ngc;
    const int64_t di = step / a.ngc, dg = step - di * a.ngc;
    uint4 h[V], d[V];
    int eh = 0, ed = 0, nv = 0;
    auto load = [&](int64_t ii, int64_t gg, uint4(&hh)[V], uint4(&dd)[V], int &e_h, int &e_d, int &n) {
        const int64_t j0 = gg * E;
        n = (int)min((int64_t)V, (a.cols - j0) >> 4);
#pragma unroll
        for (int v = 0; v < V; ++v) {
            hh[v] = v < n ? *reinterpret_cast<const uint4 *>(a.h + ii * a.ld_h + j0 + 16 * v) : make_uint4(0, 0, 0, 0);
            dd[v] = v < n ? *reinterpret_cast<const uint4 *>(a.dg + ii * a.ld_dg + j0 + 16 * v) : make_uint4(0, 0, 0, 0);
        }
        e_h = a.h_exp[ii * a.ngc + gg];
        e_d = a.dg_exp[ii * a.ngc + gg];
    };
    load(i, g, h, d, eh, ed, nv);
    while (true) {
        // the next group's cursor and loads first
        int64_t ni = i + di, ng = g + dg;
        if (ng >= a.ngc) ng -= a.ngc, ++ni;
        const bool more = ni < a.rows;
        uint4 h2[V], d2[V];
        int eh2 = 0, ed2 = 0, nv2 = 0;
        if (more) load(ni, ng, h2, d2, eh2, ed2, nv2);
        const int64_t j0 = g * E;
        const int sh = (eh < 0 && eh != kEZero) ? -eh : 0;
        if (sh > 21) {
            gelu_bwd_group_exact<1>(a, i, g, 16 * nv, 0, 0u);
        } else {
            // |C_h| < T is the interior; e_h >= 1 (or E_ZERO) leaves only C_h = 0 inside
            const int T = (eh >= 1 || eh == kEZero) ? 1 : (1 - eh >= 8 ? 256 : (1 << (1 - eh)));
            int xv[E];
            int amax = 0;
#pragma unroll
            for (int b = 0; b < E; ++b) {
                const uint4 &hv = h[b >> 4], &dv = d[b >> 4];
                const uint32_t hw = (b & 15) < 4 ? hv.x : (b & 15) < 8 ? hv.y : (b & 15) < 12 ? hv.z : hv.w;
                const uint32_t dw = (b & 15) < 4 ? dv.x : (b & 15) < 8 ? dv.y : (b & 15) < 12 ? dv.z : dv.w;
                const int ch = sx8(hw, b & 3), cd = sx8(dw, b & 3);
                const bool inside = ch > -T && ch < T;
                const int hi = ch <= -T ? 0 : (inside ? cd : 2 * cd);
                const int x = (hi << sh) + (inside ? cd * ch : 0);
                xv[b] = x;
                amax = max(amax, abs(x));
            }
            const int r0 = ed - 1 - sh;
            const int need = amax ? r0 + need_off32((uint32_t)amax) : kNoExp;
            const int e = finalize_exp(need);
            const int S = e == kEZero ? 0 : e - r0;
            uint32_t o[4 * V];
            if (rne_f32_ok(true, amax, S, need)) {
                const RneF32 k = rne_f32_consts(S);
#pragma unroll
                for (int q = 0; q < 4 * V; ++q)
                    o[q] = pack4b(rne_f32(xv[4 * q], k), rne_f32(xv[4 * q + 1], k), rne_f32(xv[4 * q + 2], k),
                                  rne_f32(xv[4 * q + 3], k));
            } else {
                const Shift hs = make_shift(S);
#pragma unroll
                for (int q = 0; q < 4 * V; ++q)
                    o[q] = pack4(apply_shift(xv[4 * q], hs), apply_shift(xv[4 * q + 1], hs),
                                 apply_shift(xv[4 * q + 2], hs), apply_shift(xv[4 * q + 3], hs));
            }
#pragma unroll
            for (int v = 0; v < V; ++v)
                if (v < nv)
                    *reinterpret_cast<uint4 *>(a.out + i * a.ld_out + j0 + 16 * v) =
                        make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
            a.out_exp[i * a.ngc + g] = (int8_t)e;
        }
        if (!more) break;
        i = ni, g = ng, eh = eh2, ed = ed2, nv = nv2;
#pragma unroll
        for (int v = 0; v < V; ++v) h[v] = h2[v], d[v] = d2[v];
    }
}

// GELU forward with one thread per group of V 16-byte vectors, the same traversal: the
// group exponent fixes the curve's thresholds and the interior rounding shift for all 16 V
// mantissas (the exponent is carried unchanged).
template <int V>
__global__ void __launch_bounds__(256) gelu_fwd_thread_kernel(const __grid_constant__ GeluArgs a) {
    constexpr int E = 16 * V;
    const int64_t total = a.rows * a.ngc;
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    int64_t gw = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gw >= total) return;
    int64_t i = gw / a.ngc, g = gw - i * a.ngc;
    const int64_t di = step / a.ngc, dg = step - di * a.ngc;
    uint4 h[V];
    int eh = 0, nv = 0;
    auto load = [&](int64_t ii, int64_t gg, uint4(&hh)[V], int &e_h, int &n) {
        const int64_t j0 = gg * E;
        n = (int)min((int64_t)V, (a.cols - j0) >> 4);
#pragma unroll
        for (int v = 0; v < V; ++v)
            hh[v] = v < n ? *reinterpret_cast<const uint4 *>(a.h + ii * a.ld_h + j0 + 16 * v) : make_uint4(0, 0, 0, 0);
        e_h = a.h_exp[ii * a.ngc + gg];
    };
    load(i, g, h, eh, nv);
    while (true) {
        int64_t ni = i + di, ng = g + dg;
        if (ng >= a.ngc) ng -= a.ngc, ++ni;
        const bool more = ni < a.rows;
        uint4 h2[V];
        int eh2 = 0, nv2 = 0;
        if (more) load(ni, ng, h2, eh2, nv2);
        uint32_t o[4 * V];
        if (eh == kEZero) {
#pragma unroll
            for (int q = 0; q < 4 * V; ++q) o[q] = 0u;
        } else if (eh >= 2) {  // |x| >= 4 for every nonzero C: h(x) = max(x, 0)
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const uint32_t src[4] = {h[v].x, h[v].y, h[v].z, h[v].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) o[4 * v + q] = __vmaxs4(src[q], 0u);
            }
        } else {
            const int s = 2 - eh;                              // interior: RNE(C (C + T) / 2^s)
            const int t = s - 1 >= 8 ? 256 : (1 << (s - 1));  // T = 2^(1-e); |C| < 256
            const int T = s <= 24 ? 1 << (s - 1) : 0;
            const Shift hs = make_shift(s);
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const uint32_t src[4] = {h[v].x, h[v].y, h[v].z, h[v].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    int r[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int c = sx8(src[q], b);
                        // C^2 / 2^s < 1/2 beyond s = 24: RNE(C / 2 + a positive tiny term) = floor((C + 1) / 2)
                        const int in = s <= 24 ? apply_shift(c * (c + T), hs) : (c + 1) >> 1;
                        r[b] = c <= -t ? 0 : (c >= t ? c : in);
                    }
                    o[4 * v + q] = pack4(r[0], r[1], r[2], r[3]);
                }
            }
        }
        const int64_t j0 = g * E;
#pragma unroll
        for (int v = 0; v < V; ++v)
            if (v < nv)
                *reinterpret_cast<uint4 *>(a.out + i * a.ld_out + j0 + 16 * v) =
                    make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        if (!more) break;
        i = ni, g = ng, eh = eh2, nv = nv2;
#pragma unroll
        for (int v = 0; v < V; ++v) h[v] = h2[v];
    }
}

// ------------------------------------------------------------------ requant, wide groups

// FIT of row-local groups wider than a warp can hold: one block of T threads per group,
// EPT elements per thread kept in registers between the max and the rounding pass.
// Fast FIT of a group's int32 values x with value exponents r (row + column exponent),
// for groups whose nonzero values have exponents within [rmin, rmax] and
// (rmax - rmin) + bitlen(max |x|) <= 30: with y = x * 2^(r - rmin) (exact, |y| < 2^30),
// the group exponent is e = rmin + need_off(max |y|), since need_off(|x| 2^d) =
// need_off(|x|) + d and need_off is monotone, and every mantissa is RNE(y / 2^(e - rmin)),
// one multiply-high rounding per value (floor((y + 2^(S-1) - 1 + lsb) / 2^S)).
__device__ __forceinline__ int fit_fast_shift(int y, int S, int m, int bias) {
    if (S <= 0) return y << -S;
    if (S == 1) return (y + ((y >> 1) & 1)) >> 1;
    const int t = __mulhi(y, m);
    return __mulhi(y + bias + (t & 1), m);
}
__device__ __forceinline__ bool fit_fast_ok(int rmin, int rmax, uint32_t amax) {
    return amax == 0 || (rmax - rmin) + (32 - __clz(amax)) <= 30;
}
__device__ __forceinline__ uint32_t uabs32(int v) { return v < 0 ? 0u - (uint32_t)v : (uint32_t)v; }

template <int T, int EPT>
__global__ void __launch_bounds__(T) requant_group_block_kernel(RequantArgs a) {
    const int64_t gidx = blockIdx.x;
    const int64_t i = gidx / a.ngc, g = gidx % a.ngc;
    const int64_t j0 = g * a.G;
    const int glen = (int)min((int64_t)a.G, a.cols - j0);
    const int re = a.base + (a.row_exp ? a.row_exp[idiv(i, a.row_div)] : 0);
    int64_t x[EPT];
    int r[EPT];
    int emax = kNoExp;
#pragma unroll
    for (int k = 0; k < EPT; ++k) {
        const int jj = threadIdx.x + k * T;
        x[k] = 0;
        r[k] = re;
        if (jj < glen) {
            const int64_t j = j0 + jj;
            x[k] = rq_value(a, i, j);
            r[k] = re + (a.col_exp ? a.col_exp[idiv(j, a.col_div)] : 0);
            if (x[k]) emax = max(emax, need64q(x[k], r[k], a.qb));
        }
    }
    __shared__ int red[T / 32];
    emax = warp_max(emax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = emax;
    __syncthreads();
    int m = red[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) m = max(m, red[w]);
    const int e = finalize_exp(m);
#pragma unroll
    for (int k = 0; k < EPT; ++k) {
        const int jj = threadIdx.x + k * T;
        if (jj < glen) a.out[i * a.out_ld + j0 + jj] = (int8_t)requant64(x[k], r[k], e);
    }
    if (threadIdx.x == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// FIT of row-local groups of int32 partial sums (one or more split-K slices), 4 columns
// per thread with 16-byte loads and 4-byte stores: one block of T threads per group of
// at most 16 T columns.  WIDE: more than one slice, summed in int64.  Requires cs = 1,
// G, cols, ld and out_ld multiples of 4.
template <int T, int V, bool WIDE>
__global__ void __launch_bounds__(T) requant_vec_kernel(RequantArgs a) {
    using X = typename std::conditional<WIDE, int64_t, int32_t>::type;
    const int64_t gidx = blockIdx.x;
    const int64_t i = gidx / a.ngc, g = gidx % a.ngc;
    const int64_t j0 = g * a.G;
    const int glen = (int)min((int64_t)a.G, a.cols - j0);
    const int re = a.base + (a.row_exp ? a.row_exp[idiv(i, a.row_div)] : 0);
    const bool ce4 = a.col_exp && a.col_div == 1 && ((reinterpret_cast<uintptr_t>(a.col_exp) & 3) == 0);
    X x[V][4];
    int r[V][4];
    int emax = kNoExp;
#pragma unroll
    for (int k = 0; k < V; ++k) {
        const int jj = 4 * (threadIdx.x + k * T);
#pragma unroll
        for (int t = 0; t < 4; ++t) x[k][t] = 0, r[k][t] = re;
        if (jj < glen) {
            const int64_t at = i * a.ld + j0 + jj;
            const int4 q = *reinterpret_cast<const int4 *>(a.v32 + at);
            X s0 = q.x, s1 = q.y, s2 = q.z, s3 = q.w;
            int sp = 1;
            for (; sp + 4 <= a.nsplit; sp += 4) {  // four slices in flight
                const int32_t *b = a.v32 + sp * a.split_stride + at;
                const int4 q2 = *reinterpret_cast<const int4 *>(b);
                const int4 q3 = *reinterpret_cast<const int4 *>(b + a.split_stride);
                const int4 q4 = *reinterpret_cast<const int4 *>(b + 2 * a.split_stride);
                const int4 q5 = *reinterpret_cast<const int4 *>(b + 3 * a.split_stride);
                s0 += ((X)q2.x + q3.x) + ((X)q4.x + q5.x), s1 += ((X)q2.y + q3.y) + ((X)q4.y + q5.y);
                s2 += ((X)q2.z + q3.z) + ((X)q4.z + q5.z), s3 += ((X)q2.w + q3.w) + ((X)q4.w + q5.w);
            }
            for (; sp < a.nsplit; ++sp) {
                const int4 q2 = *reinterpret_cast<const int4 *>(a.v32 + sp * a.split_stride + at);
                s0 += q2.x, s1 += q2.y, s2 += q2.z, s3 += q2.w;
            }
            x[k][0] = s0, x[k][1] = s1, x[k][2] = s2, x[k][3] = s3;
            if (ce4) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(a.col_exp + j0 + jj);
#pragma unroll
                for (int t = 0; t < 4; ++t) r[k][t] = re + sx8(w, t);
            } else if (a.col_exp) {
#pragma unroll
                for (int t = 0; t < 4; ++t) r[k][t] = re + a.col_exp[(j0 + jj + t) / a.col_div];
            }
        }
    }
    __shared__ int red[4][T / 32];
    const int wid = threadIdx.x >> 5;
    if constexpr (!WIDE) {
        // the fast exact FIT (see fit_fast_shift) when the group's value exponents are close
        int rmin = 0x7fffffff, rmax = -0x7fffffff;
        uint32_t amax = 0;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (4 * (threadIdx.x + k * T) < glen)
#pragma unroll
                for (int t = 0; t < 4; ++t) rmin = min(rmin, r[k][t]), rmax = max(rmax, r[k][t]);
#pragma unroll
            for (int t = 0; t < 4; ++t) amax = max(amax, uabs32((int)x[k][t]));
        }
        rmin = __reduce_min_sync(0xffffffffu, rmin), rmax = __reduce_max_sync(0xffffffffu, rmax);
        amax = __reduce_max_sync(0xffffffffu, amax);
        if ((threadIdx.x & 31) == 0) red[0][wid] = rmin, red[1][wid] = rmax, red[2][wid] = (int)amax;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < T / 32; ++w)
            rmin = min(rmin, red[0][w]), rmax = max(rmax, red[1][w]), amax = max(amax, (uint32_t)red[2][w]);
        if (fit_fast_ok(rmin, rmax, amax)) {
            const bool spread = rmax != rmin;
            uint32_t ymax = amax;
            if (spread) {  // y = x 2^(r - rmin) in place (exact: fewer than 31 bits)
                ymax = 0;
#pragma unroll
                for (int k = 0; k < V; ++k)
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        x[k][t] = (int)x[k][t] << ((r[k][t] - rmin) & 31);
                        ymax = max(ymax, uabs32((int)x[k][t]));
                    }
                ymax = __reduce_max_sync(0xffffffffu, ymax);
                if ((threadIdx.x & 31) == 0) red[3][wid] = (int)ymax;
                __syncthreads();
#pragma unroll
                for (int w = 0; w < T / 32; ++w) ymax = max(ymax, (uint32_t)red[3][w]);
            }
            const int e_raw = amax ? rmin + need_off32q(ymax, a.qb) : kNoExp;
            if (e_raw <= 127) {  // a capped exponent takes the saturating exact path below
                const int e = finalize_exp(e_raw);
                const int S = e == kEZero ? 0 : min(e - rmin, 31);
                const int m = S >= 2 ? 1 << (32 - S) : 0, bias = S >= 2 ? (1 << (S - 1)) - 1 : 0;
#pragma unroll
                for (int k = 0; k < V; ++k) {
                    const int jj = 4 * (threadIdx.x + k * T);
                    if (jj < glen) {
                        int o[4];
                        if (S >= 2) {
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const int v = (int)x[k][t];
                                o[t] = __mulhi(v + bias + (__mulhi(v, m) & 1), m);
                            }
                        } else {
#pragma unroll
                            for (int t = 0; t < 4; ++t) o[t] = fit_fast_shift((int)x[k][t], S, 0, 0);
                        }
                        *reinterpret_cast<uint32_t *>(a.out + i * a.out_ld + j0 + jj) = pack4s(o[0], o[1], o[2], o[3]);
                    }
                }
                if (threadIdx.x == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
                return;
            }
            if (spread)  // undo the in-place scaling for the exact path
#pragma unroll
                for (int k = 0; k < V; ++k)
#pragma unroll
                    for (int t = 0; t < 4; ++t) x[k][t] = (int)x[k][t] >> ((r[k][t] - rmin) & 31);
        }
    }
#pragma unroll
    for (int k = 0; k < V; ++k)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            if (WIDE) {
                if (x[k][t]) emax = max(emax, need64q((int64_t)x[k][t], r[k][t], a.qb));
            } else {
                const int32_t v = (int32_t)x[k][t];
                if (v) emax = max(emax, r[k][t] + need_off32q((uint32_t)(v < 0 ? -v : v), a.qb));
            }
        }
    emax = warp_max(emax);
    __syncthreads();  // the fast path's reductions may still read red[0]
    if ((threadIdx.x & 31) == 0) red[0][wid] = emax;
    __syncthreads();
    int m = red[0][0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) m = max(m, red[0][w]);
    const int e = finalize_exp(m);
#pragma unroll
    for (int k = 0; k < V; ++k) {
        const int jj = 4 * (threadIdx.x + k * T);
        if (jj < glen) {
            int o[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                o[t] = WIDE ? requant64((int64_t)x[k][t], r[k][t], e) : requant32((int32_t)x[k][t], r[k][t], e);
            *reinterpret_cast<uint32_t *>(a.out + i * a.out_ld + j0 + jj) = pack4(o[0], o[1], o[2], o[3]);
        }
    }
    if (threadIdx.x == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// FIT of row-local groups of one slice of int32 sums, one warp per group of at most
// 128 V columns: each lane holds V 16-byte vectors (4 columns each), all loaded before
// anything else, and the group's largest need is a warp reduction, so no block barrier
// sits between the loads and the stores.  Requires cs = 1, col_div = 1 (or no column
// exponents), G, cols, ld and out_ld multiples of 4.

template <int V>
__global__ void __launch_bounds__(256) requant_warp_kernel(const __grid_constant__ RequantArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t gidx = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gidx >= a.rows * a.ngc) return;
    const int64_t i = idiv(gidx, a.ngc), g = gidx - i * a.ngc;
    const int64_t j0 = g * a.G;
    const int glen = (int)min((int64_t)a.G, a.cols - j0);
    const int re = a.base + (a.row_exp ? a.row_exp[idiv(i, a.row_div)] : 0);
    int4 x[V];
    uint32_t ce[V];
#pragma unroll
    for (int k = 0; k < V; ++k) {
        const int jj = 4 * (lane + 32 * k);
        x[k] = make_int4(0, 0, 0, 0);
        ce[k] = 0;
        if (jj < glen) {
            x[k] = *reinterpret_cast<const int4 *>(a.v32 + i * a.ld + j0 + jj);
            if (a.col_exp) ce[k] = *reinterpret_cast<const uint32_t *>(a.col_exp + j0 + jj);
        }
    }
    // the group's column-exponent range (per-byte extremes of this lane's words, then the
    // warp's) and its largest magnitude
    uint32_t cmn = 0x7f7f7f7fu, cmx = 0x80808080u, amax = 0;
#pragma unroll
    for (int k = 0; k < V; ++k) {
        if (4 * (lane + 32 * k) < glen) cmn = __vmins4(cmn, ce[k]), cmx = __vmaxs4(cmx, ce[k]);
        amax = max(max(uabs32(x[k].x), uabs32(x[k].y)), max(max(uabs32(x[k].z), uabs32(x[k].w)), amax));
    }
    int rmin = min(min(sx8(cmn, 0), sx8(cmn, 1)), min(sx8(cmn, 2), sx8(cmn, 3)));
    int rmax = max(max(sx8(cmx, 0), sx8(cmx, 1)), max(sx8(cmx, 2), sx8(cmx, 3)));
    rmin = __reduce_min_sync(0xffffffffu, rmin), rmax = __reduce_max_sync(0xffffffffu, rmax);
    amax = __reduce_max_sync(0xffffffffu, amax);
    uint32_t packed[V];
    int e = kEZero;
    bool fast = fit_fast_ok(rmin, rmax, amax);
    const bool spread = rmax != rmin;
    if (fast) {
        uint32_t ymax = amax;
        if (spread) {  // y = x 2^(ce - rmin) in place (exact: fewer than 31 bits)
            ymax = 0;
#pragma unroll
            for (int k = 0; k < V; ++k) {
                int *v = reinterpret_cast<int *>(&x[k]);
#pragma unroll
                for (int t = 0; t < 4; ++t) v[t] <<= (sx8(ce[k], t) - rmin) & 31, ymax = max(ymax, uabs32(v[t]));
            }
            ymax = __reduce_max_sync(0xffffffffu, ymax);
        }
        const int e_raw = amax ? re + rmin + need_off32q(ymax, a.qb) : kNoExp;
        fast = e_raw <= 127;  // a capped exponent takes the saturating exact path
        if (fast) {
            e = finalize_exp(e_raw);
            const int S = e == kEZero ? 0 : min(e - re - rmin, 31);
            if (S >= 2) {
                const int m = 1 << (32 - S), bias = (1 << (S - 1)) - 1;
#pragma unroll
                for (int k = 0; k < V; ++k) {
                    int *v = reinterpret_cast<int *>(&x[k]);
                    int o[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) o[t] = __mulhi(v[t] + bias + (__mulhi(v[t], m) & 1), m);
                    packed[k] = pack4s(o[0], o[1], o[2], o[3]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < V; ++k) {
                    int *v = reinterpret_cast<int *>(&x[k]);
                    int o[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) o[t] = fit_fast_shift(v[t], S, 0, 0);
                    packed[k] = pack4s(o[0], o[1], o[2], o[3]);
                }
            }
        } else if (spread) {  // undo the in-place scaling for the exact path
#pragma unroll
            for (int k = 0; k < V; ++k) {
                int *v = reinterpret_cast<int *>(&x[k]);
#pragma unroll
                for (int t = 0; t < 4; ++t) v[t] >>= (sx8(ce[k], t) - rmin) & 31;
            }
        }
    }
    if (!fast) {
        int emax = kNoExp;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int v[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
                if (v[t]) emax = max(emax, re + sx8(ce[k], t) + need_off32q((uint32_t)(v[t] < 0 ? -v[t] : v[t]), a.qb));
        }
        e = finalize_exp(warp_max(emax));
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int v[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
            int o[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) o[t] = requant32(v[t], re + sx8(ce[k], t), e);
            packed[k] = pack4(o[0], o[1], o[2], o[3]);
        }
    }
#pragma unroll
    for (int k = 0; k < V; ++k) {
        const int jj = 4 * (lane + 32 * k);
        if (jj < glen) *reinterpret_cast<uint32_t *>(a.out + i * a.out_ld + j0 + jj) = packed[k];
    }
    if (lane == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// ------------------------------------------------------------------ fused activations

// ReLU6's clip bound in a group at exponent e, min(6 >> e, q_max) (Table 7): the integer
// 6 shifted right by e (left for e < 0, where 6 << 5 already exceeds q_max); the right
// shift truncates, so e = 2 gives 1 and e >= 3 gives 0.  E_ZERO groups hold zeros only.
__device__ __forceinline__ uint32_t relu6_bound4(int e) {
    int c;
    if (e == kEZero || e <= -5) c = 127;
    else if (e < 0) c = min(6 << (-e), 127);
    else c = e >= 3 ? 0 : (6 >> e);
    return (uint32_t)c * 0x01010101u;
}

__device__ __forceinline__ uint32_t relu_word(uint32_t w, uint32_t hi) { return __vmins4(__vmaxs4(w, 0u), hi); }

// An activation fused into a rounding pass (Table 7: integer operations on C, the
// exponent unchanged): act 0 none, 1 ReLU max(C, 0), 2 ReLU6 clip(C, 0, c) with c the
// bound of the output group's exponent e.
enum { ACT_NONE = 0, ACT_RELU = 1, ACT_RELU6 = 2 };
__device__ __forceinline__ uint4 apply_act(uint4 v, int act, int e) {
    if (act == ACT_NONE) return v;
    const uint32_t hi = act == ACT_RELU6 ? relu6_bound4(e) : 0x7f7f7f7fu;
    return make_uint4(relu_word(v.x, hi), relu_word(v.y, hi), relu_word(v.z, hi), relu_word(v.w, hi));
}

// FIT into groups that span all rows of a convolution output, from the Product's int16
// sums: t[i][j] is the exact sum rounded to odd at exponent e1 = tile_need - 7 of the
// output tile holding pixel i (tile_need[tile][group], kNoExp when the tile's group is
// all zero), and the group exponent e = finalize(gmax[group]) >= tile_need, so the
// mantissa is RNE(t * 2^(e1 - e)), a right shift of at least 7 bits, which equals RNE of
// the exact sum (Boldo and Melquiond, "Emulation of FMA and correctly rounded sums:
// proved algorithms using rounding to odd", IEEE Trans. Computers 57(4), 2008).  Output
// tiles are cv_rows image rows of width cv_W (cv_tiles_per_img per image of cv_P rows).
// 16 columns per thread: two 16-byte loads, one 16-byte store; cols, ld and out_ld
// multiples of 16, G a multiple of 16.
struct Ro16RoundArgs {
    const int16_t *v;
    int64_t rows, cols, ld;
    const int32_t *tile_need;  // [tiles][ngc]
    const int32_t *gmax;       // [ngc]
    int cv_W, cv_P, cv_rows, cv_tiles_per_img;
    int G;
    int64_t ngc;
    int8_t *out;
    int64_t out_ld;
    int8_t *out_exp;
    int act;  // fused activation (ACT_*)
};
// The round pass of the Product's EPI_RO16R output (one group per row spanning tiles):
// the row's group exponent e = finalize(max of its parts' needs), and every int16 t of
// part k (rounded to odd at need_k - 7) becomes RNE(t * 2^(need_k - 7 - e)), a right shift
// of at least 7 bits, which equals RNE of the exact sum (the same lemma as above).  One
// warp per row, 16 columns per lane step (part_cols a multiple of 16).
struct Ro16RowsArgs {
    const int16_t *v;
    int64_t rows, cols, ld;
    const int32_t *need;  // [rows][tn_ld]: need of (row, part), kNoExp when all zero
    int64_t tn_ld;
    int part_cols;
    int8_t *out;
    int64_t out_ld;
    int8_t *out_exp;
    int64_t out_exp_ld;
};
__device__ __forceinline__ uint4 ro16_round16(uint4 x0, uint4 x1, int tn, int e) {
    const int64_t s64 = (int64_t)e - ((int64_t)tn - 7);
    const int s = (int)(s64 > 40 ? 40 : s64);
    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t o[4];
    if (s >= 2 && s < 32) {
        const int m = 1 << (32 - s), bias = (1 << (s - 1)) - 1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int y[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int x = (int)(int16_t)(xw[2 * q + (k >> 1)] >> (16 * (k & 1)));
                y[k] = __mulhi(x + bias + (__mulhi(x, m) & 1), m);
            }
            o[q] = pack4(y[0], y[1], y[2], y[3]);
        }
    } else if (s >= 32) {
        o[0] = o[1] = o[2] = o[3] = 0u;  // |t| < 2^15: below half a unit
    } else {
        // e below the part's need only after an exponent overflow (status raised)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int y[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                y[k] = requant32((int)(int16_t)(xw[2 * q + (k >> 1)] >> (16 * (k & 1))), tn - 7, e);
            o[q] = pack4(y[0], y[1], y[2], y[3]);
        }
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}
__global__ void __launch_bounds__(256) ro16_rows_round_kernel(const __grid_constant__ Ro16RowsArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t i = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (i >= a.rows) return;
    const int32_t *nrow = a.need + i * a.tn_ld;
    const int16_t *vrow = a.v + i * a.ld;
    int8_t *orow = a.out + i * a.out_ld;
    const int64_t nchunk = a.cols / 16;
    // the first four chunks of this lane are loaded before the row's exponent is known
    constexpr int P = 4;
    uint4 x[P][2];
#pragma unroll
    for (int u = 0; u < P; ++u) {
        const int64_t c = lane + 32 * u;
        if (c < nchunk) x[u][0] = reinterpret_cast<const uint4 *>(vrow + 16 * c)[0], x[u][1] = reinterpret_cast<const uint4 *>(vrow + 16 * c)[1];
    }
    int m = kNoExp;
    for (int64_t k = lane; k < a.tn_ld; k += 32) m = max(m, nrow[k]);
    const int e = finalize_exp(warp_max(m));
    if (lane == 0) a.out_exp[i * a.out_exp_ld] = (int8_t)e;
#pragma unroll
    for (int u = 0; u < P; ++u) {
        const int64_t c = lane + 32 * u;
        if (c < nchunk)
            *reinterpret_cast<uint4 *>(orow + 16 * c) = ro16_round16(x[u][0], x[u][1], nrow[(16 * c) / a.part_cols], e);
    }
    for (int64_t c = lane + 32 * P; c < nchunk; c += 32) {
        const uint4 *src = reinterpret_cast<const uint4 *>(vrow + 16 * c);
        *reinterpret_cast<uint4 *>(orow + 16 * c) = ro16_round16(src[0], src[1], nrow[(16 * c) / a.part_cols], e);
    }
}

// One block per image row of the whole batch (the row's pixels share one output tile,
// so its tile index is worked out once), threads over (pixel, 16-column chunk); the
// rounding by s = e - (tile need - 7) bits runs on the fp32 pipe while s <= 22 (|t| < 2^15).
__global__ void __launch_bounds__(256) ro16_round_kernel(const __grid_constant__ Ro16RoundArgs a) {
    const int64_t prow = blockIdx.x;  // image row over the whole batch
    const int64_t img = idiv(prow, a.cv_P);
    const int h = (int)(prow - img * a.cv_P);
    const int64_t tile = img * a.cv_tiles_per_img + h / a.cv_rows;
    const int cv = (int)(a.cols / 16), per_row = a.cv_W * cv;
    for (int t = threadIdx.x; t < per_row; t += blockDim.x) {
        const int w = t / cv, c16 = t - w * cv;
        const int64_t i = prow * a.cv_W + w, j0 = (int64_t)c16 * 16;
        const int64_t g = idiv(j0, a.G);  // 16 | G, so one group per thread
        const int e = finalize_exp(a.gmax[g]);
        if (i == 0 && j0 == g * a.G) a.out_exp[g] = (int8_t)e;
        const int tn = a.tile_need[tile * a.ngc + g];
        const int64_t s64 = (int64_t)e - ((int64_t)tn - 7);
        const int s = (int)(s64 > 40 ? 40 : s64);
        const uint4 *src = reinterpret_cast<const uint4 *>(a.v + i * a.ld + j0);
        const uint4 x0 = src[0], x1 = src[1];
        const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        uint32_t o[4];
        if (s >= 2 && s <= 22) {
            const RneF32 k = rne_f32_consts(s);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o[q] = pack4b(rne_f32((int)(int16_t)xw[2 * q], k), rne_f32((int)xw[2 * q] >> 16, k),
                              rne_f32((int)(int16_t)xw[2 * q + 1], k), rne_f32((int)xw[2 * q + 1] >> 16, k));
        } else if (s >= 2 && s < 32) {
            const int m = 1 << (32 - s), bias = (1 << (s - 1)) - 1;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                int y[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int x = (int)(int16_t)(xw[2 * q + (kk >> 1)] >> (16 * (kk & 1)));
                    y[kk] = __mulhi(x + bias + (__mulhi(x, m) & 1), m);
                }
                o[q] = pack4(y[0], y[1], y[2], y[3]);
            }
        } else if (s >= 32) {
            o[0] = o[1] = o[2] = o[3] = 0u;  // |t| < 2^15: the value is below half a unit
        } else {
            // e below the tile's need only after an exponent overflow (status raised)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                int y[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    y[kk] = requant32((int)(int16_t)(xw[2 * q + (kk >> 1)] >> (16 * (kk & 1))), tn - 7, e);
                o[q] = pack4(y[0], y[1], y[2], y[3]);
            }
        }
        *reinterpret_cast<uint4 *>(a.out + i * a.out_ld + j0) = apply_act(make_uint4(o[0], o[1], o[2], o[3]), a.act, e);
    }
}

// Sum of split-K int32 slices, transposed: out[c][r] = sum_s in[s][r][c] (int64, row
// stride ld_out), through 32 x 32 shared tiles so that both the slice reads and the output
// writes are coalesced.
__global__ void __launch_bounds__(256) sum_slices_t_kernel(const int32_t *in, int nsplit, int64_t split_stride,
                                                           int64_t rows, int64_t cols, int64_t ld, int64_t *out,
                                                           int64_t ld_out) {
    __shared__ int64_t tile[32][33];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of 32 threads
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t r = r0 + ty + 8 * k, c = c0 + tx;
        int64_t acc = 0;
        if (r < rows && c < cols) {
            const int32_t *src = in + r * ld + c;
            int64_t a0 = 0, a1 = 0, a2 = 0, a3 = 0;  // four loads in flight
            int sp = 0;
            for (; sp + 4 <= nsplit; sp += 4) {
                a0 += src[sp * split_stride], a1 += src[(sp + 1) * split_stride];
                a2 += src[(sp + 2) * split_stride], a3 += src[(sp + 3) * split_stride];
            }
            for (; sp < nsplit; ++sp) a0 += src[sp * split_stride];
            acc = (a0 + a1) + (a2 + a3);
        }
        tile[ty + 8 * k][tx] = acc;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t c = c0 + ty + 8 * k, r = r0 + tx;
        if (c < cols && r < rows) out[c * ld_out + r] = tile[tx][ty + 8 * k];
    }
}

// Sum of split-K int32 slices in place of layout: out[r][c] = sum_s in[s][r][c], stored
// as int64 (OUT64) or int32 (the caller guarantees the sums fit).  Each thread sums four
// adjacent columns with 16-byte loads, four slices in flight (cols, ld and ld_out are
// multiples of 4; in and out 16-byte aligned).
template <bool OUT64>
__global__ void __launch_bounds__(256) sum_slices_kernel(const int32_t *in, int nsplit, int64_t split_stride,
                                                         int64_t rows, int64_t cols, int64_t ld, void *out,
                                                         int64_t ld_out) {
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 4-column vector
    const int64_t qpr = cols >> 2;
    if (q >= rows * qpr) return;
    const int64_t r = idiv(q, qpr), c = (q - r * qpr) * 4;
    const int32_t *src = in + r * ld + c;
    int64_t s0 = 0, s1 = 0, s2 = 0, s3 = 0;
    int sp = 0;
    for (; sp + 4 <= nsplit; sp += 4) {
        const int4 a = *reinterpret_cast<const int4 *>(src + sp * split_stride);
        const int4 b = *reinterpret_cast<const int4 *>(src + (sp + 1) * split_stride);
        const int4 d = *reinterpret_cast<const int4 *>(src + (sp + 2) * split_stride);
        const int4 e = *reinterpret_cast<const int4 *>(src + (sp + 3) * split_stride);
        s0 += ((int64_t)a.x + b.x) + ((int64_t)d.x + e.x), s1 += ((int64_t)a.y + b.y) + ((int64_t)d.y + e.y);
        s2 += ((int64_t)a.z + b.z) + ((int64_t)d.z + e.z), s3 += ((int64_t)a.w + b.w) + ((int64_t)d.w + e.w);
    }
    for (; sp < nsplit; ++sp) {
        const int4 a = *reinterpret_cast<const int4 *>(src + sp * split_stride);
        s0 += a.x, s1 += a.y, s2 += a.z, s3 += a.w;
    }
    if constexpr (OUT64) {
        int64_t *o = static_cast<int64_t *>(out) + r * ld_out + c;
        reinterpret_cast<longlong2 *>(o)[0] = make_longlong2(s0, s1);
        reinterpret_cast<longlong2 *>(o)[1] = make_longlong2(s2, s3);
    } else {
        int32_t *o = static_cast<int32_t *>(out) + r * ld_out + c;
        *reinterpret_cast<int4 *>(o) = make_int4((int)s0, (int)s1, (int)s2, (int)s3);
    }
}

// Per-column e* from the per-group-column maxima of the column scratch form, for up to
// two jobs (blockIdx.y): e_star[j] = the maximum of column j's group column, E_ZERO when
// every group of it is zero.
__global__ void estar_expand_kernel(const __grid_constant__ AlignPair P) {
    const AlignArgs &a = P.a[blockIdx.y];
    const int32_t *col_max = P.cm[blockIdx.y];
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j < a.cols) a.e_star[j] = (int8_t)estar_of(col_max[idiv(j, a.g_cols)]);
}

// A wait on an mbarrier that never completes, bounded by limit_ns: raises
// ICT_ERR_DEVICE_TIMEOUT and returns (self-test of the bounded-wait path).
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(b, 0, limit_ns, nullptr)) raise_status(ICT_ERR_DEVICE_TIMEOUT);
    __syncthreads();
}

// ------------------------------------------------------------------ integer SGD

struct SgdTensor {
    int8_t *w, *w_exp, *v, *v_exp;
    const int8_t *g, *g_exp;
    int64_t rows, cols, ld;
    int G;
    int64_t ngc;
    int64_t first_group;  // prefix sum of group counts over the tensor list
};

constexpr int kSgdMaxTensors = 128;

struct SgdArgs {
    int n;
    int64_t total_groups;
    int mom_mul, mom_shift, lr_mul, lr_shift;
    // largest shift of each term at which |term| stays below 2^29 (so every two-term sum
    // is below 2^30): 29 - bitlen(127 |multiplier|)
    int cap_mom, cap_lr;
    int qb;  // mantissa bits B of both FITs (|C| <= 2^(B-1) - 1)
    SgdTensor t[kSgdMaxTensors];
};

// One warp per group: v <- FIT(mom * v + g), w <- FIT(w - lr * v).
__device__ __forceinline__ void sgd_group(const SgdArgs &p, const SgdTensor &t, int64_t local,
                                          int lane) {
    const int64_t i = local / t.ngc, g = local % t.ngc;
    const int64_t ge = i * t.ngc + g;
    const int64_t j0 = g * t.G, j1 = min(t.cols, j0 + t.G);
    const int ev = t.v_exp[ge], eg = t.g_exp[ge], ew = t.w_exp[ge];
    const int pv = ev - p.mom_shift;
    // velocity
    int emax = kNoExp;
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const TwoTerm s = two_term((int64_t)p.mom_mul * t.v[i * t.ld + j], pv, t.g[i * t.ld + j], eg);
        if (s.x) emax = max(emax, need64q(s.x, s.r, p.qb));
    }
    const int ev2 = finalize_exp(warp_max(emax));
    // weight (recompute the new velocity mantissas element by element)
    const int pu = ev2 - p.lr_shift;
    emax = kNoExp;
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const TwoTerm s = two_term((int64_t)p.mom_mul * t.v[i * t.ld + j], pv, t.g[i * t.ld + j], eg);
        const int cv = requant64(s.x, s.r, ev2);
        const TwoTerm w = two_term(t.w[i * t.ld + j], ew, -(int64_t)p.lr_mul * cv, pu);
        if (w.x) emax = max(emax, need64q(w.x, w.r, p.qb));
    }
    const int ew2 = finalize_exp(warp_max(emax));
    __syncwarp();
    for (int64_t j = j0 + lane; j < j1; j += 32) {
        const TwoTerm s = two_term((int64_t)p.mom_mul * t.v[i * t.ld + j], pv, t.g[i * t.ld + j], eg);
        const int cv = requant64(s.x, s.r, ev2);
        const TwoTerm w = two_term(t.w[i * t.ld + j], ew, -(int64_t)p.lr_mul * cv, pu);
        const int cw = requant64(w.x, w.r, ew2);
        t.v[i * t.ld + j] = (int8_t)cv;  // each lane rewrites only the elements it read
        t.w[i * t.ld + j] = (int8_t)cw;
    }
    if (lane == 0) {
        t.v_exp[ge] = (int8_t)ev2;
        t.w_exp[ge] = (int8_t)ew2;
    }
}

// ---- vectorised SGD: L lanes per group, each lane holds CPL 16-byte chunks of W, V, G.

// Locates global group `gw` in the tensor list.
__device__ __forceinline__ int sgd_find(const SgdArgs &p, int64_t gw) {
    int lo = 0, hi = p.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.t[mid].first_group <= gw) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Exact SGD update of one group, element by element in int64 (two_term: exact up to a
// 32-bit exponent gap, sticky beyond), for groups whose values do not fit the int32 fast
// path.  Reads W, V, G from memory again and writes the results; each lane handles the
// elements li, li + L, ... of the group.  Rolled loops: it is rare.  Inlined: as an
// out-of-line call it made the fast path about 4 % slower (measured).
template <int L>
__device__ __forceinline__ void sgd_group_exact(const SgdArgs &p, const SgdTensor &t, int64_t row0,
                                             int64_t ge, int glen, int li, unsigned gmask) {
    const int ev = t.v_exp[ge], eg = t.g_exp[ge], ew = t.w_exp[ge];
    const int pv = ev - p.mom_shift;
    int emax = kNoExp;
    for (int j = li; j < glen; j += L) {
        const TwoTerm x = two_term((int64_t)p.mom_mul * t.v[row0 + j], pv, t.g[row0 + j], eg);
        if (x.x) emax = max(emax, need64q(x.x, x.r, p.qb));
    }
    const int ev2 = finalize_exp(group_max<L>(emax, gmask));
    const int pu = ev2 - p.lr_shift;
    emax = kNoExp;
    for (int j = li; j < glen; j += L) {
        const TwoTerm x = two_term((int64_t)p.mom_mul * t.v[row0 + j], pv, t.g[row0 + j], eg);
        const int cv = requant64(x.x, x.r, ev2);
        const TwoTerm w = two_term(t.w[row0 + j], ew, -(int64_t)p.lr_mul * cv, pu);
        if (w.x) emax = max(emax, need64q(w.x, w.r, p.qb));
    }
    const int ew2 = finalize_exp(group_max<L>(emax, gmask));
    for (int j = li; j < glen; j += L) {
        const TwoTerm x = two_term((int64_t)p.mom_mul * t.v[row0 + j], pv, t.g[row0 + j], eg);
        const int cv = requant64(x.x, x.r, ev2);
        const TwoTerm w = two_term(t.w[row0 + j], ew, -(int64_t)p.lr_mul * cv, pu);
        t.v[row0 + j] = (int8_t)cv;
        t.w[row0 + j] = (int8_t)requant64(w.x, w.r, ew2);
    }
    if (li == 0) {
        t.v_exp[ge] = (int8_t)ev2;
        t.w_exp[ge] = (int8_t)ew2;
    }
}

// Common exponent of two group terms a * 2^pa + b * 2^pb: r0 = min(pa, pb), shifts sa, sb;
// an absent term (E_ZERO, all mantissas zero) takes the other's exponent.  `small` when
// both shifted terms stay below 2^29 (int32 sums are exact and leave room for rounding).
__device__ __forceinline__ void common_exp(int pa, bool za, int pb, bool zb, int cap_a, int cap_b, int &r0,
                                           int &sa, int &sb, bool &small) {
    if (za) pa = pb;
    if (zb) pb = pa;
    r0 = min(pa, pb);
    sa = pa - r0;
    sb = pb - r0;
    small = sa <= cap_a && sb <= cap_b;
}

template <int L, int CPL, bool SINGLE>
__global__ void __launch_bounds__(256) sgd_vec_kernel(const __grid_constant__ SgdArgs p) {
    constexpr int GPW = 32 / L;  // groups per warp and pass
    const int lane = threadIdx.x & 31, sub = lane / L, li = lane % L;
    const unsigned gmask = L == 32 ? 0xffffffffu : (((1u << L) - 1u) << (sub * L));
    const int64_t nwarps = (int64_t)gridDim.x * 8;
    // a single tensor's fields live in registers for the whole kernel
    const SgdTensor &t0 = p.t[0];
    int8_t *const w0 = t0.w, *const v0 = t0.v, *const we0 = t0.w_exp, *const ve0 = t0.v_exp;
    const int8_t *const g0 = t0.g, *const ge0 = t0.g_exp;
    const int64_t ld0 = t0.ld, cols0 = t0.cols, ngc0 = t0.ngc;
    const int G0 = t0.G;
    for (int64_t base = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * GPW; base < p.total_groups;
         base += nwarps * GPW) {
        const int64_t gw = base + sub;
        if (gw >= p.total_groups) continue;  // whole groups only: lanes of a group agree
        int8_t *tw, *tv, *twe, *tve;
        const int8_t *tg, *tge;
        int64_t tld, tcols, tngc, local;
        int tG;
        if (SINGLE) {
            tw = w0, tv = v0, twe = we0, tve = ve0, tg = g0, tge = ge0;
            tld = ld0, tcols = cols0, tngc = ngc0, tG = G0, local = gw;
        } else {
            const SgdTensor &t = p.t[sgd_find(p, gw)];
            tw = t.w, tv = t.v, twe = t.w_exp, tve = t.v_exp, tg = t.g, tge = t.g_exp;
            tld = t.ld, tcols = t.cols, tngc = t.ngc, tG = t.G, local = gw - t.first_group;
        }
        // group (row i, column group gi); one column group per row needs no division
        int64_t i, gi;
        if (tngc == 1) {
            i = local, gi = 0;
        } else {
            const uint32_t l32 = (uint32_t)local, n32 = (uint32_t)tngc;  // both < 2^31
            i = l32 / n32, gi = l32 - (uint32_t)i * n32;
        }
        const int64_t ge = local;  // row-major exponent grid: i * ngc + gi
        const int64_t j0 = gi * tG;
        const int glen = (int)min((int64_t)tG, tcols - j0);
        const int ev = tve[ge], eg = tge[ge], ew = twe[ge];
        SgdTensor tt;  // for the exact path
        if (!SINGLE) tt = p.t[sgd_find(p, gw)];

        uint32_t wv[CPL][4], vv[CPL][4], gv[CPL][4];
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int off = (k * L + li) * 16;
            if (off < glen) {
                const int64_t at = i * tld + j0 + off;
                const uint4 a = *reinterpret_cast<const uint4 *>(tw + at);
                const uint4 b = *reinterpret_cast<const uint4 *>(tv + at);
                const uint4 c = *reinterpret_cast<const uint4 *>(tg + at);
                wv[k][0] = a.x, wv[k][1] = a.y, wv[k][2] = a.z, wv[k][3] = a.w;
                vv[k][0] = b.x, vv[k][1] = b.y, vv[k][2] = b.z, vv[k][3] = b.w;
                gv[k][0] = c.x, gv[k][1] = c.y, gv[k][2] = c.z, gv[k][3] = c.w;
                const int rem = glen - off;  // mask columns past the group's end
                if (rem < 16) {
#pragma unroll
                    for (int b2 = 0; b2 < 16; ++b2)
                        if (b2 >= rem) {
                            const uint32_t m = ~(0xffu << (8 * (b2 & 3)));
                            wv[k][b2 >> 2] &= m, vv[k][b2 >> 2] &= m, gv[k][b2 >> 2] &= m;
                        }
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) wv[k][q] = vv[k][q] = gv[k][q] = 0;
            }
        }

        // ---- velocity: v = mom * V + G (every byte unpacked once; sums stay in registers)
        constexpr int E = 16 * CPL;
        int r1, sa1, sb1;
        bool small1;
        common_exp(ev - p.mom_shift, ev == kEZero, eg, eg == kEZero, p.cap_mom, 22, r1, sa1, sb1, small1);
        if (!small1) {
            sgd_group_exact<L>(p, SINGLE ? p.t[0] : tt, i * tld + j0, ge, glen, li, gmask);
            continue;
        }
        int x[E];
        int ev2;
        {
            const int ma = p.mom_mul << sa1, mb = 1 << sb1;
            int hi = 0, lo = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                x[e] = sx8(vv[e >> 4][(e >> 2) & 3], e & 3) * ma + sx8(gv[e >> 4][(e >> 2) & 3], e & 3) * mb;
                hi = max(hi, x[e]);
                lo = min(lo, x[e]);
            }
            const int amax = group_max<L>(max(hi, -lo), gmask);
            ev2 = finalize_exp(amax ? r1 + need_off32q((uint32_t)amax, p.qb) : kNoExp);
            const Shift h = make_shift(ev2 == kEZero ? 0 : ev2 - r1);
            if (__any_sync(gmask, h.ls != 0)) {
#pragma unroll
                for (int e = 0; e < E; ++e) x[e] <<= h.ls;
            }
            if (h.rs >= 2) {
                // floor(v / 2^rs) = high word of v * 2^(32 - rs): the shifts run on the FMA pipe
                const int m = 1 << (32 - h.rs);
#pragma unroll
                for (int e = 0; e < E; ++e) x[e] = __mulhi(x[e] + h.bias + (__mulhi(x[e], m) & 1), m);  // v'
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) x[e] = (x[e] + h.bias + (int)bfe_u32((uint32_t)x[e], h.rs, h.om)) >> h.rs;
            }
        }

        // ---- weight: w = W - lr * v'
        int r2, sa2, sb2;
        bool small2;
        common_exp(ew, ew == kEZero, ev2 - p.lr_shift, ev2 == kEZero, 22, p.cap_lr, r2, sa2, sb2, small2);
        if (!small2) {
            sgd_group_exact<L>(p, SINGLE ? p.t[0] : tt, i * tld + j0, ge, glen, li, gmask);
            continue;
        }
        uint32_t nv[CPL][4], nw[CPL][4];
        int ew2;
        {
            const int ma = 1 << sa2, mb = -(p.lr_mul << sb2);
            int y[E];
            int hi = 0, lo = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                y[e] = sx8(wv[e >> 4][(e >> 2) & 3], e & 3) * ma + x[e] * mb;
                hi = max(hi, y[e]);
                lo = min(lo, y[e]);
            }
            const int amax = group_max<L>(max(hi, -lo), gmask);
            ew2 = finalize_exp(amax ? r2 + need_off32q((uint32_t)amax, p.qb) : kNoExp);
            const Shift h = make_shift(ew2 == kEZero ? 0 : ew2 - r2);
            if (__any_sync(gmask, h.ls != 0)) {
#pragma unroll
                for (int e = 0; e < E; ++e) y[e] <<= h.ls;
            }
            if (h.rs >= 2) {
                const int m = 1 << (32 - h.rs);
#pragma unroll
                for (int e = 0; e < E; ++e) y[e] = __mulhi(y[e] + h.bias + (__mulhi(y[e], m) & 1), m);
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) y[e] = (y[e] + h.bias + (int)bfe_u32((uint32_t)y[e], h.rs, h.om)) >> h.rs;
            }
#pragma unroll
            for (int e = 0; e < E; e += 4) {
                int r[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) r[q] = y[e + q];
                nw[e >> 4][(e >> 2) & 3] = __byte_perm(__byte_perm(r[0], r[1], 0x0040), __byte_perm(r[2], r[3], 0x0040), 0x5410);
                nv[e >> 4][(e >> 2) & 3] = __byte_perm(__byte_perm(x[e], x[e + 1], 0x0040),
                                                       __byte_perm(x[e + 2], x[e + 3], 0x0040), 0x5410);
            }
        }

        // ---- store (masked columns past the group's end are left untouched)
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int off = (k * L + li) * 16;
            if (off < glen) {
                const int64_t at = i * tld + j0 + off;
                if (glen - off >= 16) {
                    *reinterpret_cast<uint4 *>(tv + at) = make_uint4(nv[k][0], nv[k][1], nv[k][2], nv[k][3]);
                    *reinterpret_cast<uint4 *>(tw + at) = make_uint4(nw[k][0], nw[k][1], nw[k][2], nw[k][3]);
                } else {
                    for (int b2 = 0; b2 < glen - off; ++b2) {
                        tv[at + b2] = (int8_t)(nv[k][b2 >> 2] >> (8 * (b2 & 3)));
                        tw[at + b2] = (int8_t)(nw[k][b2 >> 2] >> (8 * (b2 & 3)));
                    }
                }
            }
        }
        if (li == 0) {
            tve[ge] = (int8_t)ev2;
            twe[ge] = (int8_t)ew2;
        }
    }
}

// SGD over one dense tensor whose groups are whole rows of exactly 16 L CPL elements (a
// parameter arena padded to its group width).  Each lane holds 16 CPL elements of W, V
// and G; the next group's chunks are loaded before the current group is computed.
//
// The two-term sums and their rounding run on the fp32 pipe, one code path for every
// group (so that the groups of a warp never split it).  Per group the sum is taken at the
// unit of one term (its mantissas are exact floats built from the bytes) with the other
// term's multiplier a float power-of-two multiple of mom or lr; one pair of directed FMAs
// gives each sum rounded to odd at 24 bits (ro_fma).  The group exponent follows from the
// largest magnitude's bit pattern (need_rel_f32), and RNE(x / 2^S) is one FMA onto
// 1.5 * 2^23: its result lies in [2^23, 2^24), where fp32 rounds to the nearest integer
// with ties to even, so the low byte of its bits is the int8 mantissa; since that
// rounding sits at least 16 bits above the sums' last places it equals rounding the exact
// sums.  Groups whose exponents lie more than kSgdGap apart, or whose exponent leaves the
// range, take the int64 path (sgd_group_exact).
__device__ __forceinline__ float sx8f(uint32_t w_biased, int b) {
    // byte b of w (stored with 0x80 added to every byte) as the float C: 2^23 + (C + 128) - (2^23 + 128)
    return __uint_as_float(__byte_perm(w_biased, 0x4B000000u, 0x7650 | b)) - 8388736.0f;
}
__device__ __forceinline__ float pow2f(int k) {  // 2^k for -126 <= k <= 127; 0 below
    return k < -126 ? 0.0f : __int_as_float((k + 127) << 23);
}
__device__ __forceinline__ uint32_t low_bytes4(float a, float b, float c, float d) {
    return __byte_perm(__byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040),
                       __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040), 0x5410);
}
// a * b + c rounded to odd at fp32's 24 bits: rounded down and rounded up, the two
// results are equal when the sum is exact and are neighbours otherwise, and the one whose
// last significand bit is set is the round-to-odd result (for either sign).  Rounding
// that to nearest even at a position at least two bits above its last place equals
// rounding the exact sum (Boldo and Melquiond, IEEE Trans. Computers 57(4), 2008).
__device__ __forceinline__ float ro_fma(float a, float b, float c) {
    const float lo = __fmaf_rd(a, b, c), hi = __fmaf_ru(a, b, c);
    return (__float_as_uint(lo) & 1u) ? lo : hi;
}
// need() of a positive normal float x (its bit pattern): the least S with
// RNE(x 2^-S) <= 2^(B-1) - 1, i.e. x < (2^(B-1) - 1/2) 2^S: S = E - (B - 2) for
// x = 1.f 2^E, plus one when 1.f >= 2 - 2^(1-B) (the significand field at or above
// 2^23 - 2^(24-B)).  A value rounded to odd at 24 bits gives the same S as the exact one,
// since the bound has at most B significant bits.
__device__ __forceinline__ int need_rel_f32(uint32_t xb, int qb) {
    return (int)(xb >> 23) - 127 - (qb - 2) + ((xb & 0x7FFFFFu) >= 0x800000u - (1u << (24 - qb)) ? 1 : 0);
}
// largest exponent gap between the two terms that the fp32 path takes: their multipliers
// stay normal floats and far from overflow
constexpr int kSgdGap = 100;

// L lanes per group, CPL 16-byte chunks per lane (a group is 16 L CPL elements; chunk k
// of lane li sits at element (k L + li) 16 of the group, so that each chunk index is a
// coalesced row of the warp): more chunks per lane spread the per-group work (targets,
// reductions, exponents, branches) over more elements.
template <int L, int CPL>
__global__ void __launch_bounds__(256) sgd_rows_kernel(const __grid_constant__ SgdArgs p) {
    constexpr int GPW = 32 / L, E = 16 * CPL, G = 16 * L * CPL;
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const int lane = threadIdx.x & 31, sub = lane / L, li = lane % L;
    const unsigned gmask = L == 32 ? 0xffffffffu : (((1u << L) - 1u) << (sub * L));
    const SgdTensor &t0 = p.t[0];
    int8_t *const tw = t0.w, *const tv = t0.v, *const twe = t0.w_exp, *const tve = t0.v_exp;
    const int8_t *const tg = t0.g, *const tge = t0.g_exp;
    const int64_t rows = t0.rows;
    const int64_t step = (int64_t)gridDim.x * 8 * GPW;
    int64_t r = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * GPW + sub;
    uint4 cw[CPL], cv[CPL], cg[CPL];
    int ev = 0, eg = 0, ew = 0;
    if (r < rows) {
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int64_t at = r * G + (k * L + li) * 16;
            cw[k] = *reinterpret_cast<const uint4 *>(tw + at);
            cv[k] = *reinterpret_cast<const uint4 *>(tv + at);
            cg[k] = *reinterpret_cast<const uint4 *>(tg + at);
        }
        ev = tve[r], eg = tge[r], ew = twe[r];
    }
    for (; r < rows; r += step) {
        const int64_t rn = r + step;
        uint4 nw4[CPL], nv4[CPL], ng4[CPL];
        int nev = 0, neg = 0, new_ = 0;
        if (rn < rows) {  // prefetch the next group
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                const int64_t at = rn * G + (k * L + li) * 16;
                nw4[k] = *reinterpret_cast<const uint4 *>(tw + at);
                nv4[k] = *reinterpret_cast<const uint4 *>(tv + at);
                ng4[k] = *reinterpret_cast<const uint4 *>(tg + at);
            }
            nev = tve[rn], neg = tge[rn], new_ = twe[rn];
        }
        // velocity: v = mom * V 2^(ev - mom_shift) + G 2^eg, at the unit 2^pb (the G term
        // unscaled, the other term's multiplier mom 2^(pa - pb) a float)
        int pa = ev - p.mom_shift, pb = eg;
        if (ev == kEZero) pa = pb;  // an absent term takes the other's exponent
        if (eg == kEZero) pb = pa;
        const int d1 = pa - pb;
        bool fast = d1 >= -kSgdGap && d1 <= kSgdGap;
        int ev2 = kEZero, ew2 = kEZero;
        float vq[E];  // 1.5 * 2^23 + the new velocity mantissas
        float y[E];   // the velocity sums, then the weight sums (rounded to odd at 24 bits)
        {
            uint32_t vb[4 * CPL], gb[4 * CPL];
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                vb[4 * k] = cv[k].x ^ 0x80808080u, vb[4 * k + 1] = cv[k].y ^ 0x80808080u;
                vb[4 * k + 2] = cv[k].z ^ 0x80808080u, vb[4 * k + 3] = cv[k].w ^ 0x80808080u;
                gb[4 * k] = cg[k].x ^ 0x80808080u, gb[4 * k + 1] = cg[k].y ^ 0x80808080u;
                gb[4 * k + 2] = cg[k].z ^ 0x80808080u, gb[4 * k + 3] = cg[k].w ^ 0x80808080u;
            }
            const float ma = (float)p.mom_mul * pow2f(fast ? d1 : 0);
            float amax = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                y[e] = ro_fma(sx8f(vb[e >> 2], e & 3), ma, sx8f(gb[e >> 2], e & 3));
                amax = fmaxf(amax, fabsf(y[e]));
            }
            const uint32_t ia = (uint32_t)group_max<L>((int)__float_as_uint(amax), gmask);
            const int need = pb + need_rel_f32(ia, p.qb);
            ev2 = ia ? finalize_exp(need) : kEZero;
            const int sh = ia ? ev2 - pb : 0;
            fast = fast && (ia == 0u || (ia >= 0x00800000u && need <= 127 && sh >= -126 && sh <= 126));
            const float sc = pow2f(fast ? -sh : 0);
#pragma unroll
            for (int e = 0; e < E; ++e) vq[e] = __fmaf_rn(y[e], sc, kMagic);
        }
        if (fast) {
            // weight: w = W 2^ew - lr * V' 2^(ev2 - lr_shift), at the unit 2^ew
            int pw = ew, pv = ev2 - p.lr_shift;
            if (ew == kEZero) pw = pv;
            if (ev2 == kEZero) pv = pw;
            const int d2 = pv - pw;
            fast = d2 >= -kSgdGap && d2 <= kSgdGap;
            uint32_t wb[4 * CPL];
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                wb[4 * k] = cw[k].x ^ 0x80808080u, wb[4 * k + 1] = cw[k].y ^ 0x80808080u;
                wb[4 * k + 2] = cw[k].z ^ 0x80808080u, wb[4 * k + 3] = cw[k].w ^ 0x80808080u;
            }
            const float mb = -(float)p.lr_mul * pow2f(fast ? d2 : 0);
            float amax = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                y[e] = ro_fma(vq[e] - kMagic, mb, sx8f(wb[e >> 2], e & 3));
                amax = fmaxf(amax, fabsf(y[e]));
            }
            const uint32_t ia = (uint32_t)group_max<L>((int)__float_as_uint(amax), gmask);
            const int need = pw + need_rel_f32(ia, p.qb);
            ew2 = ia ? finalize_exp(need) : kEZero;
            const int sh = ia ? ew2 - pw : 0;
            fast = fast && (ia == 0u || (ia >= 0x00800000u && need <= 127 && sh >= -126 && sh <= 126));
            const float sc = pow2f(fast ? -sh : 0);
#pragma unroll
            for (int e = 0; e < E; ++e) y[e] = __fmaf_rn(y[e], sc, kMagic);
        }
        const bool fit1 = fast, fit2 = fast;
        if (!(fit1 && fit2)) {
            sgd_group_exact<L>(p, t0, r * G, r, G, li, gmask);
        } else {
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                uint32_t ov[4], ow[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = 16 * k + 4 * q;
                    ov[q] = low_bytes4(vq[e], vq[e + 1], vq[e + 2], vq[e + 3]);
                    ow[q] = low_bytes4(y[e], y[e + 1], y[e + 2], y[e + 3]);
                }
                const int64_t at = r * G + (k * L + li) * 16;
                *reinterpret_cast<uint4 *>(tv + at) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
                *reinterpret_cast<uint4 *>(tw + at) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            if (li == 0) {
                tve[r] = (int8_t)ev2;
                twe[r] = (int8_t)ew2;
            }
        }
#pragma unroll
        for (int k = 0; k < CPL; ++k) cw[k] = nw4[k], cv[k] = nv4[k], cg[k] = ng4[k];
        ev = nev, eg = neg, ew = new_;
    }
}

__global__ void __launch_bounds__(256) sgd_warp_kernel(const __grid_constant__ SgdArgs p) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * 8;
    for (int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); gw < p.total_groups; gw += warps) {
        int lo = 0, hi = p.n - 1;  // tensor holding global group gw
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.t[mid].first_group <= gw) lo = mid;
            else hi = mid - 1;
        }
        sgd_group(p, p.t[lo], gw - p.t[lo].first_group, lane);
    }
}

}  // namespace ict

namespace ict {

// ------------------------------------------------------------------ conv weight prep

// Backward-data of a convolution contracts over (k, r, s) for each input channel c, so
// the KRSC weight is aligned per c (max over k, r, s of its group exponents) and laid
// out K-major as W'[c][(r*S + s)*K + k].
struct ConvWeightArgs {
    const int8_t *w;
    const int8_t *w_exp;
    int64_t ld, ngc;
    int g_rows, g_cols;
    int K, RS, C;
    int8_t *e_star;  // [C]
    int8_t *out;     // [C][out_ld]
    int64_t out_ld;
};

__global__ void __launch_bounds__(256) conv_wt_estar_kernel(ConvWeightArgs a) {
    const int c = blockIdx.x;
    int m = kNoExp;
    for (int idx = threadIdx.x; idx < a.K * a.RS; idx += blockDim.x) {
        const int k = idx / a.RS, rs = idx % a.RS;
        const int e = a.w_exp[(k / a.g_rows) * a.ngc + (rs * a.C + c) / a.g_cols];
        if (e != kEZero) m = max(m, e);
    }
    m = warp_max(m);
    __shared__ int red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        int v = red[0];
        for (int i = 1; i < 8; ++i) v = max(v, red[i]);
        a.e_star[c] = (int8_t)(v <= kNoExp ? kEZero : v);
    }
}

__global__ void __launch_bounds__(256) conv_wt_prep_kernel(ConvWeightArgs a) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_c = (int64_t)a.RS * a.K;
    if (idx >= per_c * a.C) return;
    const int c = (int)(idx / per_c), rem = (int)(idx % per_c);
    const int rs = rem / a.K, k = rem % a.K;
    const int e = a.w_exp[(k / a.g_rows) * a.ngc + (rs * a.C + c) / a.g_cols];
    const int v = a.w[k * a.ld + rs * a.C + c];
    const int es = a.e_star[c];
    int q = 0;
    if (e != kEZero && v != 0) q = es == e ? v : rne_shr32(v, es - e);
    a.out[c * a.out_ld + rem] = (int8_t)q;
}

// Exponent tables of a convolution's backward-weight Product: row m = tap * C + c of the
// MMA output takes X's exponent of channel c, column k takes dY's exponent of channel k.
__global__ void conv_wgrad_exp_kernel(const int8_t *x_exp, int gx, const int8_t *y_exp, int gy, int C,
                                      int RS, int K, int8_t *e_rows, int8_t *e_cols) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < RS * C) e_rows[i] = x_exp[(i % C) / gx];
    if (i < K) e_cols[i] = y_exp[i / gy];
}

__global__ void fill_i32_kernel(int32_t *p, int n, int32_t v) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) p[i] = v;
}

// zero result of an empty contraction: mantissas 0, every group E_ZERO
__global__ void zero_ce_kernel(int8_t *mant, int64_t rows, int64_t cols, int64_t ld, int8_t *exp,
                               int64_t n_exp) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < rows * cols) mant[(i / cols) * ld + i % cols] = 0;
    if (i < n_exp) exp[i] = (int8_t)kEZero;
}

}  // namespace ict
