// ict_pointwise.cuh -- pointwise primitives on (C,e) tensors, the steps either side of the
// contractions in a network block:
//   Clip: ReLU / ReLU6 forward and backward (Table 7: integer operations on the mantissa
//         C, the exponent carried through unchanged);
//   Sum:  Z = FIT(X + Y), the residual add and gradient merge (Table 6, Eq. 6).
// Source: "Memory-Efficient Integer-Only Training of Deep Neural Networks", Tables 6-7.
// All kernels stream 16-byte vectors of mantissas; a vector never straddles a group
// because group widths are multiples of 16 (or one group spans the row).
#pragma once

#include "ict_device.cuh"
#include "ict_elementwise.cuh"

namespace ict {

// ------------------------------------------------------------------ Clip (ReLU / ReLU6)

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

struct ClipArgs {
    const int8_t *x, *x_exp;  // forward input C and its exponents
    int64_t ldx;
    int gx_rows, gx_cols;
    int64_t ngcx;
    const int8_t *dy, *dy_exp;  // backward: upstream gradient
    int64_t ldy;
    int8_t *out, *out_exp;
    int64_t ldo;
    int64_t rows, cols;
    int six;
    int64_t n_exp;  // exponent bytes copied to out_exp (from x_exp forward, dy_exp backward)
};

__device__ __forceinline__ uint32_t relu_word(uint32_t w, uint32_t hi) { return __vmins4(__vmaxs4(w, 0u), hi); }
__device__ __forceinline__ uint32_t relu_mask(uint32_t w, uint32_t hi) {
    return __vcmpgts4(w, 0u) & __vcmplts4(w, hi);
}

// BWD = false: out = clip(C, 0, c), with c = 127 (a no-op bound) for ReLU.
// BWD = true: out = dY where C > 0 (ReLU) or 0 < C < c (ReLU6).
// Four vectors in flight per thread; the exponent grid is copied by the same threads.
template <bool BWD>
__global__ void __launch_bounds__(256) clip_kernel(const __grid_constant__ ClipArgs a) {
    const int64_t vpr = a.cols >> 4, nvec = a.rows * vpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t v0 = tid; v0 < nvec; v0 += 4 * stride) {
        uint4 w[4], d[4];
        uint32_t hi[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // all loads first
            const int64_t v = v0 + u * stride;
            if (v >= nvec) continue;
            const int64_t i = idiv(v, vpr), j = (v - i * vpr) << 4;
            w[u] = *reinterpret_cast<const uint4 *>(a.x + i * a.ldx + j);
            if (BWD) d[u] = *reinterpret_cast<const uint4 *>(a.dy + i * a.ldy + j);
            hi[u] = a.six ? relu6_bound4(a.x_exp[idiv(i, a.gx_rows) * a.ngcx + idiv(j, a.gx_cols)]) : 0x7f7f7f7fu;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t v = v0 + u * stride;
            if (v >= nvec) continue;
            const int64_t i = idiv(v, vpr), j = (v - i * vpr) << 4;
            uint4 r;
            if (BWD) {
                const uint32_t h = hi[u];
                auto m = [&](uint32_t x) { return a.six ? relu_mask(x, h) : __vcmpgts4(x, 0u); };
                r = make_uint4(d[u].x & m(w[u].x), d[u].y & m(w[u].y), d[u].z & m(w[u].z), d[u].w & m(w[u].w));
            } else {
                r = make_uint4(relu_word(w[u].x, hi[u]), relu_word(w[u].y, hi[u]), relu_word(w[u].z, hi[u]),
                               relu_word(w[u].w, hi[u]));
            }
            *reinterpret_cast<uint4 *>(a.out + i * a.ldo + j) = r;
        }
    }
    const int8_t *src = BWD ? a.dy_exp : a.x_exp;
    for (int64_t k = tid; k < a.n_exp; k += stride) a.out_exp[k] = src[k];
}

// ------------------------------------------------------------------ Sum (residual add)

// X, Y, Z share one group partition: row-local groups of G columns (g_rows = 1), or
// groups spanning all rows (then col_need, an int32 per group column, carries the
// largest need between the two passes).
struct SumArgs {
    const int8_t *x, *x_exp, *y, *y_exp;
    int8_t *z, *z_exp;
    int64_t ldx, ldy, ldz, rows, cols;
    int G;        // group width in columns (a multiple of 16, or the whole row)
    int64_t ngc;  // groups per row
    int32_t *col_need;
    // term weights m * 2^-s (|m| <= 512), and the largest shift of each weighted term at
    // which it stays below 2^29: 29 - bitlen(127 |m|)
    int xm, xs, ym, ys, cap_x, cap_y;
};

// The group's two weighted terms (x xm) 2^pa + (y ym) 2^pb with pa = ex - xs, pb = ey - ys,
// at a common exponent r0: x (xm << sa) + y (ym << sb).  An E_ZERO term (all its
// mantissas zero) takes the other's exponent.  fast: each weighted, shifted term stays
// below 2^29, so every sum lies below 2^30 and int32 arithmetic is exact.
struct SumShape {
    int pa, pb, r0, sa, sb, ma, mb, xm, ym;  // ma = xm 2^sa, mb = ym 2^sb (fast path)
    bool fast;
};
__device__ __forceinline__ SumShape sum_shape(int ex, int ey, const SumArgs &a) {
    SumShape s;
    s.xm = a.xm, s.ym = a.ym;
    const int px = ex - a.xs, py = ey - a.ys;
    s.pa = ex == kEZero ? py : px;
    s.pb = ey == kEZero ? s.pa : py;
    if (ex == kEZero && ey == kEZero) s.pa = s.pb = 0;
    s.r0 = min(s.pa, s.pb);
    s.sa = s.pa - s.r0;
    s.sb = s.pb - s.r0;
    s.fast = s.sa <= a.cap_x && s.sb <= a.cap_y;
    s.ma = s.fast ? s.xm * (1 << s.sa) : 0;
    s.mb = s.fast ? s.ym * (1 << s.sb) : 0;
    return s;
}

// Largest need() over one 16-byte vector pair.
__device__ __forceinline__ int sum_need16(uint4 vx, uint4 vy, const SumShape &s) {
    const uint32_t wx[4] = {vx.x, vx.y, vx.z, vx.w}, wy[4] = {vy.x, vy.y, vy.z, vy.w};
    if (s.fast) {
        uint32_t amax = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int v = sx8(wx[q], b) * s.ma + sx8(wy[q], b) * s.mb;
                amax = max(amax, (uint32_t)abs(v));
            }
        return amax ? s.r0 + need_off32(amax) : kNoExp;
    }
    int emax = kNoExp;
    for (int q = 0; q < 4; ++q)
        for (int b = 0; b < 4; ++b) {
            const TwoTerm t = two_term((int64_t)s.xm * sx8(wx[q], b), s.pa, (int64_t)s.ym * sx8(wy[q], b), s.pb);
            if (t.x) emax = max(emax, need64(t.x, t.r));
        }
    return emax;
}

// The 16 mantissas of a vector pair in a group of exponent E (not E_ZERO).
__device__ __forceinline__ uint4 sum_round16(uint4 vx, uint4 vy, const SumShape &s, int E) {
    const uint32_t wx[4] = {vx.x, vx.y, vx.z, vx.w}, wy[4] = {vy.x, vy.y, vy.z, vy.w};
    uint32_t o[4];
    if (s.fast) {
        const Shift h = make_shift(E - s.r0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int c[4];
#pragma unroll
            for (int b = 0; b < 4; ++b)
                c[b] = apply_shift(sx8(wx[q], b) * s.ma + sx8(wy[q], b) * s.mb, h);
            o[q] = pack4(c[0], c[1], c[2], c[3]);
        }
    } else {
        for (int q = 0; q < 4; ++q) {
            int c[4];
            for (int b = 0; b < 4; ++b) {
                const TwoTerm t = two_term((int64_t)s.xm * sx8(wx[q], b), s.pa, (int64_t)s.ym * sx8(wy[q], b), s.pb);
                c[b] = requant64(t.x, t.r, E);
            }
            o[q] = pack4(c[0], c[1], c[2], c[3]);
        }
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Row-local groups: L lanes per group, lane li takes the vectors li, li + L, ...  With
// CPL > 0 a lane holds its (at most CPL) vector pairs in registers between the pass that
// finds the group's largest need and the pass that rounds; CPL = 0 re-reads them (wide
// groups; the second reads hit L1/L2).
template <int L, int CPL>
__global__ void __launch_bounds__(256) sum_rows_kernel(const __grid_constant__ SumArgs a) {
    constexpr int GPW = 32 / L;
    const int lane = threadIdx.x & 31, sub = lane / L, li = lane % L;
    const unsigned gmask = L == 32 ? 0xffffffffu : (((1u << L) - 1u) << (sub * L));
    const int64_t groups = a.rows * a.ngc, nwarps = (int64_t)gridDim.x * 8;
    for (int64_t base = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * GPW; base < groups;
         base += nwarps * GPW) {
        const int64_t gidx = base + sub;
        if (gidx >= groups) continue;  // the L lanes of a group leave together
        const int64_t i = idiv(gidx, a.ngc), j0 = (gidx - i * a.ngc) * a.G;
        const int nv = (int)(min((int64_t)a.G, a.cols - j0) >> 4);
        const SumShape s = sum_shape(a.x_exp[gidx], a.y_exp[gidx], a);
        const int8_t *xr = a.x + i * a.ldx + j0, *yr = a.y + i * a.ldy + j0;
        int8_t *zr = a.z + i * a.ldz + j0;
        int emax = kNoExp;
        if constexpr (CPL > 0) {
            uint4 vx[CPL], vy[CPL];
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                const int c = li + k * L;
                if (c < nv) {
                    vx[k] = *reinterpret_cast<const uint4 *>(xr + 16 * c);
                    vy[k] = *reinterpret_cast<const uint4 *>(yr + 16 * c);
                }
            }
#pragma unroll
            for (int k = 0; k < CPL; ++k)
                if (li + k * L < nv) emax = max(emax, sum_need16(vx[k], vy[k], s));
            const int E = finalize_exp(group_max<L>(emax, gmask));
            if (li == 0) a.z_exp[gidx] = (int8_t)E;
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                const int c = li + k * L;
                if (c < nv)
                    *reinterpret_cast<uint4 *>(zr + 16 * c) =
                        E == kEZero ? make_uint4(0, 0, 0, 0) : sum_round16(vx[k], vy[k], s, E);
            }
        } else {
            for (int c = li; c < nv; c += L)
                emax = max(emax, sum_need16(*reinterpret_cast<const uint4 *>(xr + 16 * c),
                                            *reinterpret_cast<const uint4 *>(yr + 16 * c), s));
            const int E = finalize_exp(group_max<L>(emax, gmask));
            if (li == 0) a.z_exp[gidx] = (int8_t)E;
            for (int c = li; c < nv; c += L) {
                uint4 r = make_uint4(0, 0, 0, 0);
                if (E != kEZero)
                    r = sum_round16(*reinterpret_cast<const uint4 *>(xr + 16 * c),
                                    *reinterpret_cast<const uint4 *>(yr + 16 * c), s, E);
                *reinterpret_cast<uint4 *>(zr + 16 * c) = r;
            }
        }
    }
}

// Groups spanning all rows, pass 1: the largest need of every group column, reduced in
// shared memory per block and then with one atomicMax per group column in global memory
// (col_need pre-set to 0x80808080, below every need).
__global__ void __launch_bounds__(256) sum_global_need_kernel(const __grid_constant__ SumArgs a) {
    extern __shared__ int smax[];  // [ngc]
    for (int64_t g = threadIdx.x; g < a.ngc; g += blockDim.x) smax[g] = kNoExp;
    __syncthreads();
    const int64_t vpr = a.cols >> 4, nvec = a.rows * vpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
        const int64_t i = idiv(v, vpr), j = (v - i * vpr) << 4, g = idiv(j, a.G);
        const SumShape s = sum_shape(a.x_exp[g], a.y_exp[g], a);
        const int e = sum_need16(*reinterpret_cast<const uint4 *>(a.x + i * a.ldx + j),
                                 *reinterpret_cast<const uint4 *>(a.y + i * a.ldy + j), s);
        if (e > kNoExp) atomicMax(&smax[g], e);
    }
    __syncthreads();
    for (int64_t g = threadIdx.x; g < a.ngc; g += blockDim.x)
        if (smax[g] > kNoExp) atomicMax(&a.col_need[g], smax[g]);
}

// Pass 2: every vector rounded to its group column's exponent; the threads of row 0
// store the exponents.
__global__ void __launch_bounds__(256) sum_global_round_kernel(const __grid_constant__ SumArgs a) {
    const int64_t vpr = a.cols >> 4, nvec = a.rows * vpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
        const int64_t i = idiv(v, vpr), j = (v - i * vpr) << 4, g = idiv(j, a.G);
        const int m = a.col_need[g];
        const int E = finalize_exp(m <= kNoExp ? kNoExp : m);
        if (i == 0 && j == g * a.G) a.z_exp[g] = (int8_t)E;
        uint4 r = make_uint4(0, 0, 0, 0);
        if (E != kEZero)
            r = sum_round16(*reinterpret_cast<const uint4 *>(a.x + i * a.ldx + j),
                            *reinterpret_cast<const uint4 *>(a.y + i * a.ldy + j),
                            sum_shape(a.x_exp[g], a.y_exp[g], a), E);
        *reinterpret_cast<uint4 *>(a.z + i * a.ldz + j) = r;
    }
}

}  // namespace ict
