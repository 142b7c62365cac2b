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
    int act;  // activation fused into the rounding (ACT_*)
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
                        E == kEZero ? make_uint4(0, 0, 0, 0) : apply_act(sum_round16(vx[k], vy[k], s, E), a.act, E);
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
                    r = apply_act(sum_round16(*reinterpret_cast<const uint4 *>(xr + 16 * c),
                                              *reinterpret_cast<const uint4 *>(yr + 16 * c), s, E),
                                  a.act, E);
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
            r = apply_act(sum_round16(*reinterpret_cast<const uint4 *>(a.x + i * a.ldx + j),
                                      *reinterpret_cast<const uint4 *>(a.y + i * a.ldy + j),
                                      sum_shape(a.x_exp[g], a.y_exp[g], a), E),
                          a.act, E);
        *reinterpret_cast<uint4 *>(a.z + i * a.ldz + j) = r;
    }
}

// ------------------------------------------------------------------ Divide-by-constant (average pool)

// K x K average pool with stride K over NHWC activations (Table 6: "Average pool" ->
// Divide-by-constant): every output element is an exact integer S at exponent r divided
// by D = K^2 (forward: S the window's mantissa sum at the pixel-uniform exponent;
// backward: S the window's upstream gradient mantissa), rounded once by FIT into the
// output's groups.  Two passes: the largest need of every output group (int32 per
// group, pre-set to 0x80808080), then the rounding.  One thread per output element.
struct PoolArgs {
    const int8_t *in, *in_exp;
    int64_t ld_in, in_ngc;
    int in_g_rows, in_g_cols;
    int8_t *out, *out_exp;
    int64_t ld_out, out_ngc, out_rows, C;
    int out_g_rows, out_g_cols;
    int h, w, K, P, Q, D, bwd;
    int32_t *need;
};

// RNE(x 2^-t / D), exactly, for |x| < 2^16, 1 <= D <= 256 and -17 <= t <= 40.
__device__ __forceinline__ int64_t rne_div64(int64_t x, int t, int64_t D) {
    if (t > 40) return 0;  // |x| 2^-t / D < 2^-24: rounds to 0
    int64_t num = x, den = D;
    if (t <= 0) num = x * (1ll << (-t));
    else den = D << t;
    int64_t q = num / den, rem = num - q * den;  // truncating division
    if (rem < 0) q -= 1, rem += den;             // floor, 0 <= rem < den
    if (2 * rem > den || (2 * rem == den && (q & 1))) q += 1;
    return q;
}
// The smallest exponent at which RNE(x 2^(r - e) / D) fits in [-127, 127] (x != 0): from
// an exponent where the quotient still exceeds 127, step up until it fits.
__device__ __forceinline__ int need_div(int64_t x, int r, int D) {
    const int bx = 64 - __clzll(x < 0 ? -x : x), bd = 32 - __clz(D);
    for (int t = bx - bd - 8;; ++t) {
        const int64_t q = rne_div64(x, t, D);
        if (q >= -127 && q <= 127) return r + t;
    }
}

__device__ __forceinline__ void pool_value(const PoolArgs &a, int64_t i, int64_t ch, int64_t &S, int &r) {
    if (a.bwd) {  // input pixel i of image img receives its window's gradient
        const int64_t hw = (int64_t)a.h * a.w, img = i / hw, y = (i - img * hw) / a.w, x = i - img * hw - y * a.w;
        const int64_t o = (img * a.P + y / a.K) * a.Q + x / a.K;
        S = a.in[o * a.ld_in + ch];
        r = a.in_exp[(o / a.in_g_rows) * a.in_ngc + ch / a.in_g_cols];
        return;
    }
    const int64_t pq = (int64_t)a.P * a.Q, img = i / pq, p = (i - img * pq) / a.Q, q = i - img * pq - p * a.Q;
    const int8_t *src = a.in + ((img * a.h + p * a.K) * a.w + q * a.K) * a.ld_in + ch;
    int64_t sum = 0;
    for (int dy = 0; dy < a.K; ++dy)
        for (int dx = 0; dx < a.K; ++dx) sum += src[((int64_t)dy * a.w + dx) * a.ld_in];
    S = sum;
    r = a.in_exp[ch / a.in_g_cols];  // pixel-uniform exponents: one exponent row
}

__global__ void __launch_bounds__(256) pool_need_kernel(const __grid_constant__ PoolArgs a) {
    const int64_t n = a.out_rows * a.C, stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t0 = (int64_t)blockIdx.x * blockDim.x; t0 < n; t0 += stride) {  // whole warps iterate together
        const int64_t t = t0 + threadIdx.x;
        int e = kNoExp;
        int64_t g = -1;
        if (t < n) {
            const int64_t i = t / a.C, ch = t - i * a.C;
            int64_t S;
            int r;
            pool_value(a, i, ch, S, r);
            if (S) e = need_div(S, r, a.D);
            g = (i / a.out_g_rows) * a.out_ngc + ch / a.out_g_cols;
        }
        // lanes of one output group reduce together; one atomic per group and warp
        const unsigned peers = __match_any_sync(0xffffffffu, (long long)g);
        const int m = __reduce_max_sync(peers, e);
        if (g >= 0 && m > kNoExp && (threadIdx.x & 31) == __ffs(peers) - 1) atomicMax(&a.need[g], m);
    }
}

__global__ void __launch_bounds__(256) pool_round_kernel(const __grid_constant__ PoolArgs a) {
    const int64_t n = a.out_rows * a.C, stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += stride) {
        const int64_t i = t / a.C, ch = t - i * a.C;
        const int64_t g = (i / a.out_g_rows) * a.out_ngc + ch / a.out_g_cols;
        const int m = a.need[g];
        const int E = finalize_exp(m <= kNoExp ? kNoExp : m);
        if (i % a.out_g_rows == 0 && ch % a.out_g_cols == 0) a.out_exp[g] = (int8_t)E;
        int64_t S;
        int r;
        pool_value(a, i, ch, S, r);
        int c = 0;
        if (S && E != kEZero) {
            const int64_t q = rne_div64(S, E - r, a.D);
            c = q > 127 ? 127 : (q < -127 ? -127 : (int)q);
        }
        a.out[i * a.ld_out + ch] = (int8_t)c;
    }
}

// ------------------------------------------------------------------ patch embedding

// Non-overlapping P x P patches of NHWC activations gathered into rows, (dy, dx, ch)
// order, ALIGN_MAX-ed to one exponent: the largest of the activation's channel-group
// exponents (they are uniform over pixels).  The rows are the K-major operand of the
// patch-embedding Product (a P x P, stride P convolution), which then needs no
// alignment.  One thread per 16-byte output vector: P * c is a multiple of 16, so a
// vector lies inside one (dy) row segment, and it spans one channel group.
struct PatchArgs {
    const int8_t *in, *in_exp;
    int64_t ld_in;
    int g_cols;
    int64_t ngc;
    int8_t *out, *out_exp;
    int64_t ld_out, rows;
    int h, w, c, P, Hp, Wp;
};
__global__ void __launch_bounds__(256) patchify_kernel(const __grid_constant__ PatchArgs a) {
    const int64_t vpr = (int64_t)a.P * a.P * a.c / 16;  // vectors per output row
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= a.rows * vpr) return;
    const int64_t o = v / vpr, t = v - o * vpr;
    const int64_t seg = (int64_t)a.P * a.c;  // bytes of one (dy) row segment
    const int64_t dy = (16 * t) / seg, off = 16 * t - dy * seg;
    const int64_t per_img = (int64_t)a.Hp * a.Wp, img = o / per_img, pq = o - img * per_img;
    const int64_t pp = pq / a.Wp, qq = pq - pp * a.Wp;
    const int64_t pix = (img * a.h + pp * a.P + dy) * a.w + qq * a.P + off / a.c;
    const int ch = (int)(off % a.c);
    const uint4 raw = *reinterpret_cast<const uint4 *>(a.in + pix * a.ld_in + ch);
    int es = kEZero;  // the target: E_ZERO (-128) is the smallest byte
    for (int64_t g = 0; g < a.ngc; ++g) es = max(es, (int)a.in_exp[g]);
    const int eg = a.in_exp[ch / a.g_cols];
    if (v == 0) a.out_exp[0] = (int8_t)es;
    *reinterpret_cast<uint4 *>(a.out + o * a.ld_out + 16 * t) =
        eg == kEZero ? make_uint4(0, 0, 0, 0) : rne_shift16(raw, min(es - eg, 8));
}

// ------------------------------------------------------------------ depthwise convolution

// One R x S filter per channel (Table 6: "Convolution (incl. 1 x 1, depthwise)" ->
// Product; MobileNetV2's depthwise layers).  The contraction of channel ch runs over
// (r, s) of that channel only, so each sum keeps the activation's per-channel exponent:
// every output element is an exact integer S at exponent e_act[ch] + e_w[ch], rounded by
// FIT into the output's groups in two passes (the groups' needs, then the rounding).
// Activations are NHWC with exponents uniform over pixels; W [C][R*S] has one exponent
// per row.
struct DwArgs {
    const int8_t *a, *a_exp;  // X (forward) or dY (backward-data), [rows][C]
    int64_t lda;
    int a_gcols;
    const int8_t *w, *w_exp;  // W [C][R*S], w_exp[ch]
    int64_t ldw;
    int8_t *out, *out_exp;
    int64_t ldo, out_rows, out_ngc;
    int out_g_rows, out_g_cols;
    int h, w_, C, R, S, pad, stride, P, Q, bwd;
    int32_t *need;
};

__device__ __forceinline__ void dw_value(const DwArgs &a, int64_t i, int ch, int64_t &sum, int &r) {
    sum = 0;
    const int8_t *wr = a.w + (int64_t)ch * a.ldw;
    if (!a.bwd) {  // output pixel i = (img, p, q)
        const int64_t pq = (int64_t)a.P * a.Q, img = i / pq, p = (i - img * pq) / a.Q, q = i - img * pq - p * a.Q;
        for (int rr = 0; rr < a.R; ++rr) {
            const int64_t y = p * a.stride + rr - a.pad;
            if (y < 0 || y >= a.h) continue;
            for (int ss = 0; ss < a.S; ++ss) {
                const int64_t x = q * a.stride + ss - a.pad;
                if (x < 0 || x >= a.w_) continue;
                sum += (int64_t)a.a[((img * a.h + y) * a.w_ + x) * a.lda + ch] * wr[rr * a.S + ss];
            }
        }
    } else {  // input pixel i = (img, y, x) gathers every (p, q, r, s) that reads it
        const int64_t hw = (int64_t)a.h * a.w_, img = i / hw, y = (i - img * hw) / a.w_, x = i - img * hw - y * a.w_;
        for (int rr = 0; rr < a.R; ++rr) {
            const int64_t ph = y + a.pad - rr;
            if (ph < 0 || ph % a.stride) continue;
            const int64_t p = ph / a.stride;
            if (p >= a.P) continue;
            for (int ss = 0; ss < a.S; ++ss) {
                const int64_t qw = x + a.pad - ss;
                if (qw < 0 || qw % a.stride) continue;
                const int64_t q = qw / a.stride;
                if (q >= a.Q) continue;
                sum += (int64_t)a.a[((img * a.P + p) * a.Q + q) * a.lda + ch] * wr[rr * a.S + ss];
            }
        }
    }
    const int ea = a.a_exp[ch / a.a_gcols], ew = a.w_exp[ch];
    r = (ea == kEZero || ew == kEZero) ? 0 : ea + ew;
}

__global__ void __launch_bounds__(256) dw_need_kernel(const __grid_constant__ DwArgs a) {
    const int64_t n = a.out_rows * a.C, stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t0 = (int64_t)blockIdx.x * blockDim.x; t0 < n; t0 += stride) {  // whole warps iterate together
        const int64_t t = t0 + threadIdx.x;
        int e = kNoExp;
        int64_t g = -1;
        if (t < n) {
            const int64_t i = t / a.C;
            const int ch = (int)(t - i * a.C);
            int64_t sum;
            int r;
            dw_value(a, i, ch, sum, r);
            if (sum) e = need64(sum, r);
            g = (i / a.out_g_rows) * a.out_ngc + ch / a.out_g_cols;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, (long long)g);
        const int m = __reduce_max_sync(peers, e);
        if (g >= 0 && m > kNoExp && (threadIdx.x & 31) == __ffs(peers) - 1) atomicMax(&a.need[g], m);
    }
}

__global__ void __launch_bounds__(256) dw_round_kernel(const __grid_constant__ DwArgs a) {
    const int64_t n = a.out_rows * a.C, stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += stride) {
        const int64_t i = t / a.C;
        const int ch = (int)(t - i * a.C);
        const int64_t g = (i / a.out_g_rows) * a.out_ngc + ch / a.out_g_cols;
        const int m = a.need[g];
        const int E = finalize_exp(m <= kNoExp ? kNoExp : m);
        if (i % a.out_g_rows == 0 && ch % a.out_g_cols == 0) a.out_exp[g] = (int8_t)E;
        int64_t sum;
        int r;
        dw_value(a, i, ch, sum, r);
        a.out[i * a.ldo + ch] = (int8_t)(sum && E != kEZero ? requant64(sum, r, E) : 0);
    }
}

// Backward weight: one block per channel sums dY[(p,q)][ch] * X[pixel(p,q,r,s)][ch] over
// every output pixel for each of the R*S taps (int64, exact), then rounds the row of R*S
// sums by FIT (one group per row) and writes it with its exponent.
struct DwWgradArgs {
    const int8_t *dy, *dy_exp, *x, *x_exp;
    int64_t ldy, ldx;
    int dy_gcols, x_gcols;
    int8_t *out, *out_exp;
    int64_t ldo;
    int n, h, w_, C, R, S, pad, stride, P, Q;
};
constexpr int kDwMaxTaps = 49;
__global__ void __launch_bounds__(256) dw_wgrad_kernel(const __grid_constant__ DwWgradArgs a) {
    const int ch = blockIdx.x, taps = a.R * a.S;
    __shared__ long long part[8][kDwMaxTaps];
    __shared__ int emax_s;
    long long acc[kDwMaxTaps];
    for (int k = 0; k < taps; ++k) acc[k] = 0;
    const int64_t pq = (int64_t)a.P * a.Q, nout = (int64_t)a.n * pq;
    for (int64_t op = threadIdx.x; op < nout; op += blockDim.x) {
        const int dyv = a.dy[op * a.ldy + ch];
        if (!dyv) continue;
        const int64_t img = op / pq, p = (op - img * pq) / a.Q, q = op - img * pq - p * a.Q;
        for (int rr = 0; rr < a.R; ++rr) {
            const int64_t y = p * a.stride + rr - a.pad;
            if (y < 0 || y >= a.h) continue;
            for (int ss = 0; ss < a.S; ++ss) {
                const int64_t x = q * a.stride + ss - a.pad;
                if (x < 0 || x >= a.w_) continue;
                acc[rr * a.S + ss] += (long long)dyv * a.x[((img * a.h + y) * a.w_ + x) * a.ldx + ch];
            }
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int k = 0; k < taps; ++k) {
        long long v = acc[k];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) part[warp][k] = v;
    }
    if (threadIdx.x == 0) emax_s = kNoExp;
    __syncthreads();
    const int ey = a.dy_exp[ch / a.dy_gcols], ex = a.x_exp[ch / a.x_gcols];
    const int r = (ey == kEZero || ex == kEZero) ? 0 : ey + ex;
    long long total = 0;
    if (threadIdx.x < taps) {
        for (int wi = 0; wi < (int)(blockDim.x >> 5); ++wi) total += part[wi][threadIdx.x];
        if (total) atomicMax(&emax_s, need64(total, r));
    }
    __syncthreads();
    const int E = finalize_exp(emax_s);
    if (threadIdx.x < taps)
        a.out[(int64_t)ch * a.ldo + threadIdx.x] = (int8_t)(total && E != kEZero ? requant64(total, r, E) : 0);
    if (threadIdx.x == 0) a.out_exp[ch] = (int8_t)E;
}

}  // namespace ict
