// ict_lut.cuh -- the nonlinear-function primitive through lookup tables.
//
// Source: "Memory-Efficient Integer-Only Training of Deep Neural Networks".
//   Table 7 (GELU):        forward LUT_fwd[e, C]; backward (dY * LUT_bwd[e, C]) >> B_G;
//                          INT8 [30, 256]; the exponent e is carried unchanged.
//   Table 8 (output head): LUT_exp[e_x][k] = round(exp(k 2^e_x) 2^L), k in [-255, 0],
//                          L = 7, [30, 256]; LUT_log[p] = round(-log(p / 2^B) 2^Ll),
//                          p in [1, 2^B - 2], Ll = 5, [256]; built once at initialization.
// The tables cover the 30 exponents e = -26 .. 3.  Beyond them every row equals its
// nearest end row (e <= -26: exp rounds to 128 for every k, GELU to ceil(C / 2), GELU' to
// 1/2; e >= 3: exp to 0 for k < 0, GELU to max(C, 0), GELU' to the step), so a lookup
// clamps e.  GELU is x Phi(x) (Phi the standard normal CDF); B_G = 6, since the slope lies
// in about [-0.129, 1.129].
//
// The library builds the tables once per process on the host (long double libm, then
// round half to even) and passes them to its kernels as launch parameters; every block
// copies the rows it needs into shared memory first, so the kernels keep no device state.
#pragma once

#include <cmath>
#include <mutex>

#include "ict_device.cuh"
#include "ict_elementwise.cuh"

namespace ict {

constexpr int kLutELo = -26, kLutEHi = 3, kLutRows = kLutEHi - kLutELo + 1;
constexpr int kGeluBG = 6;

struct LutTables {
    uint8_t exp[kLutRows][256];   // [e - kLutELo][k + 255]
    uint8_t log[256];             // [p]; entries 0 and 255 repeat 1 and 254
    int8_t gelu_fwd[kLutRows][256];  // [e - kLutELo][C + 128]
    int8_t gelu_bwd[kLutRows][256];
};

__host__ __device__ __forceinline__ int lut_row(int e) {
    return (e < kLutELo ? kLutELo : (e > kLutEHi ? kLutEHi : e)) - kLutELo;
}

// Host: the tables, computed on first use.
inline const LutTables &lut_tables() {
    static LutTables t;
    static std::once_flag once;
    std::call_once(once, [] {
        auto rne = [](long double v) { return (long)std::nearbyint(v); };  // default mode: half to even
        const long double sqrt2 = std::sqrt((long double)2), sqrt2pi = std::sqrt(2 * (long double)M_PI);
        for (int e = kLutELo; e <= kLutEHi; ++e) {
            const long double s = std::ldexp((long double)1, e);
            for (int k = -255; k <= 0; ++k) t.exp[e - kLutELo][k + 255] = (uint8_t)rne(std::exp(k * s) * 128);
            for (int c = -128; c <= 127; ++c) {
                const long double x = c * s;
                const long double cdf = 0.5L * (1 + std::erf(x / sqrt2));
                const long double pdf = std::exp(-x * x / 2) / sqrt2pi;
                t.gelu_fwd[e - kLutELo][c + 128] = (int8_t)rne(c * cdf);
                t.gelu_bwd[e - kLutELo][c + 128] = (int8_t)rne((cdf + x * pdf) * (1 << kGeluBG));
            }
        }
        for (int p = 1; p <= 254; ++p) t.log[p] = (uint8_t)rne(-std::log((long double)p / 256) * 32);
        t.log[0] = t.log[1];
        t.log[255] = t.log[254];
    });
    return t;
}

// ------------------------------------------------------------------ GELU through its tables

struct GeluLutArgs {
    const int8_t *h, *h_exp;    // H (the forward input), exponent grid [.][ngc]
    const int8_t *dy, *dy_exp;  // backward: upstream gradient, same group partition as H
    int8_t *out, *out_exp;      // forward: GELU(H); backward: dH (same partition)
    int64_t rows, cols, ld_h, ld_dy, ld_out;
    int g_rows, g_cols;
    int64_t ngc;
    alignas(16) int8_t lut[kLutRows * 256];  // LUT_fwd or LUT_bwd (read as 16-byte vectors)
};

__device__ __forceinline__ void lut_to_smem(const int8_t *src, int8_t *dst, int n) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int i = threadIdx.x; i < n / 16; i += blockDim.x) d4[i] = s4[i];
    __syncthreads();
}

// Forward: every mantissa becomes LUT_fwd[e][C] (one 16-byte vector per thread; the
// group exponents are copied by the host call).  Requires g_cols a multiple of 16.
__global__ void __launch_bounds__(256) gelu_lut_fwd_kernel(const __grid_constant__ GeluLutArgs a) {
    __shared__ __align__(16) int8_t lut[kLutRows * 256];
    lut_to_smem(a.lut, lut, kLutRows * 256);
    const int64_t cv = a.cols / 16;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= a.rows * cv) return;
    const int64_t i = idiv(t, cv), j = (t - i * cv) * 16;
    const int e = a.h_exp[idiv(i, a.g_rows) * a.ngc + idiv(j, a.g_cols)];
    const int8_t *row = lut + lut_row(e) * 256 + 128;
    const uint4 v = *reinterpret_cast<const uint4 *>(a.h + i * a.ld_h + j);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
        o[q] = pack4(row[sx8(w[q], 0)], row[sx8(w[q], 1)], row[sx8(w[q], 2)], row[sx8(w[q], 3)]);
    *reinterpret_cast<uint4 *>(a.out + i * a.ld_out + j) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Backward: x = dY * LUT_bwd[e_H][C_H] exactly (|x| <= 127 * 72) at exponent e_dY - 6,
// FIT into dH's group (row-local groups shared by H, dY and dH).  One warp per group,
// lanes striding over its 16-byte vectors; the need pass and the rounding pass read the
// group twice (the second time from L1).  Requires g_cols a multiple of 16.
__global__ void __launch_bounds__(256) gelu_lut_bwd_kernel(const __grid_constant__ GeluLutArgs a) {
    __shared__ __align__(16) int8_t lut[kLutRows * 256];
    lut_to_smem(a.lut, lut, kLutRows * 256);
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= a.rows * a.ngc) return;
    const int64_t i = idiv(gw, a.ngc), g = gw - i * a.ngc;
    const int64_t j0 = g * a.g_cols, j1 = min(a.cols, j0 + a.g_cols);
    const int eh = a.h_exp[i * a.ngc + g], ed = a.dy_exp[i * a.ngc + g];
    const int8_t *row = lut + lut_row(eh == kEZero ? 0 : eh) * 256 + 128;
    auto products = [&](int64_t j, int (&x)[16]) {
        const uint4 hv = *reinterpret_cast<const uint4 *>(a.h + i * a.ld_h + j);
        const uint4 dv = *reinterpret_cast<const uint4 *>(a.dy + i * a.ld_dy + j);
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int q = 0; q < 16; ++q) x[q] = sx8(dw[q >> 2], q & 3) * (int)row[sx8(hw[q >> 2], q & 3)];
    };
    int amax = 0;
    for (int64_t j = j0 + 16 * lane; j < j1; j += 512) {
        int x[16];
        products(j, x);
#pragma unroll
        for (int q = 0; q < 16; ++q) amax = max(amax, abs(x[q]));
    }
    amax = warp_max(amax);
    const int r = ed - kGeluBG;
    const int e = finalize_exp(amax ? r + need_off32((uint32_t)amax) : kNoExp);
    const Shift h = make_shift(e == kEZero ? 0 : e - r);
    for (int64_t j = j0 + 16 * lane; j < j1; j += 512) {
        int x[16];
        products(j, x);
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = pack4(apply_shift(x[4 * q], h), apply_shift(x[4 * q + 1], h), apply_shift(x[4 * q + 2], h),
                         apply_shift(x[4 * q + 3], h));
        *reinterpret_cast<uint4 *>(a.out + i * a.ld_out + j) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (lane == 0) a.out_exp[i * a.ngc + g] = (int8_t)e;
}

// ------------------------------------------------------------------ output head

struct HeadArgs {
    const int8_t *z, *z_exp;  // logits [rows][cols], exponent grid of (g_rows, g_cols) groups
    int64_t rows, cols, ld_z;
    int g_rows, g_cols;
    int64_t ngc;
    const int32_t *target;    // [rows], in [0, cols)
    int32_t *loss;            // [rows]: LUT_log[clamp(p_target, 1, 254)], scale 2^-5
    int8_t *dz, *dz_exp;      // gradient of the summed loss, groups (1, gd) per row
    int64_t ld_dz;
    int gd;
    int64_t ngd;
    alignas(16) uint8_t lut_exp[kLutRows * 256];
    uint8_t lut_log[256];
};

// One warp per row of logits:
//   1. e* = the row's largest group exponent; C' = RNE(C 2^(e_g - e*)) (ALIGN_MAX);
//   2. k = C' - max C';  E = LUT_exp[e*][k];  S = sum E  (S >= 128);
//   3. p = RNE(E 2^8 / S) by integer division; loss = LUT_log[clamp(p_t, 1, 254)];
//   4. g = p - 2^8 [j = t] at exponent -8, FIT into each (1, gd) group of dZ.
// The row is read from global memory once per pass (L1 serves the repeats).
__global__ void __launch_bounds__(256) softmax_ce_kernel(const __grid_constant__ HeadArgs a) {
    __shared__ __align__(16) uint8_t lexp[kLutRows * 256];
    __shared__ uint8_t llog[256];
    lut_to_smem(reinterpret_cast<const int8_t *>(a.lut_exp), reinterpret_cast<int8_t *>(lexp), kLutRows * 256);
    if (threadIdx.x < 256) llog[threadIdx.x] = a.lut_log[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t i = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (i >= a.rows) return;
    const int8_t *ze = a.z_exp + idiv(i, a.g_rows) * a.ngc;
    int es = kNoExp;
    for (int64_t g = lane; g < a.ngc; g += 32)
        if (ze[g] != kEZero) es = max(es, (int)ze[g]);
    es = warp_max(es);
    const int erow = es <= kNoExp ? kEZero : es;
    const int8_t *zr = a.z + i * a.ld_z;
    auto aligned = [&](int64_t j) {
        const int e = ze[idiv(j, a.g_cols)];
        const int c = zr[j];
        if (e == kEZero || c == 0) return 0;
        const int d = erow - e;
        return d == 0 ? c : (d >= 8 ? 0 : rne_shr32(c, d));
    };
    int cmax = -128;
    for (int64_t j = lane; j < a.cols; j += 32) cmax = max(cmax, aligned(j));
    cmax = warp_max(cmax);
    const uint8_t *row = lexp + lut_row(erow) * 256 + 255;
    int S = 0;
    for (int64_t j = lane; j < a.cols; j += 32) S += row[aligned(j) - cmax];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    const int t = a.target[i];
    auto grad = [&](int64_t j) {
        const uint32_t num = (uint32_t)row[aligned(j) - cmax] << 8;
        uint32_t q = num / (uint32_t)S;
        const uint32_t rem2 = 2 * (num - q * (uint32_t)S);
        q += (rem2 > (uint32_t)S || (rem2 == (uint32_t)S && (q & 1))) ? 1u : 0u;
        return (int)q - (j == t ? 256 : 0);
    };
    if (lane == 0) {
        const int pt = grad(t) + 256;
        a.loss[i] = llog[pt < 1 ? 1 : (pt > 254 ? 254 : pt)];
    }
    for (int64_t g = 0; g < a.ngd; ++g) {
        const int64_t j0 = g * a.gd, j1 = min(a.cols, j0 + a.gd);
        int amax = 0;
        for (int64_t j = j0 + lane; j < j1; j += 32) amax = max(amax, abs(grad(j)));
        amax = warp_max(amax);
        const int e = finalize_exp(amax ? -8 + need_off32((uint32_t)amax) : kNoExp);
        const Shift h = make_shift(e == kEZero ? 0 : e + 8);
        for (int64_t j = j0 + lane; j < j1; j += 32) a.dz[i * a.ld_dz + j] = (int8_t)apply_shift(grad(j), h);
        if (lane == 0) a.dz_exp[i * a.ngd + g] = (int8_t)e;
    }
}

}  // namespace ict
