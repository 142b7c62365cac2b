// ict_gemm.cuh -- the (C,e) Product on the 5th-generation tensor cores.
//
//   D[m][n] = sum_k A[m][k] * B[n][k]     (int8 x int8 -> int32 in TMEM)
//   exponent(m, n) = eA[m] + eB[n]        (exponent addition of the Product)
//   then FIT into the caller's output groups, fused into the epilogue.
//
// Source: "Memory-Efficient Integer-Only Training of Deep Neural Networks", Table 6
// (convolution, linear and patch embedding are instances of the Product primitive)
// and Figure 1a (forward and backward of every layer in integer arithmetic).
//
// Structure (one CTA per SM, persistent over output tiles, 384 threads):
//   warp 0       TMA producer: A and B K-major tiles into a STAGES-deep ring of
//                swizzled shared-memory buffers (mbarrier full/empty pairs)
//   warp 1       MMA issuer: one thread issues tcgen05.mma kind::i8 (M = 128) into a
//                double-buffered TMEM accumulator; tcgen05.commit frees smem stages
//   warp 2       TMEM allocation / release
//   warps 4..7   epilogue warpgroup 0 (tiles using accumulator 0)
//   warps 8..11  epilogue warpgroup 1 (tiles using accumulator 1)
//                tcgen05.ld (thread = output row), group exponent, RNE shift, int8
//                stores of mantissas and group exponents.
// Epilogue fast path: within one output group the exponent of element (m, n) is
// eA[m] + eB[n]; with d_n = eB[n] - min_group(eB) every accumulator shifted left by d_n
// is exact below 2^30 when the group's spread is small, so the group exponent is
// need(max |x << d_n|) and every mantissa is one RNE shift of x << d_n by a per-row
// amount.  Groups with a larger spread take the exact per-element path.
// Every wait is bounded; on expiry the CTA raises ICT_ERR_DEVICE_TIMEOUT, drains its
// in-flight copies and MMAs (again with a bound), frees TMEM and exits.
#pragma once

#include "ict_device.cuh"

namespace ict {

enum EpiMode : int {
    EPI_FIT_ROW = 0,  // row-local groups (1, G) inside one tile -> int8 + exps
    EPI_I32 = 1,      // raw int32 partials to a workspace slice (split-K)
    EPI_RO16 = 2,     // groups spanning all rows: int16 sums rounded to odd at a per-tile
                      // exponent, the tile's need and the group's running max need
    EPI_RO16R = 3,    // one group per row spanning tiles: int16 sums rounded to odd at the
                      // exponent of the (row, tile part)'s need, and that need
};
// LOAD_2D         A, B: K-major rows from 2-D tensor maps (linear layers)
// LOAD_CONV       A: one filter tap of NHWC activations per K block (4-D box), B: K-major
//                 weight rows (convolution forward / backward-data)
// LOAD_CONV_WGRAD A: two (tap, 64-channel) slices of the shifted NHWC input X, B: 64
//                 channels of dY, both MN-major with output pixels as K (convolution
//                 backward-weight); BK is the largest number of pixels per K block
enum LoadMode : int { LOAD_2D = 0, LOAD_CONV = 1, LOAD_CONV_WGRAD = 2, LOAD_CONV_HALO = 3, LOAD_CONV_RING = 4 };
// LOAD_CONV_HALO  3 x 3 "same" convolutions whose image width is a multiple of 8: per tile
//                 and 64-channel block, three 4-D boxes (one per column shift of the
//                 filter), each holding the tile's rows and one halo row above and below;
//                 every tap's operand is a window of one box starting a whole number of
//                 image rows in (a multiple of the 8-row swizzle atom), so nine taps take
//                 three copies instead of nine.  The weight operand stays resident.
constexpr int kHaloSlot = 16384;  // bytes per box slot (256 rows of 64 bytes)
// LOAD_CONV_RING  the halo form with each CTA taking a contiguous run of tiles (in image
//                 order): the three boxes' image rows live in three rings of kRingBox
//                 bytes; a tile that continues the previous one (same image, next rows)
//                 loads only its new rows after the previous tile's, whose last two rows
//                 are its halo above, and a tile that does not, or that would pass the
//                 ring's end, restarts at the ring's start once the previous tile's MMAs
//                 are done.  Windows read past a tile's rows only for invalid output rows.
constexpr int kRingBox = 36864;

struct GemmParams {
    int M, N;       // output rows (MMA M side) and columns (MMA N side)
    int n_kblk;     // number of BK-wide K blocks
    int n_mtiles, n_ntiles, splits, kblk_per_split, num_units;
    const int8_t *eA;
    int eA_div;     // exponent of output row m: eA[m / eA_div]
    const int8_t *eB;
    int eB_div;     // exponent of output column n: eB[n / eB_div]
    int G;          // output group width along N
    int fast_slack; // groups whose eB spread is at most this take the fast epilogue
    int8_t *out;
    int64_t out_ld;
    int8_t *out_exp;
    int64_t out_exp_ld;
    int32_t *ws32;
    int64_t ws_ld, ws_split_stride;
    // EPI_RO16 (output groups spanning all rows): t = RO(acc * 2^(eA + eB - e1)) as int16
    // into ws16[row][ws16_ld], e1 = tile_need - 7 with tile_need the largest need() of the
    // group's elements in the tile (tile_need[m tile][group column], kNoExp when all are
    // zero), and the running max need of every group column in gmax
    int16_t *ws16;
    int64_t ws16_ld;
    int32_t *tile_need;
    int32_t *gmax;
    // EPI_RO16R: the same int16 form for one group per row spanning several tiles, with the
    // need of each (row, tile part) in tile_need[row * tn_ld + n tile * parts + part]
    int64_t tn_ld;
    // implicit-GEMM convolution: output tile = cv_rows image rows of width cv_W
    int cv_W, cv_P, cv_rows, cv_tiles_per_img, cv_cblk, cv_S, cv_pad, cv_sign;
    // conv: every K block of the weight operand held in shared memory for the whole kernel
    // (block kb at the B ring's slot kb; needs n_kblk <= STAGES); stage_tx_bytes is then A only
    int b_resident;
    // LOAD_CONV_HALO: the weight's K blocks held resident (taps x channel blocks); n_kblk
    // counts the channel blocks, one stage each
    int cv_bkblk;
    // LOAD_CONV_RING: image rows a ring holds, and the rows a tile's windows span from its
    // first row (2 + ceil(128 / W)); tmY is then the map of the continuing tiles' boxes,
    // and tmZ the int16 sums as bytes (128-byte rows, 128-byte swizzle, boxes of a full
    // tile's cv_rows * cv_W rows) for the staged RO16 stores
    int cv_ring_rows, cv_ring_span;
    // backward-weight: K block = wg_hrows image rows of every image (wg_kpix pixels), M rows
    // (tap, channel) in 64-row atoms (wg_atoms in total)
    int wg_hrows, wg_hblk, wg_kpix, wg_atoms;
    uint32_t stage_tx_bytes;
    uint64_t wait_ns, drain_ns;
    int epi;
    int qb;         // mantissa bits B of the FIT (|C| <= 2^(B-1) - 1); 8 for INT8
    int epi_split;  // 1: both epilogue warpgroups share every tile, one half of its columns each
    int nwg;        // host only: epilogue warpgroups of the instantiation to launch (2 or 4)
};

template <int BN, int BK, int STAGES, int NWG = 2, bool PAIR = false, int NACC = NWG, int STAGE = 0, int AB = 0,
          int BSLOTS = 0>
struct GemmSmem {
    static constexpr int kABytes = AB ? AB : 128 * BK;  // A bytes per stage
    static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * BK;  // a pair's CTA holds half of B
    // NACC TMEM accumulators of BN columns
    static constexpr int kTmemCols = (NACC * BN <= 32) ? 32 : (NACC * BN <= 64) ? 64 : (NACC * BN <= 128) ? 128
                                   : (NACC * BN <= 256) ? 256 : 512;
    static_assert(NACC * BN <= 512, "accumulators must fit TMEM");
    static constexpr int kOffB = STAGES * kABytes;
    static constexpr int kBSlots = BSLOTS > STAGES ? BSLOTS : STAGES;  // B slots (a resident weight may need more)
    static constexpr int kOffBar = kOffB + kBSlots * kBBytes;  // 2*STAGES + 2*NACC + 2 mbarriers
    static constexpr int kOffMisc = (kOffBar + (2 * STAGES + 2 * NACC + 2) * 8 + 15) / 16 * 16;
    static constexpr int kColInts = 2 * BN + 32;               // per epilogue warpgroup
    static constexpr int kOffCol = kOffMisc + 16;              // read with 16-byte vectors
    static constexpr int kOffRed = kOffCol + NWG * kColInts * 4;  // [NWG][8 groups][4 warps] row-need maxima
    // STAGE bytes per epilogue warpgroup of output staged for a TMA store (1024-aligned)
    static constexpr int kOffStage = (kOffRed + NWG * 32 * 4 + 1023) / 1024 * 1024;
    static constexpr int kBytes = kOffStage + NWG * STAGE + 1024;  // + alignment slack
    static_assert(kOffCol % 16 == 0 && (kColInts * 4) % 16 == 0 && (BN * 4) % 16 == 0,
                  "column tables are read as int4");
    static_assert(kABytes % 1024 == 0 && kBBytes % 512 == 0 && kOffB % 1024 == 0 && kABytes / 2 <= 16383 * 16,
                  "operand tiles must sit on their swizzle-atom boundaries");
    static_assert(kBytes <= 232448, "shared memory per block");
};


// Fast epilogue of one output group of NC x 32 columns of an accumulator row, the group
// on the fast path: y = acc * 2^d_n (d_n = column shift inside the group, |y| < 2^30),
// the group exponent from max |y|, then one RNE shift.  TMEM is read once (all NC chunks
// issued before a single wait) and the group stays in registers from the largest
// magnitude to the stores.  The multiplies and the high-half multiplies of the rounding
// shift run on the FMA pipe, leaving compares, the rounding bit and the packing to the
// ALU pipe.
// Output stores: straight to global memory, or (TS) into the warpgroup's staging rows,
// 64 bytes per output row with the 16-byte chunks in the TMA store's 64-byte swizzle order
// (chunk ^ ((row >> 1) & 3)), which also keeps the row-per-thread writes free of bank
// conflicts.  scol: the chunk's first column within the warpgroup's staged columns (64, or
// 128 as two 128 x 64 blocks, one TMA store each).
__device__ __forceinline__ void stage16(uint8_t *srow, int et, int scol, uint4 v) {
    *reinterpret_cast<uint4 *>(srow + (scol >> 6) * (128 * 64) + ((((scol >> 4) & 3) ^ ((et >> 1) & 3)) << 4)) = v;
}

template <bool MUL, int NC, bool TS = false>  // MUL = false: every column of the group has the same exponent
__device__ __forceinline__ void epi_fast(const GemmParams &p, uint32_t taddr, const int *colM, int gm,
                                         bool valid, int ea, int64_t grow, int ncol, int gcol,
                                         uint8_t *srow = nullptr, int et = 0, int scol = 0) {
    uint32_t v[32 * NC];
    if constexpr (NC == 2) {
        tmem_ld64(taddr, *reinterpret_cast<uint32_t(*)[64]>(v));
        tmem_ld_wait(*reinterpret_cast<uint32_t(*)[64]>(v));
    } else {
        tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld_wait();
    }
    // four independent max / min chains, so that the reductions overlap
    int hi[4] = {0, 0, 0, 0}, lo[4] = {0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 32 * NC; q += 4) {
        int y0 = (int)v[q], y1 = (int)v[q + 1], y2 = (int)v[q + 2], y3 = (int)v[q + 3];
        if (MUL) {
            const int4 m4 = *reinterpret_cast<const int4 *>(colM + q);
            y0 *= m4.x, y1 *= m4.y, y2 *= m4.z, y3 *= m4.w;
            v[q] = (uint32_t)y0, v[q + 1] = (uint32_t)y1, v[q + 2] = (uint32_t)y2, v[q + 3] = (uint32_t)y3;
        }
        const int c = (q >> 2) & 3;
        hi[c] = max(hi[c], max(max(y0, y1), max(y2, y3)));
        lo[c] = min(lo[c], min(min(y0, y1), min(y2, y3)));
    }
    const int h = max(max(hi[0], hi[1]), max(hi[2], hi[3])), l = min(min(lo[0], lo[1]), min(lo[2], lo[3]));
    const int amax = valid ? max(h, -l) : 0;
    const int need = amax ? ea + gm + need_off32q((uint32_t)amax, p.qb) : kNoExp;
    const int e = finalize_exp(need);
    // mantissa = RNE(y * 2^-S), S = e - ea - gm uniform over the row's group
    const int S = (e == kEZero) ? 0 : e - ea - gm;
    if (ncol < p.N && valid) p.out_exp[grow * p.out_exp_ld + gcol] = (int8_t)e;
    if (__all_sync(0xffffffffu, rne_f32_ok(valid, amax, S, need))) {
        const RneF32 k = rne_f32_consts(S);
        if (TS || valid) {
            int8_t *dst = p.out + grow * p.out_ld + ncol;
#pragma unroll
            for (int q = 0; q < 32 * NC; q += 16) {
                uint32_t r[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) r[t] = rne_f32((int)v[q + t], k);
                const uint4 w = make_uint4(pack4b(r[0], r[1], r[2], r[3]), pack4b(r[4], r[5], r[6], r[7]),
                                           pack4b(r[8], r[9], r[10], r[11]), pack4b(r[12], r[13], r[14], r[15]));
                if (TS) stage16(srow, et, scol + q, w);
                else if (ncol + q < p.N) *reinterpret_cast<uint4 *>(dst + q) = w;
            }
        }
        return;
    }
    if (__any_sync(0xffffffffu, valid && S < 0)) {
        const int lm = S < 0 ? (1 << min(-S, 30)) : 1;
#pragma unroll
        for (int q = 0; q < 32 * NC; ++q) v[q] = (uint32_t)((int)v[q] * lm);
    }
    const int rs = S > 0 ? min(S, 31) : 0;
    if (rs >= 2) {
        const int m = 1 << (32 - rs), bias = (1 << (rs - 1)) - 1;
#pragma unroll
        for (int q = 0; q < 32 * NC; q += 8) {  // eight elements per stage, stage by stage
            int t[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) t[k] = __mulhi((int)v[q + k], m);
#pragma unroll
            for (int k = 0; k < 8; ++k) t[k] = (int)v[q + k] + bias + (t[k] & 1);
#pragma unroll
            for (int k = 0; k < 8; ++k) v[q + k] = (uint32_t)__mulhi(t[k], m);
        }
    } else if (rs == 1) {
#pragma unroll
        for (int q = 0; q < 32 * NC; ++q) {
            const int y = (int)v[q];
            v[q] = (uint32_t)((y + ((y >> 1) & 1)) >> 1);
        }
    }
    if (TS || valid) {
        int8_t *dst = p.out + grow * p.out_ld + ncol;
#pragma unroll
        for (int q = 0; q < 32 * NC; q += 16) {
            const uint4 w = make_uint4(pack4s((int)v[q], (int)v[q + 1], (int)v[q + 2], (int)v[q + 3]),
                                       pack4s((int)v[q + 4], (int)v[q + 5], (int)v[q + 6], (int)v[q + 7]),
                                       pack4s((int)v[q + 8], (int)v[q + 9], (int)v[q + 10], (int)v[q + 11]),
                                       pack4s((int)v[q + 12], (int)v[q + 13], (int)v[q + 14], (int)v[q + 15]));
            if (TS) stage16(srow, et, scol + q, w);
            else if (ncol + q < p.N) *reinterpret_cast<uint4 *>(dst + q) = w;
        }
    }
}

// The same for a group of NCH x 32 columns read from TMEM twice, 32 columns at a time: the
// first pass finds the largest magnitude, the second rounds and stores.  Half the
// registers of the resident form, so that four epilogue warpgroups fit beside the
// producer and MMA warps.
template <bool MUL, int NCH, bool TS = false>
__device__ __forceinline__ void epi_two_pass(const GemmParams &p, uint32_t taddr, const int *colM, int gm,
                                             bool valid, int ea, int64_t grow, int ncol, int gcol,
                                             uint8_t *srow = nullptr, int et = 0, int scol = 0) {
    uint32_t v[32];
    int hi[4] = {0, 0, 0, 0}, lo[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        tmem_ld32(taddr + 32 * c, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
            int y0 = (int)v[q], y1 = (int)v[q + 1], y2 = (int)v[q + 2], y3 = (int)v[q + 3];
            if (MUL) {
                const int4 m4 = *reinterpret_cast<const int4 *>(colM + 32 * c + q);
                y0 *= m4.x, y1 *= m4.y, y2 *= m4.z, y3 *= m4.w;
            }
            const int k = (q >> 2) & 3;
            hi[k] = max(hi[k], max(max(y0, y1), max(y2, y3)));
            lo[k] = min(lo[k], min(min(y0, y1), min(y2, y3)));
        }
    }
    const int h = max(max(hi[0], hi[1]), max(hi[2], hi[3])), l = min(min(lo[0], lo[1]), min(lo[2], lo[3]));
    const int amax = valid ? max(h, -l) : 0;
    const int need = amax ? ea + gm + need_off32q((uint32_t)amax, p.qb) : kNoExp;
    const int e = finalize_exp(need);
    const int S = (e == kEZero) ? 0 : e - ea - gm;
    if (ncol < p.N && valid) p.out_exp[grow * p.out_exp_ld + gcol] = (int8_t)e;
    int8_t *dst = p.out + grow * p.out_ld + ncol;
    if (__all_sync(0xffffffffu, rne_f32_ok(valid, amax, S, need))) {
        const RneF32 k = rne_f32_consts(S);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            tmem_ld32(taddr + 32 * c, v);
            tmem_ld_wait();
            if (TS || valid) {
#pragma unroll
                for (int q = 0; q < 32; q += 16) {
                    uint32_t w4[4];
#pragma unroll
                    for (int t = 0; t < 16; t += 4) {
                        int4 m4 = make_int4(1, 1, 1, 1);
                        if (MUL) m4 = *reinterpret_cast<const int4 *>(colM + 32 * c + q + t);
                        w4[t >> 2] = pack4b(rne_f32((int)v[q + t] * m4.x, k), rne_f32((int)v[q + t + 1] * m4.y, k),
                                            rne_f32((int)v[q + t + 2] * m4.z, k), rne_f32((int)v[q + t + 3] * m4.w, k));
                    }
                    const uint4 w = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    if (TS) stage16(srow, et, scol + 32 * c + q, w);
                    else if (ncol + 32 * c + q < p.N) *reinterpret_cast<uint4 *>(dst + 32 * c + q) = w;
                }
            }
        }
        return;
    }
    const bool any_ls = __any_sync(0xffffffffu, valid && S < 0);
    const int lm = S < 0 ? (1 << min(-S, 30)) : 1;
    const int rs = S > 0 ? min(S, 31) : 0;
    const int m = rs >= 2 ? 1 << (32 - rs) : 0, bias = rs ? (1 << (rs - 1)) - 1 : 0;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        tmem_ld32(taddr + 32 * c, v);
        tmem_ld_wait();
        if (MUL || any_ls) {
#pragma unroll
            for (int q = 0; q < 32; q += 4) {
                int4 m4 = make_int4(lm, lm, lm, lm);
                if (MUL) {
                    const int4 c4 = *reinterpret_cast<const int4 *>(colM + 32 * c + q);
                    m4 = make_int4(c4.x * lm, c4.y * lm, c4.z * lm, c4.w * lm);
                }
                v[q] = (uint32_t)((int)v[q] * m4.x), v[q + 1] = (uint32_t)((int)v[q + 1] * m4.y);
                v[q + 2] = (uint32_t)((int)v[q + 2] * m4.z), v[q + 3] = (uint32_t)((int)v[q + 3] * m4.w);
            }
        }
        if (rs >= 2) {
#pragma unroll
            for (int q = 0; q < 32; q += 8) {
                int t[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) t[k] = __mulhi((int)v[q + k], m);
#pragma unroll
                for (int k = 0; k < 8; ++k) t[k] = (int)v[q + k] + bias + (t[k] & 1);
#pragma unroll
                for (int k = 0; k < 8; ++k) v[q + k] = (uint32_t)__mulhi(t[k], m);
            }
        } else if (rs == 1) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int y = (int)v[q];
                v[q] = (uint32_t)((y + ((y >> 1) & 1)) >> 1);
            }
        }
        if (TS || valid) {
#pragma unroll
            for (int q = 0; q < 32; q += 16) {
                const uint4 w = make_uint4(pack4s((int)v[q], (int)v[q + 1], (int)v[q + 2], (int)v[q + 3]),
                                           pack4s((int)v[q + 4], (int)v[q + 5], (int)v[q + 6], (int)v[q + 7]),
                                           pack4s((int)v[q + 8], (int)v[q + 9], (int)v[q + 10], (int)v[q + 11]),
                                           pack4s((int)v[q + 12], (int)v[q + 13], (int)v[q + 14], (int)v[q + 15]));
                if (TS) stage16(srow, et, scol + 32 * c + q, w);
                else if (ncol + 32 * c + q < p.N) *reinterpret_cast<uint4 *>(dst + 32 * c + q) = w;
            }
        }
    }
}

// OUTK (compile time, an EpiMode): which epilogue is compiled in -- the row-local FIT
// (EPI_FIT_ROW), raw int32 partial sums (EPI_I32), or the int16 round-to-odd sums of
// groups spanning all rows (EPI_RO16) -- so that each kernel keeps a small code footprint
// in the instruction cache.
// GC (compile time, FIT kernels): 1 or 2 when output groups are 32 or 64 columns wide and
// held in registers, 3 when 64-column groups are read from TMEM in two passes (fewer
// registers), so that only that fast path and the exact path are compiled in; 0 for
// other widths.
// NWG (compile time): epilogue warpgroups, each owning one TMEM accumulator (2 or 4).
// PAIR (compile time, LOAD_2D): a cluster of two CTAs computes 256 x BN tiles with
// tcgen05.mma.cta_group::2.  CTA r of the pair loads rows [r 128, r 128 + 128) of the A
// tile and [r BN/2, r BN/2 + BN/2) of the B tile into its own shared memory; both count
// their copies on the first CTA's full barrier, whose MMA thread issues the pair's MMAs
// and commits to both CTAs' barriers; each CTA's epilogue finishes its own 128 rows from
// its own TMEM and arrives on the first CTA's accumulator-empty barrier.  Per SM this
// halves the B bytes per multiply-add of a single-CTA 128 x BN tile.
// Q4 (compile time): four epilogue warpgroups share every tile, one quarter of its columns
// each, over two double-buffered accumulators (else one accumulator per warpgroup).
// With Q4 on pairs (TS), each epilogue warpgroup stages its 128 x 64 share of a tile's
// int8 output in shared memory and one of its threads writes it with a TMA store through
// tmY (the output, 64-byte swizzle, 64 x 128 boxes), instead of 16-byte stores that each
// touch 32 rows.  STG: the same for single CTAs with four warpgroups on alternate 128-wide
// tiles, each staging its whole 128 x 128 tile as two such boxes.
template <int BN, int BK, int STAGES, int LOAD, int OUTK, int GC = 0, int NWG = 2, bool PAIR = false, bool Q4 = false,
          bool STG = false>
__global__ void __launch_bounds__(128 + 128 * NWG, 1)
    gemm_ce_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmZ,
                   const __grid_constant__ GemmParams p) {
    static_assert(!Q4 || NWG == 4, "Q4: four epilogue warpgroups");
    // staged output: pairs with Q4 (64 columns per warpgroup), and single CTAs with four
    // warpgroups on alternate 128-wide tiles of 32-column groups (128 columns per warpgroup)
    constexpr bool TS1 = STG;
    static_assert(!STG || (!PAIR && !Q4 && NWG == 4 && BN == 128 && GC == 1 && LOAD == LOAD_2D && OUTK == EPI_FIT_ROW),
                  "staged single-CTA output: four warpgroups, 128-wide tiles of 32-column groups");
    constexpr bool TS = (PAIR && Q4 && OUTK == EPI_FIT_ROW) || TS1;
    constexpr int SCOLS = TS1 ? 128 : 64;  // staged columns per warpgroup
    static_assert(!TS || BN == 256 || TS1, "staged stores: 64 columns per warpgroup");
    constexpr bool RING = LOAD == LOAD_CONV_RING;
    constexpr bool HALO = LOAD == LOAD_CONV_HALO || RING;
    static_assert(!HALO || (BK == 64 && !PAIR), "halo tiles: 64-byte channel rows, single CTAs");
    static_assert(!RING || (3 * kRingBox) % STAGES == 0, "ring: the A region split evenly over the stages");
    // RING with RO16: each epilogue warpgroup stages its tile's int16 sums (128 rows of 128
    // bytes, 128-byte swizzle) for one TMA store instead of row-per-thread 16-byte stores
    constexpr bool TS16 = RING && OUTK == EPI_RO16 && NWG == 4 && BN == 64;
    using L = GemmSmem<BN, BK, STAGES, NWG, PAIR, Q4 ? 2 : NWG, TS ? 128 * SCOLS : (TS16 ? 128 * 128 : 0),
                       RING ? 3 * kRingBox / STAGES : (HALO ? 3 * kHaloSlot : 0), HALO ? 9 : 0>;
    static_assert(!PAIR || (LOAD == LOAD_2D && BN % 64 == 0), "pairs: 2-D loads, BN a multiple of 64");
    constexpr int TM = PAIR ? 256 : 128;  // rows of an output tile
    constexpr int NACC = Q4 ? 2 : NWG;
    // warpgroups sharing one tile (each takes a contiguous share of its columns)
    const int wpt = Q4 ? 4 : (p.epi_split ? 2 : 1);
    constexpr bool I32 = OUTK == EPI_I32, RO16 = OUTK == EPI_RO16, RO16R = OUTK == EPI_RO16R;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
    static_assert(BK == 128 || BK == 64 || (BK == 256 && LOAD == LOAD_CONV_WGRAD), "BK");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + L::kOffBar;           // [STAGES]
    const uint32_t bar_empty = bar_full + 8 * STAGES;       // [STAGES]
    const uint32_t bar_tfull = bar_empty + 8 * STAGES;      // [NACC]
    const uint32_t bar_tempty = bar_tfull + 8 * NACC;       // [NACC]
    const uint32_t bar_drain = bar_tempty + 8 * NACC;       // [1]
    const uint32_t bar_bres = bar_drain + 8;                // [1] resident weight operand landed
    volatile int *misc = (volatile int *)(smem + L::kOffMisc);  // [0] tmem base, [1] abort
    int *sCol = (int *)(smem + L::kOffCol);  // per epilogue warpgroup column tables
    int *sRed = (int *)(smem + L::kOffRed);  // per warpgroup: [group][warp] row-need maxima (RO16)
    uint8_t *sStage = smem + L::kOffStage;  // TS: per warpgroup, 128 rows x 64 bytes of output

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // pairs: this CTA's rank r and the pair's index; units advance pair by pair
    const uint32_t rank = PAIR ? cluster_ctarank() : 0;
    const bool leader = rank == 0;
    const int cta0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int ctas = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    // RING: the k-th unit of this CTA (u = cta0 + k ctas) is tile ring0 + k, so that its
    // tiles are contiguous (the same count of units as the strided walk)
    const int ring0 = RING ? cta0 * (p.num_units / ctas) + min(cta0, p.num_units % ctas) : 0;
    // ring position of a tile given the previous tile's (the same walk in producer and MMA)
    auto ring_pos = [&](int mt, int &pos, int &pimg, int &ph0, bool &cont) {
        const int img = mt / p.cv_tiles_per_img, h0 = (mt % p.cv_tiles_per_img) * p.cv_rows;
        cont = img == pimg && h0 == ph0 + p.cv_rows && pos + p.cv_rows + p.cv_ring_span <= p.cv_ring_rows;
        pos = cont ? pos + p.cv_rows : 0;
        pimg = img, ph0 = h0;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(bar_tfull + 8 * a, 1);
            // pairs: one local arrival per epilogue warpgroup that handles the tile, and on
            // the first CTA one more, forwarded from the second CTA's barrier
            mbar_init(bar_tempty + 8 * a, PAIR ? (leader ? wpt + 1 : wpt) : 128 * wpt);
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_bres, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (TS || RING) prefetch_tmap(&tmY);
        if (TS16) prefetch_tmap(&tmZ);
    }
    if (warp == 2) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_u32((const void *)&misc[0]), L::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32((const void *)&misc[0]), L::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();  // both CTAs' barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = (uint32_t)misc[0];
    volatile int *abort_flag = &misc[1];

    auto fail = [&]() {
        *abort_flag = 1;
        raise_status(ICT_ERR_DEVICE_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued[STAGES];
            uint32_t issued_phase[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = 0, issued_phase[s] = 0;
            const bool bres = (LOAD == LOAD_CONV || HALO) && p.b_resident;
            if (bres && blockIdx.x < p.num_units) {  // the weight operand, once
                const int nb = HALO ? p.cv_bkblk : p.n_kblk;
                mbar_expect_tx(bar_bres, (uint32_t)(nb * L::kBBytes));
                for (int kb = 0; kb < nb; ++kb)
                    tma_load_2d(sbase + L::kOffB + kb * L::kBBytes, &tmB, bar_bres, kb * BK, 0);
            }
            int r_pos = 0, r_img = -1, r_h0 = -1000000, prev_stage = -1;
            uint32_t prev_phase = 0;
            for (int u = cta0; u < p.num_units && !*abort_flag; u += ctas) {
                const int tile = RING ? ring0 + (u - cta0) / ctas : u % (p.n_mtiles * p.n_ntiles);
                const int split = RING ? 0 : u / (p.n_mtiles * p.n_ntiles);
                const int mt = tile / p.n_ntiles, nt = tile % p.n_ntiles;
                const int kb0 = split * p.kblk_per_split;
                const int kb1 = min(p.n_kblk, kb0 + p.kblk_per_split);
                int img = 0, h0 = 0;
                if (LOAD == LOAD_CONV || HALO) {
                    img = mt / p.cv_tiles_per_img;
                    h0 = (mt % p.cv_tiles_per_img) * p.cv_rows;
                }
                bool r_cont = false;
                if constexpr (RING) {
                    ring_pos(mt, r_pos, r_img, r_h0, r_cont);
                    // a restart overwrites rows that earlier tiles read: wait until the
                    // previous tile's MMAs (and so all earlier ones) are done
                    if (!r_cont && prev_stage >= 0 &&
                        !mbar_wait(bar_empty + 8 * prev_stage, prev_phase, p.wait_ns, abort_flag)) {
                        fail();
                        break;
                    }
                }
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, p.wait_ns, abort_flag)) {
                        fail();
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t sa = sbase + stage * L::kABytes;
                    const uint32_t sb = sbase + L::kOffB + stage * L::kBBytes;
                    if (LOAD == LOAD_2D && PAIR) {
                        // both CTAs' copies complete on the first CTA's full barrier, whose
                        // one arrival (with the pair's byte count) comes from that CTA
                        const uint32_t fb0 = mapa_shared(fb, 0);
                        if (leader) mbar_expect_tx(fb, p.stage_tx_bytes);
                        tma_load_2d_pair(sa, &tmA, fb0, kb * BK, mt * TM + (int)rank * 128);
                        tma_load_2d_pair(sb, &tmB, fb0, kb * BK, nt * BN + (int)rank * (BN / 2));
                    } else if (LOAD == LOAD_2D) {
                        mbar_expect_tx(fb, p.stage_tx_bytes);
                        tma_load_2d(sa, &tmA, fb, kb * BK, mt * 128);
                        tma_load_2d(sb, &tmB, fb, kb * BK, nt * BN);
                    } else if (RING) {
                        // rows h0 - 1 .. h0 + rows at ring rows r_pos .. (a restart), or only the
                        // new rows h0 + 1 .. h0 + rows after the previous tile's (a continuation)
                        const int nrows = r_cont ? p.cv_rows : p.cv_rows + 2;
                        const int drow = r_cont ? r_pos + 2 : r_pos, hsrc = r_cont ? h0 + 1 : h0 - 1;
                        mbar_expect_tx(fb, (uint32_t)(3 * nrows * p.cv_W * 64));
                        for (int s2 = 0; s2 < 3; ++s2)
                            tma_load_4d(sbase + s2 * kRingBox + drow * p.cv_W * 64, r_cont ? &tmY : &tmA, fb, kb * 64,
                                        p.cv_sign * (s2 - p.cv_pad), hsrc, img);
                    } else if (HALO) {
                        // three boxes (column shifts s - pad) of rows [hs, hs + rows + 2): every
                        // row shift r - pad is a window of them (the MMA's descriptor offset)
                        mbar_expect_tx(fb, p.stage_tx_bytes);
                        const int hs = p.cv_sign > 0 ? h0 - p.cv_pad : h0 + p.cv_pad - (p.cv_S - 1);
                        for (int s2 = 0; s2 < p.cv_S; ++s2)
                            tma_load_4d(sa + s2 * kHaloSlot, &tmA, fb, kb * 64, p.cv_sign * (s2 - p.cv_pad), hs, img);
                    } else if (LOAD == LOAD_CONV) {
                        mbar_expect_tx(fb, p.stage_tx_bytes);
                        const int tap = kb / p.cv_cblk, cb = kb % p.cv_cblk;
                        const int r = tap / p.cv_S, s = tap % p.cv_S;
                        tma_load_4d(sa, &tmA, fb, cb * 64, p.cv_sign * (s - p.cv_pad),
                                    h0 + p.cv_sign * (r - p.cv_pad), img);
                        if (!bres) tma_load_2d(sb, &tmB, fb, kb * BK, nt * BN);
                    } else {
                        // pixels of this K block: rows h1 .. h1 + hrows - 1 of image img1
                        const int img1 = kb / p.wg_hblk, h1 = (kb % p.wg_hblk) * p.wg_hrows;
                        const int a0 = 2 * mt, na = a0 + 1 < p.wg_atoms ? 2 : 1;
                        mbar_expect_tx(fb, (uint32_t)((na + 1) * p.wg_kpix * 64));
                        for (int q = 0; q < na; ++q) {
                            const int tap = (a0 + q) / p.cv_cblk, cb = (a0 + q) % p.cv_cblk;
                            const int r = tap / p.cv_S, s = tap % p.cv_S;
                            tma_load_4d(sa + q * (L::kABytes / 2), &tmA, fb, cb * 64, s - p.cv_pad,
                                        h1 + r - p.cv_pad, img1);
                        }
                        tma_load_4d(sb, &tmB, fb, nt * 64, 0, h1, img1);
                    }
                    issued[stage] = 1;
                    issued_phase[stage] = phase;
                    prev_stage = stage, prev_phase = phase;
                    if (++stage == STAGES) stage = 0, phase ^= 1;
                }
            }
            // drain: every issued copy must land before the CTA may exit (pairs: the first
            // CTA's full barriers count both CTAs' copies, and the second CTA stays until
            // the closing cluster barrier, which the first passes only after this drain)
            for (int s = 0; s < STAGES && leader; ++s)
                if (issued[s]) mbar_wait(bar_full + 8 * s, issued_phase[s], p.drain_ns, nullptr);
            if (bres && blockIdx.x < p.num_units) mbar_wait(bar_bres, 0, p.drain_ns, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && leader) {  // pairs: the first CTA issues the pair's MMAs
            constexpr bool kMN = LOAD == LOAD_CONV_WGRAD;  // both operands MN-major
            constexpr uint32_t kIdesc = idesc_i8(TM, BN, kMN, kMN);
            // pairs: the second CTA's barrier at the same offset, as a shared::cluster address
            const uint32_t peer_off = PAIR ? mapa_shared(sbase, 1) - sbase : 0;
            const int kk_per_blk = kMN ? p.wg_kpix / 32 : BK / 32;
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool any = false;
            if ((LOAD == LOAD_CONV || HALO) && p.b_resident && blockIdx.x < p.num_units &&
                !mbar_wait(bar_bres, 0, p.wait_ns, abort_flag))
                fail();
            int r_pos = 0, r_img = -1, r_h0 = -1000000;
            for (int u = cta0; u < p.num_units && !*abort_flag; u += ctas, ++it) {
                const int split = RING ? 0 : u / (p.n_mtiles * p.n_ntiles);
                bool r_cont = false;
                if constexpr (RING) ring_pos(ring0 + (u - cta0) / ctas, r_pos, r_img, r_h0, r_cont);
                const int kb0 = split * p.kblk_per_split;
                const int kb1 = min(p.n_kblk, kb0 + p.kblk_per_split);
                const int acc = it % NACC;
                if (!mbar_wait(bar_tempty + 8 * acc, ((it / NACC) & 1) ^ 1, p.wait_ns, abort_flag)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t tmem_d = tmem_base + acc * BN;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, p.wait_ns, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if constexpr (HALO) {
                        // tap (r, s): box s, starting (r or R - 1 - r) image rows in; B block
                        // (tap, channel block kb) of the resident weight
                        const uint32_t sa0 = RING ? sbase + r_pos * p.cv_W * 64 : sbase + stage * L::kABytes;
                        const int slot = RING ? kRingBox : kHaloSlot;
                        for (int r = 0; r < p.cv_S; ++r) {
                            const int rr = p.cv_sign > 0 ? r : p.cv_S - 1 - r;
                            for (int s2 = 0; s2 < p.cv_S; ++s2) {
                                const uint64_t da = smem_desc_kmajor(sa0 + s2 * slot + rr * p.cv_W * 64, BK);
                                const int bkb = (r * p.cv_S + s2) * p.cv_cblk + kb;
                                const uint64_t db = smem_desc_kmajor(sbase + L::kOffB + bkb * L::kBBytes, BK);
#pragma unroll
                                for (int kk = 0; kk < BK / 32; ++kk)
                                    umma_i8(tmem_d, da + 2 * kk, db + 2 * kk, kIdesc,
                                            (kb > kb0 || r > 0 || s2 > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                    } else if constexpr (kMN) {
                        // 32 pixels per MMA = four 8-row atoms of 64 bytes = 2048 bytes
                        const uint64_t da = smem_desc_mnmajor64(sbase + stage * L::kABytes, L::kABytes / 2);
                        const uint64_t db = smem_desc_mnmajor64(sbase + L::kOffB + stage * L::kBBytes, L::kABytes / 2);
                        for (int kk = 0; kk < kk_per_blk; ++kk)
                            umma_i8(tmem_d, da + 128 * kk, db + 128 * kk, kIdesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                    } else {
                        const uint64_t da = smem_desc_kmajor(sbase + stage * L::kABytes, BK);
                        const int bslot = (LOAD == LOAD_CONV && p.b_resident) ? kb : stage;
                        const uint64_t db = smem_desc_kmajor(sbase + L::kOffB + bslot * L::kBBytes, BK);
#pragma unroll
                        for (int kk = 0; kk < BK / 32; ++kk) {
                            if constexpr (PAIR)
                                umma_i8_pair(tmem_d, da + 2 * kk, db + 2 * kk, kIdesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                            else
                                umma_i8(tmem_d, da + 2 * kk, db + 2 * kk, kIdesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    any = true;
                    if constexpr (PAIR) {  // both CTAs' stages are free once the MMAs are done
                        umma_commit_pair(bar_empty + 8 * stage);
                        umma_commit_pair(bar_empty + 8 * stage + peer_off);
                    } else {
                        umma_commit(bar_empty + 8 * stage);
                    }
                    if (++stage == STAGES) stage = 0, phase ^= 1;
                }
                if (!ok) break;
                if constexpr (PAIR) {
                    umma_commit_pair(bar_tfull + 8 * acc);
                    umma_commit_pair(bar_tfull + 8 * acc + peer_off);
                } else {
                    umma_commit(bar_tfull + 8 * acc);
                }
            }
            if (any) {  // drain: all issued MMAs complete before TMEM is released
                if constexpr (PAIR) umma_commit_pair(bar_drain);
                else umma_commit(bar_drain);
                mbar_wait(bar_drain, 0, p.drain_ns, nullptr);
            }
        }
    } else if (PAIR && warp == 3) {
        // ------------------------------------------------------------ release forwarder
        // second CTA of a pair: once all of its epilogue warpgroups have released an
        // accumulator (its local barrier's phase for that tile), one remote arrival tells
        // the first CTA, whose MMA thread waits for it with its own warpgroups' arrivals
        if (!leader && lane == 0) {
            int it = 0;
            for (int u = cta0; u < p.num_units && !*abort_flag; u += ctas, ++it) {
                const int acc = it % NACC;
                if (!mbar_wait(bar_tempty + 8 * acc, (it / NACC) & 1, p.wait_ns, abort_flag)) {
                    fail();
                    break;
                }
                mbar_arrive_cluster(mapa_shared(bar_tempty + 8 * acc, 0));
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int wg = (warp - 4) >> 2;           // warpgroup (alternating tiles, or one column half)
        const int et = (threadIdx.x & 127);       // output row within the tile = TMEM lane
        const int quarter = warp & 3, wq = (warp - 4) & 3;
        const int bar_id = 1 + wg;
        int *colE = sCol + wg * L::kColInts;       // [BN] exponent of B row (output column)
        int *colD = colE + BN;                     // [BN] shift of the column in its group
        int *gmin = colD + BN;                     // [8]  min column exponent of each group
        int *gfast = gmin + 8;                     // [8]  group takes the fast path
        const int Gt = p.G >= p.N ? BN : p.G;      // group width inside the tile
        const int ngroups = BN / Gt;
        // the warpgroups form NWG / wpt streams of tiles; within a stream each of the wpt
        // warpgroups takes groups [g_lo, g_hi) (columns [c_lo, c_hi)) of every tile
        const int streams = NWG / wpt, stream = wg / wpt, part = wg % wpt;
        const int g_lo = part * (ngroups / wpt), g_hi = g_lo + ngroups / wpt;
        const int c_lo = part * (BN / wpt), c_hi = c_lo + BN / wpt;
        const int u_step = streams * ctas, it_step = streams;
        int it = stream;
        // The loop never tests the abort flag on its own: the 128 threads decide together
        // through a barrier reduction, so none of them can be left waiting at a barrier.
        // Units are visited as u0, u0 + u_step, ...: their (split, m tile, n tile) advance
        // incrementally, with no division per tile.
        const int NT = p.n_ntiles, MT = p.n_mtiles, T = MT * NT;
        const int u0 = cta0 + stream * ctas;
        // RING (one N tile, no split): the walk's units are tiles ring0 + k
        const int d_split = RING ? 0 : u_step / T, d_m = RING ? streams : (u_step % T) / NT;
        const int d_n = RING ? 0 : (u_step % T) % NT;
        int c_split = RING ? 0 : u0 / T, c_mt = RING ? ring0 + stream : (u0 % T) / NT;
        int c_nt = RING ? 0 : (u0 % T) % NT;  // unit being prefetched
        // group of a tile column: shift for power-of-two widths (Gt == BN: always group 0)
        const int gsh = (Gt & (Gt - 1)) == 0 ? __ffs(Gt) - 1 : -1;
        auto group_of = [&](int j) { return gsh >= 0 ? j >> gsh : j / Gt; };
        // The exponents a tile needs (two column exponents and one row exponent per
        // thread) are loaded one tile ahead, so that their latency hides behind the
        // previous tile's epilogue.
        int pf_e0 = kEZero, pf_e1 = kEZero, pf_ea = 0, pf_split = 0, pf_vr = 0, pf_n0 = 0, pf_mt = 0;
        int64_t pf_rb = 0;
        auto prefetch = [&](bool have) {
            if (!have) return;
            pf_mt = c_mt;
            if (LOAD == LOAD_CONV || HALO) {
                const int img = c_mt / p.cv_tiles_per_img;
                const int h0 = (c_mt % p.cv_tiles_per_img) * p.cv_rows;
                pf_rb = ((int64_t)img * p.cv_P + h0) * p.cv_W;
                pf_vr = min(p.cv_rows, p.cv_P - h0) * p.cv_W;
            } else {
                pf_rb = (int64_t)c_mt * TM + rank * 128;  // pairs: this CTA's half of the tile
                pf_vr = max(0, min(128, p.M - (int)pf_rb));
            }
            pf_n0 = c_nt * BN;
            pf_split = c_split;
            const int n_a = pf_n0 + et, n_b = pf_n0 + et + 128;
            pf_e0 = (et < BN && n_a < p.N) ? (int)p.eB[p.eB_div == 1 ? n_a : n_a / p.eB_div] : kEZero;
            pf_e1 = (et + 128 < BN && n_b < p.N) ? (int)p.eB[p.eB_div == 1 ? n_b : n_b / p.eB_div] : kEZero;
            const int64_t r = pf_rb + et;
            pf_ea = et < pf_vr ? (int)p.eA[p.eA_div == 1 ? r : r / p.eA_div] : 0;
            // advance the cursor to the unit after this one
            c_nt += d_n;
            if (c_nt >= NT) c_nt -= NT, ++c_mt;
            c_mt += d_m;
            if (c_mt >= MT) c_mt -= MT, ++c_split;
            c_split += d_split;
        };
        int *cmin = gfast + 8, *cmax = cmin + 8;  // [8] per 32-column chunk of the tile
        prefetch(u0 < p.num_units);
        for (int u = u0; u < p.num_units; u += u_step, it += it_step) {
            const int acc = it % NACC;
            const int64_t row_base = pf_rb;
            const int valid_rows = pf_vr, n0 = pf_n0, split = pf_split, mt = pf_mt;
            const int e0 = pf_e0, e1 = pf_e1, ea_pf = pf_ea;
            prefetch(u + u_step < p.num_units);
            // column tables of this tile (independent of the accumulator: built before waiting)
            if (et < BN) colE[et] = e0;
            if (et + 128 < BN) colE[et + 128] = e1;
            {   // min / max column exponent of each 32-column chunk (E_ZERO columns ignored)
                const int lo0 = __reduce_min_sync(0xffffffffu, e0 == kEZero ? 0x7fffffff : e0);
                const int hi0 = __reduce_max_sync(0xffffffffu, e0 == kEZero ? kNoExp : e0);
                const int lo1 = __reduce_min_sync(0xffffffffu, e1 == kEZero ? 0x7fffffff : e1);
                const int hi1 = __reduce_max_sync(0xffffffffu, e1 == kEZero ? kNoExp : e1);
                if (lane == 0) {
                    cmin[wq] = lo0, cmax[wq] = hi0;
                    if (BN > 128) cmin[4 + wq] = lo1, cmax[4 + wq] = hi1;
                }
            }
            if ((TS || TS16) && et == 0) bulk_wait_read();  // the previous tile's store has read the staging rows
            named_bar_sync(bar_id, 128);
            auto group_range = [&](int g, int &lo, int &hi) {
                lo = 0x7fffffff, hi = kNoExp;
                const int k0 = (g * Gt) >> 5, k1 = ((g + 1) * Gt) >> 5;
                for (int k = k0; k < k1; ++k) lo = min(lo, cmin[k]), hi = max(hi, cmax[k]);
            };
            if (et < ngroups) {
                int lo, hi;
                group_range(et, lo, hi);
                gmin[et] = hi <= kNoExp ? 0 : lo;
                // 2: every column has the same exponent (no column shifts); 1: fast path
                gfast[et] = (hi <= kNoExp || hi == lo) ? 2 : (hi - lo <= p.fast_slack ? 1 : 0);
            }
            for (int j = et; j < BN; j += 128) {  // 2^d of each column (fast groups: d <= 30)
                int lo, hi;
                group_range(group_of(j), lo, hi);
                const int e = j == et ? e0 : e1;
                const int d = (e == kEZero || hi <= kNoExp) ? 0 : e - lo;
                colD[j] = d <= 30 ? 1 << d : 0;
            }
            const bool ok = mbar_wait(bar_tfull + 8 * acc, (it / NACC) & 1, p.wait_ns, abort_flag);
            if (!ok) fail();
            if (named_bar_or(bar_id, 128, !ok || *abort_flag)) break;  // also publishes the tables
            tc_fence_after();

            const bool valid = et < valid_rows;
            uint8_t *srow = sStage + wg * (128 * SCOLS) + et * 64;  // TS: this thread's staged output row
            const int64_t grow = row_base + et;
            const int ea = valid ? ea_pf : 0;
            const int gcol0 = n0 / p.G;  // output group of the tile's first column
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
            uint32_t v[32];

            if constexpr (I32) {
                int32_t *dst = p.ws32 + split * p.ws_split_stride + grow * p.ws_ld + n0;
                for (int c = c_lo; c < c_hi; c += 32) {
                    tmem_ld32(taddr + c, v);
                    tmem_ld_wait();
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            if (n0 + c + 4 * q < p.N)
                                *reinterpret_cast<uint4 *>(dst + c + 4 * q) =
                                    make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
            } else if constexpr (RO16R) {
                // One group per row spanning several tiles.  Pass A: the row's largest
                // need() over this warpgroup's columns of the tile (thread-local: the thread
                // owns the row).  Pass B: every sum rounded to odd at e1 = that need - 7 as
                // int16 (|t| < 127.5 * 2^7); the streaming pass takes the row's largest need
                // over all parts as the group exponent e >= e1 + 7, and its RNE by e - e1 >= 2
                // bits equals RNE of the exact sum (Boldo and Melquiond, as for RO16).
                const int gf = gfast[0];
                int need = kNoExp;
                for (int c = c_lo; c < c_hi; c += 32) {
                    tmem_ld32(taddr + c, v);
                    tmem_ld_wait();
                    if (!valid || n0 + c >= p.N) continue;
                    if (gf) {
                        int ymax = 0, ymin = 0;
#pragma unroll
                        for (int q = 0; q < 32; q += 4) {
                            const int4 d4 = gf == 2 ? make_int4(1, 1, 1, 1) : *reinterpret_cast<const int4 *>(colD + c + q);
                            const int y0 = (int)v[q] * d4.x, y1 = (int)v[q + 1] * d4.y;
                            const int y2 = (int)v[q + 2] * d4.z, y3 = (int)v[q + 3] * d4.w;
                            ymax = max(ymax, max(max(y0, y1), max(y2, y3)));
                            ymin = min(ymin, min(min(y0, y1), min(y2, y3)));
                        }
                        const int amax = max(ymax, -ymin);
                        if (amax) need = max(need, ea + gmin[0] + need_off32q((uint32_t)amax, p.qb));
                    } else {
#pragma unroll 8
                        for (int q = 0; q < 32; ++q) {
                            const int32_t x = (int32_t)v[q];
                            if (x) need = max(need, ea + colE[c + q] + need_off32q((uint32_t)(x < 0 ? -x : x), p.qb));
                        }
                    }
                }
                if (valid) p.tile_need[grow * p.tn_ld + (n0 / BN) * wpt + part] = need;
                const int e1 = need - 7;
                auto ro = [](int y, int s) {  // floor(y / 2^s) with the sticky bit ORed in
                    if (s <= 0) return y << min(-s, 31);
                    s = min(s, 31);
                    return (y >> s) | (int)((y & ((1 << s) - 1)) != 0);
                };
                for (int c = c_lo; c < c_hi; c += 32) {
                    tmem_ld32(taddr + c, v);
                    tmem_ld_wait();
                    if (!valid || n0 + c >= p.N) continue;
                    uint32_t w[16];
                    if (need <= kNoExp) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) w[q] = 0u;
                    } else if (gf) {
                        const int s = e1 - ea - gmin[0];  // uniform over the row
#pragma unroll
                        for (int q = 0; q < 32; q += 2) {
                            const int m0 = gf == 2 ? 1 : colD[c + q], m1 = gf == 2 ? 1 : colD[c + q + 1];
                            w[q >> 1] = __byte_perm((uint32_t)ro((int)v[q] * m0, s), (uint32_t)ro((int)v[q + 1] * m1, s), 0x5410);
                        }
                    } else {
#pragma unroll 4
                        for (int q = 0; q < 32; q += 2)
                            w[q >> 1] = __byte_perm((uint32_t)ro((int)v[q], e1 - ea - colE[c + q]),
                                                    (uint32_t)ro((int)v[q + 1], e1 - ea - colE[c + q + 1]), 0x5410);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.ws16 + grow * p.ws16_ld + n0 + c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                }
            } else if constexpr (RO16) {
                // Groups spanning all rows.  Pass A: the largest need() of each group over
                // the tile's rows (row maxima, then warp maxima into sRed, then the four
                // warps').  Pass B: every sum rounded to odd at e1 = tile need - 7, so that
                // |t| < 127.5 * 2^7 fits int16 and the final rounding, a right shift by
                // e_group - e1 >= 7 >= 2 bits, equals RNE of the exact sum (rounding to odd
                // with two or more extra bits and then to nearest is correct rounding:
                // Boldo and Melquiond, IEEE Trans. Computers 57(4), 2008).
                int *red = sRed + wg * 32;
                // staged stores for whole tiles only: a box of cv_rows * cv_W rows must not reach
                // the next tile's pixels
                const bool st16 = TS16 && valid_rows == p.cv_rows * p.cv_W;
                for (int g = g_lo; g < g_hi; ++g) {
                    const int g0 = g * Gt, gf = gfast[g];
                    int need = kNoExp;
                    if (gf) {
                        int ymax = 0, ymin = 0;
                        for (int c = g0; c < g0 + Gt; c += 32) {
                            tmem_ld32(taddr + c, v);
                            tmem_ld_wait();
                            if (valid) {
#pragma unroll
                                for (int q = 0; q < 32; q += 4) {
                                    const int4 d4 = gf == 2 ? make_int4(1, 1, 1, 1) : *reinterpret_cast<const int4 *>(colD + c + q);
                                    const int y0 = (int)v[q] * d4.x, y1 = (int)v[q + 1] * d4.y;
                                    const int y2 = (int)v[q + 2] * d4.z, y3 = (int)v[q + 3] * d4.w;
                                    ymax = max(ymax, max(max(y0, y1), max(y2, y3)));
                                    ymin = min(ymin, min(min(y0, y1), min(y2, y3)));
                                }
                            }
                        }
                        const int amax = max(ymax, -ymin);
                        if (amax) need = ea + gmin[g] + need_off32((uint32_t)amax);
                    } else {
                        for (int c = g0; c < g0 + Gt; c += 32) {
                            tmem_ld32(taddr + c, v);
                            tmem_ld_wait();
                            if (valid) {
#pragma unroll 8
                                for (int q = 0; q < 32; ++q) {
                                    const int32_t x = (int32_t)v[q];
                                    if (x) need = max(need, ea + colE[c + q] + need_off32((uint32_t)(x < 0 ? -x : x)));
                                }
                            }
                        }
                    }
                    need = warp_max(need);
                    if (lane == 0) red[g * 4 + wq] = need;
                }
                named_bar_sync(bar_id, 128);
                for (int g = g_lo; g < g_hi; ++g) {
                    const int g0 = g * Gt, gf = gfast[g], gcol = gcol0 + g;
                    const int tneed = max(max(red[g * 4], red[g * 4 + 1]), max(red[g * 4 + 2], red[g * 4 + 3]));
                    if (et == 0 && n0 + g0 < p.N) {
                        p.tile_need[(int64_t)mt * p.out_exp_ld + gcol] = tneed;
                        if (tneed > kNoExp) atomicMax(p.gmax + gcol, tneed);
                    }
                    const int e1 = tneed - 7;
                    // round to odd: floor(y / 2^s) with the sticky bit ORed into the last place
                    auto ro = [](int y, int s) {
                        if (s <= 0) return y << min(-s, 31);
                        s = min(s, 31);
                        return (y >> s) | (int)((y & ((1 << s) - 1)) != 0);
                    };
                    for (int c = g0; c < g0 + Gt; c += 32) {
                        tmem_ld32(taddr + c, v);
                        tmem_ld_wait();
                        if (!valid || n0 + c >= p.N) continue;
                        uint32_t w[16];
                        if (tneed <= kNoExp) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) w[q] = 0u;
                        } else if (gf) {
                            const int s = e1 - ea - gmin[g];  // uniform over the row's group
#pragma unroll
                            for (int q = 0; q < 32; q += 2) {
                                const int m0 = gf == 2 ? 1 : colD[c + q], m1 = gf == 2 ? 1 : colD[c + q + 1];
                                w[q >> 1] = __byte_perm((uint32_t)ro((int)v[q] * m0, s), (uint32_t)ro((int)v[q + 1] * m1, s), 0x5410);
                            }
                        } else {
#pragma unroll 4
                            for (int q = 0; q < 32; q += 2)
                                w[q >> 1] = __byte_perm((uint32_t)ro((int)v[q], e1 - ea - colE[c + q]),
                                                        (uint32_t)ro((int)v[q + 1], e1 - ea - colE[c + q + 1]), 0x5410);
                        }
                        if (TS16 && st16) {  // 16-byte chunk k of the row at (k ^ (row & 7)) * 16
                            uint8_t *srow16 = sStage + wg * (128 * 128) + et * 128;
                            const int k0 = (c - c_lo) >> 3;
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                *reinterpret_cast<uint4 *>(srow16 + (((k0 + q) ^ (et & 7)) << 4)) =
                                    make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(p.ws16 + grow * p.ws16_ld + n0 + c);
#pragma unroll
                            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                        }
                    }
                }
            } else {
                for (int g = g_lo; g < g_hi; ++g) {
                    const int g0 = g * Gt;
                    const int gcol = gcol0 + g;
                    const int gf = gfast[g];
                    if (GC == 3 && gf) {  // 64-column groups, two passes over TMEM
                        if (gf == 2)
                            epi_two_pass<false, 2, TS>(p, taddr + g0, colD + g0, gmin[g], valid, ea, grow, n0 + g0, gcol,
                                                       srow, et, g0 - c_lo);
                        else
                            epi_two_pass<true, 2, TS>(p, taddr + g0, colD + g0, gmin[g], valid, ea, grow, n0 + g0, gcol,
                                                      srow, et, g0 - c_lo);
                        continue;
                    }
                    if (GC && GC < 3 && gf) {
                        constexpr int NC = GC > 0 && GC < 3 ? GC : 1;
                        if (gf == 2)
                            epi_fast<false, NC, TS>(p, taddr + g0, colD + g0, gmin[g], valid, ea, grow, n0 + g0, gcol,
                                                    srow, et, g0 - c_lo);
                        else
                            epi_fast<true, NC, TS>(p, taddr + g0, colD + g0, gmin[g], valid, ea, grow, n0 + g0, gcol,
                                                   srow, et, g0 - c_lo);
                        continue;
                    }
                    const int gm = gmin[g];
                    int e;
                    if (!GC && gf) {
                        // |x << d| < 2^30: the group exponent follows from the largest magnitude
                        int ymax = 0, ymin = 0;
                        for (int c = g0; c < g0 + Gt; c += 32) {
                            tmem_ld32(taddr + c, v);
                            tmem_ld_wait();
                            if (valid) {
#pragma unroll
                                for (int q = 0; q < 32; q += 4) {
                                    const int4 d4 = gf == 2 ? make_int4(1, 1, 1, 1) : *reinterpret_cast<const int4 *>(colD + c + q);
                                    const int y0 = (int)v[q] * d4.x, y1 = (int)v[q + 1] * d4.y;
                                    const int y2 = (int)v[q + 2] * d4.z, y3 = (int)v[q + 3] * d4.w;
                                    ymax = max(ymax, max(max(y0, y1), max(y2, y3)));
                                    ymin = min(ymin, min(min(y0, y1), min(y2, y3)));
                                }
                            }
                        }
                        const int amax = max(ymax, -ymin);
                        e = finalize_exp(amax ? ea + gm + need_off32q((uint32_t)amax, p.qb) : kNoExp);
                        // mantissa = RNE((x << d) * 2^-S), S = e - ea - gm uniform over the row
                        const int S = (e == kEZero) ? 0 : e - ea - gm;
                        const int ls = S < 0 ? -S : 0;
                        const int rs = S > 0 ? min(S, 31) : 0;
                        const int bias = rs ? (1 << (rs - 1)) - 1 : 0;
                        const int om = rs ? 1 : 0;
                        const bool any_ls = __any_sync(0xffffffffu, valid && ls != 0);
                        for (int c = g0; c < g0 + Gt; c += 32) {
                            if (Gt > 32) {
                                tmem_ld32(taddr + c, v);
                                tmem_ld_wait();
                            }
                            if (valid) {
                                uint32_t w[8];
                                const int hm = rs >= 2 ? 1 << (32 - rs) : 0;  // high-half multiplier
#pragma unroll
                                for (int q = 0; q < 32; q += 4) {
                                    const int4 d4 = gf == 2 ? make_int4(1, 1, 1, 1) : *reinterpret_cast<const int4 *>(colD + c + q);
                                    int y[4] = {(int)v[q] * d4.x, (int)v[q + 1] * d4.y,
                                                (int)v[q + 2] * d4.z, (int)v[q + 3] * d4.w};
                                    if (any_ls) {
#pragma unroll
                                        for (int t = 0; t < 4; ++t) y[t] <<= ls;
                                    }
                                    if (hm) {
#pragma unroll
                                        for (int t = 0; t < 4; ++t)
                                            y[t] = __mulhi(y[t] + bias + (__mulhi(y[t], hm) & 1), hm);
                                    } else {
#pragma unroll
                                        for (int t = 0; t < 4; ++t) y[t] = (y[t] + bias + ((y[t] >> rs) & om)) >> rs;
                                    }
                                    w[q >> 2] = pack4b(y[0], y[1], y[2], y[3]);
                                }
                                int8_t *dst = p.out + grow * p.out_ld + n0 + c;
                                if (n0 + c < p.N)
                                    *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                                if (n0 + c + 16 < p.N)
                                    *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(w[4], w[5], w[6], w[7]);
                            }
                        }
                    } else {
                        // exact per-element path: exponent eA + eB[n] per element
                        int emax = kNoExp;
                        for (int c = g0; c < g0 + Gt; c += 32) {
                            tmem_ld32(taddr + c, v);
                            tmem_ld_wait();
                            if (valid) {
#pragma unroll
                                for (int q = 0; q < 32; ++q) {
                                    const int32_t x = (int32_t)v[q];
                                    if (x) emax = max(emax, ea + colE[c + q] + need_off32q((uint32_t)(x < 0 ? -x : x), p.qb));
                                }
                            }
                        }
                        e = finalize_exp(emax);
                        for (int c = g0; c < g0 + Gt; c += 32) {
                            tmem_ld32(taddr + c, v);
                            tmem_ld_wait();
                            if (TS || valid) {
                                uint32_t w[8];
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    w[q] = pack4b(requant32((int32_t)v[4 * q], ea + colE[c + 4 * q], e),
                                                  requant32((int32_t)v[4 * q + 1], ea + colE[c + 4 * q + 1], e),
                                                  requant32((int32_t)v[4 * q + 2], ea + colE[c + 4 * q + 2], e),
                                                  requant32((int32_t)v[4 * q + 3], ea + colE[c + 4 * q + 3], e));
                                if constexpr (TS) {
                                    stage16(srow, et, c - c_lo, make_uint4(w[0], w[1], w[2], w[3]));
                                    stage16(srow, et, c - c_lo + 16, make_uint4(w[4], w[5], w[6], w[7]));
                                } else {
                                    int8_t *dst = p.out + grow * p.out_ld + n0 + c;
                                    if (n0 + c < p.N)
                                        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                                    if (n0 + c + 16 < p.N)
                                        *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(w[4], w[5], w[6], w[7]);
                                }
                            }
                        }
                    }
                    if (n0 + g0 < p.N && valid) p.out_exp[grow * p.out_exp_ld + gcol] = (int8_t)e;
                }
            }
            tc_fence_before();
            if constexpr (TS) fence_proxy_async();  // the staged rows, for the TMA store
            if constexpr (PAIR) {
                // the warpgroup's TMEM reads are done; one thread tells the first CTA (and,
                // with staged output, stores the warpgroup's share of the tile)
                named_bar_sync(bar_id, 128);
                if (et == 0) {
                    // the accumulator is free first: issuing the store can wait on the
                    // SM's TMA unit, which the next tile's MMAs must not.  The arrival is
                    // local (a remote one takes about a thousand cycles); the second CTA's
                    // warp 3 forwards its barrier's phases to the first CTA.
                    mbar_arrive(bar_tempty + 8 * acc);
                    if (TS && valid_rows > 0) {
                        tma_store_2d(&tmY, smem_u32(sStage + wg * (128 * 64)), n0 + c_lo, (int)row_base);
                        bulk_commit();
                    }
                }
            } else if constexpr (TS16) {
                // every row staged (whole tiles) and every TMEM read done: release, then one
                // thread stores the tile's int16 sums with one TMA store
                if (valid_rows == p.cv_rows * p.cv_W) fence_proxy_async();
                named_bar_sync(bar_id, 128);
                mbar_arrive(bar_tempty + 8 * acc);
                if (et == 0 && valid_rows == p.cv_rows * p.cv_W) {
                    tma_store_2d(&tmZ, smem_u32(sStage + wg * (128 * 128)), n0 * 2, (int)row_base);
                    bulk_commit();
                }
            } else if constexpr (TS) {
                // every row staged and every TMEM read done: the accumulator is released, then
                // one thread stores the warpgroup's tile, one TMA store per 64 columns
                named_bar_sync(bar_id, 128);
                mbar_arrive(bar_tempty + 8 * acc);
                if (et == 0 && valid_rows > 0) {
#pragma unroll
                    for (int b = 0; b < SCOLS / 64; ++b)
                        tma_store_2d(&tmY, smem_u32(sStage + wg * (128 * SCOLS) + b * (128 * 64)), n0 + c_lo + 64 * b,
                                     (int)row_base);
                    bulk_commit();
                }
            } else {
                mbar_arrive(bar_tempty + 8 * acc);
                named_bar_sync(bar_id, 128);  // the column tables are rewritten for the next tile
            }
        }
        if ((TS || TS16) && et == 0) bulk_wait_all();  // every staged store complete before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();  // the first CTA's MMAs read this CTA's stages and write its TMEM
    tc_fence_after();
    if (warp == 2) {
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, L::kTmemCols);
        else tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

}  // namespace ict
