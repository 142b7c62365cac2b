// ict_device.cuh -- device helpers shared by the libict kernels (sm_100a only).
//
// Integer requantisation primitives for the (C,e) format of "Memory-Efficient
// Integer-Only Training of Deep Neural Networks" (value = C * 2^e, INT8 mantissas,
// Abstract / Figure 1), and thin inline-PTX wrappers for mbarriers, TMA and the
// 5th-generation tensor core (tcgen05 / TMEM).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ict.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libict is written for sm_100a only"
#endif

namespace ict {

constexpr int kEZero = ICT_E_ZERO;
constexpr int kNoExp = -0x40000000;  // running max of need() before any nonzero member

// Sticky device status word: bit k set <=> status code k was raised on the device.
__device__ int32_t g_status;

__device__ __forceinline__ void raise_status(int code) { atomicOr(&g_status, 1 << code); }

// ------------------------------------------------------------------ need() and RNE

// need(x, r) - r for a = |x| > 0: the offset s such that RNE(x * 2^-s) fits in
// [-127, 127] and RNE(x * 2^-(s-1)) does not.  With b = bitlen(a), s = b - 7, plus one
// when the top eight bits of a are all ones (a >= 127.5 * 2^s rounds to 128).
// x / d for an index x >= 0 and d >= 1: a shift for powers of two, 32-bit division when
// both fit (64-bit division is a long emulated sequence).
__device__ __forceinline__ int64_t idiv(int64_t x, int64_t d) {
    if (d == 1) return x;
    if ((d & (d - 1)) == 0) return x >> (__ffsll(d) - 1);
    if (x <= 0x7fffffff && d <= 0x7fffffff) return (int64_t)((uint32_t)x / (uint32_t)d);
    return x / d;
}

__device__ __forceinline__ int need_off32(uint32_t a) {
    int s = 25 - __clz(a);  // bitlen - 7
    if (s > 0 && (a >> (s - 1)) == 255u) s += 1;
    return s;
}
// The same for B-bit mantissas (|C| <= q_max = 2^(B-1) - 1, Table 4's INT8..INT4):
// s = bitlen - (B - 1), plus one when the top B bits of a are all ones (a rounds to 2^(B-1)).
__device__ __forceinline__ int need_off32q(uint32_t a, int bits) {
    int s = (33 - bits) - __clz(a);
    if (s > 0 && (a >> (s - 1)) == (1u << bits) - 1u) s += 1;
    return s;
}
__device__ __forceinline__ int need_off64(uint64_t a) {
    int s = 57 - __clzll(a);
    if (s > 0 && (a >> (s - 1)) == 255ull) s += 1;
    return s;
}

__device__ __forceinline__ int need_off64q(uint64_t a, int bits) {
    int s = (65 - bits) - __clzll(a);
    if (s > 0 && (a >> (s - 1)) == (1ull << bits) - 1ull) s += 1;
    return s;
}

// RNE(x / 2^s), s >= 1; |x| < 2^31 so any s >= 32 gives 0.
__device__ __forceinline__ int32_t rne_shr32(int32_t x, int s) {
    if (s >= 32) return 0;
    int32_t q = x >> s;
    uint32_t rem = (uint32_t)x & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    return q + ((rem > half) || (rem == half && (q & 1)));
}
// RNE(x / 2^s), s >= 1; |x| < 2^62 so any s >= 63 gives 0.
__device__ __forceinline__ int64_t rne_shr64(int64_t x, int s) {
    if (s >= 63) return 0;
    int64_t q = x >> s;
    uint64_t rem = (uint64_t)x & ((1ull << s) - 1ull);
    uint64_t half = 1ull << (s - 1);
    return q + ((rem > half) || (rem == half && (q & 1)));
}

// bits [pos, pos + len) of x (len 0 gives 0)
__device__ __forceinline__ uint32_t bfe_u32(uint32_t x, uint32_t pos, uint32_t len) {
    uint32_t r;
    asm("bfe.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(pos), "r"(len));
    return r;
}

__device__ __forceinline__ int sat127(int64_t q) {
    return q > 127 ? 127 : (q < -127 ? -127 : (int)q);
}

// Mantissa of x (at exponent r) in a group of exponent e: RNE(x * 2^(r - e)).
// For a valid group r - e <= 6; larger left shifts only occur after an exponent
// overflow (status raised) and saturate.
__device__ __forceinline__ int requant32(int32_t x, int r, int e) {
    int k = r - e;
    if (x == 0) return 0;
    if (k >= 0) return sat127((int64_t)x << (k > 8 ? 8 : k));
    return sat127(rne_shr32(x, -k));
}
__device__ __forceinline__ int requant64(int64_t x, int r, int e) {
    int k = r - e;
    if (x == 0) return 0;
    if (k >= 0) return sat127((k > 8 ? (x > 0 ? 1024 : -1024) : (x << k)));
    return sat127(rne_shr64(x, -k));
}

// Group exponent from the running max of need(): E_ZERO when nothing was nonzero,
// raised to -127, and capped at 127 with ICT_ERR_EXP_RANGE.
__device__ __forceinline__ int finalize_exp(int emax) {
    if (emax <= kNoExp) return kEZero;
    if (emax < -127) return -127;
    if (emax > 127) {
        raise_status(ICT_ERR_EXP_RANGE);
        return 127;
    }
    return emax;
}

// sign-extended byte of a word: one prmt whose upper three selectors replicate the sign
// bit of the selected byte (PTX prmt, default mode: selector msb = sign replicate)
__device__ __forceinline__ int sx8(uint32_t w, int byte) {
    const uint32_t sel = (uint32_t)byte | ((uint32_t)(byte | 8) << 4) | ((uint32_t)(byte | 8) << 8) |
                         ((uint32_t)(byte | 8) << 12);
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));
    return (int)r;
}
// The low bytes of four words packed into one (three byte permutes).
__device__ __forceinline__ uint32_t pack4b(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// RNE(y * 2^-S) on the fp32 pipe, for |y| < 2^22 and 0 <= S <= 22.  The bit pattern
// 0x4B400000 + y is the float 1.5 * 2^23 + y exactly (the sum stays in the binade of unit
// spacing); one FMA by 2^-S with the addend 1.5 * 2^23 * (1 - 2^-S) (exact for S <= 22)
// gives 1.5 * 2^23 + y * 2^-S rounded once, to nearest even, at the unit.  The low byte of
// the result's bit pattern is then the rounded value in two's complement (|value| <= 128).
struct RneF32 {
    float sc, add;
};
__device__ __forceinline__ RneF32 rne_f32_consts(int S) {
    const float sc = __int_as_float((127 - S) << 23);
    return {sc, __fmaf_rn(-12582912.f, sc, 12582912.f)};
}
__device__ __forceinline__ uint32_t rne_f32(int y, RneF32 k) {
    return __float_as_uint(__fmaf_rn(__int_as_float(0x4B400000 + y), k.sc, k.add));
}
// the group may take the fp32 rounding: every magnitude below 2^22, a right shift of at
// most 22 bits, and an exponent that was not capped (a capped one saturates instead)
__device__ __forceinline__ bool rne_f32_ok(bool valid, int amax, int S, int need) {
    return !valid || (amax < (1 << 22) && S >= 0 && S <= 22 && need <= 127);
}

// Four values already within [-127, 127] packed into bytes in two conversion
// instructions (each packs two values; the second merges the first's word).
__device__ __forceinline__ uint32_t pack4s(int a, int b, int c, int d) {
    uint32_t t, r;
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(t) : "r"(d), "r"(c));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(b), "r"(a), "r"(t));
    return r;
}
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// ------------------------------------------------------------------ warp reductions

__device__ __forceinline__ int warp_max(int v, unsigned mask = 0xffffffffu) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(mask, v, o));
    return v;
}

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait that may suspend the thread for up to `hint_ns` nanoseconds while the phase
// is incomplete (it resumes as soon as the phase completes), so that waiting threads
// take no issue slots from the warps that share their scheduler.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase of the given parity: gives up after `limit_ns`
// nanoseconds, or as soon as another role has set *abort.  Returns false then.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          const volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
        if (abort && *abort) return false;
        if (globaltimer() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

// TMA tiled loads, completion signalled on an mbarrier (transaction bytes).  No
// multicast form is used anywhere in this library.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(m), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int x, int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(m), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// TMA tiled store from shared memory (bulk-group completion); coordinates must be
// non-negative, x a multiple of 16 bytes.  Rows and columns beyond the tensor are not
// written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(m), "r"(src),
                 "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk store of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until every committed bulk store of this thread is complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- tcgen05 / TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, issued by one thread.
__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier once every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// ---- pairs of CTAs (a cluster of two) sharing one tcgen05.mma.cta_group::2 tile: CTA r
// of the pair holds rows [r M/2, (r+1) M/2) of A and [r N/2, (r+1) N/2) of B in its own
// shared memory and rows [r M/2, (r+1) M/2) of the accumulator in its own TMEM.  Every
// copy is issued by the CTA that owns the destination, and every completion is signalled
// on each CTA's barrier by its own arrive.

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// arrive (release at cluster scope) on an mbarrier given by its shared::cluster address
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an mbarrier of
// the pair's first CTA (bar_cluster: a shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(m), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (both CTAs' TMEM) (+)= A * B^T for the pair, issued by one thread of the first CTA
__device__ __forceinline__ void umma_i8_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier of either CTA of the pair (bar_cluster: a shared::cluster address)
// once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
                 : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
// 64 consecutive 32-bit TMEM columns of this warp's 32 lanes (thread = lane).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]), "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]), "=r"(v[40]), "=r"(v[41]), "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]), "=r"(v[48]), "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]), "=r"(v[55]), "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]), "=r"(v[61]), "=r"(v[62]), "=r"(v[63])
        : "r"(taddr)
        : "memory");
}
// tcgen05.wait::ld that also takes the loaded registers as operands, so that no use of
// them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&v)[64]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]), "+r"(v[30]), "+r"(v[31]), "+r"(v[32]), "+r"(v[33]), "+r"(v[34]), "+r"(v[35]), "+r"(v[36]), "+r"(v[37]), "+r"(v[38]), "+r"(v[39]), "+r"(v[40]), "+r"(v[41]), "+r"(v[42]), "+r"(v[43]), "+r"(v[44]), "+r"(v[45]), "+r"(v[46]), "+r"(v[47]), "+r"(v[48]), "+r"(v[49]), "+r"(v[50]), "+r"(v[51]), "+r"(v[52]), "+r"(v[53]), "+r"(v[54]), "+r"(v[55]), "+r"(v[56]), "+r"(v[57]), "+r"(v[58]), "+r"(v[59]), "+r"(v[60]), "+r"(v[61]), "+r"(v[62]), "+r"(v[63]) :: "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also returns the OR of `pred` over the participating threads, so
// that every participant takes the same decision.
__device__ __forceinline__ int named_bar_or(int id, int nthreads, int pred) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(pred), "r"(id), "r"(nthreads)
        : "memory");
    return r;
}

// Shared-memory matrix descriptor for a K-major operand tile whose rows are
// `row_bytes` (128 or 64) wide and swizzled at that width (canonical tcgen05
// layout: 8-row atoms stacked densely, so the stride between atoms is 8 rows).
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr, int row_bytes) {
    const uint64_t sbo = (uint64_t)(8 * row_bytes) >> 4;
    const uint64_t layout = row_bytes == 128 ? 2ull : 4ull;  // SWIZZLE_128B / SWIZZLE_64B
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (sbo << 32) | (1ull << 46) |
           (layout << 61);
}
// Descriptor for an MN-major operand tile swizzled at 64 bytes: 64-byte atoms along
// M/N (LBO apart), 8 K-rows of 64 bytes each (SBO = 512 bytes between K atoms).
__device__ __forceinline__ uint64_t smem_desc_mnmajor64(uint32_t saddr, uint32_t lbo_bytes) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(512 >> 4) << 32) | (1ull << 46) | (4ull << 61);
}

// Instruction descriptor: kind::i8, signed A and B, s32 accumulate, M x N tile.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n, bool a_mn_major = false,
                                                bool b_mn_major = false) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

}  // namespace ict
