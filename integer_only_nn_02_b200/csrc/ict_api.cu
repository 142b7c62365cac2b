// ict_api.cu -- the C ABI of libict.so (declared in include/ict.h).
//
// Host side only: argument validation, workspace planning, TMA descriptor encoding and
// the composition align -> tensor-core Product -> FIT of each entry point.  Every step
// of the arithmetic runs in the kernels of ict_elementwise.cuh and ict_gemm.cuh.
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "ict_device.cuh"
#include "ict_elementwise.cuh"
#include "ict_gemm.cuh"
#include "ict_lut.cuh"
#include "ict_pointwise.cuh"

using namespace ict;

int launch_clip(const ict_tensor *X, const ict_tensor *dY, int six, ict_tensor *out, cudaStream_t s);

namespace {

// ------------------------------------------------------------------ device checks

struct DeviceInfo {
    bool checked = false;
    int status = ICT_OK;
    int sms = 0;
};
std::mutex g_mu;
DeviceInfo g_dev[64];
uint64_t g_wait_ns = 2000000000ull;  // bound of every mbarrier wait inside a kernel
const uint64_t kDrainNs = 1000000000ull;
// mantissa bits B of every FIT the linear Products, ict_requant and the SGD perform
// (q_max = 2^(B-1) - 1; ict_set_mantissa_bits), process-wide
std::atomic<int> g_mantissa_bits{8};
// entry points whose FIT is written for INT8 only refuse other mantissa widths
int int8_only() { return g_mantissa_bits.load(std::memory_order_relaxed) == 8 ? ICT_OK : ICT_ERR_LAYOUT; }
// largest channel count (contracted or produced) of the implicit-GEMM convolution
constexpr int kConvMaxChannels = 2048;

int device_info(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ICT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.checked) {
        int major = 0, minor = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ICT_ERR_CUDA;
        d.status = (major == 10 && minor == 0) ? ICT_OK : ICT_ERR_UNSUPPORTED_ARCH;
        d.sms = n;
        d.checked = true;
    }
    if (sms) *sms = d.sms;
    return d.status;
}
// SM count for planning; 148 (B200) when no device is visible (workspace queries only)
int planning_sms() {
    int sms = 0;
    if (device_info(&sms) != ICT_OK || sms <= 0) return 148;
    return sms;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? ICT_OK : ICT_ERR_CUDA; }

// number of kernels launched through this library (process-wide)
std::atomic<uint64_t> g_launches{0};
void counted(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// ---- optional per-kernel-class device timing (measurement only; off by default)
enum { KC_GEMM = 0, KC_SGD = 1, KC_ALIGN = 2, KC_REQUANT = 3, KC_GELU = 4, KC_ESTAR = 5, KC_OTHER = 6, KC_POINTWISE = 7,
       KC_N = 8 };
struct TimedLaunch {
    int kc;
    cudaEvent_t a, b;
    double work;
};
struct Timing {
    bool on = false;
    std::vector<TimedLaunch> pending;
    std::vector<cudaEvent_t> pool;
    double ms[KC_N] = {0}, work[KC_N] = {0};
    int64_t n[KC_N] = {0};
} g_timing;
std::mutex g_timing_mu;

cudaEvent_t timing_event() {
    if (!g_timing.pool.empty()) {
        cudaEvent_t e = g_timing.pool.back();
        g_timing.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets the launches issued during its lifetime with a pair of events on `s`.
struct KTimer {
    cudaEvent_t a = nullptr;
    cudaStream_t s;
    int kc;
    double work;
    KTimer(cudaStream_t s_, int kc_, double work_) : s(s_), kc(kc_), work(work_) {
        std::lock_guard<std::mutex> lk(g_timing_mu);
        if (!g_timing.on) return;
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
        a = timing_event();
        if (a) cudaEventRecord(a, s);
    }
    ~KTimer() {
        if (!a) return;
        std::lock_guard<std::mutex> lk(g_timing_mu);
        cudaEvent_t b = timing_event();
        if (!b) return;
        cudaEventRecord(b, s);
        g_timing.pending.push_back(TimedLaunch{kc, a, b, work});
    }
};

// ------------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

// int8 matrix [outer][inner] with row stride `stride` bytes; box inner x outer.
int tmap_2d(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint64_t stride,
            uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return ICT_ERR_CUDA;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {stride};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ICT_OK : ICT_ERR_CUDA;
}

// Dense NHWC int8 activations [n][h][w][c]; box 64 channels x w x rows x 1 image,
// 64-byte swizzle (one K block of the implicit GEMM).
int tmap_nhwc(CUtensorMap *m, const void *base, int n, int h, int w, int c, uint32_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return ICT_ERR_CUDA;
    cuuint64_t dims[4] = {(cuuint64_t)c, (cuuint64_t)w, (cuuint64_t)h, (cuuint64_t)n};
    cuuint64_t strides[3] = {(cuuint64_t)c, (cuuint64_t)w * c, (cuuint64_t)h * w * c};
    cuuint32_t box[4] = {64, (cuuint32_t)w, rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ICT_OK : ICT_ERR_CUDA;
}

// ------------------------------------------------------------------ tensors

int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return cdiv64(a, b) * b; }
int64_t n_grp_rows(const ict_tensor *t) { return cdiv64(t->rows, t->g_rows); }
int64_t n_grp_cols(const ict_tensor *t) { return cdiv64(t->cols, t->g_cols); }
bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }
int clamp_div(int64_t g, int64_t n) { return (int)(g < n ? g : (n > 0 ? n : 1)); }

int check_tensor(const ict_tensor *t) {
    if (!t || t->rows < 0 || t->cols < 0 || t->g_rows < 1 || t->g_cols < 1 || t->ld < t->cols)
        return ICT_ERR_INVALID_ARG;
    if (t->rows > 0 && t->cols > 0 && (!t->mant || !t->exp)) return ICT_ERR_INVALID_ARG;
    if (t->rows >= (1ll << 31) || t->cols >= (1ll << 31)) return ICT_ERR_LAYOUT;
    return ICT_OK;
}
// tensors read or written by 16-byte vectors / TMA
int check_vec(const ict_tensor *t) {
    if (!aligned16(t->mant) || (t->ld & 15)) return ICT_ERR_ALIGNMENT;
    if (t->cols & 15) return ICT_ERR_LAYOUT;
    if (t->g_cols < t->cols && (t->g_cols & 15)) return ICT_ERR_LAYOUT;
    return ICT_OK;
}
bool uniform_along_cols(const ict_tensor *t) { return t->g_cols >= t->cols; }

// ------------------------------------------------------------------ workspace

struct Ws {
    uint8_t *base;
    size_t cap, used;
    bool dry;
    void *take(size_t bytes) {
        used = (size_t)round_up((int64_t)used, 256);
        void *p = dry ? nullptr : base + used;
        used += bytes;
        return p;
    }
};
Ws make_ws(void *ws, size_t bytes, bool dry) { return Ws{(uint8_t *)ws, bytes, 0, dry}; }

// ------------------------------------------------------------------ kernel launchers

struct AlignJob {
    const ict_tensor *t;
    int axis;
    bool transpose;
    int8_t *out;
    int64_t ld;
    int8_t *e_star;
    int32_t *col_max;  // axis 0: int32 scratch [group columns] for a parallel column max
    bool given = false;  // the targets are read from e_star, not found from the tensor
};

// Arguments of one alignment job and how its target exponents are found.
struct AlignLaunch {
    AlignArgs a;
    int64_t n_exp;
    int estar;             // 0: none (row e* inside the rows kernel), 1: rows, 2: column scratch, 3: column blocks
    int64_t blocks, used;  // column scratch form
};

AlignLaunch plan_align(const AlignJob &j, int sms) {
    const ict_tensor *in = j.t;
    AlignLaunch L;
    AlignArgs &a = L.a;
    memset(&a, 0, sizeof(a));
    a.in = in->mant;
    a.in_exp = in->exp;
    a.rows = in->rows;
    a.cols = in->cols;
    a.ld = in->ld;
    a.g_rows = clamp_div(in->g_rows, in->rows);
    a.g_cols = clamp_div(in->g_cols, in->cols);
    a.ngc = n_grp_cols(in);
    a.axis = j.axis;
    a.out = j.out;
    a.out_ld = j.ld;
    a.e_star = j.e_star;
    {
        const int64_t gv = a.g_cols / 16;
        if (a.ngc == 1) a.gv_shift1 = 32;
        else if (a.g_cols % 16 == 0 && (gv & (gv - 1)) == 0) a.gv_shift1 = __builtin_ctzll((unsigned long long)gv) + 1;
    }
    L.n_exp = n_grp_rows(in) * a.ngc;
    L.blocks = L.used = 0;
    if (j.given) {  // targets fixed by the caller: no e* pass, the shift kernel reads e_star
        L.estar = 0;
        return L;
    }
    if (j.axis == 1) {
        L.estar = j.transpose ? 1 : 0;
        a.row_estar = j.transpose ? 0 : 1;  // computed inside align_rows_kernel
    } else {
        // every thread of the scratch form keeps one group column: a stride that is a
        // multiple of ngc
        // one block per SM at most, each reducing a band of at least 32 group rows
        L.blocks = std::max<int64_t>(1, std::min<int64_t>(cdiv64(n_grp_rows(in), 32), (int64_t)sms));
        L.used = L.blocks * 256;
        L.estar = (j.col_max && a.ngc <= 8192) ? 2 : 3;
        if (j.transpose && in->rows <= 4096 && a.g_cols >= 16) {
            L.estar = 0;  // few rows (a weight): each transposing block scans its columns' exponents
            a.col_scan = 1;
        }
        if (L.estar == 2) a.col_max = j.col_max;
    }
    return L;
}

// Tiles of the transposing kernels for the first n jobs of P (job 0's tiles first);
// fills P.tiles0, P.tiles1 and P.ntc.
unsigned transpose_tiles(AlignPair &P, int n) {
    int64_t t[2];
    for (int z = 0; z < 2; ++z) {
        const int64_t tc = z < n ? cdiv64(P.a[z].cols, 128) : 1, tr = z < n ? cdiv64(P.a[z].rows, 128) : 0;
        P.ntc[z] = (int)tc;
        t[z] = tc * tr;
    }
    P.tiles0 = (int)t[0];
    P.tiles1 = (int)t[1];
    return (unsigned)(t[0] + t[1]);
}

// The transposing alignment of the first n jobs of P: persistent streaming blocks (three
// per SM) unless a job scans its own column exponents, then one block per tile.  The
// streaming kernel's exact form serves jobs aligned per column from the column-max
// scratch with one group row per row and power-of-two group widths.
void launch_align_transpose(AlignPair &P, int n, int sms, cudaStream_t s) {
    const unsigned tiles = transpose_tiles(P, n);
    const bool scan = P.a[0].col_scan || (n > 1 && P.a[1].col_scan);
    if (scan) {
        align_transpose_kernel<<<tiles, 256, 0, s>>>(P);
        return;
    }
    bool exact = true;
    for (int z = 0; z < n; ++z) {
        const AlignArgs &a = P.a[z];
        exact = exact && a.axis == 0 && a.col_max && a.g_rows == 1 && a.gv_shift1 > 0;
    }
    const unsigned grid = std::min<unsigned>(tiles, (unsigned)sms * 3);
    if (exact)
        align_transpose_stream_kernel<true><<<grid, 256, 0, s>>>(P);
    else
        align_transpose_stream_kernel<false><<<grid, 256, 0, s>>>(P);
}

// Rows of 16-byte vectors, one row per segment of L lanes.  The narrowest segment whose
// lanes hold at most six vectors each (the most bytes in flight per lane) and stay nine
// tenths busy, else the busiest; NV = the row's vectors per lane rounded up to an
// instantiated count.  Rows of at most four vectors along the rows (with at most four
// groups when computing e*) take one thread per row; other rows of fewer than 8 or more
// than 192 vectors or (computing e*) more than 2 L groups, and 2^31 rows or more, go to the
// generic kernel.  Persistent grid: two blocks per SM.
int launch_align_rows(const AlignArgs &a, cudaStream_t s, int sms) {
    const int64_t vpr = a.cols / 16;
    const bool row_e = a.axis == 1 && a.row_estar;
    int L = 0;
    double best = -1.0;
    for (int l : {8, 16, 32}) {
        const int64_t per = cdiv64(vpr, l);
        if (per > 6 || (row_e && a.ngc > 2 * l)) continue;
        const double eff = (double)vpr / (double)(l * per);
        if (eff >= 0.9) { L = l; break; }
        if (eff > best + 1e-12) best = eff, L = l;
    }
    if (a.axis == 1 && vpr <= 4 && (!a.row_estar || a.ngc <= 4) && a.rows < (1ll << 31)) {  // thin rows
        const unsigned grid = (unsigned)std::min<int64_t>(cdiv64(a.rows, 256), (int64_t)sms * 8);
        align_rows_thin_kernel<<<grid, 256, 0, s>>>(a);
        return ICT_OK;
    }
    if (L == 0 || vpr < 8 || a.rows >= (1ll << 31)) {  // narrow rows: four threads per row
        align_rows_wide_kernel<<<dim3((unsigned)cdiv64(a.cols, 256), (unsigned)cdiv64(a.rows, 64)), 256, 0, s>>>(a);
        return ICT_OK;
    }
    const int64_t per = cdiv64(vpr, L);
    const int nv = per <= 2 ? 2 : per <= 3 ? 3 : per <= 4 ? 4 : 6;
    const bool exact = a.axis == 1 && a.g_rows == 1 && a.gv_shift1 > 0 && vpr == (int64_t)L * nv;
    const unsigned grid = (unsigned)std::min<int64_t>(cdiv64(a.rows, 256 / L), (int64_t)sms * 2);
#define ICT_ALIGN_ROWS(L_, NV_)                                                             \
    if (L == L_ && nv == NV_)                                                              \
        return exact ? (align_rows_kernel<L_, NV_, true><<<grid, 256, 0, s>>>(a), ICT_OK) \
                     : (align_rows_kernel<L_, NV_, false><<<grid, 256, 0, s>>>(a), ICT_OK);
#define ICT_ALIGN_ROWS_L(L_) ICT_ALIGN_ROWS(L_, 2) ICT_ALIGN_ROWS(L_, 3) ICT_ALIGN_ROWS(L_, 4) ICT_ALIGN_ROWS(L_, 6)
    ICT_ALIGN_ROWS_L(32)
    ICT_ALIGN_ROWS_L(16)
    ICT_ALIGN_ROWS_L(8)
#undef ICT_ALIGN_ROWS_L
#undef ICT_ALIGN_ROWS
    return ICT_ERR_LAYOUT;
}

// One or two alignment jobs; two jobs must both be transposing column alignments with
// scratch (the operands of a backward-weight contraction): they share one launch of the
// column e* kernel and one of the transposing kernel.
int launch_align_n(const AlignJob *jobs, int n, cudaStream_t s) {
    int sms = 148;
    device_info(&sms);
    AlignLaunch L[2];
    AlignPair P;
    memset(&P, 0, sizeof(P));
    double estar_work = 0, align_work = 0;
    for (int i = 0; i < n; ++i) {
        L[i] = plan_align(jobs[i], sms);
        P.a[i] = L[i].a;
        P.cm[i] = jobs[i].col_max;
        P.used[i] = L[i].used;
        estar_work += (double)L[i].n_exp + 8.0 * (double)L[i].a.ngc;
        align_work += 2.0 * (double)L[i].a.rows * (double)L[i].a.cols + (double)L[i].n_exp;
    }
    int launches = 0;
    if (n == 2 && jobs[0].given && jobs[1].given && jobs[0].transpose && jobs[1].transpose) {
        KTimer kt(s, KC_ALIGN, align_work);
        launch_align_transpose(P, 2, sms, s);
        counted(1);
        return launch_status();
    }
    if (n == 2 && (L[0].estar != 2 || L[1].estar != 2)) {  // not pairable on this device: one by one
        int st;
        if ((st = launch_align_n(jobs, 1, s))) return st;
        return launch_align_n(jobs + 1, 1, s);
    }
    if (n == 2) {
        for (int i = 0; i < 2; ++i)
            if (cudaMemsetAsync(jobs[i].col_max, 0x80, (size_t)L[i].a.ngc * 4, s) != cudaSuccess) return ICT_ERR_CUDA;
        {
            KTimer kt(s, KC_ESTAR, estar_work);
            const int64_t ngc = std::max(L[0].a.ngc, L[1].a.ngc);
            estar_cols_scratch_kernel<<<dim3((unsigned)std::max(L[0].blocks, L[1].blocks), 2), 256,
                                        (size_t)ngc * 4, s>>>(P);
        }
        KTimer kt(s, KC_ALIGN, align_work);
        launch_align_transpose(P, 2, sms, s);
        counted(2);
        return launch_status();
    }
    const AlignLaunch &l = L[0];
    const AlignArgs &a = l.a;
    if (l.estar == 1) {
        KTimer kt(s, KC_ESTAR, (double)l.n_exp + (double)a.rows);
        estar_rows_kernel<<<(unsigned)cdiv64(a.rows, 256), 256, 0, s>>>(a);
        ++launches;
    } else if (l.estar == 2) {
        if (cudaMemsetAsync(jobs[0].col_max, 0x80, (size_t)a.ngc * 4, s) != cudaSuccess) return ICT_ERR_CUDA;
        KTimer kt(s, KC_ESTAR, estar_work);
        estar_cols_scratch_kernel<<<(unsigned)l.blocks, 256, (size_t)a.ngc * 4, s>>>(P);
        ++launches;
    } else if (l.estar == 3) {
        KTimer kt(s, KC_ESTAR, (double)l.n_exp + (double)a.cols);
        estar_cols_kernel<<<(unsigned)a.ngc, 256, 0, s>>>(a);
        ++launches;
    }
    KTimer kt(s, KC_ALIGN, align_work);
    if (jobs[0].transpose)
        launch_align_transpose(P, 1, sms, s);
    else if (int st = launch_align_rows(a, s, sms))
        return st;
    counted(launches + 1);
    return launch_status();
}

int launch_align(const AlignJob &j, cudaStream_t s) {
    if (j.t->rows == 0 || j.t->cols == 0) return ICT_OK;
    return launch_align_n(&j, 1, s);
}

// The jobs of one call, pairing transposing column alignments with scratch.
int launch_aligns(const AlignJob *jobs, int n, cudaStream_t s) {
    auto pairable = [&](const AlignJob &j) {
        return j.axis == 0 && j.transpose && j.col_max && !j.given && j.t->rows > 0 && j.t->cols > 0 &&
               plan_align(j, planning_sms()).estar == 2;
    };
    auto given_t = [&](const AlignJob &j) { return j.given && j.transpose && j.t->rows > 0 && j.t->cols > 0; };
    int st;
    for (int i = 0; i < n;) {
        if (i + 1 < n && ((pairable(jobs[i]) && pairable(jobs[i + 1])) || (given_t(jobs[i]) && given_t(jobs[i + 1])))) {
            if ((st = launch_align_n(jobs + i, 2, s))) return st;
            i += 2;
        } else {
            if ((st = launch_align(jobs[i], s))) return st;
            ++i;
        }
    }
    return ICT_OK;
}

template <int T, int EPT>
void launch_requant_block(const RequantArgs &a, int64_t groups, cudaStream_t s) {
    requant_group_block_kernel<T, EPT><<<(unsigned)groups, T, 0, s>>>(a);
}

// FIT into row-local groups: one warp per group up to 127 elements, one block per
// group (values held in registers) for wider groups up to 4096.
int launch_requant_rows(RequantArgs a, cudaStream_t s) {
    const int64_t groups = a.rows * a.ngc;
    if (groups == 0) return ICT_OK;
    const int G = a.G;
    KTimer kt(s, KC_REQUANT, (double)a.rows * (double)a.cols * (a.v64 ? 9.0 : 4.0 * a.nsplit + 1.0));
    const bool vec = !a.v64 && a.cs == 1 && G >= 64 && G <= 4096 && G % 4 == 0 && a.cols % 4 == 0 &&
                     a.ld % 4 == 0 && a.out_ld % 4 == 0 && a.split_stride % 4 == 0 &&
                     (reinterpret_cast<uintptr_t>(a.v32) & 15) == 0 && (reinterpret_cast<uintptr_t>(a.out) & 3) == 0;
    const bool warp = vec && a.nsplit == 1 && G <= 1024 && (!a.col_exp || a.col_div == 1) &&
                      (reinterpret_cast<uintptr_t>(a.col_exp) & 3) == 0;
    if (warp) {
        const unsigned b = (unsigned)cdiv64(groups, 8);
        if (G <= 256) requant_warp_kernel<2><<<b, 256, 0, s>>>(a);
        else if (G <= 512) requant_warp_kernel<4><<<b, 256, 0, s>>>(a);
        else requant_warp_kernel<8><<<b, 256, 0, s>>>(a);
    } else if (vec) {
        const unsigned b = (unsigned)groups;
        const bool wide = a.nsplit > 1;
#define ICT_RQ_VEC(T_, V_)                                                      \
    (wide ? requant_vec_kernel<T_, V_, true><<<b, T_, 0, s>>>(a)               \
          : requant_vec_kernel<T_, V_, false><<<b, T_, 0, s>>>(a))
        if (G <= 256) ICT_RQ_VEC(64, 1);
        else if (G <= 512) ICT_RQ_VEC(128, 1);
        else if (G <= 1024) ICT_RQ_VEC(256, 1);
        else if (G <= 2048) ICT_RQ_VEC(256, 2);
        else ICT_RQ_VEC(256, 4);
#undef ICT_RQ_VEC
    } else if (G >= 128 && G <= 4096) {
        const int T = G >= 256 ? 256 : 128;
        const int ept = (G + T - 1) / T;
        if (T == 128 && ept <= 1) launch_requant_block<128, 1>(a, groups, s);
        else if (T == 128) launch_requant_block<128, 2>(a, groups, s);
        else if (ept <= 1) launch_requant_block<256, 1>(a, groups, s);
        else if (ept <= 2) launch_requant_block<256, 2>(a, groups, s);
        else if (ept <= 4) launch_requant_block<256, 4>(a, groups, s);
        else if (ept <= 8) launch_requant_block<256, 8>(a, groups, s);
        else launch_requant_block<256, 16>(a, groups, s);
    } else {
        requant_rows_kernel<<<(unsigned)cdiv64(groups, 8), 256, 0, s>>>(a);
    }
    counted(1);
    return launch_status();
}

int launch_zero(const ict_tensor *out, cudaStream_t s) {
    const int64_t n = out->rows * out->cols, ne = n_grp_rows(out) * n_grp_cols(out);
    const int64_t m = n > ne ? n : ne;
    if (m == 0) return ICT_OK;
    KTimer kt(s, KC_OTHER, (double)n + (double)ne);
    zero_ce_kernel<<<(unsigned)cdiv64(m, 256), 256, 0, s>>>(out->mant, out->rows, out->cols, out->ld,
                                                           out->exp, ne);
    counted(1);
    return launch_status();
}

// ---- tensor-core Product

constexpr int stages_for(int bn, int bk) {
    return bk == 256 ? 4
           : bk == 128 ? (bn <= 64 ? 8 : bn <= 128 ? 6 : bn <= 192 ? 5 : 4)
                       : (bn <= 64 ? 12 : bn <= 128 ? 10 : 8);
}

template <int BN, int BK, int LOAD>
int launch_gemm_t(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p, int grid,
                  cudaStream_t s, const CUtensorMap *ty = nullptr) {
    constexpr int ST = stages_for(BN, BK);
    auto run = [&](auto k, int nwg, int smem_bytes) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
            return (int)ICT_ERR_CUDA;
        k<<<grid, 128 + 128 * nwg, smem_bytes, s>>>(ta, tb, ty ? *ty : tb, tb, p);  // tmY: staged output only
        counted(1);
        return launch_status();
    };
    constexpr int kB2 = GemmSmem<BN, BK, ST, 2>::kBytes;
    if (p.epi == EPI_I32) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_I32>, 2, kB2);
    if constexpr (LOAD == LOAD_CONV_WGRAD) {
        return ICT_ERR_LAYOUT;  // backward-weight writes int32 only
    } else {
        if constexpr (LOAD == LOAD_CONV) {
            if constexpr (BN <= 128) {
                // four epilogue warpgroups on alternate tiles (four accumulators): the
                // per-tile rounding to odd is latency-bound, more warps hide it
                constexpr int kB4 = GemmSmem<BN, BK, ST, 4>::kBytes;
                if (p.epi == EPI_RO16 && p.nwg == 4) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_RO16, 0, 4>, 4, kB4);
            }
            if (p.epi == EPI_RO16) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_RO16>, 2, kB2);
        }
        if constexpr (LOAD == LOAD_2D) {
            if (p.epi == EPI_RO16R) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_RO16R>, 2, kB2);
        }
        if (p.epi != EPI_FIT_ROW) return ICT_ERR_LAYOUT;
        const int gt = p.G >= p.N ? BN : p.G;  // group width inside a tile
        if constexpr (LOAD == LOAD_2D && BN <= 128) {
            if (p.nwg == 4) {  // four epilogue warpgroups, four accumulators
                constexpr int kB4 = GemmSmem<BN, BK, ST, 4>::kBytes;
                if constexpr (BN == 128) {
                    // 32-column groups with the output staged per warpgroup (128 x 128) and
                    // written by TMA stores: four stages leave room for the staging rows
                    constexpr int ST4 = 4;
                    constexpr int kB4s = GemmSmem<BN, BK, ST4, 4, false, 4, 128 * 128>::kBytes;
                    if (gt == 32 && ty)
                        return run(gemm_ce_kernel<BN, BK, ST4, LOAD, EPI_FIT_ROW, 1, 4, false, false, true>, 4, kB4s);
                }
                if (gt == 32) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_FIT_ROW, 1, 4>, 4, kB4);
                return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_FIT_ROW, 0, 4>, 4, kB4);
            }
        }
        if (gt == 32) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_FIT_ROW, 1>, 2, kB2);
        if constexpr (LOAD == LOAD_2D) {
            if (gt == 64) return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_FIT_ROW, 2>, 2, kB2);
        }
        return run(gemm_ce_kernel<BN, BK, ST, LOAD, EPI_FIT_ROW, 0>, 2, kB2);
    }
}

// Pairs of CTAs (clusters of two) on 256 x BN tiles: the grid is even and launched with
// the cluster dimension; each CTA holds half of every B stage, so it has room for the
// stages of a BN / 2 tile.
template <int BN>
int launch_gemm_pair_t(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &ty, const GemmParams &p,
                       int grid, cudaStream_t s) {
    constexpr int ST = stages_for(BN / 2, 128);
    constexpr int ST4 = 5;  // four epilogue warpgroups stage 32 KB of output: one stage fewer
    auto run = [&](auto k, int smem_bytes, int nwg) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
            return (int)ICT_ERR_CUDA;
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3((unsigned)(128 + 128 * nwg), 1, 1);
        cfg.dynamicSmemBytes = (size_t)smem_bytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, k, ta, tb, ty, tb, p) != cudaSuccess) return (int)ICT_ERR_CUDA;
        counted(1);
        return launch_status();
    };
    constexpr int kB = GemmSmem<BN, 128, ST, 2, true>::kBytes;
    if (p.epi == EPI_I32) return run(gemm_ce_kernel<BN, 128, ST, LOAD_2D, EPI_I32, 0, 2, true>, kB, 2);
    if (p.epi != EPI_FIT_ROW) return ICT_ERR_LAYOUT;
    const int gt = p.G >= p.N ? BN : p.G;
    if constexpr (BN == 256) {
        // 32- and 64-column groups on 256-wide tiles: four epilogue warpgroups, a quarter of
        // the columns each
        constexpr int kB4 = GemmSmem<BN, 128, ST4, 4, true, 2, 128 * 64>::kBytes;
        if (gt == 32) return run(gemm_ce_kernel<BN, 128, ST4, LOAD_2D, EPI_FIT_ROW, 1, 4, true, true>, kB4, 4);
        if (gt == 64) return run(gemm_ce_kernel<BN, 128, ST4, LOAD_2D, EPI_FIT_ROW, 3, 4, true, true>, kB4, 4);
    }
    if (gt == 32) return run(gemm_ce_kernel<BN, 128, ST, LOAD_2D, EPI_FIT_ROW, 1, 2, true>, kB, 2);
    if (gt == 64) return run(gemm_ce_kernel<BN, 128, ST, LOAD_2D, EPI_FIT_ROW, 2, 2, true>, kB, 2);
    return run(gemm_ce_kernel<BN, 128, ST, LOAD_2D, EPI_FIT_ROW, 0, 2, true>, kB, 2);
}

// Convolution Products on halo tiles (RO16 epilogue, four warpgroups, three stages of
// three 16 KB box slots, the nine weight blocks resident).
template <int BN>
int launch_gemm_halo(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p, int grid, cudaStream_t s) {
    constexpr int ST = 3;
    constexpr int kB = GemmSmem<BN, 64, ST, 4, false, 4, 0, 3 * kHaloSlot, 9>::kBytes;
    auto k = gemm_ce_kernel<BN, 64, ST, LOAD_CONV_HALO, EPI_RO16, 0, 4>;
    if (p.epi != EPI_RO16 || p.nwg != 4 || p.n_ntiles != 1 || p.cv_bkblk > 9) return ICT_ERR_LAYOUT;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kB) != cudaSuccess) return ICT_ERR_CUDA;
    k<<<grid, 128 + 128 * 4, kB, s>>>(ta, tb, tb, tb, p);
    counted(1);
    return launch_status();
}

// The ring form (64-wide tiles): four stages over three rings of image rows; tm2 is the map
// of the continuing tiles' boxes, tmz the int16 sums' map for the staged stores.
int launch_gemm_ring(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tm2, const CUtensorMap &tmz,
                     const GemmParams &p, int grid, cudaStream_t s) {
    constexpr int ST = 4;
    constexpr int kB = GemmSmem<64, 64, ST, 4, false, 4, 128 * 128, 3 * kRingBox / ST, 9>::kBytes;
    auto k = gemm_ce_kernel<64, 64, ST, LOAD_CONV_RING, EPI_RO16, 0, 4>;
    if (p.epi != EPI_RO16 || p.nwg != 4 || p.n_ntiles != 1 || p.splits != 1 || p.cv_bkblk > 9) return ICT_ERR_LAYOUT;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kB) != cudaSuccess) return ICT_ERR_CUDA;
    k<<<grid, 128 + 128 * 4, kB, s>>>(ta, tb, tm2, tmz, p);
    counted(1);
    return launch_status();
}

int launch_gemm(int bn, int bk, int load, const CUtensorMap &ta, const CUtensorMap &tb,
                const GemmParams &p_in, int grid, cudaStream_t s, double ops, bool pair = false,
                const CUtensorMap *ty = nullptr, const CUtensorMap *tz = nullptr) {
    KTimer kt(s, KC_GEMM, ops);
    // both epilogue warpgroups take every tile (one column half each) when no output
    // group straddles the halves
    GemmParams p = p_in;
    const int gt = p.G >= p.N ? bn : p.G;
    const bool nwg4_ok = p.epi == EPI_FIT_ROW ||
                         (p.epi == EPI_RO16 && (load == LOAD_CONV || load == LOAD_CONV_HALO || load == LOAD_CONV_RING));
    if (p.nwg != 4 || !nwg4_ok || pair) p.nwg = 2;
    p.epi_split = p.nwg == 2 && (p.epi == EPI_I32 || p.epi == EPI_RO16R || (gt < bn && (bn / 2) % gt == 0));
    if (load == LOAD_CONV_RING) {
        if (bk != 64 || pair || bn != 64 || !ty || !tz) return ICT_ERR_LAYOUT;
        return launch_gemm_ring(ta, tb, *ty, *tz, p, grid, s);
    }
    if (load == LOAD_CONV_HALO) {
        if (bk != 64 || pair) return ICT_ERR_LAYOUT;
        if (bn == 64) return launch_gemm_halo<64>(ta, tb, p, grid, s);
        if (bn == 128) return launch_gemm_halo<128>(ta, tb, p, grid, s);
        return ICT_ERR_LAYOUT;
    }
    if (pair) {
        if (load != LOAD_2D || bk != 128 || (grid & 1)) return ICT_ERR_LAYOUT;
        const CUtensorMap &y = ty ? *ty : tb;  // the output map, for staged stores
        if (bn == 192) return launch_gemm_pair_t<192>(ta, tb, y, p, grid, s);
        if (bn == 256) return launch_gemm_pair_t<256>(ta, tb, y, p, grid, s);
        return ICT_ERR_LAYOUT;
    }
#define ICT_GEMM_CASE(BN_, BK_, LOAD_)          \
    if (bn == BN_ && bk == BK_ && load == LOAD_) \
        return launch_gemm_t<BN_, BK_, LOAD_>(ta, tb, p, grid, s, ty);
    ICT_GEMM_CASE(64, 128, LOAD_2D)
    ICT_GEMM_CASE(128, 128, LOAD_2D)
    ICT_GEMM_CASE(192, 128, LOAD_2D)
    ICT_GEMM_CASE(256, 128, LOAD_2D)
    ICT_GEMM_CASE(64, 64, LOAD_CONV)
    ICT_GEMM_CASE(128, 64, LOAD_CONV)
    ICT_GEMM_CASE(192, 64, LOAD_CONV)
    ICT_GEMM_CASE(256, 64, LOAD_CONV)
    ICT_GEMM_CASE(64, 256, LOAD_CONV_WGRAD)
#undef ICT_GEMM_CASE
    return ICT_ERR_LAYOUT;
}

int pick_bn(int64_t n) {
    if (n <= 64) return 64;
    if (n <= 128) return 128;
    if (n <= 192) return 192;
    if (n % 256 == 0) return 256;
    if (n % 192 == 0) return 192;
    if (n % 128 == 0) return 128;
    return 256;
}

// Tile width for an M x N output on `sms` SMs: among the widths that keep the output
// groups inside a tile, the one whose last wave of tiles is fullest (ties: wider).
int pick_bn_waves(int64_t M, int64_t N, int64_t G, int sms) {
    if (N <= 256) return pick_bn(N);
    int best = 0;
    double best_score = -1.0;
    const int cands[3] = {256, 192, 128};
    for (int bn : cands) {
        const bool fits = G >= N ? false : (bn % G == 0 && G % 32 == 0);
        if (!fits && G < N) continue;
        const int64_t tiles = cdiv64(M, 128) * cdiv64(N, bn);
        const int64_t waves = cdiv64(tiles, sms);
        const double eff = (double)(M * N) / (double)(waves * sms * 128 * bn);
        // widths whose halves hold whole groups let both epilogue warpgroups share a tile
        const bool halves = G >= N || (bn / 2) % G == 0;
        const double score = eff * (1.0 + 0.05 * bn / 64.0) * (halves ? 1.15 : 1.0);
        if (score > best_score) best_score = score, best = bn;
    }
    return best ? best : pick_bn(N);
}

// groups whose column exponents differ by at most this take the fast epilogue:
// |acc| <= K * 127^2 shifted left by the spread must stay below 2^30
int fast_slack_for(int64_t K) {
    const uint64_t bound = (uint64_t)K * 127u * 127u;
    int bits = 0;
    while ((bound >> bits) != 0) ++bits;
    return 30 - bits;
}

// A K-major operand of the Product: rows of int8, K contiguous, an exponent per row.
struct Operand {
    const int8_t *mant;
    int64_t rows, k, ld;
    const int8_t *exp;
    int exp_div;  // exponent of row i is exp[i / exp_div]
};

// Operand whose contracted index runs along the tensor's columns.
Operand operand_rows(const ict_tensor *t, Ws &ws, AlignJob *jobs, int *njobs) {
    if (uniform_along_cols(t))
        return Operand{t->mant, t->rows, t->cols, t->ld, t->exp, clamp_div(t->g_rows, t->rows)};
    const int64_t ld = round_up(t->cols, 16);
    int8_t *m = (int8_t *)ws.take((size_t)t->rows * ld);
    int8_t *e = (int8_t *)ws.take((size_t)t->rows);
    jobs[(*njobs)++] = AlignJob{t, 1, false, m, ld, e, nullptr};
    return Operand{m, t->rows, t->cols, ld, e, 1};
}
// Operand whose contracted index runs along the tensor's rows: aligned per column and
// transposed into K-major rows.
Operand operand_cols(const ict_tensor *t, Ws &ws, AlignJob *jobs, int *njobs) {
    const int64_t ld = round_up(t->rows, 16);
    int8_t *m = (int8_t *)ws.take((size_t)t->cols * ld);
    int8_t *e = (int8_t *)ws.take((size_t)round_up(t->cols, 16));
    int32_t *cm = (int32_t *)ws.take((size_t)n_grp_cols(t) * 4);
    jobs[(*njobs)++] = AlignJob{t, 0, true, m, ld, e, cm};
    return Operand{m, t->cols, t->rows, ld, e, 1};
}

struct ProductPlan {
    int bn, nwg, splits, kblk_per_split, n_kblk, n_mtiles, n_ntiles, units, grid;
    bool fused;
    bool pair;   // clusters of two CTAs on 256-row tiles (tcgen05 cta_group::2)
    bool ro16r;  // one output group per row across tiles: int16 rounded-to-odd sums + a round pass
    int32_t *ws32;
    int64_t ws_ld;
    int16_t *ws16;
    int64_t ws16_ld, tn_ld;
    int32_t *tneed;
};

// Tiling of D[M][N] = A[M][K] B[N][K]^T with FIT into the row-local groups of `out`.
// raw: the int32 sums are the result (no FIT), so the product always writes them to ws32.
ProductPlan plan_product(int64_t M, int64_t N, int64_t K, const ict_tensor *out, int sms,
                         bool allow_split, Ws &ws, bool raw = false) {
    ProductPlan pl;
    pl.bn = pick_bn_waves(M, N, out->g_cols, sms);
    pl.nwg = 2;
    {   // short contractions with 32-column output groups: four epilogue warpgroups (four
        // accumulators) on 128-wide tiles.  64-column groups keep a whole group in
        // registers, which leaves room for two warpgroups only; they split each tile.
        const int64_t G = out->g_cols;
        if (K <= 1024 && N % 128 == 0 && G == 32) pl.bn = 128, pl.nwg = 4;
    }
    // large Products with wide tiles run on pairs of CTAs: a 256 x BN tile per pair halves
    // the B bytes each SM draws per multiply-add.  128-wide tiles stay on single CTAs,
    // whose 128 x 128 steps measured faster than the pair's 256 x 128 ones.
    pl.pair = pl.nwg == 2 && pl.bn >= 192 && pl.bn % 64 == 0 && M >= 2048 && sms >= 2;
    const int units_per_wave = pl.pair ? sms / 2 : sms;
    pl.n_kblk = (int)cdiv64(K, 128);
    pl.n_mtiles = (int)cdiv64(M, pl.pair ? 256 : 128);
    pl.n_ntiles = (int)cdiv64(N, pl.bn);
    const int tiles = pl.n_mtiles * pl.n_ntiles;
    int splits = 1;
    if (allow_split && tiles < units_per_wave && pl.n_kblk >= 8) {
        // whole waves: as many K slices as fit next to the tiles on the SMs
        splits = (int)std::min<int64_t>(units_per_wave / tiles, pl.n_kblk / 4);
        if (splits < 1) splits = 1;
    }
    // int32 partial sums stay exact: at most 2^17 products of magnitude <= 127^2 each
    const int max_kblk = (1 << 17) / 128;
    if (cdiv64(pl.n_kblk, splits) > max_kblk) splits = (int)cdiv64(pl.n_kblk, max_kblk);
    pl.kblk_per_split = (int)cdiv64(pl.n_kblk, splits);
    pl.splits = (int)cdiv64(pl.n_kblk, pl.kblk_per_split);
    pl.units = tiles * pl.splits;
    pl.grid = pl.pair ? 2 * std::min(pl.units, units_per_wave) : std::min(pl.units, sms);
    const int64_t G = out->g_cols;
    const bool groups_in_tile = (G >= N) ? (N <= pl.bn) : (pl.bn % G == 0 && G % 32 == 0);
    pl.fused = !raw && pl.splits == 1 && groups_in_tile;
    // one group per row spanning several tiles, no split: each (row, tile half) rounds its
    // sums to odd into int16 with its own need; a streaming pass rounds to the row's group
    pl.ro16r = !raw && !pl.fused && pl.splits == 1 && G >= N && !pl.pair && pl.nwg == 2 && N % 16 == 0 &&
               out->ld % 16 == 0 && (reinterpret_cast<uintptr_t>(out->mant) & 15) == 0;
    pl.ws_ld = round_up(N, 32);
    pl.ws32 = (pl.fused || pl.ro16r) ? nullptr : (int32_t *)ws.take((size_t)pl.splits * M * pl.ws_ld * 4);
    pl.ws16 = nullptr, pl.tneed = nullptr, pl.ws16_ld = pl.tn_ld = 0;
    if (pl.ro16r) {
        pl.ws16_ld = round_up(N, 32);  // the epilogue writes 32-column chunks
        pl.ws16 = (int16_t *)ws.take((size_t)M * pl.ws16_ld * 2);
        pl.tn_ld = (int64_t)pl.n_ntiles * 2;
        pl.tneed = (int32_t *)ws.take((size_t)M * pl.tn_ld * 4);
    }
    return pl;
}

// Sums of the split-K int32 slices of a raw product into the caller's int32 / int64 buffer.
int launch_sum_slices(const ProductPlan &pl, int64_t M, int64_t N, void *acc, int bits, int64_t ld_acc,
                      cudaStream_t s) {
    const int64_t vecs = M * (N / 4);
    if (vecs == 0) return ICT_OK;
    KTimer kt(s, KC_REQUANT, (double)M * (double)N * (4.0 * pl.splits + bits / 8.0));
    const unsigned grid = (unsigned)cdiv64(vecs, 256);
    if (bits == 64)
        sum_slices_kernel<true><<<grid, 256, 0, s>>>(pl.ws32, pl.splits, M * pl.ws_ld, M, N, pl.ws_ld, acc, ld_acc);
    else
        sum_slices_kernel<false><<<grid, 256, 0, s>>>(pl.ws32, pl.splits, M * pl.ws_ld, M, N, pl.ws_ld, acc, ld_acc);
    counted(1);
    return launch_status();
}

int run_product(const Operand &A, const Operand &B, const ict_tensor *out, const ProductPlan &pl,
                cudaStream_t s, void *raw_acc = nullptr, int raw_bits = 0, int64_t raw_ld = 0) {
    const int64_t M = A.rows, N = B.rows, K = A.k;
    CUtensorMap ta, tb;
    int st;
    if ((st = tmap_2d(&ta, A.mant, K, M, A.ld, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))) return st;
    if ((st = tmap_2d(&tb, B.mant, K, N, B.ld, 128, pl.pair ? pl.bn / 2 : pl.bn, CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    // pairs with a fused FIT, and single CTAs with four epilogue warpgroups on 128-wide tiles
    // of 32-column groups: the output as 64 x 128 boxes (64-byte swizzle) for staged stores
    CUtensorMap ty;
    const bool staged = pl.fused && (pl.pair || (pl.nwg == 4 && pl.bn == 128 && out->g_cols == 32 &&
                                                 N % 128 == 0 && aligned16(out->mant) && out->ld % 16 == 0));
    if (staged && (st = tmap_2d(&ty, out->mant, N, M, out->ld, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))) return st;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = (int)M;
    p.N = (int)N;
    p.n_kblk = pl.n_kblk;
    p.n_mtiles = pl.n_mtiles;
    p.n_ntiles = pl.n_ntiles;
    p.splits = pl.splits;
    p.kblk_per_split = pl.kblk_per_split;
    p.num_units = pl.units;
    p.eA = A.exp;
    p.eA_div = A.exp_div;
    p.eB = B.exp;
    p.eB_div = B.exp_div;
    p.G = (int)std::min<int64_t>(out->g_cols, N);
    p.fast_slack = fast_slack_for(K);
    p.out = out->mant;
    p.out_ld = out->ld;
    p.out_exp = out->exp;
    p.out_exp_ld = n_grp_cols(out);
    p.ws32 = pl.ws32;
    p.ws_ld = pl.ws_ld;
    p.ws_split_stride = M * pl.ws_ld;
    p.stage_tx_bytes = (uint32_t)(pl.pair ? 2 * (128 * 128 + (pl.bn / 2) * 128) : 128 * 128 + pl.bn * 128);
    p.wait_ns = g_wait_ns;
    p.drain_ns = kDrainNs;
    p.epi = pl.fused ? EPI_FIT_ROW : (pl.ro16r ? EPI_RO16R : EPI_I32);
    p.qb = g_mantissa_bits.load(std::memory_order_relaxed);
    p.nwg = pl.nwg;
    p.ws16 = pl.ws16;
    p.ws16_ld = pl.ws16_ld;
    p.tile_need = pl.tneed;
    p.tn_ld = pl.tn_ld;
    if ((st = launch_gemm(pl.bn, 128, LOAD_2D, ta, tb, p, pl.grid, s, 2.0 * (double)M * (double)N * (double)K,
                          pl.pair, staged ? &ty : nullptr)))
        return st;
    if (pl.fused) return ICT_OK;
    if (raw_acc) return launch_sum_slices(pl, M, N, raw_acc, raw_bits, raw_ld, s);
    if (pl.ro16r) {
        Ro16RowsArgs r;
        memset(&r, 0, sizeof(r));
        r.v = pl.ws16;
        r.rows = M;
        r.cols = N;
        r.ld = pl.ws16_ld;
        r.need = pl.tneed;
        r.tn_ld = pl.tn_ld;
        r.part_cols = pl.bn / 2;
        r.out = out->mant;
        r.out_ld = out->ld;
        r.out_exp = out->exp;
        r.out_exp_ld = n_grp_cols(out);
        KTimer kt(s, KC_REQUANT, 3.0 * (double)M * (double)N);
        ro16_rows_round_kernel<<<(unsigned)cdiv64(M, 8), 256, 0, s>>>(r);
        counted(1);
        return launch_status();
    }
    RequantArgs a;
    memset(&a, 0, sizeof(a));
    a.qb = g_mantissa_bits.load(std::memory_order_relaxed);
    a.v32 = pl.ws32;
    a.nsplit = pl.splits;
    a.split_stride = M * pl.ws_ld;
    a.rows = M;
    a.cols = N;
    a.ld = pl.ws_ld;
    a.cs = 1;
    a.row_exp = A.exp;
    a.row_div = A.exp_div;
    a.col_exp = B.exp;
    a.col_div = B.exp_div;
    a.out = out->mant;
    a.out_ld = out->ld;
    a.out_exp = out->exp;
    a.G = (int)std::min<int64_t>(out->g_cols, N);
    a.ngc = n_grp_cols(out);
    return launch_requant_rows(a, s);
}

// ---- linear layer

struct LinearPlan {
    AlignJob jobs[2];
    int njobs;
    Operand A, B;
    ProductPlan pp;
    const ict_tensor *out;
    bool empty;  // K == 0: the result is zero
};

int plan_linear(int op, const ict_tensor *a, const ict_tensor *b, const ict_tensor *out, Ws &ws,
                LinearPlan *lp) {
    int st;
    if ((st = check_tensor(a)) || (st = check_tensor(b)) || (st = check_tensor(out))) return st;
    int64_t M, N, K;
    if (op == ICT_OP_LINEAR_FWD) {  // Y = X W^T
        if (a->cols != b->cols) return ICT_ERR_INVALID_ARG;
        M = a->rows, N = b->rows, K = a->cols;
    } else if (op == ICT_OP_LINEAR_BWD_DATA) {  // dX = dY W
        if (a->cols != b->rows) return ICT_ERR_INVALID_ARG;
        M = a->rows, N = b->cols, K = a->cols;
    } else if (op == ICT_OP_LINEAR_BWD_WEIGHT) {  // dW = dY^T X
        if (a->rows != b->rows) return ICT_ERR_INVALID_ARG;
        M = a->cols, N = b->cols, K = a->rows;
    } else {
        return ICT_ERR_INVALID_ARG;
    }
    if (out->rows != M || out->cols != N) return ICT_ERR_INVALID_ARG;
    if (out->g_rows != 1 && M > 1) return ICT_ERR_LAYOUT;
    if ((st = check_vec(out))) return st;
    if ((st = check_vec(a)) || (st = check_vec(b))) return st;
    lp->out = out;
    lp->njobs = 0;
    lp->empty = (K == 0);
    if (M == 0 || N == 0 || K == 0) return ICT_OK;
    if (op == ICT_OP_LINEAR_FWD) {
        lp->A = operand_rows(a, ws, lp->jobs, &lp->njobs);
        lp->B = operand_rows(b, ws, lp->jobs, &lp->njobs);
    } else if (op == ICT_OP_LINEAR_BWD_DATA) {
        lp->A = operand_rows(a, ws, lp->jobs, &lp->njobs);
        lp->B = operand_cols(b, ws, lp->jobs, &lp->njobs);
    } else {
        lp->A = operand_cols(a, ws, lp->jobs, &lp->njobs);
        lp->B = operand_cols(b, ws, lp->jobs, &lp->njobs);
    }
    lp->pp = plan_product(M, N, K, out, planning_sms(), op == ICT_OP_LINEAR_BWD_WEIGHT, ws);
    return ICT_OK;
}

int run_linear(const LinearPlan &lp, cudaStream_t s) {
    if (lp.empty) return launch_zero(lp.out, s);
    if (lp.out->rows == 0 || lp.out->cols == 0) return ICT_OK;
    int st;
    if ((st = launch_aligns(lp.jobs, lp.njobs, s))) return st;
    return run_product(lp.A, lp.B, lp.out, lp.pp, s);
}

int linear_entry(int op, const ict_tensor *a, const ict_tensor *b, ict_tensor *out, void *ws,
                 size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if (ws && ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    LinearPlan lp;
    Ws w = make_ws(ws, ws_bytes, false);
    if ((st = plan_linear(op, a, b, out, w, &lp))) return st;
    if (w.used > ws_bytes || (w.used && !ws)) return ICT_ERR_WORKSPACE;
    return run_linear(lp, (cudaStream_t)stream);
}

// ---- backward weight of a batch split across devices
//
// dW = dY^T X contracts over the batch.  With the batch split, every device aligns its
// shard to targets that hold for the whole batch (the maxima over all shards, found by
// ict_linear_bwd_weight_targets on each device and a MAX reduction between them) and
// contracts it exactly; the integer sums of all shards add up to the sums of the whole
// batch, which one FIT (ict_requant) turns into the single-device result bit for bit.

// Operand whose contracted index runs along the tensor's rows, aligned per column to
// caller-given targets and transposed into K-major rows.
Operand operand_cols_given(const ict_tensor *t, const int8_t *e_target, Ws &ws, AlignJob *jobs, int *njobs) {
    const int64_t ld = round_up(t->rows, 16);
    int8_t *m = (int8_t *)ws.take((size_t)t->cols * ld);
    AlignJob j{t, 0, true, m, ld, const_cast<int8_t *>(e_target), nullptr};
    j.given = true;
    jobs[(*njobs)++] = j;
    return Operand{m, t->cols, t->rows, ld, e_target, 1};
}

int check_split_operands(const ict_tensor *dY, const ict_tensor *X) {
    int st;
    if ((st = check_tensor(dY)) || (st = check_tensor(X))) return st;
    if (dY->rows != X->rows) return ICT_ERR_INVALID_ARG;
    if ((st = check_vec(dY)) || (st = check_vec(X))) return st;
    return ICT_OK;
}

struct TargetsPlan {
    AlignJob jobs[2];
    AlignLaunch L[2];
};

int plan_targets(const ict_tensor *dY, const ict_tensor *X, int8_t *e_dy, int8_t *e_x, Ws &ws, TargetsPlan *tp) {
    const ict_tensor *t[2] = {dY, X};
    int8_t *e[2] = {e_dy, e_x};
    for (int i = 0; i < 2; ++i) {
        int32_t *cm = (int32_t *)ws.take((size_t)n_grp_cols(t[i]) * 4);
        tp->jobs[i] = AlignJob{t[i], 0, false, nullptr, 0, e[i], cm};
        tp->L[i] = plan_align(tp->jobs[i], planning_sms());
    }
    return ICT_OK;
}

int run_targets(const TargetsPlan &tp, cudaStream_t s) {
    const int64_t K = tp.jobs[0].t->rows;
    if (K == 0) {  // no rows: every target is E_ZERO
        for (int i = 0; i < 2; ++i)
            if (tp.jobs[i].t->cols &&
                cudaMemsetAsync(tp.jobs[i].e_star, 0x80, (size_t)tp.jobs[i].t->cols, s) != cudaSuccess)
                return ICT_ERR_CUDA;
        return ICT_OK;
    }
    const bool paired = tp.L[0].estar == 2 && tp.L[1].estar == 2;
    if (!paired) {  // one block per group column, no scratch
        for (int i = 0; i < 2; ++i) {
            const AlignArgs &a = tp.L[i].a;
            KTimer kt(s, KC_ESTAR, (double)tp.L[i].n_exp + (double)a.cols);
            estar_cols_kernel<<<(unsigned)a.ngc, 256, 0, s>>>(a);
            counted(1);
        }
        return launch_status();
    }
    AlignPair P;
    memset(&P, 0, sizeof(P));
    double work = 0;
    for (int i = 0; i < 2; ++i) {
        P.a[i] = tp.L[i].a;
        P.cm[i] = tp.jobs[i].col_max;
        P.used[i] = tp.L[i].used;
        work += (double)tp.L[i].n_exp + 8.0 * (double)tp.L[i].a.ngc + (double)tp.L[i].a.cols;
        if (cudaMemsetAsync(tp.jobs[i].col_max, 0x80, (size_t)tp.L[i].a.ngc * 4, s) != cudaSuccess)
            return ICT_ERR_CUDA;
    }
    KTimer kt(s, KC_ESTAR, work);
    const int64_t ngc = std::max(P.a[0].ngc, P.a[1].ngc), cols = std::max(P.a[0].cols, P.a[1].cols);
    estar_cols_scratch_kernel<<<dim3((unsigned)std::max(tp.L[0].blocks, tp.L[1].blocks), 2), 256, (size_t)ngc * 4,
                                s>>>(P);
    estar_expand_kernel<<<dim3((unsigned)cdiv64(cols, 256), 2), 256, 0, s>>>(P);
    counted(2);
    return launch_status();
}

struct PartialPlan {
    AlignJob jobs[2];
    int njobs;
    Operand A, B;
    ProductPlan pp;
    ict_tensor shape;  // [N][K] with one group per row: tiling only, nothing is written to it
    int64_t M, N, K;
};

int plan_partial(const ict_tensor *dY, const ict_tensor *X, const int8_t *e_dy, const int8_t *e_x, Ws &ws,
                 PartialPlan *pp) {
    pp->M = dY->cols, pp->N = X->cols, pp->K = dY->rows;
    pp->njobs = 0;
    if (pp->M == 0 || pp->N == 0 || pp->K == 0) return ICT_OK;
    pp->A = operand_cols_given(dY, e_dy, ws, pp->jobs, &pp->njobs);
    pp->B = operand_cols_given(X, e_x, ws, pp->jobs, &pp->njobs);
    memset(&pp->shape, 0, sizeof(pp->shape));
    pp->shape.rows = pp->M;
    pp->shape.cols = pp->N;
    pp->shape.ld = pp->N;
    pp->shape.g_rows = 1;
    pp->shape.g_cols = (int32_t)pp->N;
    pp->pp = plan_product(pp->M, pp->N, pp->K, &pp->shape, planning_sms(), true, ws, true);
    return ICT_OK;
}

// ---- convolution (implicit GEMM, NHWC / KRSC, "same" 3x3-style, stride 1)

struct ConvPlan {
    AlignJob jobs[2];
    int njobs;
    bool weight_prep;      // backward-data: W'[c][(r,s,k)] aligned per input channel
    ConvWeightArgs wprep;
    const int8_t *a_mant;  // dense NHWC activation operand fed to TMA
    int a_c;               // its channel count (the contracted channels)
    const int8_t *eA;
    int eA_div;
    const int8_t *b_mant;  // K-major weight operand [N][taps * a_c]
    int64_t b_ld;
    const int8_t *eB;
    int eB_div;
    int64_t out_rows, out_cols;
    int bn, rows_per_tile, tiles_per_img;
    bool global_groups;
    int32_t *gmax;
    int n_gcols;
    // groups spanning all pixels: int16 sums rounded to odd at a per-tile exponent
    int16_t *ws16;
    int64_t ws16_ld;
    int32_t *tile_need;  // [m tiles][n_gcols]
};

int plan_conv(int dir, const ict_conv_desc *d, const ict_tensor *a, const ict_tensor *b,
              const ict_tensor *out, Ws &ws, ConvPlan *cp) {
    int st;
    if (!d) return ICT_ERR_INVALID_ARG;
    if ((st = check_tensor(a)) || (st = check_tensor(b)) || (st = check_tensor(out))) return st;
    if (d->n < 1 || d->h < 1 || d->w < 1 || d->c < 1 || d->k < 1 || d->r < 1 || d->s < 1 ||
        d->stride < 1 || d->pad < 0)
        return ICT_ERR_INVALID_ARG;
    if (d->stride != 1 || d->r != d->s || 2 * d->pad != d->r - 1) return ICT_ERR_LAYOUT;
    if (d->c % 64 || d->k % 64 || d->c > kConvMaxChannels || d->k > kConvMaxChannels || d->w > 128)
        return ICT_ERR_LAYOUT;
    const int64_t npix = (int64_t)d->n * d->h * d->w, RS = (int64_t)d->r * d->s;
    if (dir != ICT_CONV_FWD && dir != ICT_CONV_BWD_DATA) return ICT_ERR_INVALID_ARG;
    const int64_t act_c = dir == ICT_CONV_FWD ? d->c : d->k;  // contracted channels
    const int64_t out_c = dir == ICT_CONV_FWD ? d->k : d->c;
    if (a->rows != npix || a->cols != act_c) return ICT_ERR_INVALID_ARG;
    if (b->rows != d->k || b->cols != RS * d->c) return ICT_ERR_INVALID_ARG;
    if (out->rows != npix || out->cols != out_c) return ICT_ERR_INVALID_ARG;
    if (a->g_rows < a->rows) return ICT_ERR_LAYOUT;  // activation exponents uniform over pixels
    if ((st = check_vec(a)) || (st = check_vec(b)) || (st = check_vec(out))) return st;
    cp->global_groups = out->g_rows >= out->rows;
    if (!cp->global_groups && out->g_rows != 1) return ICT_ERR_LAYOUT;
    cp->bn = pick_bn(out_c);
    const int64_t G = out->g_cols;
    if (!(G >= out_c ? out_c <= cp->bn : (cp->bn % G == 0 && G % 32 == 0))) return ICT_ERR_LAYOUT;
    cp->out_rows = npix;
    cp->out_cols = out_c;
    cp->rows_per_tile = std::min(128 / d->w, d->h);
    cp->tiles_per_img = (int)cdiv64(d->h, cp->rows_per_tile);
    cp->a_c = (int)act_c;
    cp->njobs = 0;
    // activation operand: aligned along channels unless already uniform; dense NHWC
    if (uniform_along_cols(a) && a->ld == act_c) {
        cp->a_mant = a->mant;
        cp->eA = a->exp;
        cp->eA_div = clamp_div(a->g_rows, a->rows);
    } else {
        int8_t *m = (int8_t *)ws.take((size_t)npix * act_c);
        int8_t *e = (int8_t *)ws.take((size_t)npix);
        cp->jobs[cp->njobs++] = AlignJob{a, 1, false, m, act_c, e, nullptr};
        cp->a_mant = m;
        cp->eA = e;
        cp->eA_div = 1;
    }
    // weight operand
    cp->weight_prep = false;
    if (dir == ICT_CONV_FWD) {  // contracted (r, s, c) runs along W's rows: align per k
        if (uniform_along_cols(b)) {
            cp->b_mant = b->mant;
            cp->b_ld = b->ld;
            cp->eB = b->exp;
            cp->eB_div = clamp_div(b->g_rows, b->rows);
        } else {
            int8_t *m = (int8_t *)ws.take((size_t)b->rows * b->cols);
            int8_t *e = (int8_t *)ws.take((size_t)b->rows);
            cp->jobs[cp->njobs++] = AlignJob{b, 1, false, m, b->cols, e, nullptr};
            cp->b_mant = m;
            cp->b_ld = b->cols;
            cp->eB = e;
            cp->eB_div = 1;
        }
    } else {
        const int64_t ld = round_up(RS * d->k, 16);
        int8_t *m = (int8_t *)ws.take((size_t)d->c * ld);
        int8_t *e = (int8_t *)ws.take((size_t)d->c);
        ConvWeightArgs w;
        w.w = b->mant;
        w.w_exp = b->exp;
        w.ld = b->ld;
        w.ngc = n_grp_cols(b);
        w.g_rows = clamp_div(b->g_rows, b->rows);
        w.g_cols = clamp_div(b->g_cols, b->cols);
        w.K = d->k;
        w.RS = (int)RS;
        w.C = d->c;
        w.e_star = e;
        w.out = m;
        w.out_ld = ld;
        cp->wprep = w;
        cp->weight_prep = true;
        cp->b_mant = m;
        cp->b_ld = ld;
        cp->eB = e;
        cp->eB_div = 1;
    }
    cp->n_gcols = (int)n_grp_cols(out);
    cp->gmax = cp->global_groups ? (int32_t *)ws.take((size_t)cp->n_gcols * 4) : nullptr;
    // groups spanning all pixels: one Product pass writes int16 sums rounded to odd at a
    // per-tile exponent, every tile's need and every group's largest need; a streaming
    // pass rounds them with the groups' exponents
    cp->ws16 = nullptr;
    cp->tile_need = nullptr;
    if (cp->global_groups) {
        cp->ws16_ld = round_up(out_c, 32);
        cp->ws16 = (int16_t *)ws.take((size_t)npix * cp->ws16_ld * 2);
        cp->tile_need = (int32_t *)ws.take((size_t)d->n * cp->tiles_per_img * cp->n_gcols * 4);
    }
    return ICT_OK;
}

// phase bit 1: operand preparation and the first Product pass; bit 2: the pass that
// rounds with the groups' needs in cp.gmax (groups spanning all pixels).  3: both.

// act (ACT_*): an activation applied to the rounded output, fused into the streaming
// rounding pass of all-pixel groups, else a clip pass over the output in place.
int run_conv(int dir, const ict_conv_desc *d, const ict_tensor *out, const ConvPlan &cp, int sms,
             cudaStream_t s, int phase = 3, int act = ACT_NONE) {
    int st;
    for (int i = 0; (phase & 1) && i < cp.njobs; ++i)
        if ((st = launch_align(cp.jobs[i], s))) return st;
    if ((phase & 1) && cp.weight_prep) {
        const int64_t n = (int64_t)d->c * d->r * d->s * d->k;
        {
            KTimer kt(s, KC_ESTAR, (double)n);
            conv_wt_estar_kernel<<<d->c, 256, 0, s>>>(cp.wprep);
        }
        KTimer kt(s, KC_OTHER, 2.0 * (double)n);
        conv_wt_prep_kernel<<<(unsigned)cdiv64(n, 256), 256, 0, s>>>(cp.wprep);
        counted(2);
        if ((st = launch_status())) return st;
    }
    CUtensorMap ta, tb;
    // halo tiles: 3 x 3 filters, 64 contracted channels (the nine weight blocks resident),
    // image rows a multiple of 8 pixels (each row shift a whole number of swizzle atoms), a
    // box of rows + 2 image rows plus the MMA's overhang inside one 16 KB slot, all-pixel
    // output groups on one N tile (the four-warpgroup RO16 epilogue)
    const bool halo = cp.global_groups && d->r == 3 && d->s == 3 && d->pad == 1 && cp.a_c == 64 && d->w % 8 == 0 &&
                      (int64_t)(cp.rows_per_tile + 2) * d->w * 64 <= kHaloSlot &&
                      (int64_t)2 * d->w * 64 + 128 * 64 <= kHaloSlot && cp.bn <= 128 && cp.out_cols <= cp.bn;
    // the ring form: 64-wide tiles (the weight's nine blocks and three 56 KB rings fit), a ring
    // that holds a restarting tile's rows and windows
    const int ring_rows = (int)(kRingBox / ((int64_t)d->w * 64)), ring_span = 2 + (int)cdiv64(128, d->w);
    const bool ring = halo && cp.bn == 64 && ring_span <= ring_rows;
    CUtensorMap ta2, tz;  // ring: the continuing tiles' boxes (the tile's own rows only), the int16 sums
    if ((st = tmap_nhwc(&ta, cp.a_mant, d->n, d->h, d->w, cp.a_c, cp.rows_per_tile + (halo ? 2 : 0)))) return st;
    if (ring && (st = tmap_nhwc(&ta2, cp.a_mant, d->n, d->h, d->w, cp.a_c, cp.rows_per_tile))) return st;
    if (ring && (st = tmap_2d(&tz, cp.ws16, (uint64_t)cp.out_cols * 2, (uint64_t)cp.out_rows, (uint64_t)cp.ws16_ld * 2,
                              128, (uint32_t)(cp.rows_per_tile * d->w), CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    const int64_t ktot = (int64_t)d->r * d->s * cp.a_c;
    if ((st = tmap_2d(&tb, cp.b_mant, ktot, cp.out_cols, cp.b_ld, 64, cp.bn, CU_TENSOR_MAP_SWIZZLE_64B)))
        return st;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = (int)cp.out_rows;
    p.N = (int)cp.out_cols;
    p.n_kblk = (int)(ktot / 64);
    p.n_mtiles = d->n * cp.tiles_per_img;
    p.n_ntiles = (int)cdiv64(cp.out_cols, cp.bn);
    p.splits = 1;
    p.kblk_per_split = p.n_kblk;
    p.num_units = p.n_mtiles * p.n_ntiles;
    p.eA = cp.eA;
    p.eA_div = cp.eA_div;
    p.eB = cp.eB;
    p.eB_div = cp.eB_div;
    p.G = (int)std::min<int64_t>(out->g_cols, cp.out_cols);
    p.fast_slack = fast_slack_for(ktot);
    p.out = out->mant;
    p.out_ld = out->ld;
    p.out_exp = out->exp;
    p.out_exp_ld = cp.n_gcols;
    p.gmax = cp.gmax;
    p.cv_W = d->w;
    p.cv_P = d->h;
    p.cv_rows = cp.rows_per_tile;
    p.cv_tiles_per_img = cp.tiles_per_img;
    p.cv_cblk = cp.a_c / 64;
    p.cv_S = d->s;
    p.cv_pad = d->pad;
    p.cv_sign = dir == ICT_CONV_FWD ? 1 : -1;
    // the weight operand stays in shared memory when all its K blocks fit the B ring
    p.b_resident = p.n_ntiles == 1 && p.n_kblk <= stages_for(cp.bn, 64);
    p.stage_tx_bytes = (uint32_t)(64 * d->w * cp.rows_per_tile + (p.b_resident ? 0 : 64 * cp.bn));
    if (halo) {  // one stage per 64-channel block: three boxes of rows + 2 image rows
        p.cv_bkblk = p.n_kblk;
        p.n_kblk = p.cv_cblk;
        p.kblk_per_split = p.n_kblk;
        p.b_resident = 1;
        p.stage_tx_bytes = (uint32_t)(3 * 64 * d->w * (cp.rows_per_tile + 2));
        p.cv_ring_rows = ring_rows;
        p.cv_ring_span = ring_span;
    }
    p.qb = 8;
    p.wait_ns = g_wait_ns;
    p.drain_ns = kDrainNs;
    const int grid = std::min(p.num_units, sms);
    const double ops = 2.0 * (double)cp.out_rows * (double)cp.out_cols * (double)ktot;
    if (!cp.global_groups) {
        p.epi = EPI_FIT_ROW;
        if ((st = launch_gemm(cp.bn, 64, LOAD_CONV, ta, tb, p, grid, s, ops))) return st;
        return act == ACT_NONE ? ICT_OK : launch_clip(out, nullptr, act == ACT_RELU6, const_cast<ict_tensor *>(out), s);
    }
    if (phase & 1) {
        {
            KTimer kt(s, KC_OTHER, 4.0 * (double)cp.n_gcols);
            fill_i32_kernel<<<(unsigned)cdiv64(cp.n_gcols, 256), 256, 0, s>>>(cp.gmax, cp.n_gcols, kNoExp);
        }
        counted(1);
    }
    p.epi = EPI_RO16;
    p.nwg = cp.bn <= 128 ? 4 : 2;
    p.ws16 = cp.ws16;
    p.ws16_ld = cp.ws16_ld;
    p.tile_need = cp.tile_need;
    if ((phase & 1) && (st = launch_gemm(cp.bn, 64, ring ? LOAD_CONV_RING : (halo ? LOAD_CONV_HALO : LOAD_CONV), ta, tb,
                                         p, grid, s, ops, false, ring ? &ta2 : nullptr, ring ? &tz : nullptr)))
        return st;
    if (!(phase & 2)) return ICT_OK;
    Ro16RoundArgs r;
    r.v = cp.ws16;
    r.rows = cp.out_rows;
    r.cols = cp.out_cols;
    r.ld = cp.ws16_ld;
    r.tile_need = cp.tile_need;
    r.gmax = cp.gmax;
    r.cv_W = d->w;
    r.cv_P = d->h;
    r.cv_rows = cp.rows_per_tile;
    r.cv_tiles_per_img = cp.tiles_per_img;
    r.G = p.G;
    r.ngc = cp.n_gcols;
    r.out = out->mant;
    r.out_ld = out->ld;
    r.out_exp = out->exp;
    r.act = act;
    const int64_t image_rows = cp.out_rows / d->w;  // one block per image row of the batch
    KTimer kt(s, KC_REQUANT, 3.0 * (double)cp.out_rows * (double)cp.out_cols);
    ro16_round_kernel<<<(unsigned)image_rows, 256, 0, s>>>(r);
    counted(1);
    return launch_status();
}

// ---- convolution backward-weight: dW[k][(r,s,c)] = sum over output pixels of
// dY[pix][k] * X[pix shifted by (r,s)][c], both NHWC operands read MN-major by TMA

struct WgradPlan {
    int hrows, hblk, kpix, atoms, mtiles, ntiles, splits, kblk_per_split, n_kblk, units;
    int64_t M, N, ws_ld;
    int32_t *partial;
    int64_t *sums64;  // [N][sums_ld] slice sums
    int64_t sums_ld;
    int8_t *e_rows, *e_cols;
};

int plan_wgrad(const ict_conv_desc *d, const ict_tensor *dY, const ict_tensor *X, const ict_tensor *dW,
               int sms, Ws &ws, WgradPlan *wp) {
    int st;
    if ((st = check_tensor(dY)) || (st = check_tensor(X)) || (st = check_tensor(dW))) return st;
    if (d->stride != 1 || d->r != d->s || 2 * d->pad != d->r - 1) return ICT_ERR_LAYOUT;
    if (d->c % 64 || d->k % 64 || d->w > 256) return ICT_ERR_LAYOUT;
    const int64_t npix = (int64_t)d->n * d->h * d->w, RS = (int64_t)d->r * d->s;
    if (dY->rows != npix || dY->cols != d->k || X->rows != npix || X->cols != d->c) return ICT_ERR_INVALID_ARG;
    if (dW->rows != d->k || dW->cols != RS * d->c) return ICT_ERR_INVALID_ARG;
    if (dY->g_rows < dY->rows || X->g_rows < X->rows) return ICT_ERR_LAYOUT;  // uniform over pixels
    if (dY->ld != d->k || X->ld != d->c) return ICT_ERR_LAYOUT;                // dense NHWC
    if (dW->g_rows != 1 && dW->rows > 1) return ICT_ERR_LAYOUT;
    if ((st = check_vec(dY)) || (st = check_vec(X)) || (st = check_vec(dW))) return st;
    // K block: whole image rows, a multiple of 32 pixels, at most 256
    wp->hrows = 0;
    for (int h = 1; d->w * h <= 256; ++h)  // rows past the image end are zero-filled
        if ((d->w * h) % 32 == 0) { wp->hrows = h; break; }
    if (!wp->hrows) return ICT_ERR_LAYOUT;
    wp->kpix = d->w * wp->hrows;
    wp->hblk = (int)cdiv64(d->h, wp->hrows);
    wp->n_kblk = d->n * wp->hblk;
    wp->atoms = (int)(RS * d->c / 64);
    wp->mtiles = (wp->atoms + 1) / 2;
    wp->ntiles = d->k / 64;
    const int tiles = wp->mtiles * wp->ntiles;
    int splits = std::max(1, std::min(sms / tiles, wp->n_kblk / 4));
    // int32 partials stay exact: pixels per slice times 127^2 below 2^31
    const int max_kblk = std::max(1, (int)(((1ll << 31) - 1) / (16129ll * wp->kpix)));
    if (cdiv64(wp->n_kblk, splits) > max_kblk) splits = (int)cdiv64(wp->n_kblk, max_kblk);
    wp->kblk_per_split = (int)cdiv64(wp->n_kblk, splits);
    wp->splits = (int)cdiv64(wp->n_kblk, wp->kblk_per_split);
    wp->units = tiles * wp->splits;
    wp->M = RS * d->c;
    wp->N = d->k;
    wp->ws_ld = round_up(wp->N, 32);
    wp->partial = (int32_t *)ws.take((size_t)wp->splits * wp->M * wp->ws_ld * 4);
    wp->sums64 = (int64_t *)ws.take((size_t)wp->M * wp->N * 8);
    wp->sums_ld = wp->M;
    wp->e_rows = (int8_t *)ws.take((size_t)wp->M);
    wp->e_cols = (int8_t *)ws.take((size_t)wp->N);
    return ICT_OK;
}

// sums_only: the int64 sums (and the exponent vectors) are the result; no FIT.
int run_wgrad(const ict_conv_desc *d, const ict_tensor *dY, const ict_tensor *X, const ict_tensor *dW,
              const WgradPlan &wp, int sms, cudaStream_t s, bool sums_only = false) {
    int st;
    const int RS = d->r * d->s;
    {
        KTimer kt(s, KC_OTHER, 2.0 * (double)(wp.M + wp.N));
        conv_wgrad_exp_kernel<<<(unsigned)cdiv64(std::max<int64_t>(wp.M, wp.N), 256), 256, 0, s>>>(
            X->exp, clamp_div(X->g_cols, X->cols), dY->exp, clamp_div(dY->g_cols, dY->cols), d->c, RS, d->k,
            wp.e_rows, wp.e_cols);
    }
    counted(1);
    if ((st = launch_status())) return st;
    CUtensorMap ta, tb;
    if ((st = tmap_nhwc(&ta, X->mant, d->n, d->h, d->w, d->c, wp.hrows))) return st;
    if ((st = tmap_nhwc(&tb, dY->mant, d->n, d->h, d->w, d->k, wp.hrows))) return st;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = (int)wp.M;
    p.N = (int)wp.N;
    p.n_kblk = wp.n_kblk;
    p.n_mtiles = wp.mtiles;
    p.n_ntiles = wp.ntiles;
    p.splits = wp.splits;
    p.kblk_per_split = wp.kblk_per_split;
    p.num_units = wp.units;
    p.eA = wp.e_rows;
    p.eA_div = 1;
    p.eB = wp.e_cols;
    p.eB_div = 1;
    p.G = (int)wp.N;
    p.ws32 = wp.partial;
    p.ws_ld = wp.ws_ld;
    p.ws_split_stride = wp.M * wp.ws_ld;
    p.cv_cblk = d->c / 64;
    p.cv_S = d->s;
    p.cv_pad = d->pad;
    p.wg_hrows = wp.hrows;
    p.wg_hblk = wp.hblk;
    p.wg_kpix = wp.kpix;
    p.wg_atoms = wp.atoms;
    p.wait_ns = g_wait_ns;
    p.drain_ns = kDrainNs;
    p.epi = EPI_I32;
    if ((st = launch_gemm(64, 256, LOAD_CONV_WGRAD, ta, tb, p, std::min(wp.units, sms), s,
                          2.0 * (double)wp.M * (double)wp.N * (double)d->n * d->h * d->w)))
        return st;
    // dW[k][j] = sum over slices of partial[j][k]: the slices are summed and transposed
    // into int64 sums64[k][j], then FIT per row k with exponent e_cols[k] + e_rows[j]
    {
        KTimer kt(s, KC_REQUANT, 4.0 * (double)wp.splits * (double)wp.M * (double)wp.N + 8.0 * (double)wp.M * wp.N);
        sum_slices_t_kernel<<<dim3((unsigned)cdiv64(wp.N, 32), (unsigned)cdiv64(wp.M, 32)), 256, 0, s>>>(
            wp.partial, wp.splits, wp.M * wp.ws_ld, wp.M, wp.N, wp.ws_ld, wp.sums64, wp.sums_ld);
        counted(1);
        if ((st = launch_status())) return st;
    }
    if (sums_only) return ICT_OK;
    RequantArgs a;
    memset(&a, 0, sizeof(a));
    a.qb = 8;  // convolution: INT8 only
    a.v64 = wp.sums64;
    a.nsplit = 1;
    a.rows = wp.N;
    a.cols = wp.M;
    a.ld = wp.sums_ld;
    a.cs = 1;
    a.row_exp = wp.e_cols;
    a.row_div = 1;
    a.col_exp = wp.e_rows;
    a.col_div = 1;
    a.out = dW->mant;
    a.out_ld = dW->ld;
    a.out_exp = dW->exp;
    a.G = clamp_div(dW->g_cols, dW->cols);
    a.ngc = n_grp_cols(dW);
    return launch_requant_rows(a, s);
}

// ---- SGD

int fill_sgd_tensor(ict_tensor *W, ict_tensor *V, const ict_tensor *G, SgdTensor *t) {
    int st;
    if ((st = check_tensor(W)) || (st = check_tensor(V)) || (st = check_tensor(G))) return st;
    if (W->rows != V->rows || W->rows != G->rows || W->cols != V->cols || W->cols != G->cols)
        return ICT_ERR_INVALID_ARG;
    if (W->g_cols != V->g_cols || W->g_cols != G->g_cols) return ICT_ERR_INVALID_ARG;
    if ((W->g_rows != 1 || V->g_rows != 1 || G->g_rows != 1) && W->rows > 1) return ICT_ERR_LAYOUT;
    if (W->ld != V->ld || W->ld != G->ld) return ICT_ERR_LAYOUT;
    t->w = W->mant;
    t->w_exp = W->exp;
    t->v = V->mant;
    t->v_exp = V->exp;
    t->g = G->mant;
    t->g_exp = G->exp;
    t->rows = W->rows;
    t->cols = W->cols;
    t->ld = W->ld;
    t->G = clamp_div(W->g_cols, W->cols);
    t->ngc = n_grp_cols(W);
    return ICT_OK;
}

int check_sgd_params(const ict_sgd_params *p) {
    if (!p) return ICT_ERR_INVALID_ARG;
    if (p->mom_shift < 0 || p->mom_shift > 62 || p->lr_shift < 0 || p->lr_shift > 62) return ICT_ERR_INVALID_ARG;
    if (p->mom_mul < -65535 || p->mom_mul > 65535 || p->lr_mul < -65535 || p->lr_mul > 65535)
        return ICT_ERR_INVALID_ARG;
    return ICT_OK;
}

template <int L, int CPL>
int launch_sgd_vec(const SgdArgs &a, int sms, cudaStream_t s) {
    constexpr int gpb = 8 * (32 / L);  // groups per block and pass
    const int64_t blocks = std::min<int64_t>(cdiv64(a.total_groups, gpb), (int64_t)sms * 8);
    if (a.n == 1)
        sgd_vec_kernel<L, CPL, true><<<(unsigned)blocks, 256, 0, s>>>(a);
    else
        sgd_vec_kernel<L, CPL, false><<<(unsigned)blocks, 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

int bitlen_u64(uint64_t v) {
    int b = 0;
    while (v >> b) ++b;
    return b;
}

// Vectorised kernel when every tensor shares one group width G (a multiple of 16, at
// most 2048): L lanes per group, CPL 16-byte chunks per lane; else one warp per group.
int run_sgd(SgdArgs &a, int sms, cudaStream_t s) {
    if (a.total_groups == 0) return ICT_OK;
    double elems = 0;
    for (int i = 0; i < a.n; ++i) elems += (double)a.t[i].rows * (double)a.t[i].cols;
    KTimer kt(s, KC_SGD, 5.0 * elems + 5.0 * (double)a.total_groups);
    bool vec = true;
    const int G = a.t[0].G;
    for (int i = 0; i < a.n; ++i)
        vec = vec && a.t[i].G == G && (a.t[i].ld & 15) == 0 && aligned16(a.t[i].w) && aligned16(a.t[i].v) &&
              aligned16(a.t[i].g);
    vec = vec && G % 16 == 0 && G <= 2048;
    const SgdTensor &t0 = a.t[0];
    // one dense tensor, one group per row of 16 L CPL elements: the prefetching kernel,
    // two chunks per lane where the group allows (groups of 32 to 1024 elements)
    const int Lr = G / 16;
    if (vec && a.n == 1 && t0.ngc == 1 && t0.cols == t0.G && t0.ld == t0.G && Lr >= 1 && Lr <= 32 &&
        (Lr & (Lr - 1)) == 0) {
        const int CPL = (Lr >= 2 && Lr <= 64) ? 2 : 1, L = Lr / CPL;
        const int64_t gpb = 8 * (32 / L);
        const unsigned blocks = (unsigned)std::min<int64_t>(cdiv64(a.total_groups, gpb), (int64_t)sms * 8);
        bool done = true;
        if (CPL == 2) {
            switch (L) {
                case 1: sgd_rows_kernel<1, 2><<<blocks, 256, 0, s>>>(a); break;
                case 2: sgd_rows_kernel<2, 2><<<blocks, 256, 0, s>>>(a); break;
                case 4: sgd_rows_kernel<4, 2><<<blocks, 256, 0, s>>>(a); break;
                case 8: sgd_rows_kernel<8, 2><<<blocks, 256, 0, s>>>(a); break;
                case 16: sgd_rows_kernel<16, 2><<<blocks, 256, 0, s>>>(a); break;
                default: done = false;
            }
        } else {
            switch (L) {
                case 1: sgd_rows_kernel<1, 1><<<blocks, 256, 0, s>>>(a); break;
                case 32: sgd_rows_kernel<32, 1><<<blocks, 256, 0, s>>>(a); break;
                default: done = false;
            }
        }
        if (done) {
            counted(1);
            return launch_status();
        }
    }
    if (vec) {
        const int chunks = G / 16;
        if (chunks <= 1) return launch_sgd_vec<1, 1>(a, sms, s);
        if (chunks <= 2) return launch_sgd_vec<2, 1>(a, sms, s);
        if (chunks <= 4) return launch_sgd_vec<4, 1>(a, sms, s);
        if (chunks <= 8) return launch_sgd_vec<8, 1>(a, sms, s);
        if (chunks <= 16) return launch_sgd_vec<16, 1>(a, sms, s);
        if (chunks <= 32) return launch_sgd_vec<32, 1>(a, sms, s);
        if (chunks <= 64) return launch_sgd_vec<32, 2>(a, sms, s);
        if (chunks <= 128) return launch_sgd_vec<32, 4>(a, sms, s);
    }
    const int64_t blocks = std::min<int64_t>(cdiv64(a.total_groups, 8), (int64_t)sms * 16);
    sgd_warp_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

// ---- allocation-free forward Product: fixed scratch inside the library

// One array per device that loads the library; host code must not pass its name to a
// kernel (on the host it is only a stand-in), so its device address is looked up with
// cudaGetSymbolAddress, with the device current, and kept per device together with the
// context it belongs to: after a device reset the module is loaded again (possibly at
// another address) in a new context, and the next call looks the address up again.
static __device__ __align__(256) uint8_t g_noalloc_scratch[ICT_NOALLOC_SCRATCH_BYTES];
struct NoallocSlot {
    void *ctx;
    void *addr;
};
NoallocSlot g_noalloc_slot[64];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (CtxGetCurrentFn)ptr;
    }
    return fn;
}

int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ICT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return ICT_ERR_CUDA;
    CUcontext ctx = nullptr;  // NULL until the runtime has made a context current on this thread
    if (get_ctx(&ctx) != CUDA_SUCCESS) return ICT_ERR_CUDA;
    NoallocSlot &slot = g_noalloc_slot[dev];
    if (!ctx || !slot.addr || slot.ctx != (void *)ctx) {
        void *p = nullptr;  // the lookup makes the device's primary context current
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ICT_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return ICT_ERR_CUDA;
        slot.ctx = (void *)ctx;
        slot.addr = p;
    }
    *out = slot.addr;
    return ICT_OK;
}

}  // namespace

// ====================================================================== C ABI

// Split-batch convolution, forward and backward-data with groups spanning all pixels:
// phase 1 writes this shard's largest need per group column into `need` (the int32 sums
// stay in ws), phase 2 rounds with the needs given (after the MAX over the shards).
int conv_split(int dir, const ict_conv_desc *d, const ict_tensor *a, const ict_tensor *b, const ict_tensor *out,
               int32_t *need, void *ws, size_t ws_bytes, void *stream, int phase) {
    int st, sms = 0;
    if ((st = device_info(&sms))) return st;
    if ((st = int8_only())) return st;
    if ((dir != ICT_CONV_FWD && dir != ICT_CONV_BWD_DATA) || !need) return ICT_ERR_INVALID_ARG;
    if (ws && ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    Ws w = make_ws(ws, ws_bytes, false);
    ConvPlan cp;
    if ((st = plan_conv(dir, d, a, b, out, w, &cp))) return st;
    if (!cp.global_groups) return ICT_ERR_LAYOUT;  // pixel-local groups: no exchange, call the whole Product
    if (w.used > ws_bytes || (w.used && !ws)) return ICT_ERR_WORKSPACE;
    cp.gmax = need;
    return run_conv(dir, d, out, cp, sms, (cudaStream_t)stream, phase);
}

// ---- pointwise primitives (ReLU / ReLU6, Sum)

// A tensor streamed by 16-byte vectors whose groups never straddle a vector.
int check_pointwise(const ict_tensor *t) {
    int st;
    if ((st = check_tensor(t))) return st;
    return check_vec(t);
}
bool same_groups(const ict_tensor *a, const ict_tensor *b) {
    return a->rows == b->rows && a->cols == b->cols && clamp_div(a->g_rows, a->rows) == clamp_div(b->g_rows, b->rows) &&
           clamp_div(a->g_cols, a->cols) == clamp_div(b->g_cols, b->cols);
}
unsigned stream_grid(int64_t nvec, int per_thread) {
    int sms = 148;
    device_info(&sms);
    const int64_t want = cdiv64(nvec, 256 * (int64_t)per_thread);
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
}

int launch_clip(const ict_tensor *X, const ict_tensor *dY, int six, ict_tensor *out, cudaStream_t s) {
    ClipArgs a;
    memset(&a, 0, sizeof(a));
    a.x = X->mant;
    a.x_exp = X->exp;
    a.ldx = X->ld;
    a.gx_rows = clamp_div(X->g_rows, X->rows);
    a.gx_cols = clamp_div(X->g_cols, X->cols);
    a.ngcx = n_grp_cols(X);
    if (dY) {
        a.dy = dY->mant;
        a.dy_exp = dY->exp;
        a.ldy = dY->ld;
    }
    a.out = out->mant;
    a.out_exp = out->exp;
    a.ldo = out->ld;
    a.rows = X->rows;
    a.cols = X->cols;
    a.six = six;
    a.n_exp = n_grp_rows(out) * n_grp_cols(out);
    const int64_t nvec = a.rows * (a.cols >> 4);
    if (std::max(nvec, a.n_exp) == 0) return ICT_OK;
    KTimer kt(s, KC_POINTWISE, (double)a.rows * (double)a.cols * (dY ? 3.0 : 2.0) + 2.0 * (double)a.n_exp);
    const unsigned grid = stream_grid(std::max(nvec, a.n_exp), 4);
    if (dY) clip_kernel<true><<<grid, 256, 0, s>>>(a);
    else clip_kernel<false><<<grid, 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

// Sum operands: one shape and one group partition, row-local (g_rows = 1) or spanning
// all rows; group columns a multiple of 16 wide unless one spans the row.
int check_sum(const ict_tensor *X, const ict_tensor *Y, const ict_tensor *Z, bool *global) {
    int st;
    if ((st = check_pointwise(X)) || (st = check_pointwise(Y)) || (st = check_pointwise(Z))) return st;
    if (X->rows != Y->rows || X->cols != Y->cols || X->rows != Z->rows || X->cols != Z->cols)
        return ICT_ERR_INVALID_ARG;
    if (!same_groups(X, Y) || !same_groups(X, Z)) return ICT_ERR_LAYOUT;
    const int gr = clamp_div(X->g_rows, X->rows);
    *global = X->rows > 1 && gr >= X->rows;
    if (gr != 1 && !*global) return ICT_ERR_LAYOUT;
    if (*global && n_grp_cols(X) > 8192) return ICT_ERR_LAYOUT;
    return ICT_OK;
}

// Average pool K x K, stride K: geometry checks and the arguments of both directions.
int plan_pool(bool bwd, const ict_tensor *in, int n, int h, int w, int K, const ict_tensor *out, PoolArgs *a) {
    int st;
    if ((st = check_tensor(in)) || (st = check_tensor(out))) return st;
    if (n < 1 || h < 1 || w < 1 || K < 1 || K > 16 || h % K || w % K) return ICT_ERR_INVALID_ARG;
    const int64_t P = h / K, Q = w / K, big = (int64_t)n * h * w, small = (int64_t)n * P * Q;
    if (in->rows != (bwd ? small : big) || out->rows != (bwd ? big : small) || in->cols != out->cols)
        return ICT_ERR_INVALID_ARG;
    if (!bwd && in->rows > 0 && in->g_rows < in->rows) return ICT_ERR_LAYOUT;  // pixel-uniform exponents
    memset(a, 0, sizeof(*a));
    a->in = in->mant, a->in_exp = in->exp, a->ld_in = in->ld, a->in_ngc = n_grp_cols(in);
    a->in_g_rows = clamp_div(in->g_rows, in->rows), a->in_g_cols = clamp_div(in->g_cols, in->cols);
    a->out = out->mant, a->out_exp = out->exp, a->ld_out = out->ld, a->out_ngc = n_grp_cols(out);
    a->out_g_rows = clamp_div(out->g_rows, out->rows), a->out_g_cols = clamp_div(out->g_cols, out->cols);
    a->out_rows = out->rows, a->C = out->cols;
    a->h = h, a->w = w, a->K = K, a->P = (int)P, a->Q = (int)Q, a->D = K * K, a->bwd = bwd;
    return ICT_OK;
}
int64_t pool_groups(const PoolArgs &a) { return cdiv64(a.out_rows, a.out_g_rows) * a.out_ngc; }

int run_pool(PoolArgs a, void *ws, size_t ws_bytes, cudaStream_t s) {
    const int64_t n = a.out_rows * a.C, groups = pool_groups(a);
    if (n == 0) return ICT_OK;
    if (!ws || ((uintptr_t)ws & 255) || ws_bytes < (size_t)groups * 4) return ICT_ERR_WORKSPACE;
    a.need = (int32_t *)ws;
    if (cudaMemsetAsync(a.need, 0x80, (size_t)groups * 4, s) != cudaSuccess) return ICT_ERR_CUDA;
    // algorithmic bytes: every input mantissa read once, every output written once
    const double bytes = a.bwd ? (double)n + (double)n / a.D : (double)n * (a.D + 1.0);
    KTimer kt(s, KC_POINTWISE, bytes);
    const unsigned grid = stream_grid(n, 1);
    pool_need_kernel<<<grid, 256, 0, s>>>(a);
    pool_round_kernel<<<grid, 256, 0, s>>>(a);
    counted(2);
    return launch_status();
}

int sum_entry(const ict_tensor *X, int32_t x_mul, int32_t x_shift, const ict_tensor *Y, int32_t y_mul,
              int32_t y_shift, ict_tensor *Z, int act, void *ws, size_t ws_bytes, void *stream);

extern "C" {

const char *ict_status_string(int32_t status) {
    switch (status) {
        case ICT_OK: return "ICT_OK";
        case ICT_ERR_INVALID_ARG: return "ICT_ERR_INVALID_ARG";
        case ICT_ERR_LAYOUT: return "ICT_ERR_LAYOUT";
        case ICT_ERR_ALIGNMENT: return "ICT_ERR_ALIGNMENT";
        case ICT_ERR_WORKSPACE: return "ICT_ERR_WORKSPACE";
        case ICT_ERR_UNSUPPORTED_ARCH: return "ICT_ERR_UNSUPPORTED_ARCH";
        case ICT_ERR_CUDA: return "ICT_ERR_CUDA";
        case ICT_ERR_DEVICE_TIMEOUT: return "ICT_ERR_DEVICE_TIMEOUT";
        case ICT_ERR_EXP_RANGE: return "ICT_ERR_EXP_RANGE";
        default: return "ICT_ERR_UNKNOWN";
    }
}

const char *ict_version(void) { return "libict 0.1 sm_100a"; }

uint64_t ict_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t ict_timing_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timing.on = on != 0;
    return ICT_OK;
}

int32_t ict_timing_read(int32_t kernel_class, double *ms_total, int64_t *launches, double *work,
                        int32_t reset) {
    if (kernel_class < 0 || kernel_class >= KC_N) return ICT_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_timing_mu);
    for (const TimedLaunch &t : g_timing.pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(t.b) != cudaSuccess || cudaEventElapsedTime(&ms, t.a, t.b) != cudaSuccess)
            return ICT_ERR_CUDA;
        g_timing.ms[t.kc] += ms;
        g_timing.n[t.kc] += 1;
        g_timing.work[t.kc] += t.work;
        g_timing.pool.push_back(t.a);
        g_timing.pool.push_back(t.b);
    }
    g_timing.pending.clear();
    if (ms_total) *ms_total = g_timing.ms[kernel_class];
    if (launches) *launches = g_timing.n[kernel_class];
    if (work) *work = g_timing.work[kernel_class];
    if (reset) {
        for (int k = 0; k < KC_N; ++k) g_timing.ms[k] = g_timing.work[k] = 0, g_timing.n[k] = 0;
    }
    return ICT_OK;
}

int32_t ict_get_device_status(int32_t *host_out, void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return ICT_ERR_CUDA;
    int32_t v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return ICT_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return ICT_ERR_CUDA;
    if (host_out) *host_out = v;
    if (v & (1 << ICT_ERR_DEVICE_TIMEOUT)) return ICT_ERR_DEVICE_TIMEOUT;
    if (v & (1 << ICT_ERR_EXP_RANGE)) return ICT_ERR_EXP_RANGE;
    return ICT_OK;
}

int32_t ict_selftest_wait_timeout(uint64_t limit_ns, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if (limit_ns == 0) return ICT_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
    counted(1);
    return launch_status();
}

int32_t ict_set_wait_limit_ns(uint64_t ns) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_wait_ns = ns ? ns : 2000000000ull;
    return ICT_OK;
}

int32_t ict_set_mantissa_bits(int32_t bits) {
    if (bits < 2 || bits > 8) return ICT_ERR_INVALID_ARG;
    g_mantissa_bits.store(bits, std::memory_order_relaxed);
    return ICT_OK;
}
int32_t ict_get_mantissa_bits(void) { return g_mantissa_bits.load(std::memory_order_relaxed); }

int32_t ict_requant(const void *vals, int32_t val_bits, int64_t rows, int64_t cols, int64_t ld_vals,
                    int32_t base_exp, const int8_t *row_exp, const int8_t *col_exp,
                    ict_tensor *out, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_tensor(out))) return st;
    if (val_bits != 32 && val_bits != 64) return ICT_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld_vals < cols || out->rows != rows || out->cols != cols)
        return ICT_ERR_INVALID_ARG;
    if (rows && cols && !vals) return ICT_ERR_INVALID_ARG;
    if (out->g_rows != 1 && rows > 1) return ICT_ERR_LAYOUT;
    RequantArgs a;
    memset(&a, 0, sizeof(a));
    a.qb = g_mantissa_bits.load(std::memory_order_relaxed);
    a.v32 = val_bits == 32 ? (const int32_t *)vals : nullptr;
    a.v64 = val_bits == 64 ? (const int64_t *)vals : nullptr;
    a.nsplit = 1;
    a.rows = rows;
    a.cols = cols;
    a.ld = ld_vals;
    a.cs = 1;
    a.base = base_exp;
    a.row_exp = row_exp;
    a.row_div = 1;
    a.col_exp = col_exp;
    a.col_div = 1;
    a.out = out->mant;
    a.out_ld = out->ld;
    a.out_exp = out->exp;
    a.G = clamp_div(out->g_cols, cols);
    a.ngc = n_grp_cols(out);
    return launch_requant_rows(a, (cudaStream_t)stream);
}

int32_t ict_align(const ict_tensor *in, int32_t axis, int32_t transpose, int8_t *out_mant,
                  int64_t ld_out, int8_t *e_star, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_tensor(in))) return st;
    if ((axis != 0 && axis != 1) || !out_mant || !e_star) return ICT_ERR_INVALID_ARG;
    if ((st = check_vec(in))) return st;
    if (!aligned16(out_mant) || (ld_out & 15)) return ICT_ERR_ALIGNMENT;
    if (ld_out < (transpose ? round_up(in->rows, 16) : in->cols)) return ICT_ERR_INVALID_ARG;
    return launch_align(AlignJob{in, axis, transpose != 0, out_mant, ld_out, e_star, nullptr},
                        (cudaStream_t)stream);
}

size_t ict_linear_workspace(int32_t op, const ict_tensor *a, const ict_tensor *b,
                            const ict_tensor *out) {
    LinearPlan lp;
    Ws w = make_ws(nullptr, 0, true);
    if (plan_linear(op, a, b, out, w, &lp) != ICT_OK) return 0;
    return w.used;
}

int32_t ict_linear_fwd(const ict_tensor *X, const ict_tensor *W, ict_tensor *Y, void *ws,
                       size_t ws_bytes, void *stream) {
    return linear_entry(ICT_OP_LINEAR_FWD, X, W, Y, ws, ws_bytes, stream);
}
int32_t ict_linear_fwd_noalloc(const ict_tensor *X, const ict_tensor *W, ict_tensor *Y, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    LinearPlan lp;
    Ws dry = make_ws(nullptr, 0, true);
    if ((st = plan_linear(ICT_OP_LINEAR_FWD, X, W, Y, dry, &lp))) return st;
    if (dry.used > ICT_NOALLOC_SCRATCH_BYTES) return ICT_ERR_WORKSPACE;
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch))) return st;
    return linear_entry(ICT_OP_LINEAR_FWD, X, W, Y, scratch, ICT_NOALLOC_SCRATCH_BYTES, stream);
}

int32_t ict_linear_bwd_data(const ict_tensor *dY, const ict_tensor *W, ict_tensor *dX, void *ws,
                            size_t ws_bytes, void *stream) {
    return linear_entry(ICT_OP_LINEAR_BWD_DATA, dY, W, dX, ws, ws_bytes, stream);
}
int32_t ict_linear_bwd_weight(const ict_tensor *dY, const ict_tensor *X, ict_tensor *dW, void *ws,
                              size_t ws_bytes, void *stream) {
    return linear_entry(ICT_OP_LINEAR_BWD_WEIGHT, dY, X, dW, ws, ws_bytes, stream);
}

size_t ict_linear_bwd_weight_partial_workspace(const ict_tensor *dY, const ict_tensor *X) {
    if (check_split_operands(dY, X) != ICT_OK) return 0;
    Ws wt = make_ws(nullptr, 0, true), wp = make_ws(nullptr, 0, true);
    TargetsPlan tp;
    PartialPlan pp;
    plan_targets(dY, X, nullptr, nullptr, wt, &tp);
    plan_partial(dY, X, nullptr, nullptr, wp, &pp);
    return std::max<size_t>(std::max(wt.used, wp.used), 256);
}
int32_t ict_linear_bwd_weight_targets(const ict_tensor *dY, const ict_tensor *X, int8_t *e_dy, int8_t *e_x,
                                      void *ws, size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_split_operands(dY, X))) return st;
    if ((dY->cols && !e_dy) || (X->cols && !e_x)) return ICT_ERR_INVALID_ARG;
    if (!ws || ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    Ws w = make_ws(ws, ws_bytes, false);
    TargetsPlan tp;
    plan_targets(dY, X, e_dy, e_x, w, &tp);
    if (w.used > ws_bytes) return ICT_ERR_WORKSPACE;
    return run_targets(tp, (cudaStream_t)stream);
}
int32_t ict_linear_bwd_weight_partial(const ict_tensor *dY, const ict_tensor *X, const int8_t *e_dy,
                                      const int8_t *e_x, void *acc, int32_t acc_bits, int64_t ld_acc,
                                      void *ws, size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_split_operands(dY, X))) return st;
    const int64_t M = dY->cols, N = X->cols, K = dY->rows;
    if (acc_bits != 32 && acc_bits != 64) return ICT_ERR_INVALID_ARG;
    if (ld_acc < N || (M && N && !acc) || (M && !e_dy) || (N && !e_x)) return ICT_ERR_INVALID_ARG;
    if (!aligned16(acc) || (ld_acc & 3)) return ICT_ERR_ALIGNMENT;
    if (acc_bits == 32 && K * 127 * 127 >= (int64_t(1) << 31)) return ICT_ERR_LAYOUT;
    if (ws && ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    if (M == 0 || N == 0) return ICT_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (K == 0) {  // empty shard: its sums are zero
        if (cudaMemsetAsync(acc, 0, (size_t)((M - 1) * ld_acc + N) * (acc_bits / 8), s) != cudaSuccess)
            return ICT_ERR_CUDA;
        return ICT_OK;
    }
    Ws w = make_ws(ws, ws_bytes, false);
    PartialPlan pp;
    plan_partial(dY, X, e_dy, e_x, w, &pp);
    if (w.used > ws_bytes || !ws) return ICT_ERR_WORKSPACE;
    if ((st = launch_aligns(pp.jobs, pp.njobs, s))) return st;
    return run_product(pp.A, pp.B, &pp.shape, pp.pp, s, acc, acc_bits, ld_acc);
}
size_t ict_conv_workspace(int32_t dir, const ict_conv_desc *d) {
    if (!d || d->n < 1 || d->h < 1 || d->w < 1 || d->c < 1 || d->k < 1 || d->r < 1 || d->s < 1)
        return 0;
    if (dir == ICT_CONV_BWD_WEIGHT) {
        // the plan's own sizes: int32 partial slices and the exponent tables
        ict_tensor dY{nullptr, nullptr, (int64_t)d->n * d->h * d->w, d->k, d->k, INT32_MAX, 32};
        ict_tensor X{nullptr, nullptr, (int64_t)d->n * d->h * d->w, d->c, d->c, INT32_MAX, 32};
        ict_tensor dW{nullptr, nullptr, d->k, (int64_t)d->r * d->s * d->c, (int64_t)d->r * d->s * d->c, 1,
                      d->r * d->s * d->c};
        static int8_t dummy[16] __attribute__((aligned(16)));
        dY.mant = X.mant = dW.mant = dummy;
        dY.exp = X.exp = dW.exp = dummy;
        WgradPlan wp;
        Ws w = make_ws(nullptr, 0, true);
        if (plan_wgrad(d, &dY, &X, &dW, planning_sms(), w, &wp) != ICT_OK) return 0;
        return w.used;
    }
    // worst case: activation aligned copy + its exponents, the prepared weight, gmax
    const int64_t npix = (int64_t)d->n * d->h * d->w;
    const int64_t act_c = dir == ICT_CONV_FWD ? d->c : d->k;
    const int64_t RS = (int64_t)d->r * d->s;
    Ws w = make_ws(nullptr, 0, true);
    w.take((size_t)npix * act_c);
    w.take((size_t)npix);
    w.take((size_t)std::max<int64_t>(d->k * RS * d->c, d->c * round_up(RS * d->k, 16)));
    w.take((size_t)std::max(d->k, d->c));
    w.take((size_t)std::max(d->k, d->c) * 4);
    // groups spanning all pixels: int16 sums and the per-tile needs
    const int64_t out_c = dir == ICT_CONV_FWD ? d->k : d->c;
    w.take((size_t)npix * round_up(out_c, 32) * 2);
    const int64_t rows_per_tile = std::max(1, std::min(128 / std::max(d->w, 1), d->h));
    w.take((size_t)d->n * cdiv64(d->h, rows_per_tile) * cdiv64(out_c, 16) * 4);
    return w.used;
}

int32_t ict_conv_implicit_gemm(int32_t dir, const ict_conv_desc *d, const ict_tensor *a,
                               const ict_tensor *b, ict_tensor *out, void *ws, size_t ws_bytes,
                               void *stream) {
    int st, sms = 0;
    if ((st = device_info(&sms))) return st;
    if ((st = int8_only())) return st;
    if (ws && ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    Ws w = make_ws(ws, ws_bytes, false);
    if (dir == ICT_CONV_BWD_WEIGHT) {
        if (!d) return ICT_ERR_INVALID_ARG;
        WgradPlan wp;
        if ((st = plan_wgrad(d, a, b, out, sms, w, &wp))) return st;
        if (w.used > ws_bytes || (w.used && !ws)) return ICT_ERR_WORKSPACE;
        return run_wgrad(d, a, b, out, wp, sms, (cudaStream_t)stream);
    }
    ConvPlan cp;
    if ((st = plan_conv(dir, d, a, b, out, w, &cp))) return st;
    if (w.used > ws_bytes || (w.used && !ws)) return ICT_ERR_WORKSPACE;
    return run_conv(dir, d, out, cp, sms, (cudaStream_t)stream);
}

int32_t ict_conv_fwd_act(const ict_conv_desc *d, const ict_tensor *X, const ict_tensor *W, ict_tensor *Y,
                         int32_t act, void *ws, size_t ws_bytes, void *stream) {
    int st, sms = 0;
    if ((st = device_info(&sms))) return st;
    if ((st = int8_only())) return st;
    if (act < ACT_NONE || act > ACT_RELU6) return ICT_ERR_INVALID_ARG;
    if (ws && ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    Ws w = make_ws(ws, ws_bytes, false);
    ConvPlan cp;
    if ((st = plan_conv(ICT_CONV_FWD, d, X, W, Y, w, &cp))) return st;
    if (w.used > ws_bytes || (w.used && !ws)) return ICT_ERR_WORKSPACE;
    return run_conv(ICT_CONV_FWD, d, Y, cp, sms, (cudaStream_t)stream, 3, act);
}
int32_t ict_conv_split_begin(int32_t dir, const ict_conv_desc *d, const ict_tensor *a, const ict_tensor *b,
                             ict_tensor *out, int32_t *need, void *ws, size_t ws_bytes, void *stream) {
    return conv_split(dir, d, a, b, out, need, ws, ws_bytes, stream, 1);
}
int32_t ict_conv_split_end(int32_t dir, const ict_conv_desc *d, const ict_tensor *a, const ict_tensor *b,
                           ict_tensor *out, const int32_t *need, void *ws, size_t ws_bytes, void *stream) {
    return conv_split(dir, d, a, b, out, const_cast<int32_t *>(need), ws, ws_bytes, stream, 2);
}
int32_t ict_conv_bwd_weight_partial(const ict_conv_desc *d, const ict_tensor *dY, const ict_tensor *X,
                                    int64_t *acc, int64_t ld_acc, int8_t *e_k, int8_t *e_rsc, void *ws,
                                    size_t ws_bytes, void *stream) {
    int st, sms = 0;
    if ((st = device_info(&sms))) return st;
    if ((st = int8_only())) return st;
    if (!d || !acc || !e_k || !e_rsc) return ICT_ERR_INVALID_ARG;
    if (ws && ((uintptr_t)ws & 255)) return ICT_ERR_WORKSPACE;
    const int64_t RSC = (int64_t)d->r * d->s * d->c;
    if (ld_acc < RSC || ((uintptr_t)acc & 7)) return ICT_ERR_INVALID_ARG;
    static int8_t shape_only[16] __attribute__((aligned(16)));  // dW's shape for the plan; never written
    ict_tensor dW{shape_only, shape_only, d->k, RSC, RSC, 1, (int32_t)RSC};
    Ws w = make_ws(ws, ws_bytes, false);
    WgradPlan wp;
    if ((st = plan_wgrad(d, dY, X, &dW, sms, w, &wp))) return st;
    if (w.used > ws_bytes || (w.used && !ws)) return ICT_ERR_WORKSPACE;
    wp.sums64 = acc;
    wp.sums_ld = ld_acc;
    wp.e_rows = e_rsc;
    wp.e_cols = e_k;
    return run_wgrad(d, dY, X, &dW, wp, sms, (cudaStream_t)stream, true);
}

int32_t ict_sgd_momentum_step(ict_tensor *W, ict_tensor *V, const ict_tensor *G,
                              const ict_sgd_params *p, void *stream) {
    ict_tensor *Ws_[1] = {W}, *Vs_[1] = {V};
    const ict_tensor *Gs_[1] = {G};
    return ict_sgd_momentum_step_multi(1, Ws_, Vs_, Gs_, p, stream);
}

int32_t ict_sgd_momentum_step_multi(int32_t n_tensors, ict_tensor *const *W, ict_tensor *const *V,
                                    const ict_tensor *const *G, const ict_sgd_params *p,
                                    void *stream) {
    int st, sms = 0;
    if ((st = device_info(&sms))) return st;
    if (n_tensors < 1 || n_tensors > kSgdMaxTensors || !W || !V || !G) return ICT_ERR_INVALID_ARG;
    if ((st = check_sgd_params(p))) return st;
    SgdArgs a;  // passed whole as the kernel's parameter block (about 12 KB)
    memset(&a, 0, sizeof(a));
    a.qb = g_mantissa_bits.load(std::memory_order_relaxed);
    a.n = n_tensors;
    a.mom_mul = p->mom_mul;
    a.mom_shift = p->mom_shift;
    a.lr_mul = p->lr_mul;
    a.lr_shift = p->lr_shift;
    a.cap_mom = 29 - bitlen_u64(127ull * (uint64_t)std::abs(p->mom_mul));
    a.cap_lr = 29 - bitlen_u64(127ull * (uint64_t)std::abs(p->lr_mul));
    int64_t total = 0;
    for (int i = 0; i < n_tensors; ++i) {
        if ((st = fill_sgd_tensor(W[i], V[i], G[i], &a.t[i]))) return st;
        a.t[i].first_group = total;
        total += a.t[i].rows * a.t[i].ngc;
    }
    a.total_groups = total;
    return run_sgd(a, sms, (cudaStream_t)stream);
}

int32_t ict_gelu_fwd(const ict_tensor *H, ict_tensor *out, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_tensor(H)) || (st = check_tensor(out))) return st;
    if (out->rows != H->rows || out->cols != H->cols || out->g_rows != H->g_rows ||
        out->g_cols != H->g_cols)
        return ICT_ERR_INVALID_ARG;
    if ((st = check_vec(H)) || (st = check_vec(out))) return st;
    if (H->rows == 0 || H->cols == 0) return ICT_OK;
    GeluArgs a;
    memset(&a, 0, sizeof(a));
    a.h = H->mant;
    a.h_exp = H->exp;
    a.out = out->mant;
    a.rows = H->rows;
    a.cols = H->cols;
    a.ld_h = H->ld;
    a.ld_out = out->ld;
    a.g_rows = clamp_div(H->g_rows, H->rows);
    a.g_cols = clamp_div(H->g_cols, H->cols);
    a.ngc = n_grp_cols(H);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t ne = (size_t)(n_grp_rows(H) * n_grp_cols(H));
    if (cudaMemcpyAsync(out->exp, H->exp, ne, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return ICT_ERR_CUDA;
    const int64_t vecs = H->rows * (H->cols / 16);
    KTimer kt(s, KC_GELU, 2.0 * (double)H->rows * (double)H->cols + 2.0 * (double)ne);
    const int G = (int)a.g_cols;
    if (a.g_rows == 1 && (G == 16 || G == 32 || G == 64)) {  // one thread per group
        int sms = 148;
        device_info(&sms);
        const unsigned blocks = (unsigned)std::min<int64_t>(cdiv64(H->rows * a.ngc, 256), (int64_t)sms * 4);
        if (G == 16) gelu_fwd_thread_kernel<1><<<blocks, 256, 0, s>>>(a);
        else if (G == 32) gelu_fwd_thread_kernel<2><<<blocks, 256, 0, s>>>(a);
        else gelu_fwd_thread_kernel<4><<<blocks, 256, 0, s>>>(a);
    } else {
        gelu_fwd_kernel<<<(unsigned)cdiv64(vecs, 256), 256, 0, s>>>(a);
    }
    counted(1);
    return launch_status();
}

int32_t ict_gelu_bwd(const ict_tensor *H, const ict_tensor *dG, ict_tensor *dH, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    if ((st = check_tensor(H)) || (st = check_tensor(dG)) || (st = check_tensor(dH))) return st;
    if (dG->rows != H->rows || dG->cols != H->cols || dH->rows != H->rows || dH->cols != H->cols)
        return ICT_ERR_INVALID_ARG;
    if ((H->g_rows != 1 || dG->g_rows != 1 || dH->g_rows != 1) && H->rows > 1) return ICT_ERR_LAYOUT;
    if (H->g_cols != dG->g_cols || H->g_cols != dH->g_cols) return ICT_ERR_LAYOUT;
    if (H->rows == 0 || H->cols == 0) return ICT_OK;
    GeluArgs a;
    memset(&a, 0, sizeof(a));
    a.h = H->mant;
    a.h_exp = H->exp;
    a.dg = dG->mant;
    a.dg_exp = dG->exp;
    a.out = dH->mant;
    a.out_exp = dH->exp;
    a.rows = H->rows;
    a.cols = H->cols;
    a.ld_h = H->ld;
    a.ld_dg = dG->ld;
    a.ld_out = dH->ld;
    a.g_rows = 1;
    a.g_cols = clamp_div(H->g_cols, H->cols);
    a.ngc = n_grp_cols(H);
    const int64_t groups = H->rows * a.ngc;
    cudaStream_t s = (cudaStream_t)stream;
    const int G = a.g_cols;
    KTimer kt(s, KC_GELU, 3.0 * (double)H->rows * (double)H->cols + 3.0 * (double)groups);
    const bool vec = check_vec(H) == ICT_OK && check_vec(dG) == ICT_OK && check_vec(dH) == ICT_OK &&
                     G % 16 == 0 && G <= 512 && ((G / 16) & (G / 16 - 1)) == 0;
    if (vec && (G == 16 || G == 32 || G == 64)) {  // one thread per group
        int sms = 148;
        device_info(&sms);
        const unsigned blocks = (unsigned)std::min<int64_t>(cdiv64(groups, 256), (int64_t)sms * 4);
        if (G == 16) gelu_bwd_thread_kernel<1><<<blocks, 256, 0, s>>>(a);
        else if (G == 32) gelu_bwd_thread_kernel<2><<<blocks, 256, 0, s>>>(a);
        else gelu_bwd_thread_kernel<4><<<blocks, 256, 0, s>>>(a);
    } else if (vec) {
        int sms = 148;
        device_info(&sms);
        const int L = G / 16, gpb = 8 * (32 / L);
        const unsigned blocks = (unsigned)std::min<int64_t>(cdiv64(groups, gpb), (int64_t)sms * 8);
        switch (L) {
            case 1: gelu_bwd_vec_kernel<1><<<blocks, 256, 0, s>>>(a); break;
            case 2: gelu_bwd_vec_kernel<2><<<blocks, 256, 0, s>>>(a); break;
            case 4: gelu_bwd_vec_kernel<4><<<blocks, 256, 0, s>>>(a); break;
            case 8: gelu_bwd_vec_kernel<8><<<blocks, 256, 0, s>>>(a); break;
            case 16: gelu_bwd_vec_kernel<16><<<blocks, 256, 0, s>>>(a); break;
            default: gelu_bwd_vec_kernel<32><<<blocks, 256, 0, s>>>(a); break;
        }
    } else {
        gelu_bwd_kernel<<<(unsigned)cdiv64(groups, 8), 256, 0, s>>>(a);
    }
    counted(1);
    return launch_status();
}

// ---- nonlinear functions through lookup tables (Tables 7 and 8)

int32_t ict_lut_tables(uint8_t *lut_exp, uint8_t *lut_log, int8_t *gelu_fwd, int8_t *gelu_bwd) {
    const LutTables &t = lut_tables();
    if (lut_exp) memcpy(lut_exp, t.exp, sizeof(t.exp));
    if (lut_log) memcpy(lut_log, t.log, sizeof(t.log));
    if (gelu_fwd) memcpy(gelu_fwd, t.gelu_fwd, sizeof(t.gelu_fwd));
    if (gelu_bwd) memcpy(gelu_bwd, t.gelu_bwd, sizeof(t.gelu_bwd));
    return ICT_OK;
}

int32_t ict_gelu_lut_fwd(const ict_tensor *H, ict_tensor *out, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_tensor(H)) || (st = check_tensor(out))) return st;
    if (out->rows != H->rows || out->cols != H->cols || out->g_rows != H->g_rows || out->g_cols != H->g_cols)
        return ICT_ERR_INVALID_ARG;
    if ((st = check_pointwise(H)) || (st = check_pointwise(out))) return st;
    if (H->rows == 0 || H->cols == 0) return ICT_OK;
    GeluLutArgs a;
    memset(&a, 0, offsetof(GeluLutArgs, lut));
    a.h = H->mant;
    a.h_exp = H->exp;
    a.out = out->mant;
    a.rows = H->rows;
    a.cols = H->cols;
    a.ld_h = H->ld;
    a.ld_out = out->ld;
    a.g_rows = clamp_div(H->g_rows, H->rows);
    a.g_cols = clamp_div(H->g_cols, H->cols);
    a.ngc = n_grp_cols(H);
    memcpy(a.lut, lut_tables().gelu_fwd, sizeof(a.lut));
    cudaStream_t s = (cudaStream_t)stream;
    const size_t ne = (size_t)(n_grp_rows(H) * n_grp_cols(H));
    if (cudaMemcpyAsync(out->exp, H->exp, ne, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return ICT_ERR_CUDA;
    KTimer kt(s, KC_GELU, 2.0 * (double)H->rows * (double)H->cols + 2.0 * (double)ne);
    gelu_lut_fwd_kernel<<<(unsigned)cdiv64(H->rows * (H->cols / 16), 256), 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

int32_t ict_gelu_lut_bwd(const ict_tensor *H, const ict_tensor *dY, ict_tensor *dH, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    if ((st = check_tensor(H)) || (st = check_tensor(dY)) || (st = check_tensor(dH))) return st;
    if (dY->rows != H->rows || dY->cols != H->cols || dH->rows != H->rows || dH->cols != H->cols)
        return ICT_ERR_INVALID_ARG;
    if ((H->g_rows != 1 || dY->g_rows != 1 || dH->g_rows != 1) && H->rows > 1) return ICT_ERR_LAYOUT;
    if (H->g_cols != dY->g_cols || H->g_cols != dH->g_cols) return ICT_ERR_LAYOUT;
    if ((st = check_pointwise(H)) || (st = check_pointwise(dY)) || (st = check_pointwise(dH))) return st;
    if (H->rows == 0 || H->cols == 0) return ICT_OK;
    GeluLutArgs a;
    memset(&a, 0, offsetof(GeluLutArgs, lut));
    a.h = H->mant;
    a.h_exp = H->exp;
    a.dy = dY->mant;
    a.dy_exp = dY->exp;
    a.out = dH->mant;
    a.out_exp = dH->exp;
    a.rows = H->rows;
    a.cols = H->cols;
    a.ld_h = H->ld;
    a.ld_dy = dY->ld;
    a.ld_out = dH->ld;
    a.g_rows = 1;
    a.g_cols = clamp_div(H->g_cols, H->cols);
    a.ngc = n_grp_cols(H);
    memcpy(a.lut, lut_tables().gelu_bwd, sizeof(a.lut));
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t groups = H->rows * a.ngc;
    KTimer kt(s, KC_GELU, 3.0 * (double)H->rows * (double)H->cols + 3.0 * (double)groups);
    gelu_lut_bwd_kernel<<<(unsigned)cdiv64(groups, 8), 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

int32_t ict_softmax_ce(const ict_tensor *Z, const int32_t *target, int32_t *loss, ict_tensor *dZ, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    if ((st = check_tensor(Z)) || (st = check_tensor(dZ))) return st;
    if (!target || !loss || dZ->rows != Z->rows || dZ->cols != Z->cols) return ICT_ERR_INVALID_ARG;
    if (dZ->g_rows != 1 && dZ->rows > 1) return ICT_ERR_LAYOUT;
    if (Z->rows == 0 || Z->cols == 0) return ICT_OK;
    HeadArgs a;
    memset(&a, 0, offsetof(HeadArgs, lut_exp));
    a.z = Z->mant;
    a.z_exp = Z->exp;
    a.rows = Z->rows;
    a.cols = Z->cols;
    a.ld_z = Z->ld;
    a.g_rows = clamp_div(Z->g_rows, Z->rows);
    a.g_cols = clamp_div(Z->g_cols, Z->cols);
    a.ngc = n_grp_cols(Z);
    a.target = target;
    a.loss = loss;
    a.dz = dZ->mant;
    a.dz_exp = dZ->exp;
    a.ld_dz = dZ->ld;
    a.gd = clamp_div(dZ->g_cols, dZ->cols);
    a.ngd = n_grp_cols(dZ);
    memcpy(a.lut_exp, lut_tables().exp, sizeof(a.lut_exp));
    memcpy(a.lut_log, lut_tables().log, sizeof(a.lut_log));
    cudaStream_t s = (cudaStream_t)stream;
    KTimer kt(s, KC_OTHER, 2.0 * (double)Z->rows * (double)Z->cols + 8.0 * (double)Z->rows);
    softmax_ce_kernel<<<(unsigned)cdiv64(Z->rows, 8), 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

int32_t ict_relu_fwd(const ict_tensor *X, int32_t six, ict_tensor *Z, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_pointwise(X)) || (st = check_pointwise(Z))) return st;
    if (six != 0 && six != 1) return ICT_ERR_INVALID_ARG;
    if (six && (st = int8_only())) return st;  // ReLU6's bound min(6 >> e, q_max) is written for INT8
    if (Z->rows != X->rows || Z->cols != X->cols) return ICT_ERR_INVALID_ARG;
    if (!same_groups(X, Z)) return ICT_ERR_LAYOUT;
    return launch_clip(X, nullptr, six, Z, (cudaStream_t)stream);
}
int32_t ict_relu_bwd(const ict_tensor *X, const ict_tensor *dY, int32_t six, ict_tensor *dX, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if (six && (st = int8_only())) return st;
    if ((st = check_pointwise(X)) || (st = check_pointwise(dY)) || (st = check_pointwise(dX))) return st;
    if (six != 0 && six != 1) return ICT_ERR_INVALID_ARG;
    if (dY->rows != X->rows || dY->cols != X->cols || dX->rows != X->rows || dX->cols != X->cols)
        return ICT_ERR_INVALID_ARG;
    if (!same_groups(dY, dX)) return ICT_ERR_LAYOUT;
    return launch_clip(X, dY, six, dX, (cudaStream_t)stream);
}
size_t ict_sum_workspace(const ict_tensor *X, const ict_tensor *Y, const ict_tensor *Z) {
    bool global = false;
    if (check_sum(X, Y, Z, &global) != ICT_OK) return 0;
    return global ? (size_t)round_up(n_grp_cols(X) * 4, 256) : 0;
}
int32_t ict_sum(const ict_tensor *X, const ict_tensor *Y, ict_tensor *Z, void *ws, size_t ws_bytes, void *stream) {
    return sum_entry(X, 1, 0, Y, 1, 0, Z, ACT_NONE, ws, ws_bytes, stream);
}
int32_t ict_sum_act(const ict_tensor *X, const ict_tensor *Y, ict_tensor *Z, int32_t act, void *ws,
                    size_t ws_bytes, void *stream) {
    if (act < ACT_NONE || act > ACT_RELU6) return ICT_ERR_INVALID_ARG;
    return sum_entry(X, 1, 0, Y, 1, 0, Z, act, ws, ws_bytes, stream);
}
int32_t ict_sum_scaled(const ict_tensor *X, int32_t x_mul, int32_t x_shift, const ict_tensor *Y, int32_t y_mul,
                       int32_t y_shift, ict_tensor *Z, void *ws, size_t ws_bytes, void *stream) {
    return sum_entry(X, x_mul, x_shift, Y, y_mul, y_shift, Z, ACT_NONE, ws, ws_bytes, stream);
}
int32_t ict_patchify(const ict_tensor *X, int32_t n, int32_t h, int32_t w, int32_t P, ict_tensor *out,
                     void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = check_tensor(X)) || (st = check_tensor(out))) return st;
    if (n < 1 || h < 1 || w < 1 || P < 1 || h % P || w % P) return ICT_ERR_INVALID_ARG;
    const int64_t c = X->cols, rows = (int64_t)n * (h / P) * (w / P), K = (int64_t)P * P * c;
    if (X->rows != (int64_t)n * h * w || out->rows != rows || out->cols != K) return ICT_ERR_INVALID_ARG;
    if (X->g_rows < X->rows) return ICT_ERR_LAYOUT;  // exponents uniform over pixels
    const int g_cols = clamp_div(X->g_cols, X->cols);
    // 16-byte vectors: each inside one channel group and one row segment
    if ((P * c) % 16 || !(g_cols >= c || (c % 16 == 0 && g_cols % 16 == 0))) return ICT_ERR_LAYOUT;
    if (out->g_rows < out->rows || out->g_cols < out->cols) return ICT_ERR_LAYOUT;  // one exponent
    if (c % 16 && X->ld != c) return ICT_ERR_LAYOUT;  // narrow channels: pixels must be packed
    if (!aligned16(X->mant) || (c % 16 == 0 && (X->ld & 15)) || !aligned16(out->mant) || (out->ld & 15))
        return ICT_ERR_ALIGNMENT;
    PatchArgs a;
    memset(&a, 0, sizeof(a));
    a.in = X->mant, a.in_exp = X->exp, a.ld_in = X->ld, a.g_cols = g_cols, a.ngc = n_grp_cols(X);
    a.out = out->mant, a.out_exp = out->exp, a.ld_out = out->ld, a.rows = rows;
    a.h = h, a.w = w, a.c = (int)c, a.P = P, a.Hp = h / P, a.Wp = w / P;
    const int64_t vecs = rows * (K / 16);
    if (vecs == 0) return ICT_OK;
    cudaStream_t s = (cudaStream_t)stream;
    KTimer kt(s, KC_ALIGN, 2.0 * (double)rows * (double)K);
    patchify_kernel<<<(unsigned)cdiv64(vecs, 256), 256, 0, s>>>(a);
    counted(1);
    return launch_status();
}

size_t ict_depthwise_workspace(int32_t dir, const ict_conv_desc *d, const ict_tensor *out) {
    if (!d || !out || dir == ICT_CONV_BWD_WEIGHT) return 256;
    return (size_t)round_up(std::max<int64_t>(n_grp_rows(out) * n_grp_cols(out) * 4, 1), 256);
}
int32_t ict_depthwise(int32_t dir, const ict_conv_desc *d, const ict_tensor *a, const ict_tensor *b,
                      ict_tensor *out, void *ws, size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    if (!d || (st = check_tensor(a)) || (st = check_tensor(b)) || (st = check_tensor(out)))
        return d ? st : ICT_ERR_INVALID_ARG;
    if (d->n < 1 || d->h < 1 || d->w < 1 || d->c < 1 || d->k != d->c || d->r < 1 || d->s < 1 || d->stride < 1 ||
        d->pad < 0 || d->r * d->s > kDwMaxTaps)
        return ICT_ERR_INVALID_ARG;
    const int64_t P = (d->h + 2 * d->pad - d->r) / d->stride + 1, Q = (d->w + 2 * d->pad - d->s) / d->stride + 1;
    if (P < 1 || Q < 1) return ICT_ERR_INVALID_ARG;
    const int64_t C = d->c, RS = (int64_t)d->r * d->s;
    const int64_t npix_in = (int64_t)d->n * d->h * d->w, npix_out = (int64_t)d->n * P * Q;
    cudaStream_t s = (cudaStream_t)stream;
    if (dir == ICT_CONV_BWD_WEIGHT) {  // a = dY, b = X, out = dW [C][R*S]
        if (a->rows != npix_out || a->cols != C || b->rows != npix_in || b->cols != C) return ICT_ERR_INVALID_ARG;
        if (out->rows != C || out->cols != RS) return ICT_ERR_INVALID_ARG;
        if (a->g_rows < a->rows || b->g_rows < b->rows) return ICT_ERR_LAYOUT;  // pixel-uniform exponents
        if ((out->g_rows != 1 && C > 1) || out->g_cols < RS) return ICT_ERR_LAYOUT;  // one group per row
        DwWgradArgs w;
        memset(&w, 0, sizeof(w));
        w.dy = a->mant, w.dy_exp = a->exp, w.ldy = a->ld, w.dy_gcols = clamp_div(a->g_cols, a->cols);
        w.x = b->mant, w.x_exp = b->exp, w.ldx = b->ld, w.x_gcols = clamp_div(b->g_cols, b->cols);
        w.out = out->mant, w.out_exp = out->exp, w.ldo = out->ld;
        w.n = d->n, w.h = d->h, w.w_ = d->w, w.C = (int)C, w.R = d->r, w.S = d->s, w.pad = d->pad;
        w.stride = d->stride, w.P = (int)P, w.Q = (int)Q;
        KTimer kt(s, KC_OTHER, (double)npix_out * C + (double)npix_in * C + (double)C * RS);
        dw_wgrad_kernel<<<(unsigned)C, 256, 0, s>>>(w);
        counted(1);
        return launch_status();
    }
    if (dir != ICT_CONV_FWD && dir != ICT_CONV_BWD_DATA) return ICT_ERR_INVALID_ARG;
    const bool bwd = dir == ICT_CONV_BWD_DATA;
    if (a->rows != (bwd ? npix_out : npix_in) || a->cols != C) return ICT_ERR_INVALID_ARG;
    if (b->rows != C || b->cols != RS) return ICT_ERR_INVALID_ARG;
    if (out->rows != (bwd ? npix_in : npix_out) || out->cols != C) return ICT_ERR_INVALID_ARG;
    if (a->g_rows < a->rows) return ICT_ERR_LAYOUT;                 // pixel-uniform exponents
    if ((b->g_rows != 1 && C > 1) || b->g_cols < RS) return ICT_ERR_LAYOUT;  // one exponent per filter
    DwArgs x;
    memset(&x, 0, sizeof(x));
    x.a = a->mant, x.a_exp = a->exp, x.lda = a->ld, x.a_gcols = clamp_div(a->g_cols, a->cols);
    x.w = b->mant, x.w_exp = b->exp, x.ldw = b->ld;
    x.out = out->mant, x.out_exp = out->exp, x.ldo = out->ld, x.out_rows = out->rows, x.out_ngc = n_grp_cols(out);
    x.out_g_rows = clamp_div(out->g_rows, out->rows), x.out_g_cols = clamp_div(out->g_cols, out->cols);
    x.h = d->h, x.w_ = d->w, x.C = (int)C, x.R = d->r, x.S = d->s, x.pad = d->pad, x.stride = d->stride;
    x.P = (int)P, x.Q = (int)Q, x.bwd = bwd;
    const int64_t groups = n_grp_rows(out) * n_grp_cols(out), n = out->rows * C;
    if (n == 0) return ICT_OK;
    if (!ws || ((uintptr_t)ws & 255) || ws_bytes < (size_t)groups * 4) return ICT_ERR_WORKSPACE;
    x.need = (int32_t *)ws;
    if (cudaMemsetAsync(x.need, 0x80, (size_t)groups * 4, s) != cudaSuccess) return ICT_ERR_CUDA;
    KTimer kt(s, KC_OTHER, (double)(bwd ? npix_out : npix_in) * C + (double)n + (double)C * RS);
    const unsigned grid = stream_grid(n, 1);
    dw_need_kernel<<<grid, 256, 0, s>>>(x);
    dw_round_kernel<<<grid, 256, 0, s>>>(x);
    counted(2);
    return launch_status();
}

}  // extern "C"

int sum_entry(const ict_tensor *X, int32_t x_mul, int32_t x_shift, const ict_tensor *Y, int32_t y_mul,
              int32_t y_shift, ict_tensor *Z, int act, void *ws, size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    if (x_mul < -512 || x_mul > 512 || y_mul < -512 || y_mul > 512 || x_shift < 0 || y_shift < 0 ||
        x_shift > 64 || y_shift > 64)
        return ICT_ERR_INVALID_ARG;
    bool global = false;
    if ((st = check_sum(X, Y, Z, &global))) return st;
    cudaStream_t s = (cudaStream_t)stream;
    SumArgs a;
    memset(&a, 0, sizeof(a));
    a.x = X->mant, a.x_exp = X->exp, a.ldx = X->ld;
    a.y = Y->mant, a.y_exp = Y->exp, a.ldy = Y->ld;
    a.z = Z->mant, a.z_exp = Z->exp, a.ldz = Z->ld;
    a.rows = X->rows, a.cols = X->cols;
    a.G = clamp_div(X->g_cols, X->cols);
    a.ngc = n_grp_cols(X);
    a.xm = x_mul, a.xs = x_shift, a.ym = y_mul, a.ys = y_shift;
    a.act = act;
    auto cap = [](int m) {
        const uint32_t v = 127u * (uint32_t)(m < 0 ? -m : m);
        int bits = 0;
        while ((v >> bits) != 0) ++bits;
        return 29 - bits;
    };
    a.cap_x = cap(x_mul), a.cap_y = cap(y_mul);
    const int64_t n = a.rows * a.cols;
    if (n == 0) return ICT_OK;
    if (global) {
        const size_t need = (size_t)a.ngc * 4;
        if (!ws || ((uintptr_t)ws & 255) || ws_bytes < need) return ICT_ERR_WORKSPACE;
        a.col_need = (int32_t *)ws;
        if (cudaMemsetAsync(a.col_need, 0x80, need, s) != cudaSuccess) return ICT_ERR_CUDA;
        KTimer kt(s, KC_POINTWISE, 5.0 * (double)n + 3.0 * (double)a.ngc);
        const unsigned grid = stream_grid(a.rows * (a.cols >> 4), 2);
        sum_global_need_kernel<<<grid, 256, (size_t)a.ngc * 4, s>>>(a);
        sum_global_round_kernel<<<grid, 256, 0, s>>>(a);
        counted(2);
        return launch_status();
    }
    KTimer kt(s, KC_POINTWISE, 3.0 * (double)n + 3.0 * (double)(a.rows * a.ngc));
    const int64_t nv = cdiv64(a.G, 16);  // vectors per group
    const int64_t groups = a.rows * a.ngc;
#define ICT_SUM_ROWS(L_, CPL_)                                                              \
    {                                                                                       \
        const int64_t blocks = cdiv64(groups, 8 * (32 / L_));                               \
        sum_rows_kernel<L_, CPL_><<<(unsigned)std::min<int64_t>(blocks, 148 * 16), 256, 0, s>>>(a); \
    }
    if (nv <= 1) ICT_SUM_ROWS(1, 1)
    else if (nv <= 2) ICT_SUM_ROWS(2, 1)
    else if (nv <= 4) ICT_SUM_ROWS(4, 1)
    else if (nv <= 8) ICT_SUM_ROWS(8, 1)
    else if (nv <= 16) ICT_SUM_ROWS(16, 1)
    else if (nv <= 32) ICT_SUM_ROWS(32, 1)
    else if (nv <= 64) ICT_SUM_ROWS(32, 2)
    else if (nv <= 128) ICT_SUM_ROWS(32, 4)
    else ICT_SUM_ROWS(32, 0)
#undef ICT_SUM_ROWS
    counted(1);
    return launch_status();
}

extern "C" {

size_t ict_avgpool_workspace(int32_t dir, const ict_tensor *in, int32_t n, int32_t h, int32_t w, int32_t K,
                             const ict_tensor *out) {
    PoolArgs a;
    if (plan_pool(dir == 1, in, n, h, w, K, out, &a) != ICT_OK) return 0;
    return (size_t)round_up(std::max<int64_t>(pool_groups(a) * 4, 1), 256);
}
int32_t ict_avgpool_fwd(const ict_tensor *X, int32_t n, int32_t h, int32_t w, int32_t K, ict_tensor *Y, void *ws,
                        size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    PoolArgs a;
    if ((st = plan_pool(false, X, n, h, w, K, Y, &a))) return st;
    return run_pool(a, ws, ws_bytes, (cudaStream_t)stream);
}
int32_t ict_avgpool_bwd(const ict_tensor *dY, int32_t n, int32_t h, int32_t w, int32_t K, ict_tensor *dX, void *ws,
                        size_t ws_bytes, void *stream) {
    int st;
    if ((st = device_info(nullptr))) return st;
    if ((st = int8_only())) return st;
    PoolArgs a;
    if ((st = plan_pool(true, dY, n, h, w, K, dX, &a))) return st;
    return run_pool(a, ws, ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
