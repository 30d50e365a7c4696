// C entry points of libtern: argument checks on the host, then dispatch to
// the kernels.  Nothing here allocates device memory.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "tern_internal.cuh"

namespace tern {

Options g_opt;

namespace {
thread_local char t_err[512] = "";
std::mutex g_dev_mu;
DeviceInfo g_dev_cache[64];
bool g_dev_valid[64];
}  // namespace

void clear_error() { t_err[0] = '\0'; }

tern_status fail(tern_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return st;
}

tern_status cuda_fail(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return TERN_OK;
    return fail(TERN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

tern_status current_device(DeviceInfo *out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(TERN_ERR_DEVICE, "device ordinal %d out of range", dev);
    // The tensor maps are encoded through the driver API, which needs a
    // context current in the calling thread; a host thread whose first CUDA
    // call is one of ours has none yet.  cudaFree(nullptr) binds the device's
    // primary context when no context is current (and leaves a current one
    // alone), once per thread and device.
    thread_local bool t_bound[64] = {};
    if (!t_bound[dev]) {
        e = cudaFree(nullptr);
        if (e != cudaSuccess) return cuda_fail(e, "binding the device context");
        t_bound[dev] = true;
    }
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!g_dev_valid[dev]) {
        DeviceInfo d;
        d.device = dev;
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
        int smem = 0;
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        d.max_smem_optin = static_cast<size_t>(smem);
        g_dev_cache[dev] = d;
        g_dev_valid[dev] = true;
    }
    *out = g_dev_cache[dev];
    if (out->major != 10 || out->minor != 0)
        return fail(TERN_ERR_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                    out->major, out->minor);
    return TERN_OK;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;
}  // namespace

// Resolves cuTensorMapEncodeTiled from the driver once per process.
static bool resolve_encode() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

tern_status encode_tiled_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                            uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                            CUtensorMapSwizzle swizzle) {
    if (!resolve_encode())
        return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(g_encode_err));
    std::memset(map, 0, sizeof(*map));
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return TERN_OK;
}

tern_status encode_tiled_3d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, const uint64_t dims[3],
                            const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle) {
    if (!resolve_encode())
        return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(g_encode_err));
    std::memset(map, 0, sizeof(*map));
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t str[2] = {strides[0], strides[1]};
    const cuuint32_t bx[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, dt, 3, const_cast<void *>(base), d, str, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", static_cast<int>(r));
    return TERN_OK;
}

}  // namespace tern

using namespace tern;

namespace {

// Smallest M sent to the tensor-core kernel by default; below it the
// bandwidth kernel runs in chunks of eight token rows.
constexpr int64_t kTensorCoreMinM = 32;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tern_status check_nk(int64_t N, int64_t K) {
    if (N < 1) return fail(TERN_ERR_SHAPE, "N must be >= 1 (got %lld)", static_cast<long long>(N));
    if (K < kGroup || K % kGroup != 0)
        return fail(TERN_ERR_SHAPE, "K must be a positive multiple of 128 (got %lld)",
                    static_cast<long long>(K));
    if (N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 30))
        return fail(TERN_ERR_SHAPE, "N or K too large (N=%lld, K=%lld)", static_cast<long long>(N),
                    static_cast<long long>(K));
    if (N * K > (int64_t(1) << 46))
        return fail(TERN_ERR_SHAPE, "N*K too large");
    return TERN_OK;
}

tern_status check_mat(const void *x, const void *slots, const void *scales, const void *y) {
    if (!x || !slots || !scales || !y) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(x)) return fail(TERN_ERR_ALIGN, "x is not 16-byte aligned");
    if (!aligned16(slots)) return fail(TERN_ERR_ALIGN, "slots is not 16-byte aligned");
    if (!aligned16(scales)) return fail(TERN_ERR_ALIGN, "scales is not 16-byte aligned");
    if (!aligned16(y)) return fail(TERN_ERR_ALIGN, "y is not 16-byte aligned");
    return TERN_OK;
}

// Streaming-multiprocessor count of the current device (148 on B200 when no
// device is visible, so that sizes can be planned on a machine without one).
int planning_sms() {
    DeviceInfo dev;
    if (current_device(&dev) == TERN_OK) return dev.sms;
    clear_error();
    return 148;
}

// Bandwidth kernels (M <= 8).  Default: the TMA-staged mma.sync kernel,
// the fastest measured so far; the knob selects the others for comparison.
// (Values 1 and 5 named two kernels that were measured, kept for comparison
// and then removed.)
enum { kVarDefault = 0, kVarTma = 2, kVarTc = 3, kVarPc = 4, kVarPcTok = 6 };

bool use_tc(int M) { return g_opt.gemv_variant == kVarTc && M <= 4; }

tern_status launch_bandwidth(const MatDesc *d, int count, int M, void *workspace, size_t ws_bytes,
                             cudaStream_t s) {
    // The persistent step kernel where its shape rules hold, as measured on
    // B200 against the per-matrix kernels: at one and two token rows (digit
    // form) for every decode shape alone and grouped (M = 1: head 5120 x
    // 151936 39 against 52 us; M = 2: gate 9.8 against 13.1 us, a decode
    // layer 22.9 against 28.1 us), and at five to eight rows for groups of
    // four products or more, which it reads once where the per-matrix kernel
    // takes two passes of four rows (a decode layer at M = 8: 56.7 against
    // 64.2 us; single products stay on the per-matrix kernels, 5-10 % faster).
    const bool step_m = M <= 2 || (M >= 5 && count >= 4);
    if (g_opt.gemv_variant == kVarDefault && step_m && gemv_step_supports(d, count, M, 0, gemv_step_digit_form(M, 0)))
        return launch_gemv_step(d, count, M, 0, gemv_step_digit_form(M, 0), s);
    if (use_tc(M)) return launch_gemv_tc(d, count, M, workspace, ws_bytes, s);
    // Default: the producer/consumer kernel where its shape rules hold (K a
    // multiple of 1024, x fits its shared memory), else the TMA-staged one.
    if ((g_opt.gemv_variant == kVarPc || g_opt.gemv_variant == kVarDefault || g_opt.gemv_variant == kVarPcTok) &&
        gemv_pc_supports(d, count, M, g_opt.gemv_variant == kVarPcTok))
        return launch_gemv_pc(d, count, M, g_opt.gemv_variant == kVarPcTok, s);
    // M = 5..8 whose x does not fit the token-per-column kernel: two launches
    // of the group-per-column kernel (4 + M - 4 token rows), each reading the
    // weights once.
    if (g_opt.gemv_variant == kVarDefault && M > 4 && gemv_pc_supports(d, count, 4, false) &&
        count <= TERN_MAX_GROUP) {
        MatDesc lo[TERN_MAX_GROUP], hi[TERN_MAX_GROUP];
        for (int i = 0; i < count; i++) {
            lo[i] = d[i];
            hi[i] = d[i];
            hi[i].x = d[i].x + static_cast<size_t>(4) * d[i].K;
            hi[i].y = d[i].y + static_cast<size_t>(4) * d[i].N;
        }
        tern_status st = launch_gemv_pc(lo, count, 4, false, s);
        if (st != TERN_OK) return st;
        return launch_gemv_pc(hi, count, M - 4, false, s);
    }
    return launch_gemv_tma(d, count, M, s);
}

size_t bandwidth_workspace(const MatDesc *d, int count, int M) {
    if (!use_tc(M)) return 0;
    return gemv_tc_workspace_bytes(d, count, M, planning_sms());
}

MatDesc mat(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y, int64_t N,
            int64_t K) {
    MatDesc d;
    d.x = reinterpret_cast<const __half *>(x);
    d.slots = slots;
    d.scales = reinterpret_cast<const __half *>(scales);
    d.y = reinterpret_cast<__half *>(y);
    d.N = static_cast<int>(N);
    d.K = static_cast<int>(K);
    return d;
}

}  // namespace

extern "C" {

int tern_version(void) { return 100; }

const char *tern_status_string(int status) {
    switch (status) {
        case TERN_OK: return "ok";
        case TERN_ERR_INVALID_ARG: return "invalid argument";
        case TERN_ERR_ALIGN: return "misaligned pointer";
        case TERN_ERR_SHAPE: return "unsupported shape";
        case TERN_ERR_WORKSPACE: return "workspace too small";
        case TERN_ERR_CUDA: return "CUDA error";
        case TERN_ERR_TIMEOUT: return "device wait timed out";
        case TERN_ERR_DEVICE: return "unsupported device";
        case TERN_ERR_GUARD: return "in-kernel index check failed";
        default: return "unknown status";
    }
}

const char *tern_last_error(void) { return t_err; }

size_t tern_slots_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < kGroup || K % kGroup != 0) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K / 4);
}

size_t tern_scales_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < kGroup || K % kGroup != 0) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K / kGroup) * 2;
}

size_t tern_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || check_nk(N, K) != TERN_OK) {
        clear_error();
        return 0;
    }
    MatDesc d = mat(nullptr, nullptr, nullptr, nullptr, N, K);
    size_t best = 0;
    for (int64_t m0 = 0; m0 < M && M <= 8; m0 += 8) {
        const int mc = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
        best = std::max(best, bandwidth_workspace(&d, 1, mc));
    }
    return best;
}

size_t tern_gemv_grouped_workspace_bytes(const tern_gemv_desc *descs, int32_t count, int64_t M) {
    if (!descs || count < 1 || count > TERN_MAX_GROUP || M < 1 || M > 8) return 0;
    MatDesc d[TERN_MAX_GROUP];
    for (int i = 0; i < count; i++) {
        if (check_nk(descs[i].N, descs[i].K) != TERN_OK) {
            clear_error();
            return 0;
        }
        d[i] = mat(nullptr, nullptr, nullptr, nullptr, descs[i].N, descs[i].K);
    }
    return bandwidth_workspace(d, count, static_cast<int>(M));
}

tern_status tern_pack_g128(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K,
                           uint8_t *slots_out, uint16_t *scales_out, int32_t *invalid_count,
                           void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    if (!codes || !scales_in || !slots_out || !scales_out)
        return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(codes)) return fail(TERN_ERR_ALIGN, "codes is not 16-byte aligned");
    if (!aligned16(slots_out)) return fail(TERN_ERR_ALIGN, "slots_out is not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(scales_in) | reinterpret_cast<uintptr_t>(scales_out)) & 1u)
        return fail(TERN_ERR_ALIGN, "scales are not 2-byte aligned");
    if ((reinterpret_cast<uintptr_t>(invalid_count) & 3u) != 0)
        return fail(TERN_ERR_ALIGN, "invalid_count is not 4-byte aligned");
    return launch_pack(codes, scales_in, N, K, slots_out, scales_out, invalid_count,
                       static_cast<cudaStream_t>(stream));
}

tern_status tern_unpack_g128(const uint8_t *slots, int64_t N, int64_t K, int8_t *codes_out,
                             void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    if (!slots || !codes_out) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(slots) || !aligned16(codes_out))
        return fail(TERN_ERR_ALIGN, "slots and codes_out must be 16-byte aligned");
    return launch_unpack(slots, N, K, codes_out, static_cast<cudaStream_t>(stream));
}

tern_status tern_gemm(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y,
                      int64_t M, int64_t N, int64_t K, void *workspace, size_t ws_bytes,
                      void *stream) {
    clear_error();
    if (M < 1) return fail(TERN_ERR_SHAPE, "M must be >= 1 (got %lld)", static_cast<long long>(M));
    if (M > (int64_t(1) << 24)) return fail(TERN_ERR_SHAPE, "M too large");
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    st = check_mat(x, slots, scales, y);
    if (st != TERN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t min_m = g_opt.gemm_min_m > 0 ? g_opt.gemm_min_m : kTensorCoreMinM;
    const bool tensor = (g_opt.gemm_path == 2) || (g_opt.gemm_path != 1 && M > 8 && M >= min_m);
    if (tensor) return launch_gemm_tc(mat(x, slots, scales, y, N, K), static_cast<int>(M), s);
    // Bandwidth kernel, eight token rows per launch (weights re-read per chunk).
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mc = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
        MatDesc d = mat(x + m0 * K, slots, scales, y + m0 * N, N, K);
        st = launch_bandwidth(&d, 1, mc, workspace, ws_bytes, s);
        if (st != TERN_OK) return st;
    }
    return TERN_OK;
}

tern_status tern_gemv(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y,
                      int64_t N, int64_t K, void *workspace, size_t ws_bytes, void *stream) {
    return tern_gemm(x, slots, scales, y, 1, N, K, workspace, ws_bytes, stream);
}

tern_status tern_gemv_noalloc(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y,
                              int64_t N, int64_t K, void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    st = check_mat(x, slots, scales, y);
    if (st != TERN_OK) return st;
    return gemv_noalloc(mat(x, slots, scales, y, N, K), static_cast<cudaStream_t>(stream));
}

tern_status tern_embed_gather(const int32_t *ids, int64_t M, const uint8_t *slots, const uint16_t *scales,
                              int64_t V, int64_t K, uint16_t *out, int32_t *bad_count, void *stream) {
    clear_error();
    if (M < 0) return fail(TERN_ERR_SHAPE, "M must be >= 0 (got %lld)", static_cast<long long>(M));
    tern_status st = check_nk(V, K);
    if (st != TERN_OK) return st;
    if (V > 0x7FFFFFFFll || M > 0x7FFFFFFFll) return fail(TERN_ERR_SHAPE, "V and M must fit in int32");
    if (!ids || !slots || !scales || !out) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if ((reinterpret_cast<uintptr_t>(ids) & 3u) || (reinterpret_cast<uintptr_t>(bad_count) & 3u))
        return fail(TERN_ERR_ALIGN, "ids and bad_count must be 4-byte aligned");
    if (!aligned16(slots) || !aligned16(out)) return fail(TERN_ERR_ALIGN, "slots and out must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(scales) & 1u) return fail(TERN_ERR_ALIGN, "scales are not 2-byte aligned");
    if (M == 0) return TERN_OK;
    return launch_embed(ids, M, slots, scales, V, K, out, bad_count, static_cast<cudaStream_t>(stream));
}

namespace {
// Products whose M rows of x do not fit in shared memory beside the rings run
// as K segments of whole 1024-k units that do, in calls of their own: segment
// 0 (with every product that fits) writes y, each later segment adds its sum
// to y.  Each weight is still read once.  At most kMaxSeg segments: each one
// rounds the running sum to fp16 once more (at most 2^-11 of sum |x w| each),
// and four roundings, 1.95e-3 of sum |x w|, stay within the 2e-3 tolerance.
// Fills seg[s][0..n[s]) for segments s < nseg_max (everything in segment 0
// when every product fits).
constexpr int kMaxSeg = 4;
tern_status plan_step_segments(const MatDesc *d, int count, int m, int fmt, bool x8, const char *name,
                               MatDesc (&seg)[8][TERN_MAX_STEP], int (&n)[8], int &nseg_max) {
    nseg_max = 1;
    for (int s = 0; s < 8; s++) n[s] = 0;
    const int unit_bytes = fmt == 0 ? 256 : (fmt == 1 ? 128 : 208);  // weight bytes of one 1024-k row unit
    for (int i = 0; i < count; i++) {
        if (gemv_step_fits(d[i].K, m, fmt, x8)) {
            seg[0][n[0]++] = d[i];
            continue;
        }
        const int B = d[i].K / 1024;
        int bfit = B - 1;
        while (bfit > 0 && !gemv_step_fits(bfit * 1024, m, fmt, x8)) bfit--;
        if (bfit == 0) return fail(TERN_ERR_SHAPE, "%s: M x 1024 too large for shared memory", name);
        const int nseg = (B + bfit - 1) / bfit;
        if (nseg > kMaxSeg)
            return fail(TERN_ERR_SHAPE, "%s: K=%d needs more than %d segments at M=%d", name, d[i].K, kMaxSeg, m);
        nseg_max = std::max(nseg_max, nseg);
        for (int sgi = 0; sgi < nseg; sgi++) {
            const int u0 = sgi * B / nseg, u1 = (sgi + 1) * B / nseg;
            MatDesc e = d[i];
            e.x = d[i].x + static_cast<size_t>(u0) * 1024;
            e.slots = d[i].slots + static_cast<size_t>(u0) * unit_bytes;
            e.scales = d[i].scales + static_cast<size_t>(u0) * (1024 / kGroup);
            e.K = (u1 - u0) * 1024;
            e.kfull = d[i].K;
            e.accum = sgi > 0;
            seg[sgi][n[sgi]++] = e;
        }
    }
    for (int sgi = 0; sgi < nseg_max; sgi++) {
        if (n[sgi] == 0) continue;
        if (!gemv_step_supports(seg[sgi], n[sgi], m, fmt, x8))
            return fail(TERN_ERR_SHAPE, "%s: M x K too large for shared memory", name);
    }
    return TERN_OK;
}

tern_status gemv_step_api(const tern_gemv_desc *descs, int32_t count, int64_t M, int fmt, const char *name,
                          void *stream) {
    clear_error();
    if (!descs) return fail(TERN_ERR_INVALID_ARG, "descs is NULL");
    if (count < 1 || count > TERN_MAX_STEP)
        return fail(TERN_ERR_INVALID_ARG, "count must be 1..%d (got %d)", TERN_MAX_STEP, count);
    const int mmax = fmt == 1 ? 4 : 8;
    if (M < 1 || M > mmax)
        return fail(TERN_ERR_SHAPE, "%s takes M in 1..%d (got %lld)", name, mmax, static_cast<long long>(M));
    thread_local MatDesc d[TERN_MAX_STEP];  // per host thread: calls may run concurrently
    for (int i = 0; i < count; i++) {
        tern_status st = check_nk(descs[i].N, descs[i].K);
        if (st != TERN_OK) return st;
        if (descs[i].K % 1024 != 0)
            return fail(TERN_ERR_SHAPE, "%s needs K a multiple of 1024 (descriptor %d has K=%lld)", name, i,
                        static_cast<long long>(descs[i].K));
        st = check_mat(descs[i].x, descs[i].slots, descs[i].scales, descs[i].y);
        if (st != TERN_OK) return st;
        d[i] = mat(descs[i].x, descs[i].slots, descs[i].scales, descs[i].y, descs[i].N, descs[i].K);
    }
    const int m = static_cast<int>(M);
    cudaStream_t st_ = static_cast<cudaStream_t>(stream);
    // The digit form by default (M <= 4); a call whose products the digit
    // form cannot cut into at most kMaxSeg K segments (its staged x takes
    // twice the room) runs in the fp16 form instead.
    bool x8 = gemv_step_digit_form(m, fmt);
    thread_local MatDesc seg[8][TERN_MAX_STEP];
    int nseg_max = 1, n[8] = {0};
    tern_status st = plan_step_segments(d, count, m, fmt, x8, name, seg, n, nseg_max);
    if (st == TERN_ERR_SHAPE && x8) {
        x8 = false;
        st = plan_step_segments(d, count, m, fmt, x8, name, seg, n, nseg_max);
    }
    if (st != TERN_OK) return st;
    for (int sgi = 0; sgi < nseg_max; sgi++) {
        if (n[sgi] == 0) continue;
        st = launch_gemv_step(seg[sgi], n[sgi], m, fmt, x8, st_);
        if (st != TERN_OK) return st;
    }
    return TERN_OK;
}
}  // namespace

tern_status tern_gemv_step(const tern_gemv_desc *descs, int32_t count, int64_t M, void *stream) {
    return gemv_step_api(descs, count, M, 0, "tern_gemv_step", stream);
}

tern_status tern_step_plan(const int64_t *N, const int64_t *K, int32_t count, int64_t M, int32_t grid,
                           int32_t *first_tile) {
    clear_error();
    if (M < 1 || M > 8) return fail(TERN_ERR_SHAPE, "M must be in [1, 8] (got %lld)", static_cast<long long>(M));
    return gemv_step_plan(N, K, count, static_cast<int>(M), grid, first_tile);
}

tern_status tern_b1_gemv_step(const tern_gemv_desc *descs, int32_t count, int64_t M, void *stream) {
    return gemv_step_api(descs, count, M, 1, "tern_b1_gemv_step", stream);
}

tern_status tern_t5_gemv_step(const tern_gemv_desc *descs, int32_t count, int64_t M, void *stream) {
    return gemv_step_api(descs, count, M, 2, "tern_t5_gemv_step", stream);
}

size_t tern_t5_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < kGroup || K % kGroup != 0) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(t5_row_bytes(K));
}

tern_status tern_t5_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bytes_out,
                         uint16_t *scales_out, int32_t *invalid_count, void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    if (!codes || !scales_in || !bytes_out || !scales_out) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(codes)) return fail(TERN_ERR_ALIGN, "codes is not 16-byte aligned");
    if (!aligned16(bytes_out)) return fail(TERN_ERR_ALIGN, "bytes_out is not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(scales_in) | reinterpret_cast<uintptr_t>(scales_out)) & 1u)
        return fail(TERN_ERR_ALIGN, "scales are not 2-byte aligned");
    if ((reinterpret_cast<uintptr_t>(invalid_count) & 3u) != 0)
        return fail(TERN_ERR_ALIGN, "invalid_count is not 4-byte aligned");
    return launch_pack_t5(codes, scales_in, N, K, bytes_out, scales_out, invalid_count,
                          static_cast<cudaStream_t>(stream));
}

tern_status tern_t5_unpack(const uint8_t *bytes, int64_t N, int64_t K, int8_t *codes_out, void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    if (!bytes || !codes_out) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(bytes) || !aligned16(codes_out)) return fail(TERN_ERR_ALIGN, "bytes and codes_out must be 16-byte aligned");
    return launch_unpack_t5(bytes, N, K, codes_out, static_cast<cudaStream_t>(stream));
}

tern_status tern_b1_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bits_out,
                         uint16_t *scales_out, int32_t *invalid_count, void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    if (!codes || !scales_in || !bits_out || !scales_out) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(codes)) return fail(TERN_ERR_ALIGN, "codes is not 16-byte aligned");
    if (!aligned16(bits_out)) return fail(TERN_ERR_ALIGN, "bits_out is not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(scales_in) | reinterpret_cast<uintptr_t>(scales_out)) & 1u)
        return fail(TERN_ERR_ALIGN, "scales are not 2-byte aligned");
    if ((reinterpret_cast<uintptr_t>(invalid_count) & 3u) != 0)
        return fail(TERN_ERR_ALIGN, "invalid_count is not 4-byte aligned");
    return launch_pack_b1(codes, scales_in, N, K, bits_out, scales_out, invalid_count,
                          static_cast<cudaStream_t>(stream));
}

tern_status tern_b1_unpack(const uint8_t *bits, int64_t N, int64_t K, int8_t *codes_out, void *stream) {
    clear_error();
    tern_status st = check_nk(N, K);
    if (st != TERN_OK) return st;
    if (!bits || !codes_out) return fail(TERN_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(bits) || !aligned16(codes_out)) return fail(TERN_ERR_ALIGN, "bits and codes_out must be 16-byte aligned");
    return launch_unpack_b1(bits, N, K, codes_out, static_cast<cudaStream_t>(stream));
}

tern_status tern_gemv_grouped(const tern_gemv_desc *descs, int32_t count, int64_t M,
                              void *workspace, size_t ws_bytes, void *stream) {
    clear_error();
    if (!descs) return fail(TERN_ERR_INVALID_ARG, "descs is NULL");
    if (count < 1 || count > TERN_MAX_GROUP)
        return fail(TERN_ERR_INVALID_ARG, "count must be 1..%d (got %d)", TERN_MAX_GROUP, count);
    if (M < 1 || M > 8) return fail(TERN_ERR_SHAPE, "grouped product takes M in 1..8 (got %lld)",
                                    static_cast<long long>(M));
    MatDesc d[TERN_MAX_GROUP];
    for (int i = 0; i < count; i++) {
        tern_status st = check_nk(descs[i].N, descs[i].K);
        if (st != TERN_OK) return st;
        st = check_mat(descs[i].x, descs[i].slots, descs[i].scales, descs[i].y);
        if (st != TERN_OK) return st;
        d[i] = mat(descs[i].x, descs[i].slots, descs[i].scales, descs[i].y, descs[i].N, descs[i].K);
    }
    return launch_bandwidth(d, count, static_cast<int>(M), workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

tern_status tern_sync_status(void *stream) {
    clear_error();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int v = 0, w = 0, u = 0;
    tern_status st = read_gemm_status(true, &v);
    if (st != TERN_OK) return st;
    st = read_gemv_status(true, &w);
    if (st != TERN_OK) return st;
    st = read_gemvtc_status(true, &u);
    if (st != TERN_OK) return st;
    unsigned int z = 0;
    st = read_gemvpc_status(true, &z);
    if (st != TERN_OK) return st;
    unsigned int t6 = 0;
    st = read_gemvstep_status(true, &t6);
    if (st != TERN_OK) return st;
    if (v == 0) v = w;
    if (v == 0) v = u;
    if (v == 0) v = z;
    if (v == 0) v = t6;
    if (v != 0) return fail(static_cast<tern_status>(v), "a kernel gave up a bounded wait on the device");
    unsigned int guard = 0;
    st = read_gemvstep_guard(true, &guard);
    if (st != TERN_OK) return st;
    if (guard != 0) return fail(TERN_ERR_GUARD, "%u in-kernel index checks failed (debug build)", guard);
    return TERN_OK;
}

tern_status tern_set_option(int option, int64_t value) {
    clear_error();
    if (value < 0 || value > 100000000) return fail(TERN_ERR_INVALID_ARG, "option value %lld", static_cast<long long>(value));
    switch (option) {
        case TERN_OPT_GEMV_KSPLIT: g_opt.gemv_ksplit = static_cast<int>(value); return TERN_OK;
        case TERN_OPT_GEMV_CLUSTER: g_opt.gemv_cluster = static_cast<int>(value); return TERN_OK;
        case TERN_OPT_GEMV_CTAS: g_opt.gemv_ctas = static_cast<int>(value); return TERN_OK;
        case TERN_OPT_GEMM_PATH:
            if (value > 2) return fail(TERN_ERR_INVALID_ARG, "gemm path %lld", static_cast<long long>(value));
            g_opt.gemm_path = static_cast<int>(value);
            return TERN_OK;
        case TERN_OPT_GEMM_MIN_M: g_opt.gemm_min_m = static_cast<int>(value); return TERN_OK;
        case TERN_OPT_GEMV_VARIANT:
            if (value > 6 || value == 1 || value == 5)
                return fail(TERN_ERR_INVALID_ARG, "gemv variant %lld", static_cast<long long>(value));
            g_opt.gemv_variant = static_cast<int>(value);
            return TERN_OK;
        case TERN_OPT_GEMV_GRID: g_opt.gemv_grid = static_cast<int>(value); return TERN_OK;
        case TERN_OPT_GEMV_PREFETCH: g_opt.gemv_prefetch = static_cast<int>(value); return TERN_OK;
        case TERN_OPT_STEP_FORM:
            if (value > 2) return fail(TERN_ERR_INVALID_ARG, "step form %lld", static_cast<long long>(value));
            g_opt.step_form = static_cast<int>(value);
            return TERN_OK;
        case TERN_OPT_TEST_STALL_US:
            g_gemm_skip_loads = value > 0 ? 1 : 0;
            g_gemm_timeout_ns = value > 0 ? static_cast<unsigned long long>(value) * 1000ull : 1000000000ull;
            return TERN_OK;
        default: return fail(TERN_ERR_INVALID_ARG, "unknown option %d", option);
    }
}

}  // extern "C"
