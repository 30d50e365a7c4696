// Compute-bound ternary-g128 prefill product on the 5th-generation tensor
// cores (tcgen05, sm_100a).
//
// What it computes: y[m][n] = sum_k x[m][k] * s[n][k/128] * t[n][k] for large
// M (prompt processing is compute-bound: "Bonsai 27B ternary / 1-bit
// quantization", ThakiCloud blog, section "Throughput and speculative
// decoding"), with the weights read from the 2-bit slots and the group scale
// applied inside the product ("Ternary-Bonsai-27B" model summary, aitrends.kr,
// section "Technical features").
//
// Design.  The MMA computes the transposed tile D[n][m] = sum_k W[n][k] x[m][k]:
//  * A operand = 128 weight rows x 64 k per step, held in TENSOR MEMORY.  Two
//    of the 256 unpack threads share a weight row, one half of the step each:
//    one 8-byte load brings 32 codes, two instructions per pair turn them
//    into exact fp16 t (the LOP3/HFMA2 construction of the bandwidth kernel),
//    a byte permute puts them in k order, one HMUL2 applies the row's fp16
//    group scale (s*t is exact: t is -1, 0 or +1), and one tcgen05.st writes
//    16 columns.  Two unpack warps per tensor-memory lane quarter (one per
//    half) let one hide the other's latencies, and a warp announces a stage
//    one k step late, so that its store completes while it unpacks the next.  The unpacked weights never
//    touch shared memory or HBM.
//  * B operand = 256 token rows x 64 k of x, brought by TMA into shared memory
//    in the 128-byte-swizzled K-major layout the MMA reads directly.
//  * D = 128 x 256 fp32 accumulator in tensor memory; one thread issues
//    tcgen05.mma (M=128, N=256, K=16) four times per k step.
//  * Producer (TMA), MMA issuer and unpack warps run a 4-stage mbarrier
//    pipeline; the unpack warps then drain D with tcgen05.ld and write fp16
//    (the two warps of a lane quarter take 128 token columns each).
//  * Every wait is bounded: past the limit the waiting thread records
//    TERN_ERR_TIMEOUT in a device-side status word, the CTA stops issuing
//    work, waits (bounded) for its own copies and MMAs in flight, releases its
//    tensor memory and exits.
#include <cstring>

#include "tern_internal.cuh"

namespace tern {

// Device-side record of a bounded wait in this kernel that gave up (read and
// cleared by tern_sync_status).
__device__ unsigned int g_tern_device_status;

namespace {

constexpr int kTN = 128;       // weight rows per tile (MMA M)
constexpr int kTM = 256;       // token rows per tile (MMA N)
constexpr int kBK = 64;        // k per pipeline step (one 128-byte swizzle row of fp16)
constexpr int kStages = 4;
constexpr int kThreads = 320;  // warp 0: TMA, warp 1: MMA + TMEM owner, warps 2..9: unpack + epilogue
constexpr int kUnpackWarps = 8;
constexpr int kXStageBytes = kTM * kBK * 2;  // 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol = 0;        // accumulator: columns [0, 256)
constexpr uint32_t kACol = 256;      // A stages: 32 columns each
constexpr int kRingK = 4;            // k steps of slot bytes prefetched per unpack thread
// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B fp16, both
// K-major, N = 256 (bits 17-22 = N>>3), M = 128 (bits 24-28 = M>>4).
constexpr uint32_t kIdesc = (1u << 4) | ((kTM >> 3) << 17) | ((kTN >> 4) << 24);

struct GemmParams {
    const uint8_t *slots;
    const __half *scales;
    __half *y;
    int M, N, K;
    unsigned long long timeout_ns;
    int skip_loads;  // test only: never issue the TMA loads (exercises the timeout path)
};

// Bounded wait on phase `parity`.  On timeout: record it and raise the CTA abort flag.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned long long deadline,
                                          volatile int *abort_flag) {
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (globaltimer() > deadline) {
            atomicExch(&g_tern_device_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, M=128, N=256, K=16.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(kIdesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 16 codes of one slot word -> 8 fp16 pairs in k order, each times s (exact).
// out[c] = {s*t[2c], s*t[2c+1]} for c = 0..7.
__device__ __forceinline__ void unpack_word_scaled(uint32_t w, uint32_t s2, uint32_t *out) {
    uint32_t p[8];  // p[j] = {t[j], t[j+8]}
    unpack_word(w, p);
#pragma unroll
    for (int c = 0; c < 4; c++) {
        out[c] = hmul2_u32(prmt(p[2 * c], p[2 * c + 1], 0x5410u), s2);      // {t[2c],   t[2c+1]}
        out[c + 4] = hmul2_u32(prmt(p[2 * c], p[2 * c + 1], 0x7632u), s2);  // {t[2c+8], t[2c+9]}
    }
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms.
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xs = smem;                                               // kStages x 32 KB
    uint64_t *full_x = reinterpret_cast<uint64_t *>(smem + kStages * kXStageBytes);
    uint64_t *full_a = full_x + kStages;
    uint64_t *empty = full_a + kStages;
    uint64_t *d_full = empty + kStages;
    uint64_t *mma_done = d_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTN, m0 = blockIdx.y * kTM;
    const int nk = p.K / kBK;
    const unsigned long long deadline = globaltimer() + p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full_x[s], 1);
            mbar_init(&full_a[s], kUnpackWarps);
            mbar_init(&empty[s], 1);
        }
        mbar_init(d_full, 1);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&xmap) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer: x tiles ----------------
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < nk; i++) {
                const int s = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, deadline, abort_flag)) break;
                if (p.skip_loads) continue;
                mbar_expect_tx(&full_x[s], kXStageBytes);
                tma_load_2d(xs + s * kXStageBytes, &xmap, i * kBK, m0, &full_x[s]);
                issued = i + 1;
            }
            if (*abort_flag) {
                // Let the copies this thread started land before the CTA exits.
                const unsigned long long dl2 = globaltimer() + p.timeout_ns;
                for (int i = (issued > kStages ? issued - kStages : 0); i < issued; i++) {
                    int dummy = 0;
                    volatile int *never = &dummy;
                    mbar_wait(&full_x[i % kStages], (i / kStages) & 1, dl2, never);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int i = 0;
            for (; i < nk; i++) {
                const int s = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                if (!mbar_wait(&full_x[s], ph, deadline, abort_flag)) break;
                if (!mbar_wait(&full_a[s], ph, deadline, abort_flag)) break;
                tc_fence_after();
                const uint32_t xaddr = smem_u32(xs + s * kXStageBytes);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; kk++) {
                    tc_mma_ts(tmem + kDCol, tmem + kACol + s * (kBK / 2) + kk * 8,
                              smem_desc_sw128(xaddr + kk * 32), (i | kk) != 0);
                }
                tc_commit(&empty[s]);
            }
            tc_commit(d_full);
            tc_commit(mma_done);
            // All MMAs this thread issued must finish before tensor memory is freed.
            const unsigned long long dl2 = globaltimer() + p.timeout_ns;
            int dummy = 0;
            mbar_wait(mma_done, 0, dl2, &dummy);
        }
    } else {
        // ---------------- unpack (A producer), then epilogue ----------------
        const int q = warp & 3;         // tensor-memory lane quarter this warp may access
        const int hh = (warp - 2) >> 2;  // which half of a k step (32 codes, 16 columns) it unpacks
        const int row = q * 32 + lane;
        const int n = n0 + row;
        const int nld = n < p.N ? n : p.N - 1;
        const int K4 = p.K >> 2;
        const int G = p.K / kGroup;
        const uint8_t *srow = p.slots + static_cast<size_t>(nld) * K4;
        const unsigned short *scrow = reinterpret_cast<const unsigned short *>(p.scales) + static_cast<size_t>(nld) * G;
        uint2 ring[kRingK];
        uint32_t sring[kRingK];
        const uint8_t *hrow = srow + hh * 8;
#pragma unroll
        for (int u = 0; u < kRingK; u++) {
            if (u < nk) {
                ring[u] = __ldg(reinterpret_cast<const uint2 *>(hrow + u * 16));
                sring[u] = __ldg(scrow + (u * kBK) / kGroup);
            }
        }
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        bool ok = true;
        // A stage is announced to the MMA issuer one k step late: the store
        // into tensor memory of step i completes while step i + 1 is
        // unpacked, then the warp waits for it and arrives on step i's
        // barrier (before waiting for step i + 1's stage to be free).
        int pending = -1;
        auto announce = [&]() {
            if (pending < 0) return;
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_a[pending]);
            pending = -1;
        };
        for (int ib = 0; ib < nk && ok; ib += kRingK) {
#pragma unroll
            for (int u = 0; u < kRingK; u++) {
                const int i = ib + u;
                if (i < nk && ok) {
                    const int s = i % kStages;
                    const uint32_t ph = (i / kStages) & 1;
                    const uint2 wv = ring[u];
                    const uint32_t sc = sring[u];
                    if (i + kRingK < nk) {
                        ring[u] = __ldg(reinterpret_cast<const uint2 *>(hrow + (i + kRingK) * 16));
                        sring[u] = __ldg(scrow + ((i + kRingK) * kBK) / kGroup);
                    }
                    uint32_t v[16];
                    const uint32_t s2 = sc | (sc << 16);
                    unpack_word_scaled(wv.x, s2, v);
                    unpack_word_scaled(wv.y, s2, v + 8);
                    announce();
                    // tcgen05.st is warp-collective: take the decision warp-wide.
                    ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1, deadline, abort_flag));
                    if (ok) {
                        tc_fence_after();
                        tmem_st_x16(tmem + lane_base + kACol + s * (kBK / 2) + hh * 16, v);
                        pending = s;
                    }
                }
            }
        }
        if (ok) {
            announce();
        } else {
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");  // no store left in flight
        }
        // Epilogue: D[row][token] -> y[m0 + token][n]
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(d_full, 0, deadline, abort_flag) && !*abort_flag);
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = hh * (kTM / 2); c0 < (hh + 1) * (kTM / 2); c0 += 32) {
                uint32_t v[32];
                tmem_ld_x32(tmem + lane_base + kDCol + c0, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (n < p.N) {
#pragma unroll
                    for (int j = 0; j < 32; j++) {
                        const int m = m0 + c0 + j;
                        if (m < p.M) p.y[static_cast<size_t>(m) * p.N + n] = __float2half_rn(__uint_as_float(v[j]));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

bool g_gemm_attr[64];

}  // namespace

unsigned long long g_gemm_timeout_ns = 1000000000ull;  // 1 s
int g_gemm_skip_loads = 0;

tern_status launch_gemm_tc(const MatDesc &d, int M, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    CUtensorMap xmap;
    st = encode_tiled_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d.x, static_cast<uint64_t>(d.K),
                         static_cast<uint64_t>(M), static_cast<uint64_t>(d.K) * 2, kBK, kTM,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TERN_OK) return st;

    const size_t smem = static_cast<size_t>(kStages) * kXStageBytes + 1024 + 256;
    if (smem > dev.max_smem_optin) return fail(TERN_ERR_DEVICE, "needs %zu B shared memory", smem);
    if (!g_gemm_attr[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
        g_gemm_attr[dev.device] = true;
    }
    GemmParams p;
    p.slots = d.slots;
    p.scales = d.scales;
    p.y = d.y;
    p.M = M;
    p.N = d.N;
    p.K = d.K;
    p.timeout_ns = g_gemm_timeout_ns;
    p.skip_loads = g_gemm_skip_loads;
    const dim3 grid((d.N + kTN - 1) / kTN, (M + kTM - 1) / kTM);
    if (grid.y > 65535u) return fail(TERN_ERR_SHAPE, "M too large for one launch");
    gemm_tc_kernel<<<grid, kThreads, smem, stream>>>(xmap, p);
    return cuda_fail(cudaGetLastError(), "gemm kernel launch");
}

tern_status read_gemm_status(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_device_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_device_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    }
    *out = v;
    return TERN_OK;
}

}  // namespace tern
