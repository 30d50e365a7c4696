// Bandwidth-bound ternary-g128 product for M = 1..8 token rows on the
// 5th-generation tensor cores, with the weights unpacked straight into tensor
// memory at one logic instruction per pair of weights.
//
// What it computes: y[m][n] = sum_k x[m][k] * s[n][k/128] * t[n][k] with t
// read straight from the 2-bit slots and the group scale applied inside the
// product ("Ternary-Bonsai-27B" model summary, aitrends.kr, section
// "Technical features"); decode is bound by memory bandwidth ("Bonsai 27B
// ternary / 1-bit quantization", ThakiCloud blog, section "Throughput and
// speculative decoding").
//
// Arithmetic (exact up to the fp32 accumulation):
//  * A slot word holds 16 codes c = t + 1; "pair j" of a word is field j of
//    both 16-bit halves.  w & (0x00030003 << 2j') (j' = j for j < 5, the word
//    shifted right by 10 for j >= 5) is an fp16 pair of subnormals
//    c * 4^j' * 2^-24.  Each tcgen05.mma (K = 16) takes pair j of the eight
//    words of a scale group, so it sees one factor 4^j'; the B operand holds
//    x * 2^(E - 2j') (E = min(8, 15 - e), e the binary exponent of max|x|: an
//    exact power-of-two scaling).  Every product is c * x * 2^(E-24).
//  * t = c - 1: lane 31 of every warp reads an all-ones word (code 1 = t 0)
//    instead of a weight row, so its accumulator is D(ones) from the very same
//    MMA; subtracting it (one shuffle) makes an all-zero weight row exactly 0.
//    A tile is therefore 124 weight rows (4 warps x 31) on 128 TMEM lanes.
//  * Each thread owns one weight row: per group it loads 8 words (two 16-byte
//    shared loads), forms 64 registers with 72 ALU instructions and writes
//    them to tensor memory with one tcgen05.st; one thread issues the 8 MMAs
//    (M = 128, N = 16, K = 16, fp32 in TMEM); the same threads read the group's
//    accumulator back two groups later and add s * (D - D(ones)) in fp32.
//
// Per CTA (one per SM): two warpgroups, each with 4 unpack warps, a TMA
// producer warp (2 boxes of 128 rows x 512 k of slots + 128 x 8 scales per
// 1024-k slice), a builder warp (the B operand of the slice: M token rows of
// x, class-scaled, in the 128-byte-swizzled K-major layout; token rows 8-15
// of the N = 16 operand alias rows 0-7 through a zero row-group stride) and an
// MMA warp.  The CTA owns a run of tiles; its (tile, slice) units are split in
// half between the warpgroups, and the one tile they may share is summed in
// fixed order at the end.  Every wait is bounded.
#include <algorithm>
#include <cstring>

#include "tern_internal.cuh"

namespace tern {

// Device-side record of a bounded wait in this kernel that gave up.
__device__ unsigned int g_tern_gemvtm_status;

namespace {

constexpr int kRowsPerWarp = 31;
constexpr int kTileRows = 4 * kRowsPerWarp;     // 124 weight rows per tile
constexpr int kSG = 8;                          // scale groups per slice (1024 k)
constexpr int kBoxBytes = 128 * 128;            // 128 rows x 128 B (512 k)
constexpr int kStageTx = 2 * kBoxBytes + 128 * kSG * 2;
constexpr int kBRing = 2;
constexpr int kBSlice = kSG * 2048;             // 8 groups x 2 atoms x 8 rows x 128 B
constexpr uint32_t kTmemCols = 512;

// Shape of a CTA with WGS warpgroups.  Each warpgroup owns 512 / WGS tensor
// memory columns: an A ring of 64-column buffers and a D ring of 16-column
// accumulators; groups in flight are bounded by the A ring, and the drain
// runs kLag groups behind the unpack.
template <int WGS>
struct Cfg {
    static constexpr int kStages = WGS == 2 ? 2 : 4;    // slot stages per warpgroup
    static constexpr int kARing = WGS == 2 ? 3 : 6;
    static constexpr int kDRing = WGS == 2 ? 4 : 8;
    static constexpr int kLag = WGS == 2 ? 2 : 5;
    static constexpr int kThreads = WGS * 7 * 32;
    static constexpr uint32_t kCols = kTmemCols / WGS;
    static constexpr uint32_t kDBase = kARing * 64;     // first D column
    static_assert(kARing * 64 + kDRing * 16 <= static_cast<int>(kCols), "tensor memory");
    static_assert(kDRing >= kLag + 2, "D ring");
};
constexpr int kMaxDesc = TERN_MAX_GROUP;
// kind::f16 instruction descriptor: D fp32, A/B fp16 K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

struct alignas(64) MDesc {
    CUtensorMap smap;   // slots uint8 [N][K/4], box 128 B x 128 rows, 128-byte swizzle
    CUtensorMap cmap;   // scales fp16 [N][K/128], box 8 x 128, no swizzle
    const __half *x;    // [M][K]
    __half *y;          // [M][N]
    int N, K, B;        // B = K / 1024 slices per row
    int ntile;          // ceil(N / 124)
    int c_begin, c_count;
};

struct MParams {
    MDesc d[kMaxDesc];
    int count, M;
    int skip_loads;
    unsigned long long timeout_ns;
};

template <int WGS>
struct Smem {
    using C = Cfg<WGS>;
    uint8_t slot[WGS][C::kStages][2][kBoxBytes];  // 1024-aligned boxes (first member)
    uint8_t bsl[WGS][kBRing][kBSlice];            // B operand slices, 1024-aligned atoms
    uint16_t scl[WGS][C::kStages][128][kSG];
    uint32_t ones[32];                            // 128 bytes of code-1 words
    float part[WGS][128][8];                      // the tile the warpgroups may share
    uint64_t slot_full[WGS][C::kStages], slot_empty[WGS][C::kStages];
    uint64_t b_full[WGS][kBRing], b_empty[WGS][kBRing];
    uint64_t a_full[WGS][C::kARing], a_empty[WGS][C::kARing];
    uint64_t d_full[WGS][C::kDRing], d_empty[WGS][C::kDRing];
    uint64_t mma_done[WGS];
    int part_tile[WGS];
    unsigned int emax;
    uint32_t tmem_base;
};

__device__ __forceinline__ bool tm_wait(uint64_t *bar, uint32_t parity, unsigned long long deadline) {
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() > deadline) {
            atomicExch(&g_tern_gemvtm_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

// K-major, 128-byte swizzle, version 1; the row-group stride is 0, so rows
// 8-15 of the operand read rows 0-7 again.
__device__ __forceinline__ uint64_t desc_b(uint32_t addr) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {"
        "%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, "
        "%33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, "
        "%49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};"
        ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]),
        "r"(v[32]), "r"(v[33]), "r"(v[34]), "r"(v[35]), "r"(v[36]), "r"(v[37]), "r"(v[38]), "r"(v[39]),
        "r"(v[40]), "r"(v[41]), "r"(v[42]), "r"(v[43]), "r"(v[44]), "r"(v[45]), "r"(v[46]), "r"(v[47]),
        "r"(v[48]), "r"(v[49]), "r"(v[50]), "r"(v[51]), "r"(v[52]), "r"(v[53]), "r"(v[54]), "r"(v[55]),
        "r"(v[56]), "r"(v[57]), "r"(v[58]), "r"(v[59]), "r"(v[60]), "r"(v[61]), "r"(v[62]), "r"(v[63])
        : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld<1>(uint32_t taddr, uint32_t (&v)[1]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v[0]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<2>(uint32_t taddr, uint32_t (&v)[2]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<4>(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// The (tile, slice) units of one warpgroup: the CTA owns tiles [t0, t1) of
// its matrix; unit u = slice u % B of tile t0 + u / B; warpgroup w takes units
// [w * U / WGS, (w + 1) * U / WGS).
struct Units {
    int t0, u0, u1, B;
    __device__ void init(const MDesc &d, int lc, int wg, int nwg) {
        t0 = static_cast<int>((static_cast<long long>(lc) * d.ntile) / d.c_count);
        const int t1 = static_cast<int>((static_cast<long long>(lc + 1) * d.ntile) / d.c_count);
        B = d.B;
        const int U = (t1 - t0) * B;
        u0 = (U * wg) / nwg;
        u1 = (U * (wg + 1)) / nwg;
    }
    __device__ int tile(int u) const { return t0 + u / B; }
    __device__ int slice(int u) const { return u - (u / B) * B; }
};

template <int MT, int WGS>
__global__ void __launch_bounds__(Cfg<WGS>::kThreads, 1) gemv_tmem_kernel(const __grid_constant__ MParams p) {
    using C = Cfg<WGS>;
    constexpr int kWG = WGS, kStages = C::kStages, kARing = C::kARing, kDRing = C::kDRing, kLag = C::kLag;
    constexpr int kThreads = C::kThreads;
    constexpr uint32_t kWGCols = C::kCols, kDBase = C::kDBase;
    // warp roles: [0, 4*WGS) unpack (warpgroup w = warp / 4), then WGS producers,
    // WGS builders and WGS MMA issuers
    constexpr int kProd = 4 * WGS, kBuild = 5 * WGS, kMma = 6 * WGS;
    extern __shared__ uint8_t smem_raw[];
    Smem<WGS> &sm = *reinterpret_cast<Smem<WGS> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M;
    int di = 0;
#pragma unroll 1
    while (di + 1 < p.count && static_cast<int>(blockIdx.x) >= p.d[di + 1].c_begin) di++;
    const MDesc &d = p.d[di];
    const int lc = blockIdx.x - d.c_begin;
    const int wg = warp < kProd ? (warp >> 2) : ((warp - kProd) % WGS);

    if (threadIdx.x == 0) {
        for (int w = 0; w < kWG; w++) {
            for (int s = 0; s < kStages; s++) {
                mbar_init(&sm.slot_full[w][s], 1);
                mbar_init(&sm.slot_empty[w][s], 4);
            }
            for (int b = 0; b < kBRing; b++) {
                mbar_init(&sm.b_full[w][b], 1);
                mbar_init(&sm.b_empty[w][b], 1);
            }
            for (int a = 0; a < kARing; a++) {
                mbar_init(&sm.a_full[w][a], 4);
                mbar_init(&sm.a_empty[w][a], 1);
            }
            for (int e = 0; e < kDRing; e++) {
                mbar_init(&sm.d_full[w][e], 1);
                mbar_init(&sm.d_empty[w][e], 4);
            }
            mbar_init(&sm.mma_done[w], 1);
            sm.part_tile[w] = -1;
        }
        sm.emax = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // B slices start at zero: token rows >= M are never written afterwards.
    for (int i = threadIdx.x; i < kWG * kBRing * kBSlice / 16; i += kThreads)
        reinterpret_cast<uint4 *>(&sm.bsl[0][0][0])[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x < 32) sm.ones[threadIdx.x] = 0x55555555u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == kMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    __syncthreads();
    // E from the largest finite |x| of all token rows (every thread helps).
    {
        unsigned int mx = 0;
        const int n8 = M * d.K / 8;
        for (int i = threadIdx.x; i < n8; i += kThreads) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(d.x) + i);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; e++) mx = __vmaxu2(mx, __vminu2(wv[e] & 0x7FFF7FFFu, 0x7BFF7BFFu));
        }
        mx = max(mx & 0xFFFFu, mx >> 16);
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) atomicMax(&sm.emax, mx);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const int ex = max(static_cast<int>(sm.emax >> 10), 1) - 15;
    const int E = min(8, 15 - ex);
    const uint32_t tmem = sm.tmem_base + wg * kWGCols;
    const unsigned long long deadline = globaltimer() + p.timeout_ns;
    Units un;
    un.init(d, lc, wg, WGS);

    if (warp >= kProd && warp < kBuild) {
        // ======================= TMA producer =======================
        if (lane == 0) {
            bool dead = p.skip_loads != 0;
            int issued = 0;
            for (int u = un.u0; u < un.u1 && !dead; u++) {
                const int i = u - un.u0, st = i % kStages;
                dead = !tm_wait(&sm.slot_empty[wg][st], ((i / kStages) & 1) ^ 1, deadline);
                if (dead) break;
                const int tile = un.tile(u), sl = un.slice(u);
                mbar_expect_tx(&sm.slot_full[wg][st], kStageTx);
                tma_load_2d(&sm.slot[wg][st][0][0], &d.smap, sl * 256, tile * kTileRows, &sm.slot_full[wg][st]);
                tma_load_2d(&sm.slot[wg][st][1][0], &d.smap, sl * 256 + 128, tile * kTileRows, &sm.slot_full[wg][st]);
                tma_load_2d(&sm.scl[wg][st][0][0], &d.cmap, sl * kSG, tile * kTileRows, &sm.slot_full[wg][st]);
                issued++;
            }
            // The copies still in flight must land before the CTA exits (bounded).
            const unsigned long long dl2 = globaltimer() + p.timeout_ns;
            for (int i = (issued > kStages ? issued - kStages : 0); i < issued; i++)
                tm_wait(&sm.slot_full[wg][i % kStages], (i / kStages) & 1, dl2);
        }
    } else if (warp >= kBuild && warp < kMma) {
        // ======================= B builder =======================
        // Item (m, group j, word quad wq): x[m][128j + 64wq .. +64) of the
        // slice gives, for every pair i, one 16-byte chunk of the operand of
        // mma i: {x[16w + i], x[16w + i + 8]} for the four words w of the quad.
        uint32_t fac[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const int e = E - 2 * (i < 5 ? i : i - 5);  // in [-8, 8]
            const uint32_t h = static_cast<uint32_t>(15 + e) << 10;
            fac[i] = h | (h << 16);
        }
        bool dead = false;
        for (int u = un.u0; u < un.u1 && !dead; u++) {
            const int i = u - un.u0, bb = i % kBRing;
            bool ok = true;
            if (lane == 0) ok = tm_wait(&sm.b_empty[wg][bb], ((i / kBRing) & 1) ^ 1, deadline);
            dead = !__shfl_sync(0xffffffffu, ok, 0);
            if (dead) break;
            const int k0 = un.slice(u) * 1024;
            uint8_t *base = &sm.bsl[wg][bb][0];
            for (int it = lane; it < M * 16; it += 32) {
                const int m = it >> 4, j = (it >> 1) & 7, wq = it & 1;
                const uint4 *src = reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(m) * d.K + k0 + j * 128 + wq * 64);
                uint32_t r[4][8];
#pragma unroll
                for (int w = 0; w < 4; w++) {
                    const uint4 a = __ldg(src + 2 * w), b = __ldg(src + 2 * w + 1);
                    r[w][0] = a.x; r[w][1] = a.y; r[w][2] = a.z; r[w][3] = a.w;
                    r[w][4] = b.x; r[w][5] = b.y; r[w][6] = b.z; r[w][7] = b.w;
                }
                uint8_t *gb = base + j * 2048 + m * 128;
#pragma unroll
                for (int pi = 0; pi < 8; pi++) {
                    const uint32_t sel = (pi & 1) ? 0x7632u : 0x5410u;
                    uint4 o;
                    o.x = hmul2(prmt(r[0][pi >> 1], r[0][4 + (pi >> 1)], sel), fac[pi]);
                    o.y = hmul2(prmt(r[1][pi >> 1], r[1][4 + (pi >> 1)], sel), fac[pi]);
                    o.z = hmul2(prmt(r[2][pi >> 1], r[2][4 + (pi >> 1)], sel), fac[pi]);
                    o.w = hmul2(prmt(r[3][pi >> 1], r[3][4 + (pi >> 1)], sel), fac[pi]);
                    const int c16 = (pi & 3) * 2 + wq;
                    *reinterpret_cast<uint4 *>(gb + (pi >> 2) * 1024 + ((c16 ^ m) << 4)) = o;
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.b_full[wg][bb]);
        }
    } else if (warp >= kMma) {
        // ======================= MMA issuer =======================
        if (lane == 0) {
            bool dead = false;
            int f = 0;
            for (int u = un.u0; u < un.u1 && !dead; u++) {
                const int i = u - un.u0, bb = i % kBRing;
                dead = !tm_wait(&sm.b_full[wg][bb], (i / kBRing) & 1, deadline);
                const uint32_t bbase = smem_u32(&sm.bsl[wg][bb][0]);
                for (int j = 0; j < kSG && !dead; j++, f++) {
                    const int ab = f % kARing, db = f % kDRing;
                    dead = !tm_wait(&sm.a_full[wg][ab], (f / kARing) & 1, deadline) ||
                           !tm_wait(&sm.d_empty[wg][db], ((f / kDRing) & 1) ^ 1, deadline);
                    if (dead) break;
                    fence_after();
#pragma unroll
                    for (int pi = 0; pi < 8; pi++)
                        mma_f16(tmem + kDBase + db * 16, tmem + ab * 64 + pi * 8,
                                desc_b(bbase + j * 2048 + (pi >> 2) * 1024 + (pi & 3) * 32), pi > 0);
                    commit(&sm.a_empty[wg][ab]);
                    commit(&sm.d_full[wg][db]);
                }
                if (!dead) commit(&sm.b_empty[wg][bb]);
            }
            // nothing may be in flight when the tensor memory is freed
            commit(&sm.mma_done[wg]);
            tm_wait(&sm.mma_done[wg], 0, globaltimer() + p.timeout_ns);
        }
    } else {
        // ======================= unpack + drain =======================
        const int q = warp & 3;                       // tensor-memory lane quarter
        const bool ones = lane == kRowsPerWarp;       // this lane computes D(ones)
        const int rt = q * kRowsPerWarp + lane;       // row in the tile (lane < 31)
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const float post = ldexpf(1.0f, 24 - E);
        const int N = d.N;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; m++) acc[m] = 0.f;
        uint4 sc_cur = make_uint4(0, 0, 0, 0), sc_prev = sc_cur;  // this row's 8 scales, current / previous unit
        int cur_u = un.u0 - 1;
        int f = 0, fd = 0;
        bool dead = false;

        // Reads back the accumulator of group fd (two groups behind) and adds it.
        auto drain = [&]() {
            const int db = fd % kDRing;
            bool ok = !dead;
            if (ok) ok = __all_sync(0xffffffffu, tm_wait(&sm.d_full[wg][db], (fd / kDRing) & 1, deadline));
            dead = !ok;
            const int u = un.u0 + fd / kSG, j = fd % kSG;
            if (ok) {
                fence_after();
                uint32_t v[MT];
                tmem_ld<MT>(tmem + lane_off + kDBase + db * 16, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.d_empty[wg][db]);
                const uint4 sc = (u == cur_u) ? sc_cur : sc_prev;
                const uint32_t sw = (j < 2) ? sc.x : (j < 4) ? sc.y : (j < 6) ? sc.z : sc.w;
                const float s = __half2float(__ushort_as_half(static_cast<unsigned short>((j & 1) ? (sw >> 16) : sw)));
#pragma unroll
                for (int m = 0; m < MT; m++) {
                    const float o = __shfl_sync(0xffffffffu, __uint_as_float(v[m]), kRowsPerWarp);
                    acc[m] = fmaf(s, __uint_as_float(v[m]) - o, acc[m]);
                }
            }
            fd++;
            if (j == kSG - 1 && (un.slice(u) == un.B - 1 || u == un.u1 - 1)) {
                // ---- this warpgroup's part of a tile is complete ----
                const int tile = un.tile(u);
                const bool whole = un.slice(u) == un.B - 1 && (u - un.slice(u) >= un.u0);
                const int row = tile * kTileRows + rt;
                if (whole) {
                    if (!dead && !ones && row < N) {
#pragma unroll
                        for (int m = 0; m < MT; m++)
                            if (m < M) d.y[static_cast<size_t>(m) * N + row] = __float2half_rn(acc[m] * post);
                    }
                } else {
                    if (!ones) {
#pragma unroll
                        for (int m = 0; m < MT; m++) sm.part[wg][rt][m] = acc[m] * post;
                    }
                    if (q == 0 && lane == 0) sm.part_tile[wg] = dead ? -2 : tile;
                }
#pragma unroll
                for (int m = 0; m < MT; m++) acc[m] = 0.f;
            }
        };

        for (int u = un.u0; u < un.u1; u++) {
            const int i = u - un.u0, st = i % kStages;
            bool ok = !dead;
            if (ok) ok = __all_sync(0xffffffffu, tm_wait(&sm.slot_full[wg][st], (i / kStages) & 1, deadline));
            dead = !ok;
            sc_prev = sc_cur;
            cur_u = u;
            sc_cur = ones ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4 *>(&sm.scl[wg][st][rt][0]);
            // lane 31 reads the 128-byte all-ones row for both boxes
            const uint8_t *rowp = ones ? reinterpret_cast<const uint8_t *>(&sm.ones[0]) : &sm.slot[wg][st][0][0] + rt * 128;
            const int box_stride = ones ? 0 : kBoxBytes;
            const int sw = ones ? 0 : (rt & 7);
#pragma unroll 1
            for (int j = 0; j < kSG; j++) {
                if (!dead) {
                    const uint8_t *bp = rowp + (j >> 2) * box_stride;
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(bp + (((2 * (j & 3)) ^ sw) << 4));
                    const uint4 w1 = *reinterpret_cast<const uint4 *>(bp + (((2 * (j & 3) + 1) ^ sw) << 4));
                    if (j == kSG - 1) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.slot_empty[wg][st]);
                    }
                    const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    uint32_t v[64];
#pragma unroll
                    for (int w = 0; w < 8; w++) {
                        const uint32_t a = wd[w], a5 = wd[w] >> 10;
                        v[0 * 8 + w] = a & 0x00030003u;
                        v[1 * 8 + w] = a & 0x000C000Cu;
                        v[2 * 8 + w] = a & 0x00300030u;
                        v[3 * 8 + w] = a & 0x00C000C0u;
                        v[4 * 8 + w] = a & 0x03000300u;
                        v[5 * 8 + w] = a5 & 0x00030003u;
                        v[6 * 8 + w] = a5 & 0x000C000Cu;
                        v[7 * 8 + w] = a5 & 0x00300030u;
                    }
                    const int ab = f % kARing;
                    ok = __all_sync(0xffffffffu, tm_wait(&sm.a_empty[wg][ab], ((f / kARing) & 1) ^ 1, deadline));
                    dead = !ok;
                    if (ok) {
                        fence_after();
                        tmem_st64(tmem + lane_off + ab * 64, v);
                        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                        fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.a_full[wg][ab]);
                    }
                }
                f++;
                if (f - fd > kLag) drain();
            }
        }
        while (fd < f) drain();

        // ---- the tile shared by the two warpgroups: summed in fixed order ----
        named_bar_sync(1, 4 * WGS * 32);
        if (WGS == 2 && wg == 0 && !ones) {
            const int t = sm.part_tile[0];
            if (t >= 0 && t == sm.part_tile[WGS - 1]) {
                const int row = t * kTileRows + rt;
                if (row < N) {
#pragma unroll
                    for (int m = 0; m < MT; m++)
                        if (m < M)
                            d.y[static_cast<size_t>(m) * N + row] =
                                __float2half_rn(sm.part[0][rt][m] + sm.part[WGS - 1][rt][m]);
                }
            }
        }
    }

    fence_before();
    __syncthreads();
    if (warp == kMma) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem_base), "r"(kTmemCols));
    }
}

bool g_attr_tm[64][4][2];

int tm_mt(int M) { return M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : 8)); }

}  // namespace

bool gemv_tmem_supports(const MatDesc *md, int count, int M) {
    if (M < 1 || M > 8 || count < 1 || count > kMaxDesc) return false;
    for (int i = 0; i < count; i++)
        if (md[i].K % 1024 != 0) return false;
    return true;
}

tern_status launch_gemv_tmem(const MatDesc *md, int count, int M, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    if (!gemv_tmem_supports(md, count, M)) return fail(TERN_ERR_SHAPE, "tensor-memory kernel: unsupported shape");
    const int MT = tm_mt(M);
    // warpgroups per CTA: 2 by default, 1 with TERN_OPT_GEMV_CTAS = 1
    const int wgs = g_opt.gemv_ctas == 1 ? 1 : 2;
    auto pick = [&](auto k1, auto k2, auto k4, auto k8) { return MT == 1 ? k1 : (MT == 2 ? k2 : (MT == 4 ? k4 : k8)); };
    auto kern = wgs == 2 ? pick(gemv_tmem_kernel<1, 2>, gemv_tmem_kernel<2, 2>, gemv_tmem_kernel<4, 2>, gemv_tmem_kernel<8, 2>)
                         : pick(gemv_tmem_kernel<1, 1>, gemv_tmem_kernel<2, 1>, gemv_tmem_kernel<4, 1>, gemv_tmem_kernel<8, 1>);
    const int mi = MT == 1 ? 0 : (MT == 2 ? 1 : (MT == 4 ? 2 : 3));
    const size_t smem = (wgs == 2 ? sizeof(Smem<2>) : sizeof(Smem<1>)) + 1024;
    const int threads = wgs == 2 ? Cfg<2>::kThreads : Cfg<1>::kThreads;
    if (smem > dev.max_smem_optin) return fail(TERN_ERR_DEVICE, "needs %zu B shared memory", smem);
    if (!g_attr_tm[dev.device][mi][wgs - 1]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemv tmem)");
        g_attr_tm[dev.device][mi][wgs - 1] = true;
    }
    // One CTA per SM (it owns all 512 tensor-memory columns).  CTAs go to the
    // matrices in proportion to their (tile, slice) units: start from one each
    // and hand the rest to the matrix whose CTAs carry the most; never more
    // CTAs than tiles; then drop CTAs that do not lower their matrix's load.
    long long cap = static_cast<long long>(dev.sms);
    if (g_opt.gemv_grid > 0) cap = std::min<long long>(cap, g_opt.gemv_grid);
    cap = std::max<long long>(cap, count);
    int ntile[kMaxDesc];
    long long cl[kMaxDesc];
    long long used = 0;
    for (int i = 0; i < count; i++) {
        ntile[i] = (md[i].N + kTileRows - 1) / kTileRows;
        cl[i] = 1;
        used++;
    }
    auto load = [&](int i, long long c) {
        return ((ntile[i] + c - 1) / c) * static_cast<long long>(md[i].K / 1024);
    };
    while (used < cap) {
        int worst = -1;
        long long wv = -1;
        for (int i = 0; i < count; i++) {
            if (cl[i] >= ntile[i]) continue;
            const long long l = load(i, cl[i]);
            if (l > wv) {
                wv = l;
                worst = i;
            }
        }
        if (worst < 0) break;
        cl[worst]++;
        used++;
    }
    for (int i = 0; i < count; i++)
        while (cl[i] > 1 && load(i, cl[i] - 1) == load(i, cl[i])) cl[i]--;

    MParams p;
    std::memset(&p, 0, sizeof(p));
    p.count = count;
    p.M = M;
    p.skip_loads = g_gemm_skip_loads;
    p.timeout_ns = g_gemm_timeout_ns;
    int next = 0;
    for (int i = 0; i < count; i++) {
        MDesc &g = p.d[i];
        st = encode_tiled_2d(&g.smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots, static_cast<uint64_t>(md[i].K / 4),
                             static_cast<uint64_t>(md[i].N), static_cast<uint64_t>(md[i].K / 4), 128, 128,
                             CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TERN_OK) return st;
        const int G = md[i].K / kGroup;
        st = encode_tiled_2d(&g.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, md[i].scales, static_cast<uint64_t>(G),
                             static_cast<uint64_t>(md[i].N), static_cast<uint64_t>(G) * 2, kSG, 128,
                             CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != TERN_OK) return st;
        g.x = md[i].x;
        g.y = md[i].y;
        g.N = md[i].N;
        g.K = md[i].K;
        g.B = md[i].K / 1024;
        g.ntile = ntile[i];
        g.c_begin = next;
        g.c_count = static_cast<int>(cl[i]);
        next += g.c_count;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(next));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_fail(e, "gemv tmem kernel launch");
    return TERN_OK;
}

tern_status read_gemvtm_status(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_gemvtm_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_gemvtm_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    }
    *out = v;
    return TERN_OK;
}

}  // namespace tern
