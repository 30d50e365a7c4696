// Bandwidth-bound ternary-g128 product for M = 1..8 token rows on the
// 5th-generation tensor cores (tcgen05).
//
// What it computes: y[m][n] = sum_k x[m][k] * s[n][k/128] * t[n][k] with t
// read straight from the 2-bit slots and the group scale applied inside the
// product ("Ternary-Bonsai-27B" model summary, aitrends.kr, section
// "Technical features"); decode is bound by memory bandwidth ("Bonsai 27B
// ternary / 1-bit quantization", ThakiCloud blog, section "Throughput and
// speculative decoding"), so everything is organised around streaming the
// slots once at the lowest instruction cost per weight.
//
// Why tensor cores for an M <= 8 product: at the measured HBM bandwidth an SM
// has to retire ~86 weights per cycle with 4 instruction issues per cycle,
// and turning two 2-bit codes into an exact fp16 pair already costs two
// instructions (LOP3 + HFMA2).  Doing the multiply-adds on the CUDA cores, or
// even with per-warp mma.sync (which needs per-warp B-fragment loads, scale
// shuffles and MMA issues), leaves too few issue slots.  Here each thread owns
// one weight row: its unpacked codes go to tensor memory with one tcgen05.st
// per 64 weights, and a single thread issues the MMAs, so the unpack is almost
// the only per-weight work.
//
// Per warpgroup (128 threads = 128 weight rows of a tile) the pipeline is:
//  * producer warp: TMA of 128 rows x 512 k of slots (16 KB, 128-byte swizzle)
//    into a 3-stage ring; builds the B operand of every scale group (16 token
//    rows x 128 k of x, rows >= M zero) in the k order the unpack produces
//    (pairs k, k+8 of each 16-weight word), loading x one stage ahead;
//  * unpack warps: per group, two 16-byte shared loads, LOP3+HFMA2 per pair,
//    tcgen05.st of 64 columns (A operand, t exact in fp16);
//  * MMA thread: 8 x tcgen05.mma (M=128, N=16, K=16, fp32) per group into its
//    own accumulator of a 4-deep ring;
//  * the unpack warps drain each group's accumulator two groups later with
//    tcgen05.ld and add s * D in fp32 (the scale stays out of the fp16 path).
// Work items are 128 rows x (a multiple of 512 k); a tile split over several
// items is reduced through the caller's workspace: partials in fixed order by
// the last item to arrive (per-tile arrival counter, reset after use), so the
// result does not depend on scheduling.  Every wait is bounded.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "tern_internal.cuh"

namespace tern {

// Device-side record of a bounded wait in this kernel that gave up.
__device__ unsigned int g_tern_gemvtc_status;

namespace {

constexpr int kRows = 128;                      // tile rows = MMA M
constexpr int kTok = 16;                        // MMA N: token columns (rows >= M of B are zero)
constexpr int kGPS = 4;                         // scale groups per slot stage (512 k = 128 B per row)
constexpr int kSlotStages = 3;
constexpr int kSlotStageBytes = kRows * 128;    // 16 KB
constexpr int kBBytes = kTok * 128 * 2;         // 4 KB: x of one group in the MMA's B layout
constexpr int kRingB = 2, kRingD = 4;
constexpr int kLag = 2;                         // groups between unpacking and draining
constexpr int kSRing = 4;                       // stages of scales held (drain lag + 2 ahead)
constexpr int kWG = 2;                          // warpgroups per CTA
constexpr int kWarpsPerWG = 6;                  // 4 unpack + producer + MMA
constexpr int kThreads = kWG * kWarpsPerWG * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWGCols = 256;               // per WG: A ring at +0/+64, D ring at +128 + 16 d
constexpr int kMaxDesc = TERN_MAX_GROUP;
constexpr int kMaxTcRows = 4;                   // token rows handled by this kernel
// The workspace starts with a fixed-size block of per-tile arrival counters,
// then the partial sums.  Fixed so that the counters of every call land on
// counters (zeroed) and never on another call's leftover partials.
constexpr int kMaxSplitTiles = 32768;
constexpr size_t kCounterBytes = static_cast<size_t>(kMaxSplitTiles) * 4;
// kind::f16 instruction descriptor: D fp32, A/B fp16 K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | ((kTok >> 3) << 17) | ((kRows >> 4) << 24);

struct alignas(64) CDesc {
    CUtensorMap map;        // slots uint8 [N][K/4], box 128 B x 128 rows, 128-byte swizzle
    const __half *x;        // [M][K]
    const __half *scales;   // [N][G]
    __half *y;              // [M][N]
    int N, K, G;
    int ntile;              // ceil(N / 128)
    int parts;              // items per tile (K split)
    int spp;                // slot stages per part (4 groups each)
    int item_begin;         // first global item index of this matrix
    int tile_ws;            // first tile counter of this matrix in the workspace
    long long pslot;        // first partial slot of this matrix
};

struct CParams {
    CDesc d[kMaxDesc];
    int count, M;
    int total_items;
    int wg_slots;             // warpgroups in the grid
    unsigned int *counters;   // per split tile, zero between calls
    float *partials;          // [slot][128 rows][MT]
    unsigned long long timeout_ns;
    int skip_loads;
};

struct Smem {
    uint8_t slot[kWG][kSlotStages][kSlotStageBytes];  // 1024-aligned (first member)
    uint8_t bbuf[kWG][kRingB][kBBytes];
    uint64_t slot_full[kWG][kSlotStages], slot_empty[kWG][kSlotStages];
    uint64_t a_full[kWG][2], a_empty[kWG][2];
    uint64_t b_full[kWG][kRingB], b_empty[kWG][kRingB];
    uint64_t d_full[kWG][kRingD], d_empty[kWG][kRingD];
    uint64_t mma_done[kWG];
    unsigned short sring[kWG][kSRing][kRows][kGPS];  // per-thread scale ring
    uint32_t tmem_base;
    int last_flag[kWG];
};

__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, unsigned long long deadline) {
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() > deadline) {
            atomicExch(&g_tern_gemvtc_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
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

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(kIdesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

// K-major, 128-byte swizzle, 8-row groups 1024 bytes apart, version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void tmem_st_x64(uint32_t taddr, const uint32_t (&v)[64]) {
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
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Position of an item in the launch: matrix, tile, part, stage range.
struct ItemPos {
    int di, tile, part;
    int s0, ns;  // first slot stage (in units of 4 groups) and stage count
};

__device__ __forceinline__ ItemPos locate(const CParams &p, int item) {
    int di = 0;
    while (di + 1 < p.count && item >= p.d[di + 1].item_begin) di++;
    const CDesc &d = p.d[di];
    const int local = item - d.item_begin;
    ItemPos r;
    r.di = di;
    r.tile = local / d.parts;
    r.part = local - r.tile * d.parts;
    const int nst = (d.G + kGPS - 1) / kGPS;  // stages of a full row
    r.s0 = r.part * d.spp;
    r.ns = min(d.spp, nst - r.s0);
    return r;
}

// Walks the flat sequence of (item, stage) of one warpgroup.
struct Cursor {
    int item, stage;  // current item index and stage within it
    ItemPos pos;
    bool valid;
    __device__ void init(const CParams &p, int first) {
        item = first;
        stage = 0;
        valid = item < p.total_items;
        if (valid) pos = locate(p, item);
    }
    // Advance one stage; returns true when the item changed.
    __device__ bool next_stage(const CParams &p) {
        if (++stage < pos.ns) return false;
        stage = 0;
        item += p.wg_slots;
        valid = item < p.total_items;
        if (valid) pos = locate(p, item);
        return true;
    }
};

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_tc_kernel(const __grid_constant__ CParams p) {
    static_assert(MT == 1 || MT == 2 || MT == 4, "token tile");
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // warps [0,4) WG0 unpack, [4,8) WG1 unpack, 8/9 producers, 10/11 MMA issuers
    const int wg = warp < 8 ? (warp >> 2) : ((warp - 8) & 1);
    const int M = p.M;
    const unsigned long long deadline = globaltimer() + p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kWG; w++) {
            for (int s = 0; s < kSlotStages; s++) {
                mbar_init(&sm.slot_full[w][s], 1);
                mbar_init(&sm.slot_empty[w][s], 4);
            }
            for (int a = 0; a < 2; a++) {
                mbar_init(&sm.a_full[w][a], 4);
                mbar_init(&sm.a_empty[w][a], 1);
            }
            for (int b = 0; b < kRingB; b++) {
                mbar_init(&sm.b_full[w][b], 1);
                mbar_init(&sm.b_empty[w][b], 1);
            }
            for (int d = 0; d < kRingD; d++) {
                mbar_init(&sm.d_full[w][d], 1);
                mbar_init(&sm.d_empty[w][d], 4);
            }
            mbar_init(&sm.mma_done[w], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // B buffers start at zero: token rows >= M are never written afterwards.
    for (int i = threadIdx.x; i < kWG * kRingB * kBBytes / 16; i += kThreads)
        reinterpret_cast<uint4 *>(&sm.bbuf[0][0][0])[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 10) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base + wg * kWGCols;
    const int first_item = blockIdx.x * kWG + wg;

    if (warp >= 8 && warp < 10) {
        // ======================= producer warp =======================
        Cursor cs;  // slot stream
        cs.init(p, first_item);
        int fs_issue = 0;
        bool dead = false;
        auto issue_stage = [&]() {
            if (!cs.valid) return;
            const int slot = fs_issue % kSlotStages;
            if (lane == 0) {
                dead = dead || !tc_wait(&sm.slot_empty[wg][slot], ((fs_issue / kSlotStages) & 1) ^ 1, deadline);
                if (!dead && !p.skip_loads) {
                    const CDesc &d = p.d[cs.pos.di];
                    mbar_expect_tx(&sm.slot_full[wg][slot], kSlotStageBytes);
                    tma_load_2d(&sm.slot[wg][slot][0], &d.map, (cs.pos.s0 + cs.stage) * 128, cs.pos.tile * kRows,
                                &sm.slot_full[wg][slot]);
                }
            }
            dead = __shfl_sync(0xffffffffu, dead, 0);
            fs_issue++;
            cs.next_stage(p);
        };
        for (int s = 0; s < kSlotStages; s++) issue_stage();

        // B stream: x of stage k is loaded during stage k-1 (registers), then
        // permuted into the MMA layout group by group.
        constexpr int kPairs = (MT * 8 + 31) / 32;  // (token row, 16-k block) pairs per lane per group
        uint4 xr[kGPS][kPairs][2];
        Cursor cb;
        cb.init(p, first_item);
        auto load_x = [&](const Cursor &c) {
#pragma unroll
            for (int j = 0; j < kGPS; j++)
#pragma unroll
                for (int i = 0; i < kPairs; i++) {
                    xr[j][i][0] = make_uint4(0, 0, 0, 0);
                    xr[j][i][1] = make_uint4(0, 0, 0, 0);
                    const int pr = lane + 32 * i;
                    const int m = pr >> 3, b = pr & 7;
                    if (c.valid && m < M) {
                        const CDesc &d = p.d[c.pos.di];
                        const int k = ((c.pos.s0 + c.stage) * kGPS + j) * kGroup + b * 16;
                        if (k < d.K) {
                            const uint4 *src = reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(m) * d.K + k);
                            xr[j][i][0] = __ldg(src);
                            xr[j][i][1] = __ldg(src + 1);
                        }
                    }
                }
        };
        load_x(cb);
        int fb = 0;  // flat group counter of the B stream
        while (cb.valid && !dead) {
            uint4 cur[kGPS][kPairs][2];
#pragma unroll
            for (int j = 0; j < kGPS; j++)
#pragma unroll
                for (int i = 0; i < kPairs; i++) {
                    cur[j][i][0] = xr[j][i][0];
                    cur[j][i][1] = xr[j][i][1];
                }
            Cursor nxt = cb;
            nxt.next_stage(p);
            load_x(nxt);
#pragma unroll
            for (int j = 0; j < kGPS; j++) {
                const int rb = fb % kRingB;
                if (lane == 0) dead = dead || !tc_wait(&sm.b_empty[wg][rb], ((fb / kRingB) & 1) ^ 1, deadline);
                dead = __shfl_sync(0xffffffffu, dead, 0);
                if (dead) break;
                uint8_t *bb = &sm.bbuf[wg][rb][0];
#pragma unroll
                for (int i = 0; i < kPairs; i++) {
                    const int pr = lane + 32 * i;
                    const int m = pr >> 3, b = pr & 7;
                    if (m < M) {
                        const uint4 lo = cur[j][i][0], hi = cur[j][i][1];  // x[16b .. 16b+7], x[16b+8 .. 16b+15]
                        uint4 o0, o1;
                        o0.x = prmt(lo.x, hi.x, 0x5410u);  // {x0, x8}
                        o0.y = prmt(lo.x, hi.x, 0x7632u);  // {x1, x9}
                        o0.z = prmt(lo.y, hi.y, 0x5410u);  // {x2, x10}
                        o0.w = prmt(lo.y, hi.y, 0x7632u);  // {x3, x11}
                        o1.x = prmt(lo.z, hi.z, 0x5410u);  // {x4, x12}
                        o1.y = prmt(lo.z, hi.z, 0x7632u);  // {x5, x13}
                        o1.z = prmt(lo.w, hi.w, 0x5410u);  // {x6, x14}
                        o1.w = prmt(lo.w, hi.w, 0x7632u);  // {x7, x15}
                        // 16-byte chunks 2b and 2b+1 of the permuted group; atom = 64 k
                        const int atom = b >> 2;
                        const int r = m & 7;
                        uint8_t *rowp = bb + atom * 2048 + (m >> 3) * 1024 + r * 128;
                        const int c0 = (2 * b) & 7, c1 = (2 * b + 1) & 7;
                        *reinterpret_cast<uint4 *>(rowp + ((c0 ^ r) << 4)) = o0;
                        *reinterpret_cast<uint4 *>(rowp + ((c1 ^ r) << 4)) = o1;
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.b_full[wg][rb]);
                fb++;
                if (j == kGPS - 1) issue_stage();  // the ring slot of the stage just finished frees next
            }
            cb = nxt;
        }
        // Let this warp's copies in flight land before leaving (bounded).
        if (dead && lane == 0) {
            const unsigned long long dl2 = globaltimer() + p.timeout_ns;
            for (int f = (fs_issue > kSlotStages ? fs_issue - kSlotStages : 0); f < fs_issue; f++)
                tc_wait(&sm.slot_full[wg][f % kSlotStages], (f / kSlotStages) & 1, dl2);
        }
    } else if (warp >= 10) {
        // ======================= MMA issuer =======================
        if (lane == 0) {
            Cursor c;
            c.init(p, first_item);
            int f = 0;
            bool dead = false;
            while (c.valid && !dead) {
                for (int j = 0; j < kGPS && !dead; j++) {
                    const int ab = f & 1, rb = f % kRingB, db = f % kRingD;
                    dead = !tc_wait(&sm.a_full[wg][ab], (f >> 1) & 1, deadline) ||
                           !tc_wait(&sm.b_full[wg][rb], (f / kRingB) & 1, deadline) ||
                           !tc_wait(&sm.d_empty[wg][db], ((f / kRingD) & 1) ^ 1, deadline);
                    if (dead) break;
                    tc_fence_after();
                    const uint32_t bbase = smem_u32(&sm.bbuf[wg][rb][0]);
#pragma unroll
                    for (int kk = 0; kk < 8; kk++)
                        tc_mma(tmem + 128 + db * kTok, tmem + ab * 64 + kk * 8,
                               desc_sw128(bbase + (kk >> 2) * 2048 + (kk & 3) * 32), kk > 0);
                    tc_commit(&sm.a_empty[wg][ab]);
                    tc_commit(&sm.b_empty[wg][rb]);
                    tc_commit(&sm.d_full[wg][db]);
                    f++;
                }
                c.next_stage(p);
            }
            tc_commit(&sm.mma_done[wg]);
            tc_wait(&sm.mma_done[wg], 0, globaltimer() + p.timeout_ns);
        }
    } else {
        // ======================= unpack + drain warps =======================
        const int q = warp & 3;  // tensor-memory lane quarter
        const int r = q * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        Cursor cu, cd, csc;  // unpack stream, drain stream, scale prefetch stream
        cu.init(p, first_item);
        cd = cu;
        csc = cu;
        int fu = 0, fd = 0, fsu = 0, fsd = 0;  // flat group / stage counters of unpack and drain
        int dj = 0;                            // group within the drain's stage
        bool dead = false;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; m++) acc[m] = 0.f;
        uint2 spre = make_uint2(0, 0);  // scales of the stage two ahead (4 x fp16)
        auto load_scales = [&](const Cursor &c) -> uint2 {
            uint2 v = make_uint2(0, 0);
            if (!c.valid) return v;
            const CDesc &d = p.d[c.pos.di];
            const int row = min(c.pos.tile * kRows + r, d.N - 1);
            const int g0 = (c.pos.s0 + c.stage) * kGPS;
            const unsigned short *sp = reinterpret_cast<const unsigned short *>(d.scales) + static_cast<size_t>(row) * d.G;
            unsigned short h[4];
#pragma unroll
            for (int j = 0; j < 4; j++) h[j] = (g0 + j < d.G) ? __ldg(sp + g0 + j) : static_cast<unsigned short>(0);
            v.x = h[0] | (static_cast<uint32_t>(h[1]) << 16);
            v.y = h[2] | (static_cast<uint32_t>(h[3]) << 16);
            return v;
        };
        auto put_scales = [&](int stage_idx, uint2 v) {
            uint2 *dst = reinterpret_cast<uint2 *>(&sm.sring[wg][stage_idx % kSRing][r][0]);
            *dst = v;
        };
        // prologue: stages 0 and 1 of scales into the ring, stage 2 in flight
        put_scales(0, load_scales(csc));
        csc.next_stage(p);
        put_scales(1, load_scales(csc));
        csc.next_stage(p);
        spre = load_scales(csc);
        csc.next_stage(p);

        auto drain_one = [&]() {
            const int db = fd % kRingD;
            bool ok = !dead;
            if (ok) ok = __all_sync(0xffffffffu, tc_wait(&sm.d_full[wg][db], (fd / kRingD) & 1, deadline));
            dead = !ok;
            uint32_t v[MT];
#pragma unroll
            for (int m = 0; m < MT; m++) v[m] = 0;
            if (ok) {
                tc_fence_after();
                tmem_ld<MT>(tmem + lane_base + 128 + db * kTok, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.d_empty[wg][db]);
                const float s = __half2float(__ushort_as_half(sm.sring[wg][fsd % kSRing][r][dj]));
#pragma unroll
                for (int m = 0; m < MT; m++) acc[m] = fmaf(s, __uint_as_float(v[m]), acc[m]);
            }
            fd++;
            if (++dj == kGPS) {
                dj = 0;
                fsd++;
                const int tile = cd.pos.tile, di = cd.pos.di, part = cd.pos.part;
                if (cd.next_stage(p)) {
                    // ---- end of an item: store, or hand the partial to the last arriver ----
                    const CDesc &d = p.d[di];
                    const int row = tile * kRows + r;
                    if (d.parts == 1) {
                        if (!dead && row < d.N) {
#pragma unroll
                            for (int m = 0; m < MT; m++)
                                if (m < M) d.y[static_cast<size_t>(m) * d.N + row] = __float2half_rn(acc[m]);
                        }
                    } else {
                        float *mine = p.partials + ((d.pslot + static_cast<long long>(tile) * d.parts + part) * kRows + r) * MT;
#pragma unroll
                        for (int m = 0; m < MT; m++) mine[m] = acc[m];
                        __threadfence();
                        named_bar_sync(1 + wg, 128);
                        if (r == 0) {
                            int last = 0;
                            if (!dead) {
                                const unsigned int old = atomicAdd(p.counters + d.tile_ws + tile, 1u);
                                last = (old == static_cast<unsigned int>(d.parts - 1));
                            }
                            sm.last_flag[wg] = last;
                        }
                        named_bar_sync(1 + wg, 128);
                        if (sm.last_flag[wg]) {
                            __threadfence();
                            float sum[MT];
#pragma unroll
                            for (int m = 0; m < MT; m++) sum[m] = 0.f;
                            const float *base = p.partials + ((d.pslot + static_cast<long long>(tile) * d.parts) * kRows + r) * MT;
                            for (int pp = 0; pp < d.parts; pp++) {
#pragma unroll
                                for (int m = 0; m < MT; m++) sum[m] += __ldcg(base + static_cast<long long>(pp) * kRows * MT + m);
                            }
                            if (row < d.N) {
#pragma unroll
                                for (int m = 0; m < MT; m++)
                                    if (m < M) d.y[static_cast<size_t>(m) * d.N + row] = __float2half_rn(sum[m]);
                            }
                            if (r == 0) p.counters[d.tile_ws + tile] = 0u;  // ready for the next call
                        }
                    }
#pragma unroll
                    for (int m = 0; m < MT; m++) acc[m] = 0.f;
                }
            }
        };

        while (cu.valid) {
            // ---- one slot stage: 4 scale groups ----
            const int slot = fsu % kSlotStages;
            put_scales(fsu + 2, spre);
            spre = load_scales(csc);
            csc.next_stage(p);
            bool ok = !dead;
            if (ok) ok = __all_sync(0xffffffffu, tc_wait(&sm.slot_full[wg][slot], (fsu / kSlotStages) & 1, deadline));
            dead = !ok;
            const uint8_t *rowp = &sm.slot[wg][slot][0] + r * 128;
            const int sw = r & 7;
#pragma unroll 1
            for (int j = 0; j < kGPS; j++) {
                if (!dead) {
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(rowp + (((2 * j) ^ sw) << 4));
                    const uint4 w1 = *reinterpret_cast<const uint4 *>(rowp + (((2 * j + 1) ^ sw) << 4));
                    if (j == kGPS - 1) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.slot_empty[wg][slot]);
                    }
                    uint32_t v[64];
                    unpack_word(w0.x, *reinterpret_cast<uint32_t(*)[8]>(&v[0]));
                    unpack_word(w0.y, *reinterpret_cast<uint32_t(*)[8]>(&v[8]));
                    unpack_word(w0.z, *reinterpret_cast<uint32_t(*)[8]>(&v[16]));
                    unpack_word(w0.w, *reinterpret_cast<uint32_t(*)[8]>(&v[24]));
                    unpack_word(w1.x, *reinterpret_cast<uint32_t(*)[8]>(&v[32]));
                    unpack_word(w1.y, *reinterpret_cast<uint32_t(*)[8]>(&v[40]));
                    unpack_word(w1.z, *reinterpret_cast<uint32_t(*)[8]>(&v[48]));
                    unpack_word(w1.w, *reinterpret_cast<uint32_t(*)[8]>(&v[56]));
                    const int ab = fu & 1;
                    ok = __all_sync(0xffffffffu, tc_wait(&sm.a_empty[wg][ab], ((fu >> 1) & 1) ^ 1, deadline));
                    dead = !ok;
                    if (ok) {
                        tc_fence_after();
                        tmem_st_x64(tmem + lane_base + ab * 64, v);
                        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.a_full[wg][ab]);
                    }
                }
                fu++;
                if (fu - fd > kLag) drain_one();
            }
            fsu++;
            cu.next_stage(p);
        }
        while (fd < fu) drain_one();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 10) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem_base), "r"(kTmemCols));
    }
}

bool g_attr_tc[64][4];

}  // namespace

struct Plan {
    int spp[kMaxDesc];
    int parts[kMaxDesc];
    int ntile[kMaxDesc];
    int total_items;
    long long partial_slots;
    int split_tiles;
};

static Plan make_plan(const MatDesc *md, int count, int wg_slots, bool allow_split) {
    // Choose the item size (a multiple of 4 groups) that balances best: the
    // makespan is ceil(items / warpgroups) items of roughly equal size.
    Plan best{};
    double best_cost = 1e300;
    const int cands[] = {4, 8, 12, 16, 24, 32, 48, 64, 1 << 20};
    for (int target : cands) {
        if (!allow_split && target != (1 << 20)) continue;
        Plan pl{};
        long long items = 0, work = 0, max_item = 0;
        for (int i = 0; i < count; i++) {
            const int G = md[i].K / kGroup;
            const int nst = (G + kGPS - 1) / kGPS;
            const int spp = std::min(nst, std::max(1, target / kGPS));
            pl.spp[i] = spp;
            pl.parts[i] = (nst + spp - 1) / spp;
            pl.ntile[i] = (md[i].N + kRows - 1) / kRows;
            items += static_cast<long long>(pl.ntile[i]) * pl.parts[i];
            work += static_cast<long long>(pl.ntile[i]) * nst;
            max_item = std::max<long long>(max_item, spp);
        }
        // makespan estimate in stages: rounds of the largest item, plus a
        // per-item overhead (pipeline ramp, reduction) of about one stage
        const long long rounds = (items + wg_slots - 1) / wg_slots;
        const double avg_item = static_cast<double>(work) / items;
        const double cost = rounds * (avg_item + 1.0) + (max_item - avg_item);
        if (cost < best_cost) {
            best_cost = cost;
            best = pl;
            best.total_items = static_cast<int>(std::min<long long>(items, 0x7fffffff));
        }
    }
    best.partial_slots = 0;
    best.split_tiles = 0;
    for (int i = 0; i < count; i++) {
        if (best.parts[i] > 1) {
            best.partial_slots += static_cast<long long>(best.ntile[i]) * best.parts[i];
            best.split_tiles += best.ntile[i];
        }
    }
    return best;
}

size_t gemv_tc_workspace_bytes(const MatDesc *md, int count, int M, int sms) {
    if (M < 1 || M > kMaxTcRows) return 0;
    const int MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
    const Plan pl = make_plan(md, count, sms * kWG, true);
    if (pl.split_tiles == 0 || pl.split_tiles > kMaxSplitTiles) return 0;
    return kCounterBytes + static_cast<size_t>(pl.partial_slots) * kRows * MT * sizeof(float);
}

tern_status launch_gemv_tc(const MatDesc *md, int count, int M, void *workspace, size_t ws_bytes,
                           cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    if (count < 1 || count > kMaxDesc) return fail(TERN_ERR_INVALID_ARG, "descriptor count %d", count);
    if (M < 1 || M > kMaxTcRows) return fail(TERN_ERR_SHAPE, "tensor-core bandwidth kernel takes 1..4 rows, got %d", M);
    const int MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
    auto kern = MT == 1 ? gemv_tc_kernel<1> : (MT == 2 ? gemv_tc_kernel<2> : gemv_tc_kernel<4>);
    const int mi = MT == 1 ? 0 : (MT == 2 ? 1 : 2);
    const size_t smem = sizeof(Smem) + 1024;
    if (smem > dev.max_smem_optin) return fail(TERN_ERR_DEVICE, "needs %zu B shared memory", smem);
    if (!g_attr_tc[dev.device][mi]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemv tc)");
        g_attr_tc[dev.device][mi] = true;
    }
    const int grid = dev.sms;  // one CTA per SM (it owns all 512 tensor-memory columns)
    const size_t need = gemv_tc_workspace_bytes(md, count, M, dev.sms);
    const bool split = workspace != nullptr && need > 0 && ws_bytes >= need;
    const Plan pl = make_plan(md, count, grid * kWG, split);

    CParams p;
    std::memset(&p, 0, sizeof(p));
    p.count = count;
    p.M = M;
    p.total_items = pl.total_items;
    p.wg_slots = grid * kWG;
    p.timeout_ns = g_gemm_timeout_ns;
    p.skip_loads = g_gemm_skip_loads;
    if (split && pl.split_tiles > 0) {
        p.counters = static_cast<unsigned int *>(workspace);
        p.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kCounterBytes);
    }
    int item = 0, tiles_ws = 0;
    long long pslot = 0;
    for (int i = 0; i < count; i++) {
        CDesc &g = p.d[i];
        st = encode_tiled_2d(&g.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots, static_cast<uint64_t>(md[i].K / 4),
                             static_cast<uint64_t>(md[i].N), static_cast<uint64_t>(md[i].K / 4), 128, kRows,
                             CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TERN_OK) return st;
        g.x = md[i].x;
        g.scales = md[i].scales;
        g.y = md[i].y;
        g.N = md[i].N;
        g.K = md[i].K;
        g.G = md[i].K / kGroup;
        g.ntile = pl.ntile[i];
        g.parts = pl.parts[i];
        g.spp = pl.spp[i];
        g.item_begin = item;
        g.tile_ws = tiles_ws;
        g.pslot = pslot;
        item += g.ntile * g.parts;
        if (g.parts > 1) {
            tiles_ws += g.ntile;
            pslot += static_cast<long long>(g.ntile) * g.parts;
        }
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_fail(e, "gemv tc kernel launch");
    return TERN_OK;
}

tern_status read_gemvtc_status(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_gemvtc_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_gemvtc_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    }
    *out = v;
    return TERN_OK;
}

}  // namespace tern

// ---------------------------------------------------------------------------
// Entry-point variant that allocates nothing: the M = 1 product of this
// kernel with its split-K scratch (arrival counters + partial sums) taken from
// a fixed area compiled into the library instead of a caller workspace.  It
// serves callers that may not allocate device memory on their own: code that
// runs while a CUDA graph is being captured into a pool the caller does not
// control, runtimes that forbid allocation after start-up (real-time or
// certified deployments), and plug-ins hosted by a framework that owns all
// device memory.  The area is shared by every call on a device, so calls that
// may overlap on the GPU (different streams, or graphs launched concurrently)
// race on it; callers must serialise them.
namespace tern {

// Largest scratch the no-allocation entry point can use, per device.  Every
// GPU that loads this library reserves it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64];
}  // namespace

tern_status gemv_noalloc(const MatDesc &d, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    // (current_device refuses ordinals outside [0, 64); checked again here,
    // where the per-device table is indexed)
    if (dev.device < 0 || dev.device >= 64) return fail(TERN_ERR_DEVICE, "device ordinal %d out of range", dev.device);
    void *scratch = nullptr;
    {
        // One-time set-up per device, with that device current: the host can
        // only use the symbol's device address, never the symbol itself.
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (g_noalloc_ptr[dev.device] == nullptr) {
            void *ptr = nullptr;
            cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
            g_noalloc_ptr[dev.device] = ptr;
        }
        scratch = g_noalloc_ptr[dev.device];
    }
    const size_t need = gemv_tc_workspace_bytes(&d, 1, 1, dev.sms);
    if (need > kNoAllocScratchBytes)
        return fail(TERN_ERR_WORKSPACE,
                    "N=%d K=%d needs %zu bytes of scratch; the no-allocation entry point has %zu", d.N, d.K, need,
                    kNoAllocScratchBytes);
    if (need == 0) return launch_gemv_tc(&d, 1, 1, nullptr, 0, stream);
    // The area keeps the previous call's contents: clear the arrival counters,
    // the only part that must start at zero (the partial sums are overwritten).
    cudaError_t e = cudaMemsetAsync(scratch, 0, kCounterBytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "clearing no-allocation scratch");
    return launch_gemv_tc(&d, 1, 1, scratch, kNoAllocScratchBytes, stream);
}

}  // namespace tern
