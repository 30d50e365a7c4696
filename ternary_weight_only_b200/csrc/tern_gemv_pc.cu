// Bandwidth-bound ternary-g128 product for M = 1..8 token rows: producer /
// consumer form of the TMA-staged mma.sync kernel, for K a multiple of 1024.
//
// What it computes: y[m][n] = sum_k x[m][k] * s[n][k/128] * t[n][k] with t
// read straight from the 2-bit slots and the group scale applied inside the
// product ("Ternary-Bonsai-27B" model summary, aitrends.kr, section
// "Technical features"); decode is bound by memory bandwidth ("Bonsai 27B
// ternary / 1-bit quantization", ThakiCloud blog, section "Throughput and
// speculative decoding").
//
// Arithmetic (mma.sync m16n8k16, weight rows as A, token rows as B, fp32
// accumulate, group scale applied in fp32) with a one-instruction unpack:
//  * A slot word holds 16 codes; its "pair j" is field j of both 16-bit halves
//    (weights j and j+8).  One AND with 0x00030003 << 2j' (j' = j for j < 5,
//    j - 5 on the word shifted right by 10 for j >= 5) leaves an fp16 pair
//    whose halves are the subnormals c * 4^j' * 2^-24: exact, no offset.
//  * Every mma takes pair j of the lane's four words, so one mma sees one
//    factor 4^j'.  The staged x carries the inverse: the B operand of pair j
//    is x * 2^(E - 2j'), an exact power-of-two scaling for E = min(8, 15 - e),
//    e the binary exponent of max|x| (no overflow; for max|x| < 256 nothing
//    is rounded).  Each product is then c * x * 2^(E-24), exact in fp32.
//  * t = c - 1, so a group's sum is D(codes) - D(all ones); D(all ones) is
//    computed per group and token once per CTA with the very same mma chain,
//    so an all-zero row of weights gives exactly 0.  The fp32 accumulator is
//    multiplied by 2^(24-E) at the end of a tile.
// One CTA per SM: twelve consumer warps and one producer warp (13 warps, at
// most four on a scheduler, so 128 registers a thread).  Each consumer owns a
// private ring of `ns` stages; a stage is one "slice" of 16 weight rows x
// 1024 k: two 128-byte-swizzled TMA boxes of slots (2 x 2 KB) and one TMA box
// of the matching 16 x 8 fp16 scales (256 B, which needs the scale rows to be
// a multiple of 16 bytes, i.e. K a multiple of 1024).  Lane c of the producer
// warp refills consumer c's ring as soon as a stage is free, polling with
// non-blocking waits, so no consumer waits for another.
#include <algorithm>
#include <cstring>

#include "tern_internal.cuh"
#include "tern_unpack_mma.cuh"

namespace tern {

// Device-side record of a bounded wait in this kernel that gave up.
__device__ unsigned int g_tern_gemvpc_status;

namespace {

// Consumer warps: twelve fed by one producer warp (token-per-column form), or
// sixteen that load their own rings (group-per-column form).
constexpr int kConsTok = 12, kConsGC = 16;
__host__ __device__ constexpr int ncons(bool gc) { return gc ? kConsGC : kConsTok; }
__host__ __device__ constexpr int nthreads(bool gc) { return gc ? kConsGC * 32 : (kConsTok + 1) * 32; }
constexpr int kRows = 16;                       // tile rows (mma M)
constexpr int kSG = 8;                          // scale groups per slice (1024 k)
constexpr int kBox = 128;                       // bytes per row of one slot box (4 groups)
constexpr int kSlotBytes = kRows * kBox * 2;    // 4 KB
constexpr int kScaleBytes = kRows * kSG * 2;    // 256 B
constexpr int kMaxNS = 4;                       // ring stages per consumer, at most
constexpr int kGroupK = 128;
__host__ __device__ constexpr int barbytes(bool gc) { return 2 * ncons(gc) * kMaxNS * 8; }
// partial tiles, two per consumer: float4 per lane, or (group-per-column form,
// after the sum over the four lanes of a row) float2 per mma row g
__host__ __device__ constexpr int recbytes(bool gc) { return gc ? ncons(gc) * 2 * 16 * 16 : ncons(gc) * 2 * 32 * 4 * 4; }
constexpr size_t kSmemBudget = 232448;          // opt-in shared memory per block on sm_100
constexpr int kMaxDesc = TERN_MAX_GROUP;

struct alignas(64) PDesc {
    CUtensorMap smap;   // slots as uint8 [K/512][N][128], box 128 B x 16 rows x 2, 128-byte swizzle
    CUtensorMap cmap;   // scales fp16 [N][K/128], box 8 x 16, no swizzle
    const __half *x;    // [M][K]
    __half *y;          // [M][N]
    int N, K, B;        // B = K / 1024 slices per row
    int ntile;          // ceil(N / 16)
    int c_begin, c_count;  // CTAs of this matrix
};

struct PParams {
    PDesc d[kMaxDesc];
    int count, M;
    unsigned int smem_usable;  // dynamic shared memory past the 1024-byte alignment
    int kmax;           // largest K of the launch (sizes the all-ones table)
    int xs_halves;
    int skip_loads;
    int pf;             // L2 prefetch distance in units (0: none)
    unsigned long long timeout_ns;
};

// Bytes before the staged x: barriers, partial tiles, tile ids, maxima, d1.
__host__ __device__ constexpr uint32_t fixed_bytes(int kmax, bool gc) {
    return barbytes(gc) + recbytes(gc) + 2 * ncons(gc) * 4 + 16 * 4 + (static_cast<uint32_t>(kmax / kGroupK) * 8 + 16) * 4;
}
// Dynamic shared memory for rings of ns stages beside xs_halves of staged x
// (+1024 for the alignment of the start).
size_t smem_bytes(int ns, int xs_halves, int kmax, bool gc) {
    const size_t ring_off = (fixed_bytes(kmax, gc) + static_cast<size_t>(xs_halves) * 2 + 1023) & ~size_t(1023);
    return 1024 + ring_off + static_cast<size_t>(ncons(gc)) * ns * (kSlotBytes + kScaleBytes);
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool pc_wait(uint64_t *bar, uint32_t parity, unsigned long long deadline) {
    while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
        if (globaltimer() > deadline) {
            atomicExch(&g_tern_gemvpc_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
            return false;
        }
    }
    return true;
}


// Work of warp w (consumer w, or producer lane w) of CTA lc of a matrix: the
// CTA owns tiles [t0, t1) (balanced to one tile), whose (tile, slice) units
// in tile-major order are split evenly over the consumer warps: units
// [u0, u1), unit u = slice u % B of tile t0 + u / B.
struct Range {
    int t0, u0, u1;
    __device__ void init(const PDesc &d, int lc, int w, int kCons) {
        t0 = static_cast<int>((static_cast<long long>(lc) * d.ntile) / d.c_count);
        const int t1 = static_cast<int>((static_cast<long long>(lc + 1) * d.ntile) / d.c_count);
        const int U = (t1 - t0) * d.B;
        u0 = (U * w) / kCons;
        u1 = (U * (w + 1)) / kCons;
    }
};

// GC (M = 1 only): the eight B columns carry the eight scale groups of a
// slice instead of eight token rows, so one set of B fragments serves all
// eight groups (see gc_note below).
template <int MT, bool GC>
__global__ void __launch_bounds__(nthreads(GC), 1) gemv_pc_kernel(const __grid_constant__ PParams p) {
    constexpr int kCons = ncons(GC);
    // Layout width of the staged x: token rows, or the eight groups of a slice.
    constexpr int XT = GC ? 8 : MT;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned start (offset arithmetic on the shared array keeps the
    // compiler's knowledge that every derived pointer is shared memory)
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int M = p.M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int di = 0;
#pragma unroll 1
    while (di + 1 < p.count && static_cast<int>(blockIdx.x) >= p.d[di + 1].c_begin) di++;
    const PDesc &d = p.d[di];
    const int lc = blockIdx.x - d.c_begin;
    const int B = d.B;

    uint64_t *full = reinterpret_cast<uint64_t *>(base);  // [kCons][kMaxNS]
    uint64_t *empty = full + kCons * kMaxNS;
    float *rec = reinterpret_cast<float *>(empty + kCons * kMaxNS);  // partial tiles (recbytes)
    int *rec_tile = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(rec) + recbytes(GC));  // [kCons][2]
    unsigned int *wmax = reinterpret_cast<unsigned int *>(rec_tile + 2 * kCons);  // [kCons]
    // [lane q][2 G + 4]: two floats per group, rows padded so that the four
    // lanes q of a quarter warp read distinct banks (group-per-column form:
    // one float per group)
    float *d1 = reinterpret_cast<float *>(wmax + 16);
    __half *xs = reinterpret_cast<__half *>(d1 + (p.kmax / kGroupK) * 8 + 16);
    // The rings take what is left after this CTA's own staged x (a grouped
    // launch is sized for its largest K; CTAs of smaller K get deeper rings).
    const uint32_t ring_off = (fixed_bytes(p.kmax, GC) + static_cast<uint32_t>(MT) * d.K * 2 + 1023u) & ~1023u;
    const int ns = min(kMaxNS, static_cast<int>((p.smem_usable - ring_off) / (kCons * (kSlotBytes + kScaleBytes))));
    uint8_t *slot_ring = base + ring_off;                        // [kCons][ns][4096], 1024-aligned boxes
    uint8_t *scale_ring = slot_ring + kCons * ns * kSlotBytes;   // [kCons][ns][256]

    if (threadIdx.x == 0) {
        for (int i = 0; i < kCons * kMaxNS; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const unsigned long long deadline = globaltimer() + p.timeout_ns;
    // Programmatic dependent launch: the next launch in the stream may start
    // its CTAs as SMs free up.  It prefetches only weights (which no GEMV
    // writes) before its grid-dependency wait, and reads x and writes y after.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kCons) {
        // ======================= producer warp =======================
        // Lane c (< kCons) feeds consumer warp c its units in order, one ring
        // stage each.
        Range r;
        int u = 0, s = 0, issued = 0;
        uint32_t ph = 0;
        bool done = true;
        // (the group-per-column form loads its own rings: nothing to do here)
        if (lane < kCons && !p.skip_loads && !GC) {
            r.init(d, lc, lane, kCons);
            u = r.u0;
            done = u >= r.u1;
        }
        uint8_t *my_slots = slot_ring + lane * ns * kSlotBytes;
        uint8_t *my_scales = scale_ring + lane * ns * kScaleBytes;
        uint64_t *my_full = full + lane * kMaxNS;
        uint64_t *my_empty = empty + lane * kMaxNS;
        // L2 prefetch `pf` units ahead of the ring (the ring itself covers the
        // next ns units): the later TMA loads then hit L2.
        auto prefetch = [&](int v) {
            const int tile = r.t0 + v / B;
            const int kbx = v - (v / B) * B;
            tma_prefetch_3d(&d.smap, 0, tile * kRows, kbx * 2);
            tma_prefetch_2d(&d.cmap, kbx * kSG, tile * kRows);
        };
        if (!done && p.pf > ns)
            for (int v = u + ns; v < r.u1 && v < u + p.pf; v++) prefetch(v);
        while (__any_sync(0xffffffffu, !done)) {
            bool progressed = false;
            if (!done) {
                if (mbar_test_wait(&my_empty[s], ph ^ 1)) {
                    const int tile = r.t0 + u / B;
                    const int kbx = u - (u / B) * B;
                    mbar_expect_tx(&my_full[s], kSlotBytes + kScaleBytes);
                    tma_load_3d(my_slots + s * kSlotBytes, &d.smap, 0, tile * kRows, kbx * 2, &my_full[s]);
                    tma_load_2d(my_scales + s * kScaleBytes, &d.cmap, kbx * kSG, tile * kRows, &my_full[s]);
                    if (p.pf > ns && u + p.pf < r.u1) prefetch(u + p.pf);
                    issued++;
                    if (++s == ns) {
                        s = 0;
                        ph ^= 1;
                    }
                    progressed = true;
                    done = ++u >= r.u1;
                } else if (globaltimer() > deadline) {
                    atomicExch(&g_tern_gemvpc_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
                    done = true;
                }
            }
            if (!__any_sync(0xffffffffu, progressed)) __nanosleep(128);
        }
        // The last min(ns, issued) stages are the only ones that can still be
        // in flight: they must land before the CTA exits, also when the
        // consumer gave up on them (bounded; normally already complete).
        const unsigned long long dl2 = globaltimer() + p.timeout_ns;
        for (int i = 0; i < ns && i < issued; i++) {
            const int uu = issued - 1 - i;
            pc_wait(&my_full[uu % ns], (uu / ns) & 1, dl2);
        }
    } else {
        // ======================= consumer warps =======================
        const int K = d.K, N = d.N;
        const int nthr = kCons * 32;
        Range r;
        r.init(d, lc, warp, kCons);
        uint8_t *my_slots = slot_ring + warp * ns * kSlotBytes;
        uint8_t *my_scales = scale_ring + warp * ns * kScaleBytes;
        uint64_t *my_full = full + warp * kMaxNS;
        uint64_t *my_empty = empty + warp * kMaxNS;
        // Group-per-column form: lane 0 loads the warp's own ring (unit v into
        // stage `st`); the first ns units go out before the grid-dependency
        // wait (weights are never written by a preceding launch).
        // (tile, slice) of the next unit to issue, advanced by increments
        int is_tile = r.t0 + r.u0 / B, is_kb = r.u0 - (r.u0 / B) * B;
        auto issue = [&](int st) {
            if (lane == 0) {
                mbar_expect_tx(&my_full[st], kSlotBytes + kScaleBytes);
                tma_load_3d(my_slots + st * kSlotBytes, &d.smap, 0, is_tile * kRows, is_kb * 2, &my_full[st]);
                tma_load_2d(my_scales + st * kScaleBytes, &d.cmap, is_kb * kSG, is_tile * kRows, &my_full[st]);
            }
            if (++is_kb == B) {
                is_kb = 0;
                is_tile++;
            }
        };
        int issued_end = r.u0;  // units [r.u0, issued_end) have been issued
        if (GC && !p.skip_loads) {
            issued_end = min(r.u0 + ns, r.u1);
            for (int v = r.u0; v < issued_end; v++) issue(v - r.u0);
        }
        // x may be the output of the preceding launch: wait for it to finish.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // (1) E from the largest finite |x| of all token rows.
        {
            unsigned int mx = 0;
            for (int idx = threadIdx.x; idx < M * K / 8; idx += nthr) {
                const uint4 v = *reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(idx) * 8);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; e++) mx = __vmaxu2(mx, __vminu2(wv[e] & 0x7FFF7FFFu, 0x7BFF7BFFu));
            }
            mx = max(mx & 0xFFFFu, mx >> 16);
            mx = __reduce_max_sync(0xffffffffu, mx);
            if (lane == 0) wmax[warp] = mx;
            if (lane < 2) rec_tile[warp * 2 + lane] = -1;
        }
        named_bar_sync(1, nthr);
        unsigned int mx = 0;
#pragma unroll
        for (int i = 0; i < kCons; i++) mx = max(mx, wmax[i]);
        // binary exponent of max|x| (subnormal and zero count as -14)
        const int ex = max(static_cast<int>(mx >> 10), 1) - 15;
        const int E = min(8, 15 - ex);
        // (2) stage x in pair order, pair j scaled by 2^(E - 2j').
        {
            // factor pairs for elements (2i, 2i+1) of an 8-element run: 2^(E - 2j'),
            // as fp16x2 (exact powers of two); the multiply rounds only subnormal results
            uint32_t fac2[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int e0 = E - 2 * (2 * i < 5 ? 2 * i : 2 * i - 5);
                const int e1 = E - 2 * (2 * i + 1 < 5 ? 2 * i + 1 : 2 * i + 1 - 5);
                fac2[i] = (static_cast<uint32_t>(15 + e0) << 10) | (static_cast<uint32_t>(15 + e1) << 26);
            }
            const int per_m = K / 8;
            // GC: MT token rows (M real, the rest zero) and 8 / MT groups per
            // set share the eight columns: column (G % GPB) * MT + m of set G / GPB
            constexpr int GPB = GC ? 8 / MT : 1;
            for (int idx = threadIdx.x; idx < (GC ? MT : M) * per_m; idx += nthr) {
                const int m = idx / per_m, c8 = idx - m * per_m;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (m < M) v = *reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(m) * K + c8 * 8);
                const uint32_t pr[4] = {v.x, v.y, v.z, v.w};
                const int kl = c8 * 8;
                const int gk = kl >> 7;
                const int di = GC ? xs_pair_index<8>((gk % GPB) * MT + m, ((gk / GPB) << 7) | (kl & 127))
                                  : xs_pair_index<MT>(m, kl);
                unsigned short *dst = reinterpret_cast<unsigned short *>(xs + di);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    uint32_t h2;
                    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(h2) : "r"(pr[i]), "r"(fac2[i]));
                    // element e = 2i + t lands at chunk e / 2 = i, slot t * 4
                    dst[i * XT * 32] = static_cast<unsigned short>(h2);
                    dst[i * XT * 32 + 4] = static_cast<unsigned short>(h2 >> 16);
                }
            }
        }
        named_bar_sync(1, nthr);
        const int g = lane >> 2, q = lane & 3;
        const int gx = g < M ? g : M - 1;
        const int G = K / kGroupK;
        constexpr int kGroupHalves = XT * 4 * 32;
        const __half *xlane = xs + ((GC ? g : gx) * 4 + q) * 8;
        // (3) the all-ones pass: D(ones) per group and B column (token).  GC:
        // one chain per slice gives all eight groups, column n = group n;
        // stored as d1[group].
        if (GC) {
            // one chain per set: d1[set * 8 + column]
            for (int sl = warp; sl < G * MT / kSG; sl += kCons) {
                float c[4];
                group_mma<8>(c, kOnes, kOnes, kOnes, kOnes, xlane + sl * kGroupHalves);
                if (g == 0) *reinterpret_cast<float2 *>(d1 + sl * kSG + 2 * q) = make_float2(c[0], c[1]);
            }
        } else {
            for (int grp = warp; grp < G; grp += kCons) {
                float c[4];
                group_mma<MT>(c, kOnes, kOnes, kOnes, kOnes, xlane + grp * kGroupHalves);
                if (g == 0) *reinterpret_cast<float2 *>(d1 + q * (2 * G + 4) + grp * 2) = make_float2(c[0], c[1]);
            }
        }
        named_bar_sync(1, nthr);

        const int row = tile_row(g);
        const float4 qm = make_float4(q == 0 ? 1.f : 0.f, q == 1 ? 1.f : 0.f, q == 2 ? 1.f : 0.f, q == 3 ? 1.f : 0.f);
        const float2 qh = make_float2(q < 2 ? 1.f : 0.f, q < 2 ? 0.f : 1.f);
        // Group-per-column form: lanes q < kGcLanes hold complete sums after
        // the tile's lane reduction; lane (g, q) stores v = (row g: tokens t0,
        // t1; row g+8: tokens t0, t1) with t0 = 2q, t1 = 2q + 1 (MT = 4),
        // t0 = 0, t1 = 1 (MT = 2) or only token 0 from v.x, v.z (MT = 1).
        constexpr int kGcLanes = MT == 4 ? 2 : 1;
        auto gc_store = [&](int tile, float4 v) {
            if (q >= kGcLanes) return;
            const int n0 = tile * kRows + row, n1 = n0 + 8;
            const int t0 = MT == 4 ? 2 * q : 0, t1 = t0 + 1;
            if (n0 < N) {
                if (t0 < M) d.y[static_cast<size_t>(t0) * N + n0] = __float2half_rn(v.x);
                if (MT > 1 && t1 < M) d.y[static_cast<size_t>(t1) * N + n0] = __float2half_rn(v.y);
            }
            if (n1 < N) {
                if (t0 < M) d.y[static_cast<size_t>(t0) * N + n1] = __float2half_rn(v.z);
                if (MT > 1 && t1 < M) d.y[static_cast<size_t>(t1) * N + n1] = __float2half_rn(v.w);
            }
        };
        uint32_t off[4];
#pragma unroll
        for (int j = 0; j < 4; j++) off[j] = row * kBox + (((2 * j + (q >> 1)) ^ (row & 7)) << 4) + (q & 1) * 8;
        const float *d1lane = d1 + q * (2 * G + 4);
        const float post = ldexpf(1.0f, 24 - E);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        int s = 0;
        uint32_t ph = 0;
        bool dead = false;
        int dead_u = r.u1, dead_s = 0;
        uint32_t dead_ph = 0;
        int tl = r.u0 / B;                 // tile (relative to t0) being accumulated
        int kb = r.u0 - tl * B;            // its next slice
        const int kb_first = kb;           // first slice of the first tile
        for (int u = r.u0; u < r.u1; u++) {
            bool ok = !dead;
            if (ok) ok = __all_sync(0xffffffffu, pc_wait(&my_full[s], ph, deadline));
            if (!ok && !dead) {
                dead_u = u;
                dead_s = s;
                dead_ph = ph;
            }
            dead = dead || !ok;
            if (ok && GC) {
                // gc_note: the slice's B fragments carry (group, token) pairs
                // (gcm_slice); weight group G runs its eight-mma chain into its
                // own accumulator, of which only its own columns are kept.
                const uint8_t *sl = my_slots + s * kSlotBytes;
                const uint8_t *scb = my_scales + s * kScaleBytes;
                // scales of the lane's groups (rows `row`, `row` + 8), read before
                // the stage is refilled: MT = 1 groups 2q, 2q+1; otherwise one
                // group per set h (4h + q, or 2h + q/2)
                __half2 sh[MT == 1 ? 2 : MT];
                if (MT == 1) {
                    sh[0] = *reinterpret_cast<const __half2 *>(scb + row * 16 + 4 * q);
                    sh[MT == 1 ? 1 : 0] = *reinterpret_cast<const __half2 *>(scb + (row + 8) * 16 + 4 * q);
                } else {
#pragma unroll
                    for (int h = 0; h < MT; h++) {
                        const int grp = MT == 2 ? 4 * h + q : 2 * h + (q >> 1);
                        sh[h] = __halves2half2(*reinterpret_cast<const __half *>(scb + row * 16 + 2 * grp),
                                               *reinterpret_cast<const __half *>(scb + (row + 8) * 16 + 2 * grp));
                    }
                }
                // All eight groups' words first, then the mmas field by field
                // (j outer, group inner): eight independent accumulation chains
                // between two dependent mmas.
                uint32_t wd[kSG][4];
#pragma unroll
                for (int G8 = 0; G8 < kSG; G8++) {
                    const uint8_t *bx = sl + (G8 >> 2) * (kRows * kBox);
                    const uint2 a = *reinterpret_cast<const uint2 *>(bx + off[G8 & 3]);
                    const uint2 b = *reinterpret_cast<const uint2 *>(bx + off[G8 & 3] + 8 * kBox);
                    wd[G8][0] = a.x;  // row g,   word 2q
                    wd[G8][1] = b.x;  // row g+8, word 2q
                    wd[G8][2] = a.y;  // row g,   word 2q+1
                    wd[G8][3] = b.y;  // row g+8, word 2q+1
                }
                // Everything this unit needs from the stage is in registers:
                // refill it now, so that the next load is in flight during the
                // mmas below (the warp barrier orders the reads before the
                // proxy fence and the copy that overwrites the stage).
                __syncwarp();
                if (issued_end < r.u1) {
                    if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    issue(s);
                    issued_end++;
                }
                float out[MT][4];
                gcm_slice<MT>(wd, xlane + kb * MT * kGroupHalves, qm, qh, out);
                // acc[0..1] = row g, columns 2q, 2q+1; acc[2..3] = row g+8
#pragma unroll
                for (int h = 0; h < MT; h++) {
                    const float2 on = *reinterpret_cast<const float2 *>(d1 + (kb * MT + h) * kSG + 2 * q);
                    float sa0, sa1, sb0, sb1;
                    if (MT == 1) {
                        const float2 fa = __half22float2(sh[0]), fb = __half22float2(sh[MT == 1 ? 1 : 0]);
                        sa0 = fa.x; sa1 = fa.y; sb0 = fb.x; sb1 = fb.y;
                    } else {
                        const float2 f = __half22float2(sh[h]);
                        sa0 = sa1 = f.x;
                        sb0 = sb1 = f.y;
                    }
                    acc[0] = fmaf(sa0, out[h][0] - on.x, acc[0]);
                    acc[1] = fmaf(sa1, out[h][1] - on.y, acc[1]);
                    acc[2] = fmaf(sb0, out[h][2] - on.x, acc[2]);
                    acc[3] = fmaf(sb1, out[h][3] - on.y, acc[3]);
                }
            } else if (ok) {
                const uint8_t *sl = my_slots + s * kSlotBytes;
                const uint8_t *scb = my_scales + s * kScaleBytes;
                const int grp0 = kb * kSG;
                const __half *xg = xlane + grp0 * kGroupHalves;
                const float *dg = d1lane + grp0 * 2;
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    // four groups of one 512-k box: their scales (rows row, row+8)
                    // and all-ones sums come in with four vector loads
                    const uint2 sa4 = *reinterpret_cast<const uint2 *>(scb + row * 16 + h * 8);
                    const uint2 sb4 = *reinterpret_cast<const uint2 *>(scb + (row + 8) * 16 + h * 8);
                    const float4 o01 = *reinterpret_cast<const float4 *>(dg + h * 8);
                    const float4 o23 = *reinterpret_cast<const float4 *>(dg + h * 8 + 4);
                    const uint8_t *bx = sl + h * (kRows * kBox);
                    const __half *xh = xg + h * 4 * kGroupHalves;
                    const float ox[4] = {o01.x, o01.z, o23.x, o23.z};
                    const float oy[4] = {o01.y, o01.w, o23.y, o23.w};
                    const uint32_t sav[2] = {sa4.x, sa4.y}, sbv[2] = {sb4.x, sb4.y};
#pragma unroll
                    for (int jj = 0; jj < 4; jj++) {
                        const uint2 a = *reinterpret_cast<const uint2 *>(bx + off[jj]);
                        const uint2 b = *reinterpret_cast<const uint2 *>(bx + off[jj] + 8 * kBox);
                        float c[4];
                        group_mma<MT>(c, a.x, a.y, b.x, b.y, xh + jj * kGroupHalves);
                        const uint32_t wa = sav[jj >> 1], wb = sbv[jj >> 1];
                        const float sa = __half2float(__ushort_as_half(static_cast<unsigned short>((jj & 1) ? (wa >> 16) : wa)));
                        const float sb = __half2float(__ushort_as_half(static_cast<unsigned short>((jj & 1) ? (wb >> 16) : wb)));
                        acc[0] = fmaf(sa, c[0] - ox[jj], acc[0]);
                        acc[1] = fmaf(sa, c[1] - oy[jj], acc[1]);
                        acc[2] = fmaf(sb, c[2] - ox[jj], acc[2]);
                        acc[3] = fmaf(sb, c[3] - oy[jj], acc[3]);
                    }
                }
            }
            // Release the stage (the group-per-column form released it above).
            // A warp that gave up a wait stops arriving, so its producer lane
            // gives up too.
            if (!(GC && ok)) {
                __syncwarp();
                if (lane == 0 && !dead) mbar_arrive(&my_empty[s]);
            }
            if (++s == ns) {
                s = 0;
                ph ^= 1;
            }
            ++kb;
            if (kb == B || u + 1 == r.u1) {
                // ---- this warp's part of a tile is complete ----
                const int tile = r.t0 + tl;
                const bool whole = kb == B && (tl != r.u0 / B || kb_first == 0);
                if (GC) {
                    // sum the lanes q that hold other groups of the same tokens
                    // (all four for MT <= 2, the pair q, q ^ 2 for MT = 4)
                    if (MT == 1) {
                        acc[0] += acc[1];
                        acc[2] += acc[3];
                        acc[1] = acc[3] = 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        if (MT <= 2) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 1);
                        acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 2);
                    }
                }
                const float v0 = acc[0] * post, v1 = acc[1] * post, v2 = acc[2] * post, v3 = acc[3] * post;
                if (GC) {
                    if (whole) {
                        if (!dead) gc_store(tile, make_float4(v0, v1, v2, v3));
                    } else {
                        const int slot = (tl == r.u0 / B) ? 0 : 1;
                        if (q < kGcLanes)
                            *reinterpret_cast<float4 *>(rec + (((warp * 2 + slot) * 8 + g) * 2 + q) * 4) =
                                make_float4(v0, v1, v2, v3);
                        if (lane == 0) rec_tile[warp * 2 + slot] = dead ? -2 : tile;
                    }
                } else if (whole) {
                    if (!dead) {
                        const int n0 = tile * kRows + row, n1 = n0 + 8;
                        const int m0 = 2 * q, m1 = 2 * q + 1;
                        if (m0 < M) {
                            if (n0 < N) d.y[static_cast<size_t>(m0) * N + n0] = __float2half_rn(v0);
                            if (n1 < N) d.y[static_cast<size_t>(m0) * N + n1] = __float2half_rn(v2);
                        }
                        if (m1 < M) {
                            if (n0 < N) d.y[static_cast<size_t>(m1) * N + n0] = __float2half_rn(v1);
                            if (n1 < N) d.y[static_cast<size_t>(m1) * N + n1] = __float2half_rn(v3);
                        }
                    }
                } else {
                    // A tile shared with neighbouring warps: keep the partial
                    // (slot 0 = the range's first tile, slot 1 = its last).
                    const int slot = (tl == r.u0 / B) ? 0 : 1;
                    *reinterpret_cast<float4 *>(rec + ((warp * 2 + slot) * 32 + lane) * 4) = make_float4(v0, v1, v2, v3);
                    if (lane == 0) rec_tile[warp * 2 + slot] = dead ? -2 : tile;
                }
                acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                kb = 0;
                tl++;
            }
        }
        // A warp that gave up may still have copies of its own in flight
        // (group-per-column form): they must land before the CTA exits.
        if (GC && dead) {
            const unsigned long long dl2 = globaltimer() + p.timeout_ns;
            int st = dead_s;
            uint32_t phs = dead_ph;
            for (int v = dead_u; v < issued_end; v++) {
                pc_wait(&my_full[st], phs, dl2);
                if (++st == ns) {
                    st = 0;
                    phs ^= 1;
                }
            }
        }
        // ---- tiles split over several warps: summed in warp order by the
        // first warp that holds a part ----
        named_bar_sync(1, nthr);
#pragma unroll 1
        for (int slot = 0; slot < 2; slot++) {
            const int tile = rec_tile[warp * 2 + slot];
            if (tile < 0) continue;
            bool owner = true;
            for (int w2 = 0; w2 < warp; w2++)
                if (rec_tile[w2 * 2] == tile || rec_tile[w2 * 2 + 1] == tile) owner = false;
            if (!owner) continue;
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            bool bad = false;
            for (int w2 = warp; w2 < kCons; w2++) {
                for (int s2 = 0; s2 < 2; s2++) {
                    if (rec_tile[w2 * 2 + s2] != tile) continue;
                    if (GC) {
                        if (q < kGcLanes) {
                            const float4 o = *reinterpret_cast<const float4 *>(rec + (((w2 * 2 + s2) * 8 + g) * 2 + q) * 4);
                            sum.x += o.x; sum.y += o.y; sum.z += o.z; sum.w += o.w;
                        }
                    } else {
                        const float4 o = *reinterpret_cast<const float4 *>(rec + ((w2 * 2 + s2) * 32 + lane) * 4);
                        sum.x += o.x; sum.y += o.y; sum.z += o.z; sum.w += o.w;
                    }
                }
            }
            // a part that gave up is marked -2; then the tile is not stored
            for (int w2 = 0; w2 < kCons; w2++)
                if (rec_tile[w2 * 2] == -2 || rec_tile[w2 * 2 + 1] == -2) bad = true;
            if (bad) continue;
            if (GC) {
                gc_store(tile, sum);
                continue;
            }
            const int n0 = tile * kRows + row, n1 = n0 + 8;
            const int m0 = 2 * q, m1 = 2 * q + 1;
            if (m0 < M) {
                if (n0 < N) d.y[static_cast<size_t>(m0) * N + n0] = __float2half_rn(sum.x);
                if (n1 < N) d.y[static_cast<size_t>(m0) * N + n1] = __float2half_rn(sum.z);
            }
            if (m1 < M) {
                if (n0 < N) d.y[static_cast<size_t>(m1) * N + n0] = __float2half_rn(sum.y);
                if (n1 < N) d.y[static_cast<size_t>(m1) * N + n1] = __float2half_rn(sum.w);
            }
        }
    }
}

bool g_attr_pc[64][7];
int g_occ_pc[64][7];

int pc_mt(int M) { return M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : 8)); }

// Kernel instance for M token rows: M <= 4 takes the group-per-column form
// (M = 3 padded to 4) unless `token_columns` asks for the token-per-column
// form; M = 5..8 always take the latter.
using PcKernel = void (*)(PParams);
PcKernel pc_kernel(int M, bool token_columns, int *index, bool *gc) {
    const int MT = pc_mt(M);
    *gc = MT <= 4 && !token_columns;
    if (*gc) {
        *index = MT == 1 ? 4 : (MT == 2 ? 5 : 6);
        return MT == 1 ? gemv_pc_kernel<1, true> : (MT == 2 ? gemv_pc_kernel<2, true> : gemv_pc_kernel<4, true>);
    }
    *index = MT == 1 ? 0 : (MT == 2 ? 1 : (MT == 4 ? 2 : 3));
    return MT == 1 ? gemv_pc_kernel<1, false>
                   : (MT == 2 ? gemv_pc_kernel<2, false> : (MT == 4 ? gemv_pc_kernel<4, false> : gemv_pc_kernel<8, false>));
}

}  // namespace

bool gemv_pc_supports(const MatDesc *md, int count, int M, bool token_columns) {
    if (M < 1 || M > 8) return false;
    int kmax = 0;
    for (int i = 0; i < count; i++) {
        if (md[i].K % 1024 != 0) return false;
        kmax = std::max(kmax, md[i].K);
    }
    // x is staged whole per CTA; at least two ring stages must fit beside it.
    const bool gc = pc_mt(M) <= 4 && !token_columns;
    // (the group-per-column form refills a stage as soon as it is read, so
    // one stage per warp still overlaps loads with the mmas)
    return smem_bytes(gc ? 1 : 2, pc_mt(M) * kmax, kmax, gc) <= kSmemBudget;
}

tern_status launch_gemv_pc(const MatDesc *md, int count, int M, bool token_columns, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    if (count < 1 || count > kMaxDesc) return fail(TERN_ERR_INVALID_ARG, "descriptor count %d", count);
    if (!gemv_pc_supports(md, count, M, token_columns))
        return fail(TERN_ERR_SHAPE, "producer/consumer kernel: unsupported shape");
    const int MT = pc_mt(M);
    int mi = 0;
    bool gc = false;
    const PcKernel kern = pc_kernel(M, token_columns, &mi, &gc);
    int kmax = 0;
    for (int i = 0; i < count; i++) kmax = std::max(kmax, md[i].K);
    const int xs_halves = MT * kmax;
    const size_t budget = std::min<size_t>(kSmemBudget, dev.max_smem_optin);
    // The whole budget: every CTA sizes its rings (2..4 stages) from what its
    // own staged x leaves.
    const size_t smem = std::min(budget, smem_bytes(kMaxNS, MT * 1024, kmax, gc));
    const int ns_min = gc ? 1 : 2;
    if (smem_bytes(ns_min, xs_halves, kmax, gc) > smem)
        return fail(TERN_ERR_SHAPE, "needs %zu B of shared memory", smem_bytes(ns_min, xs_halves, kmax, gc));
    if (!g_attr_pc[dev.device][mi]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(dev.max_smem_optin));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemv pc)");
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nthreads(gc), static_cast<size_t>(kSmemBudget));
        if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
        if (occ < 1) return fail(TERN_ERR_SHAPE, "producer/consumer kernel does not fit on an SM");
        g_occ_pc[dev.device][mi] = occ;
        g_attr_pc[dev.device][mi] = true;
    }
    // One CTA per SM (a CTA holds most of the SM's shared memory).  Each
    // matrix gets CTAs in proportion to its slices: start from one each and
    // hand the rest, one at a time, to the matrix whose CTAs carry the most
    // (tiles per CTA, rounded up, x slices per tile); never more CTAs than tiles.
    long long cap = static_cast<long long>(dev.sms);
    if (g_opt.gemv_grid > 0) cap = std::min<long long>(cap, g_opt.gemv_grid);
    cap = std::max<long long>(cap, count);
    int ntile[kMaxDesc];
    long long cl[kMaxDesc];
    long long used = 0;
    for (int i = 0; i < count; i++) {
        ntile[i] = (md[i].N + kRows - 1) / kRows;
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
    // Then trim CTAs that do not lower their matrix's largest load.
    for (int i = 0; i < count; i++)
        while (cl[i] > 1 && load(i, cl[i] - 1) == load(i, cl[i])) cl[i]--;

    PParams p;
    std::memset(&p, 0, sizeof(p));
    p.count = count;
    p.M = M;
    p.smem_usable = static_cast<unsigned int>(smem - 1024);
    p.kmax = kmax;
    p.xs_halves = xs_halves;
    p.skip_loads = g_gemm_skip_loads;
    p.pf = g_opt.gemv_prefetch;
    p.timeout_ns = g_gemm_timeout_ns;
    int next = 0;
    for (int i = 0; i < count; i++) {
        PDesc &g = p.d[i];
        // The slot matrix seen as [K/512 chunks][N rows][128 bytes]: one copy
        // brings both 512-k boxes of a slice (chunk stride 128 B, row stride K/4 B).
        const uint64_t sdims[3] = {static_cast<uint64_t>(kBox), static_cast<uint64_t>(md[i].N),
                                   static_cast<uint64_t>(md[i].K / 512)};
        const uint64_t sstr[2] = {static_cast<uint64_t>(md[i].K / 4), static_cast<uint64_t>(kBox)};
        const uint32_t sbox[3] = {static_cast<uint32_t>(kBox), static_cast<uint32_t>(kRows), 2};
        st = encode_tiled_3d(&g.smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots, sdims, sstr, sbox,
                             CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TERN_OK) return st;
        const int G = md[i].K / kGroup;
        st = encode_tiled_2d(&g.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, md[i].scales, static_cast<uint64_t>(G),
                             static_cast<uint64_t>(md[i].N), static_cast<uint64_t>(G) * 2, kSG, kRows,
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
    cfg.blockDim = dim3(nthreads(gc));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_fail(e, "gemv pc kernel launch");
    return TERN_OK;
}

tern_status read_gemvpc_status(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_gemvpc_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_gemvpc_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    }
    *out = v;
    return TERN_OK;
}

}  // namespace tern
