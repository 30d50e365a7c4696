// Bandwidth-bound ternary-g128 product for M = 1..8 token rows, TMA-staged.
//
// What it computes: y[m][n] = sum_k x[m][k] * s[n][k/128] * t[n][k] with t
// read straight from the 2-bit slots and the group scale applied inside the
// product ("Ternary-Bonsai-27B" model summary, aitrends.kr, section
// "Technical features"); decode is bound by memory bandwidth ("Bonsai 27B
// ternary / 1-bit quantization", ThakiCloud blog, section "Throughput and
// speculative decoding"), so the kernel is built around the weight stream.
//
// Design (B200, sm_100a):
//  * Work unit = a "slice": 16 weight rows x 512 k (4 scale groups) = 2 KB of
//    slots, one TMA box from a 2-D tensor map over the slot matrix, written
//    into shared memory with the 128-byte swizzle so that the lanes' 8-byte
//    fragment loads hit distinct banks.
//  * Every warp runs its own 3-stage ring of slices (lane 0 issues the TMA
//    loads and refills a stage as soon as the warp has read it), so an SM
//    with 2-3 CTAs keeps 96-144 KB of weight loads in flight without spending
//    registers on them; the per-row fp16 scales ride along in a
//    2-register-per-lane ring of plain loads issued three slices ahead.
//  * Unpack: one LOP3 + one HFMA2 per pair of weights gives exact fp16 t; the
//    multiply-accumulate runs on the tensor cores (mma.sync m16n8k16, fp32
//    accumulate) with the 16 weight rows as the A operand straight from
//    registers and the M <= 8 token rows as the B operand, staged once per CTA
//    in shared memory in the order the unpack produces (see xs_index).  Each
//    scale group's 16 x M partial is scaled by s in fp32.
//  * Partition: a tile (16 rows) is split along K between P warps of a CTA
//    (reduced through shared memory in a fixed order) and, when x would not
//    fit in shared memory, between the S CTAs of a thread-block cluster
//    (reduced through distributed shared memory in a fixed order).  The host
//    picks P and the CTA count of every matrix of a grouped call so that the
//    slowest CTA has the least work: results are deterministic and no global
//    scratch memory is used.
//  * Waits on the TMA barriers are bounded; a warp that gives up records
//    TERN_ERR_TIMEOUT, stops loading and computing but keeps taking part in
//    its CTA's barriers, and drains its own copies before exiting.
#include <algorithm>
#include <cstring>

#include "tern_internal.cuh"

namespace tern {

// Device-side record of a bounded wait in this kernel that gave up.
__device__ unsigned int g_tern_gemv_status;

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kNS = 3;             // stages per warp
constexpr int kSliceRows = 16;
constexpr int kSliceBytes = 128;   // per row: 512 weights
constexpr int kSliceGroups = 4;    // scale groups per slice
constexpr int kStageBytes = kSliceRows * kSliceBytes;  // 2 KB
constexpr int kMaxDesc = TERN_MAX_GROUP;

struct alignas(64) TDesc {
    CUtensorMap map;  // slots as uint8 [N][K/4], box 128 x 16, 128-byte swizzle
    const __half *x;
    const __half *scales;
    __half *y;
    int N, K, G, B;   // B = ceil(G / 4) slices along K
    int ntile;        // ceil(N / 16)
    int P;            // warps per tile (K split inside a CTA)
    int cl_begin;     // first cluster owned by this matrix
    int cl_count;     // clusters owned by this matrix
};

struct TParams {
    TDesc d[kMaxDesc];
    int count;
    int M;            // token rows, 1..8
    int S;            // CTAs per cluster (K split across CTAs)
    int xs_halves;    // capacity of the x staging area (halves)
    int skip_loads;   // test only: issue no loads (exercises the timeout path)
    unsigned long long timeout_ns;
};

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, unsigned long long deadline) {
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() > deadline) {
            atomicExch(&g_tern_gemv_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
            return false;
        }
    }
    return true;
}

// Tile row handled as mma row g (and g + 8): even rows for g < 4, odd rows for
// g >= 4.  With the 128-byte swizzle this makes the 16 lanes of each half-warp
// read 16 distinct 8-byte bank pairs (four rows 2 apart cover all eight swizzle
// phases of the two 16-byte chunks of a scale group).
__device__ __forceinline__ int tile_row(int g) { return g < 4 ? 2 * g : 2 * g - 7; }

// MINB = resident CTAs per SM the register budget is sized for (2 or 3).
template <int MT, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) gemv_tma_kernel(const __grid_constant__ TParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = smem;                                                   // [warp][stage] 2 KB each
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kWarps * kNS * kStageBytes);  // [warp][stage]
    __half *xs = reinterpret_cast<__half *>(full + kWarps * kNS);
    float *red = reinterpret_cast<float *>(xs + p.xs_halves);                // [2][warp][lane][4]
    float *cpart = red + 2 * kWarps * 32 * 4;                                 // [2][slot][lane][4]

    const int S = p.S, M = p.M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int row = tile_row(g);
    const int cl = blockIdx.x / S;
    const int rank = (S > 1) ? static_cast<int>(cluster_ctarank()) : 0;

    int di = 0;
#pragma unroll 1
    while (di + 1 < p.count && cl >= p.d[di + 1].cl_begin) di++;
    const TDesc &d = p.d[di];
    const int N = d.N, K = d.K, G = d.G;
    const int P = d.P;

    // K range of this CTA (whole slices), then of this warp.
    const int bA = (d.B * rank) / S, bB = (d.B * (rank + 1)) / S;
    const int nbc = bB - bA;
    const int spc = kWarps / P;  // tiles a CTA works on at once
    const int slot = warp / P, part = warp % P;
    const int b0 = bA + (nbc * part) / P, b1 = bA + (nbc * (part + 1)) / P;
    const int nb = b1 - b0;  // >= 1 (host guarantees P * S <= B)

    const int lc = cl - d.cl_begin;
    const int stride = d.cl_count * spc;
    const int tile0 = lc * spc + slot;
    const int lead = d.ntile - lc * spc;
    const int nit = lead > 0 ? (lead + stride - 1) / stride : 0;  // uniform in the CTA and the cluster
    const int total = nit * nb;

    uint64_t *wfull = full + warp * kNS;
    uint8_t *wst = stages + warp * kNS * kStageBytes;
    if (lane == 0) {
        for (int s = 0; s < kNS; s++) mbar_init(&wfull[s], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();

    // Issue stream: slice (is_it, is_b) goes next.  Lane 0 issues the TMA;
    // every lane loads its two scales of that slice (rows row and row + 8,
    // group q of the slice; 0 beyond K so that padded groups contribute 0).
    int is_it = 0, is_b = 0;
    uint32_t n_issued = 0;  // 8 bits per stage: loads issued into it (lane 0)
    const unsigned short *sc = reinterpret_cast<const unsigned short *>(d.scales);
    auto issue_next = [&](int stage, uint32_t &sa, uint32_t &sb) {
        const int tile = tile0 + is_it * stride;
        const bool ok = is_it < nit && tile < d.ntile;
        if (ok && lane == 0 && !p.skip_loads) {
            mbar_expect_tx(&wfull[stage], kStageBytes);
            tma_load_2d(wst + stage * kStageBytes, &d.map, (b0 + is_b) * kSliceBytes, tile * kSliceRows,
                        &wfull[stage]);
            n_issued += 1u << (8 * stage);
        }
        const int grp = (b0 + is_b) * kSliceGroups + q;
        sa = sb = 0;
        if (ok && grp < G) {
            const int r0 = min(tile * kSliceRows + row, N - 1);
            const int r1 = min(tile * kSliceRows + row + 8, N - 1);
            sa = __ldg(sc + static_cast<size_t>(r0) * G + grp);
            sb = __ldg(sc + static_cast<size_t>(r1) * G + grp);
        }
        if (++is_b == nb) {
            is_b = 0;
            is_it++;
        }
    };

    uint32_t sra[kNS], srb[kNS];
#pragma unroll
    for (int s = 0; s < kNS; s++) issue_next(s, sra[s], srb[s]);

    // Stage this CTA's K range of x in fragment order (overlaps the first
    // loads); groups past K are zero so that padded slices contribute 0.
    const int gA = bA * kSliceGroups;
    {
        const int gB = bB * kSliceGroups;
        const int per_m = (gB - gA) * (kGroup / 8);
        for (int idx = threadIdx.x; idx < M * per_m; idx += kThreads) {
            const int m = idx / per_m, c8 = idx - m * per_m;
            const int k = gA * kGroup + c8 * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (k < K) v = *reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(m) * K + k);
            const __half *hv = reinterpret_cast<const __half *>(&v);
#pragma unroll
            for (int e = 0; e < 8; e++) xs[xs_index(m, c8 * 8 + e, MT)] = hv[e];
        }
    }
    __syncthreads();

    // Per-lane swizzled byte offsets of its 8-byte fragment of group j (row
    // `row`; row + 8 is 1024 bytes further with the same swizzle phase).
    uint32_t off[kSliceGroups];
#pragma unroll
    for (int j = 0; j < kSliceGroups; j++)
        off[j] = row * kSliceBytes + (((2 * j + (q >> 1)) ^ (row & 7)) << 4) + (q & 1) * 8;

    // B column g holds token min(g, M-1): columns past M repeat the last token
    // (never stored), so every lane loads unconditionally.
    const int gx = g < M ? g : M - 1;
    const __half *xlane = xs + (gx * 4 + q) * 16;  // fragment of word 0, group 0
    constexpr int kGroupHalves = 2 * MT * 64;    // x halves per scale group
    constexpr int kWordHalves = MT * 64;         // word 1 of a group is this far
    const int shfl_base = lane & ~3;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int c_it = 0, c_b = 0, buf = 0;
    bool dead = false;  // this warp gave up a wait: no more loads, computes or stores
    const unsigned long long deadline = globaltimer() + p.timeout_ns;

#pragma unroll 1
    for (int fb = 0; fb < total; fb += kNS) {
#pragma unroll
        for (int u = 0; u < kNS; u++) {
            const int f = fb + u;
            if (f < total) {
                const int tile = tile0 + c_it * stride;
                const bool live = tile < d.ntile;
                if (live && !dead) {
                    dead = !__all_sync(0xffffffffu, wait_bounded(&wfull[u], (f / kNS) & 1, deadline));
                }
                if (live && !dead) {
                    const uint8_t *st = wst + u * kStageBytes;
                    const __half *xg = xlane + ((b0 + c_b) * kSliceGroups - gA) * kGroupHalves;
                    const float fa = __half2float(__ushort_as_half(static_cast<unsigned short>(sra[u])));
                    const float fb2 = __half2float(__ushort_as_half(static_cast<unsigned short>(srb[u])));
#pragma unroll
                    for (int j = 0; j < kSliceGroups; j++) {
                        const uint2 a = *reinterpret_cast<const uint2 *>(st + off[j]);
                        const uint2 b = *reinterpret_cast<const uint2 *>(st + off[j] + 1024);
                        const __half *xb = xg + j * kGroupHalves;
                        const uint4 x0 = *reinterpret_cast<const uint4 *>(xb);
                        const uint4 x1 = *reinterpret_cast<const uint4 *>(xb + 8);
                        const uint4 x2 = *reinterpret_cast<const uint4 *>(xb + kWordHalves);
                        const uint4 x3 = *reinterpret_cast<const uint4 *>(xb + kWordHalves + 8);
                        float c[4];
                        {
                            uint32_t ta[8], tb[8];
                            unpack_word(a.x, ta);
                            unpack_word(b.x, tb);
                            mma_16816_zc(c, ta[0], tb[0], ta[1], tb[1], x0.x, x0.y);
                            mma_16816(c, ta[2], tb[2], ta[3], tb[3], x0.z, x0.w);
                            mma_16816(c, ta[4], tb[4], ta[5], tb[5], x1.x, x1.y);
                            mma_16816(c, ta[6], tb[6], ta[7], tb[7], x1.z, x1.w);
                        }
                        {
                            uint32_t ta[8], tb[8];
                            unpack_word(a.y, ta);
                            unpack_word(b.y, tb);
                            mma_16816(c, ta[0], tb[0], ta[1], tb[1], x2.x, x2.y);
                            mma_16816(c, ta[2], tb[2], ta[3], tb[3], x2.z, x2.w);
                            mma_16816(c, ta[4], tb[4], ta[5], tb[5], x3.x, x3.y);
                            mma_16816(c, ta[6], tb[6], ta[7], tb[7], x3.z, x3.w);
                        }
                        const float sa = __shfl_sync(0xffffffffu, fa, shfl_base | j);
                        const float sb = __shfl_sync(0xffffffffu, fb2, shfl_base | j);
                        acc[0] = fmaf(sa, c[0], acc[0]);
                        acc[1] = fmaf(sa, c[1], acc[1]);
                        acc[2] = fmaf(sb, c[2], acc[2]);
                        acc[3] = fmaf(sb, c[3], acc[3]);
                    }
                }
                // Stage u is free again: refill it with the slice kNS ahead.
                __syncwarp();
                if (!dead) issue_next(u, sra[u], srb[u]);
                if (++c_b == nb) {
                    // ---- end of this warp's share of a tile: reduce and store ----
                    float v[4] = {acc[0], acc[1], acc[2], acc[3]};
                    bool writer = true;
                    if (P > 1 || S > 1) {
                        float *rb = red + ((buf * kWarps + warp) * 32 + lane) * 4;
                        *reinterpret_cast<float4 *>(rb) = make_float4(v[0], v[1], v[2], v[3]);
                        if (S > 1) __syncthreads();
                        else named_bar_sync(1 + slot, 32 * P);
                        writer = (part == 0);
                        if (writer) {
                            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                            for (int pp = 0; pp < P; pp++) {
                                const float4 o = *reinterpret_cast<const float4 *>(
                                    red + ((buf * kWarps + slot * P + pp) * 32 + lane) * 4);
                                sum.x += o.x; sum.y += o.y; sum.z += o.z; sum.w += o.w;
                            }
                            v[0] = sum.x; v[1] = sum.y; v[2] = sum.z; v[3] = sum.w;
                        }
                        if (S > 1) {
                            float *cp = cpart + ((buf * kWarps + slot) * 32 + lane) * 4;
                            if (writer) *reinterpret_cast<float4 *>(cp) = make_float4(v[0], v[1], v[2], v[3]);
                            cluster_sync_all();
                            writer = writer && rank == 0;
                            if (writer) {
                                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                                const uint32_t addr = smem_u32(cp);
                                for (int rr = 0; rr < S; rr++) {
                                    const float4 o = ld_shared_cluster_f4(mapa_shared(addr, rr));
                                    sum.x += o.x; sum.y += o.y; sum.z += o.z; sum.w += o.w;
                                }
                                v[0] = sum.x; v[1] = sum.y; v[2] = sum.z; v[3] = sum.w;
                            }
                        }
                        buf ^= 1;
                    }
                    if (writer && live && !dead) {
                        const int n0 = tile * kSliceRows + row, n1 = n0 + 8;
                        const int m0 = 2 * q, m1 = 2 * q + 1;
                        if (m0 < M) {
                            if (n0 < N) d.y[static_cast<size_t>(m0) * N + n0] = __float2half_rn(v[0]);
                            if (n1 < N) d.y[static_cast<size_t>(m0) * N + n1] = __float2half_rn(v[2]);
                        }
                        if (m1 < M) {
                            if (n0 < N) d.y[static_cast<size_t>(m1) * N + n0] = __float2half_rn(v[1]);
                            if (n1 < N) d.y[static_cast<size_t>(m1) * N + n1] = __float2half_rn(v[3]);
                        }
                    }
                    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                    c_b = 0;
                    c_it++;
                }
            }
        }
    }
    if (dead && lane == 0) {
        // Let this warp's copies in flight land before the CTA's memory is
        // released: wait (bounded) for the phase of the last load into each stage.
        const unsigned long long dl2 = globaltimer() + p.timeout_ns;
        for (int s = 0; s < kNS; s++) {
            const uint32_t n = (n_issued >> (8 * s)) & 0xFFu;
            if (n > 0) wait_bounded(&wfull[s], (n - 1) & 1, dl2);
        }
    }
    if (S > 1) cluster_sync_all();
}

bool g_attr_done[64][8];
int g_occ[64][8][256];

}  // namespace

namespace {
// Per-CTA work (slices per warp) with P warps per tile and c CTAs (clusters).
long long cta_work(int ntile, int nb_cta, int P, long long c, int warps) {
    const long long spc = warps / P;
    const long long rounds = (ntile + c * spc - 1) / (c * spc);
    return rounds * ((nb_cta + P - 1) / P);
}
}  // namespace

tern_status plan_partition(const int *ntile, const int *nbc, const int *nbmin, int count, int warps,
                           long long cap, int forced_P, int *Pout, long long *cl_out) {
    // For every matrix choose P (warps per 16-row tile, a divisor of `warps`) and its
    // CTA count so that the largest per-CTA work is as small as possible with
    // at most `cap` CTAs (clusters) in total: binary search on that bound, then
    // hand leftover CTAs to the matrices whose CTAs work longest.
    auto best_for = [&](int i, long long tau, int *Pc) -> long long {
        long long best = -1;
        for (int P = 1; P <= warps; P++) {
            if (warps % P != 0) continue;  // every slot of P warps is whole
            if (forced_P > 0 && P != forced_P) continue;
            if (P > nbmin[i]) continue;  // every warp's part keeps at least one slice
            const long long per_tile = (nbc[i] + P - 1) / P;
            if (per_tile > tau) continue;
            const long long rounds = tau / per_tile;
            const long long spc = warps / P;
            const long long c = (ntile[i] + rounds * spc - 1) / (rounds * spc);
            if (best < 0 || c < best || (c == best && P > *Pc)) {
                best = c;
                *Pc = P;
            }
        }
        return best;
    };
    long long lo = 1, hi = 1;
    for (int i = 0; i < count; i++) hi = std::max<long long>(hi, static_cast<long long>(ntile[i]) * nbc[i]);
    while (lo < hi) {
        const long long mid = (lo + hi) / 2;
        long long need = 0;
        bool ok = true;
        for (int i = 0; i < count && ok; i++) {
            int P = 1;
            const long long c = best_for(i, mid, &P);
            if (c < 0) ok = false;
            else need += c;
        }
        if (ok && need <= cap) hi = mid;
        else lo = mid + 1;
    }
    long long used = 0;
    for (int i = 0; i < count; i++) {
        int P = 1;
        const long long c = best_for(i, lo, &P);
        if (c < 0) return fail(TERN_ERR_SHAPE, "no valid k split for matrix %d", i);
        Pout[i] = P;
        cl_out[i] = c;
        used += c;
    }
    while (used < cap) {
        int worst = -1;
        long long wv = -1;
        for (int i = 0; i < count; i++) {
            const long long w = cta_work(ntile[i], nbc[i], Pout[i], cl_out[i], warps);
            const long long spc = warps / Pout[i];
            if (cl_out[i] * spc >= ntile[i]) continue;  // already one tile per slot
            if (w > wv) {
                wv = w;
                worst = i;
            }
        }
        if (worst < 0) break;
        const long long before = cta_work(ntile[worst], nbc[worst], Pout[worst], cl_out[worst], warps);
        const long long after = cta_work(ntile[worst], nbc[worst], Pout[worst], cl_out[worst] + 1, warps);
        if (after >= before) break;
        cl_out[worst]++;
        used++;
    }
    return TERN_OK;
}

tern_status launch_gemv_tma(const MatDesc *md, int count, int M, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    if (count < 1 || count > kMaxDesc) return fail(TERN_ERR_INVALID_ARG, "descriptor count %d", count);
    if (M < 1 || M > 8) return fail(TERN_ERR_SHAPE, "bandwidth kernel takes 1..8 rows, got %d", M);

    int bmin = 1 << 30, bmax = 0;
    for (int i = 0; i < count; i++) {
        const int B = (md[i].K / kGroup + kSliceGroups - 1) / kSliceGroups;
        bmin = std::min(bmin, B);
        bmax = std::max(bmax, B);
    }
    // Cluster split along K only when x would not fit next to the stages.
    int S = 1;
    const int MT = M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : 8));
    // Register budget: 2 CTAs per SM (128 registers) unless the knob asks for 3.
    const bool two = g_opt.gemv_ctas != 3;
    using KernFn = void (*)(TParams);
    KernFn kern;
    if (two) kern = MT == 1 ? gemv_tma_kernel<1, 2> : (MT == 2 ? gemv_tma_kernel<2, 2> : (MT == 4 ? gemv_tma_kernel<4, 2> : gemv_tma_kernel<8, 2>));
    else kern = MT == 1 ? gemv_tma_kernel<1, 3> : (MT == 2 ? gemv_tma_kernel<2, 3> : (MT == 4 ? gemv_tma_kernel<4, 3> : gemv_tma_kernel<8, 3>));
    auto xs_bytes = [&](int s) {
        return static_cast<long long>(MT) * ((bmax + s - 1) / s) * kSliceGroups * kGroup * 2;
    };
    while (S < 8 && S * 2 <= bmin && xs_bytes(S) > 96 * 1024) S *= 2;
    if (g_opt.gemv_cluster > 0) S = g_opt.gemv_cluster;
    if (S != 1 && S != 2 && S != 4 && S != 8) return fail(TERN_ERR_INVALID_ARG, "cluster size %d", S);
    if (S > bmin) return fail(TERN_ERR_SHAPE, "cluster size %d exceeds the %d k-slices of K", S, bmin);

    const int xs_halves = static_cast<int>(xs_bytes(S) / 2);
    const size_t smem = 1024 + static_cast<size_t>(kWarps) * kNS * kStageBytes + kWarps * kNS * 8 +
                        static_cast<size_t>(xs_halves) * 2 + 2 * kWarps * 32 * 4 * sizeof(float) +
                        (S > 1 ? 2 * kWarps * 32 * 4 * sizeof(float) : 0);
    if (smem > dev.max_smem_optin) return fail(TERN_ERR_SHAPE, "needs %zu B of shared memory", smem);
    const int mi = (MT == 1 ? 0 : (MT == 2 ? 1 : (MT == 4 ? 2 : 3))) + (two ? 4 : 0);
    if (!g_attr_done[dev.device][mi]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(dev.max_smem_optin));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        g_attr_done[dev.device][mi] = true;
    }
    const int skb = static_cast<int>((smem + 1023) / 1024);
    int occ = (skb < 256) ? g_occ[dev.device][mi][skb] : 0;
    if (occ == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, skb * 1024);
        if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
        if (skb < 256) g_occ[dev.device][mi][skb] = occ;
    }
    if (occ < 1) return fail(TERN_ERR_SHAPE, "kernel does not fit on an SM (smem %zu)", smem);
    if (g_opt.gemv_ctas > 0) occ = std::min(occ, g_opt.gemv_ctas);
    const long long cap = std::max<long long>(count, static_cast<long long>(dev.sms) * occ / S);

    int ntile[kMaxDesc], nbc[kMaxDesc], nbmin[kMaxDesc], Pch[kMaxDesc];
    long long cl_count[kMaxDesc];
    for (int i = 0; i < count; i++) {
        ntile[i] = (md[i].N + kSliceRows - 1) / kSliceRows;
        const int B = (md[i].K / kGroup + kSliceGroups - 1) / kSliceGroups;
        nbc[i] = (B + S - 1) / S;  // slices of the widest CTA range
        nbmin[i] = B / S;          // ... and of the narrowest
    }
    st = plan_partition(ntile, nbc, nbmin, count, kWarps, cap, g_opt.gemv_ksplit, Pch, cl_count);
    if (st != TERN_OK) return st;

    TParams p;  // copied into the launch by cudaLaunchKernelEx
    std::memset(&p, 0, sizeof(p));
    p.count = count;
    p.M = M;
    p.S = S;
    p.xs_halves = xs_halves;
    p.timeout_ns = g_gemm_timeout_ns;
    p.skip_loads = g_gemm_skip_loads;
    int next = 0;
    for (int i = 0; i < count; i++) {
        TDesc &g = p.d[i];
        st = encode_tiled_2d(&g.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots, static_cast<uint64_t>(md[i].K / 4),
                             static_cast<uint64_t>(md[i].N), static_cast<uint64_t>(md[i].K / 4), kSliceBytes,
                             kSliceRows, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != TERN_OK) return st;
        g.x = md[i].x;
        g.scales = md[i].scales;
        g.y = md[i].y;
        g.N = md[i].N;
        g.K = md[i].K;
        g.G = md[i].K / kGroup;
        g.B = (g.G + kSliceGroups - 1) / kSliceGroups;
        g.ntile = ntile[i];
        g.P = Pch[i];
        g.cl_begin = next;
        g.cl_count = static_cast<int>(cl_count[i]);
        next += g.cl_count;
    }
    const long long grid = static_cast<long long>(next) * S;
    if (grid > 0x7fffffffLL) return fail(TERN_ERR_SHAPE, "grid too large");

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (S > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_fail(e, "gemv kernel launch");
    return TERN_OK;
}

tern_status read_gemv_status(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_gemv_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_gemv_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    }
    *out = v;
    return TERN_OK;
}

}  // namespace tern
