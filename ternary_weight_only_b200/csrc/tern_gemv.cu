// Bandwidth-bound ternary-g128 product for M = 1..8 token rows.
//
// What it computes: y[m][n] = sum_k x[m][k] * s[n][k/128] * t[n][k] with
// t in {-1,0,+1} read straight from the 2-bit slots ("Ternary-Bonsai-27B"
// model summary, aitrends.kr, section "Technical features": the kernels
// consume the packed slots directly and apply the group scale inside the
// matmul; decode is bound by memory bandwidth: "Bonsai 27B ternary / 1-bit
// quantization", ThakiCloud blog, section "Throughput and speculative
// decoding").  The small-M case is the verify pass of speculative decoding
// (same section), which reads the weights once for all M rows.
//
// Design (B200, sm_100a):
//  * The weights are the only large stream (0.2656 B/weight).  Every lane
//    keeps kRing groups of its slot bytes in flight in a register ring
//    (8-byte loads, 4 lanes cover one 32-byte sector of a row), so one SM
//    holds ~48 KB of loads in flight without staging through shared memory.
//  * Unpacking costs two instructions per pair of weights: one LOP3 places
//    two 2-bit codes into the mantissas of an fp16 pair whose exponent makes
//    it 1024 + c*4^j, and one HFMA2 with constants (4^-j, -(1024*4^-j + 1))
//    turns that into t = c - 1 exactly (every intermediate is exact in fp16).
//  * The multiply-add runs on the tensor cores (mma.sync m16n8k16, fp32
//    accumulate): 16 weight rows form the A operand straight from registers,
//    the M <= 8 token rows form the B operand.  This is not for FLOPs -- the
//    B side is mostly empty at M = 1 -- but because the tensor pipe absorbs
//    the 16x8x16 multiply-adds in one instruction, which leaves the issue
//    slots for the unpack.  All products t*x are exact; one tile of 16
//    rows x 128 k (one scale group) is reduced inside the tensor core, then
//    scaled by s in fp32.
//  * The dot product does not care which k sits in which MMA slot, so each
//    lane feeds the codes in the order its LOP3 produces them (pairs k, k+8
//    of a 16-weight word) and x is staged once per CTA in shared memory in
//    that same order ("fragment order"), so each B fragment is one 128-bit
//    shared load with no bank conflicts.
//  * Long K is split between the warps of a CTA (KS) and, when x would not
//    fit in shared memory or the matrix has few rows, between the CTAs of a
//    thread-block cluster (S), reduced through distributed shared memory in
//    a fixed order: deterministic, no global scratch, no atomics.
#include <algorithm>
#include <cstring>

#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRing = 6;  // scale groups in flight per lane
constexpr int kMaxDesc = TERN_MAX_GROUP;

struct GDesc {
    const __half *x;
    const uint8_t *slots;
    const __half *scales;
    __half *y;
    int N, K, G;
    int ntile;     // ceil(N / 16)
    int cl_begin;  // first cluster owned by this matrix
    int cl_count;  // clusters owned by this matrix
};

struct GParams {
    GDesc d[kMaxDesc];
    int count;
    int M;          // token rows, 1..8
    int S;          // CTAs per cluster (split of K across CTAs)
    int KS;         // warps per tile inside a CTA (split of K across warps)
    int xs_halves;  // size of the x staging area
};

struct Item {
    uint2 a, b;          // slot bytes of rows g and g+8 for one scale group
    uint32_t sa, sb;     // their fp16 scales (low 16 bits)
};

__global__ void __launch_bounds__(kThreads, 2) gemv_mma_kernel(const __grid_constant__ GParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int S = p.S, KS = p.KS, M = p.M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int cl = blockIdx.x / S;
    const int rank = (S > 1) ? static_cast<int>(cluster_ctarank()) : 0;

    int di = 0;
#pragma unroll 1
    while (di + 1 < p.count && cl >= p.d[di + 1].cl_begin) di++;
    const GDesc &d = p.d[di];
    const int N = d.N, K = d.K, G = d.G;
    const int K4 = K >> 2;

    // K range of this CTA (whole scale groups), then of this warp.
    const int gA = (G * rank) / S, gB = (G * (rank + 1)) / S;
    const int ngc = gB - gA;
    const int spc = kWarps / KS;  // tiles a CTA works on at once
    const int slot = warp / KS, part = warp % KS;
    const int gp0 = gA + (ngc * part) / KS, gp1 = gA + (ngc * (part + 1)) / KS;
    const int ng = gp1 - gp0;  // >= 1 (host guarantees KS * S <= G)

    const int lc = cl - d.cl_begin;
    const int stride = d.cl_count * spc;
    const int tile0 = lc * spc + slot;
    const int lead = d.ntile - lc * spc;  // tiles left for slot 0 of this CTA
    const int nit = lead > 0 ? (lead + stride - 1) / stride : 0;  // uniform in the CTA
    const int total = nit * ng;

    __half *xs = reinterpret_cast<__half *>(smem);
    float *red = reinterpret_cast<float *>(smem + static_cast<size_t>(p.xs_halves) * 2);
    float *cpart = red + 2 * kWarps * 32 * 4;

    auto load_item = [&](int f, Item &it) {
        const int itn = f / ng;
        const int grp = gp0 + (f - itn * ng);
        const int tile = tile0 + itn * stride;
        if (f < total && tile < d.ntile) {
            const int r0 = min(tile * 16 + g, N - 1);
            const int r1 = min(tile * 16 + g + 8, N - 1);
            it.a = ldg_nc_u2(d.slots + static_cast<size_t>(r0) * K4 + grp * 32 + q * 8);
            it.b = ldg_nc_u2(d.slots + static_cast<size_t>(r1) * K4 + grp * 32 + q * 8);
            it.sa = __ldg(reinterpret_cast<const unsigned short *>(d.scales) +
                          static_cast<size_t>(r0) * G + grp);
            it.sb = __ldg(reinterpret_cast<const unsigned short *>(d.scales) +
                          static_cast<size_t>(r1) * G + grp);
        } else {
            it.a = make_uint2(0x55555555u, 0x55555555u);
            it.b = it.a;
            it.sa = it.sb = 0;
        }
    };

    // Put the first kRing groups of slot bytes in flight before staging x.
    Item ring[kRing];
#pragma unroll
    for (int u = 0; u < kRing; u++) load_item(u, ring[u]);

    // Stage this CTA's K range of x in fragment order.
    {
        const int KC = ngc * kGroup;
        const int per_m = KC / 8;
        for (int idx = threadIdx.x; idx < M * per_m; idx += kThreads) {
            const int m = idx / per_m, c8 = idx - m * per_m;
            const uint4 v = *reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(m) * K +
                                                             static_cast<size_t>(gA) * kGroup + c8 * 8);
            const __half *hv = reinterpret_cast<const __half *>(&v);
#pragma unroll
            for (int e = 0; e < 8; e++) xs[xs_index(m, c8 * 8 + e, M)] = hv[e];
        }
    }
    __syncthreads();

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int cgi = 0, cit = 0, buf = 0;
    const bool has_x = g < M;
    const int xw_stride = M * 64;  // halves between word 0 and word 1 of a group

#pragma unroll 1
    for (int fb = 0; fb < total; fb += kRing) {
#pragma unroll
        for (int u = 0; u < kRing; u++) {
            const int f = fb + u;
            if (f < total) {
                const Item it = ring[u];
                load_item(f + kRing, ring[u]);
                const int tile = tile0 + cit * stride;
                if (tile < d.ntile) {
                    const int grp_l = gp0 + cgi - gA;
                    const __half *xb = xs + ((grp_l * 2 * M + g) * 4 + q) * 16;
                    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0, x2 = x0, x3 = x0;
                    if (has_x) {
                        x0 = *reinterpret_cast<const uint4 *>(xb);
                        x1 = *reinterpret_cast<const uint4 *>(xb + 8);
                        x2 = *reinterpret_cast<const uint4 *>(xb + xw_stride);
                        x3 = *reinterpret_cast<const uint4 *>(xb + xw_stride + 8);
                    }
                    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
                    {
                        uint32_t ta[8], tb[8];
                        unpack_word(it.a.x, ta);
                        unpack_word(it.b.x, tb);
                        mma_16816(c0, ta[0], tb[0], ta[1], tb[1], x0.x, x0.y);
                        mma_16816(c0, ta[2], tb[2], ta[3], tb[3], x0.z, x0.w);
                        mma_16816(c0, ta[4], tb[4], ta[5], tb[5], x1.x, x1.y);
                        mma_16816(c0, ta[6], tb[6], ta[7], tb[7], x1.z, x1.w);
                    }
                    {
                        uint32_t ta[8], tb[8];
                        unpack_word(it.a.y, ta);
                        unpack_word(it.b.y, tb);
                        mma_16816(c1, ta[0], tb[0], ta[1], tb[1], x2.x, x2.y);
                        mma_16816(c1, ta[2], tb[2], ta[3], tb[3], x2.z, x2.w);
                        mma_16816(c1, ta[4], tb[4], ta[5], tb[5], x3.x, x3.y);
                        mma_16816(c1, ta[6], tb[6], ta[7], tb[7], x3.z, x3.w);
                    }
                    const float sa = __half2float(__ushort_as_half(static_cast<unsigned short>(it.sa)));
                    const float sb = __half2float(__ushort_as_half(static_cast<unsigned short>(it.sb)));
                    acc[0] = fmaf(sa, c0[0] + c1[0], acc[0]);
                    acc[1] = fmaf(sa, c0[1] + c1[1], acc[1]);
                    acc[2] = fmaf(sb, c0[2] + c1[2], acc[2]);
                    acc[3] = fmaf(sb, c0[3] + c1[3], acc[3]);
                }
                if (++cgi == ng) {
                    // ---- end of this warp's share of a tile: reduce and store ----
                    float v[4] = {acc[0], acc[1], acc[2], acc[3]};
                    bool writer = true;
                    if (KS > 1 || S > 1) {
                        float *rb = red + ((buf * kWarps + warp) * 32 + lane) * 4;
                        *reinterpret_cast<float4 *>(rb) = make_float4(v[0], v[1], v[2], v[3]);
                        __syncthreads();
                        writer = (part == 0);
                        if (writer) {
                            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                            for (int pp = 0; pp < KS; pp++) {
                                const float4 o = *reinterpret_cast<const float4 *>(
                                    red + ((buf * kWarps + slot * KS + pp) * 32 + lane) * 4);
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
                                const uint32_t a = smem_u32(cp);
                                for (int rr = 0; rr < S; rr++) {
                                    const float4 o = ld_shared_cluster_f4(mapa_shared(a, rr));
                                    sum.x += o.x; sum.y += o.y; sum.z += o.z; sum.w += o.w;
                                }
                                v[0] = sum.x; v[1] = sum.y; v[2] = sum.z; v[3] = sum.w;
                            }
                        }
                        buf ^= 1;
                    }
                    if (writer && tile < d.ntile) {
                        const int n0 = tile * 16 + g, n1 = n0 + 8;
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
                    cgi = 0;
                    cit++;
                }
            }
        }
    }
    // No CTA of a cluster may leave while another can still read its cpart.
    if (S > 1) cluster_sync_all();
}

bool g_attr_done[64];
int g_occ[64][256];

int pow2_at_least(double v, int lo, int hi) {
    int r = lo;
    while (r < hi && r < v) r *= 2;
    return r;
}

}  // namespace

tern_status launch_gemv_mma(const MatDesc *md, int count, int M, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    if (count < 1 || count > kMaxDesc) return fail(TERN_ERR_INVALID_ARG, "descriptor count %d", count);
    if (M < 1 || M > 8) return fail(TERN_ERR_SHAPE, "bandwidth kernel takes 1..8 rows, got %d", M);

    int gmin = 1 << 30, gmax = 0;
    long long tiles = 0;
    for (int i = 0; i < count; i++) {
        const int G = md[i].K / kGroup;
        gmin = std::min(gmin, G);
        gmax = std::max(gmax, G);
        tiles += (md[i].N + 15) / 16;
    }

    // Cluster split: keep the staged x slice within 96 KB so two CTAs fit per SM.
    int S = 1;
    while (S < 8 && S * 2 <= gmin &&
           static_cast<long long>(M) * ((gmax + S - 1) / S) * kGroup * 2 > 96 * 1024)
        S *= 2;
    if (g_opt.gemv_cluster > 0) S = g_opt.gemv_cluster;
    if (S != 1 && S != 2 && S != 4 && S != 8) return fail(TERN_ERR_INVALID_ARG, "cluster size %d", S);
    if (S > gmin) return fail(TERN_ERR_SHAPE, "cluster size %d exceeds K/128 = %d", S, gmin);

    const int xs_halves = M * ((gmax + S - 1) / S) * kGroup;
    const size_t smem = static_cast<size_t>(xs_halves) * 2 + 2 * kWarps * 32 * 4 * sizeof(float) +
                        (S > 1 ? 2 * kWarps * 32 * 4 * sizeof(float) : 0);
    if (smem > dev.max_smem_optin)
        return fail(TERN_ERR_SHAPE, "x slice needs %zu B of shared memory", smem);
    if (dev.device >= 0 && dev.device < 64 && !g_attr_done[dev.device]) {
        cudaError_t e = cudaFuncSetAttribute(gemv_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(dev.max_smem_optin));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        g_attr_done[dev.device] = true;
    }
    // Resident CTAs per SM for this shared-memory size (cached: the query is
    // not a stream operation, but caching keeps graph capture cheap).
    const int skb = static_cast<int>((smem + 1023) / 1024);
    int occ = (skb < 256) ? g_occ[dev.device][skb] : 0;
    cudaError_t e = cudaSuccess;
    if (occ == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_mma_kernel, kThreads, skb * 1024);
        if (e != cudaSuccess) return cuda_fail(e, "occupancy query");
        if (skb < 256) g_occ[dev.device][skb] = occ;
    }
    if (occ < 1) return fail(TERN_ERR_SHAPE, "kernel does not fit on an SM (smem %zu)", smem);
    if (g_opt.gemv_ctas > 0) occ = std::min(occ, g_opt.gemv_ctas);
    const long long cap_ctas = static_cast<long long>(dev.sms) * occ;

    // Warps sharing a tile along K: enough (tile, part) work items to fill the
    // resident warps about twice over.
    int KS = pow2_at_least(2.0 * cap_ctas * kWarps / (static_cast<double>(tiles) * S), 1, 8);
    while (KS > 1 && KS * S > gmin) KS /= 2;
    if (g_opt.gemv_ksplit > 0) KS = g_opt.gemv_ksplit;
    if (KS != 1 && KS != 2 && KS != 4 && KS != 8) return fail(TERN_ERR_INVALID_ARG, "k-split %d", KS);
    if (KS * S > gmin) return fail(TERN_ERR_SHAPE, "k-split %d x cluster %d exceeds K/128 = %d", KS, S, gmin);

    GParams p;
    std::memset(&p, 0, sizeof(p));
    p.count = count;
    p.M = M;
    p.S = S;
    p.KS = KS;
    p.xs_halves = xs_halves;
    const int spc = kWarps / KS;
    const long long cap_clusters = std::max<long long>(1, cap_ctas / S);
    long long want_total = 0;
    long long want[kMaxDesc];
    double work_total = 0;
    for (int i = 0; i < count; i++) {
        const int nt = (md[i].N + 15) / 16;
        want[i] = (nt + spc - 1) / spc;
        want_total += want[i];
        work_total += static_cast<double>(nt) * (md[i].K / kGroup);
    }
    int next = 0;
    for (int i = 0; i < count; i++) {
        const int nt = (md[i].N + 15) / 16;
        long long c = want[i];
        if (want_total > cap_clusters) {
            const double share = static_cast<double>(nt) * (md[i].K / kGroup) / work_total;
            c = std::max<long long>(1, std::min<long long>(want[i], static_cast<long long>(share * cap_clusters + 0.5)));
        }
        GDesc &g = p.d[i];
        g.x = md[i].x;
        g.slots = md[i].slots;
        g.scales = md[i].scales;
        g.y = md[i].y;
        g.N = md[i].N;
        g.K = md[i].K;
        g.G = md[i].K / kGroup;
        g.ntile = nt;
        g.cl_begin = next;
        g.cl_count = static_cast<int>(c);
        next += static_cast<int>(c);
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
    e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel, p);
    if (e != cudaSuccess) return cuda_fail(e, "gemv kernel launch");
    return TERN_OK;
}

}  // namespace tern
