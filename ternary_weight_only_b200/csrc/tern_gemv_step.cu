// One persistent launch for a whole decode step of M = 1 ternary-g128
// products: many independent matrices (every projection of every layer and
// the output head) streamed by all SMs as one flat list of weight tiles.
//
// What it computes: y_i[n] = sum_k x_i[k] * s_i[n][k/128] * t_i[n][k] for
// every matrix i, with t read straight from the 2-bit slots and the group
// scale applied inside the product ("Ternary-Bonsai-27B" model summary,
// aitrends.kr, section "Technical features").  Generation speed is set by the
// bytes read per token ("Bonsai 27B ternary / 1-bit quantization",
// ThakiCloud blog, section "Throughput and speculative decoding"): one launch
// for the step removes the per-launch start-up and drain of every SM, which
// per-matrix launches pay once per matrix.
//
// Work split: the tiles (16 weight rows) of all matrices, in order, form one
// list; the host cuts it into one contiguous range per CTA with equal
// numbers of 1024-k units (slices).  Inside a CTA each matrix's part is a
// "piece": its x is staged once (all warps), its units are split evenly over
// the sixteen warps, and tiles shared by two warps are summed in warp order
// after the piece (deterministic, no atomics, no scratch).
//
// Loads: every warp keeps its own ring of ns stages; a stage is one unit, two
// 128-byte-swizzled boxes of 16 slot rows x 128 bytes (one 3-D tensor copy)
// plus the 16 x 8 fp16 scales (one 2-D tensor copy), completing on the
// stage's mbarrier.  The tensor maps travel in the kernel parameters, which
// bounds one launch to kMaxPer matrices; the host splits longer lists into
// several launches.  The ring runs ahead across piece boundaries: weights
// never depend on the preceding launch or piece.
//
// Arithmetic: the group-per-column mma.sync form (tern_unpack_mma.cuh), or,
// at one to four token rows, the digit form below (all three storages).
//
// Digit form (X8): mma.sync m16n8k32 with unsigned 8-bit weights and signed
// 8-bit activations, exact 32-bit integer sums.  One AND of a slot word with
// 0x03030303 << 2f leaves four bytes c * 4^f (field f of each byte: weights
// 4b + f), so one instruction unpacks four weights and no shift is needed.
// The activations become integers on a fixed point per 128-k group and token
// row: X = rint(x * 2^(eC - 2f)) with eC = 29 - floor(log2 max|x|) of the
// group, so the field factor 4^f cancels and |X| < 2^30; X is split into
// four signed base-256 digits, and the eight mma columns carry (group or
// token, digit) pairs (four token rows: two column sets of two tokens, fed
// by the same unpacked weights).  Every X of an element within 2^13 of its group's
// largest |x| is exact; smaller ones are off by at most 2^-24 of that largest
// |x| (below the rounding of an fp32 sum).  A group's integer sums per digit
// are exact, t = c - 1 is restored by starting each chain at minus the same
// chain on the all-ones word, and the two digits a lane holds are joined as
// d0 + 256 d1 (no overflow: |d| < 2^21) before one conversion to fp32 and
// the multiply by the group scale and 2^(16 h - eC).
//
// The same kernel serves the 1-bit variant (weights in {-1, +1}, one bit
// each, fp16 scale per 128 weights: "Bonsai 27B ternary / 1-bit
// quantization", ThakiCloud blog, sections "What it is" and "How compression
// works"), template parameter F = 1: a stage's weights are one 128-byte-
// swizzled box of 16 rows x 128 bytes (1024 k), the unpack is b1_slice, and
// a group's sum is 2 D(bits) - D(all ones).
//
// F = 2 serves the five-per-byte packing (base-3 digits, 26 bytes per
// 128-weight group; tern.h): a stage is one box of 16 rows x 208 bytes (1024
// k, no swizzle), and every lane turns its bytes into the 2-bit codes of the
// ternary slot words in registers -- an 8-byte window per group and row (the
// lane's 32 weights start at byte 0, 6, 12 or 19 of the group, digit 0, 2, 4
// or 1), each byte through a 256-entry table of its five codes (replicated
// per lane so that the 32 lookups of a warp hit 32 distinct banks), the eight
// 10-bit results joined and shifted by the digit offset -- after which the
// ternary arithmetic runs unchanged.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "tern_internal.cuh"
#include "tern_unpack_mma.cuh"

namespace tern {

// Device-side record of a bounded wait in this kernel that gave up.
__device__ unsigned int g_tern_gemvstep_status;
// Failed in-kernel index checks (debug build; see TERN_GUARD).
__device__ unsigned int g_tern_gemvstep_guard;

namespace {

constexpr int kW = 16;                    // warps per CTA, all consumers
constexpr int kThreads = kW * 32;
constexpr int kRows = 16;                 // tile rows (mma M)
constexpr int kSG = 8;                    // scale groups per unit (1024 k)
constexpr int kBox = 128;                 // bytes per row of one slot box (512 k)
constexpr int kScaleStage = kRows * kSG * 2;           // 256
constexpr int kT5Row = 208;              // five-per-byte bytes of one row of a unit (8 x 26)
// weight bytes of one stage (16 rows x 1024 k): 2-bit slots (two boxes), bits, or base-3 bytes
__host__ __device__ constexpr int slot_stage(int f) {
    return f == 0 ? kRows * kBox * 2 : (f == 1 ? kRows * kBox : kRows * kT5Row);
}
// the five-per-byte code table: 256 entries x 32 lanes x 4 bytes
__host__ __device__ constexpr int lut_bytes(int f) { return f == 2 ? 256 * 32 * 4 : 0; }
__host__ __device__ constexpr int stage_bytes(int f) { return slot_stage(f) + kScaleStage; }
constexpr int kMaxNS = 4;
constexpr int kMaxCtas = 160;
constexpr int kMaxPer = 96;               // matrices per launch (parameter space)
constexpr size_t kSmemBudget = 232448;

struct SDesc {
    const __half *x;
    __half *y;
    int N, K;
    int tile0;   // first tile of this matrix in the flat tile list
    int ntile;   // ceil(N / 16)
    int xs;      // row stride of x (elements): K, or the full row of a K segment
    int accum;   // add the result to y (a K segment after the first) instead of writing it
};

struct alignas(64) SMaps {
    CUtensorMap smap;   // slots as uint8 [K/512][N][128], box 128 B x 16 rows x 2, 128-byte swizzle
                        // (1-bit: bits as uint8 [N][K/8], box 128 B x 16 rows, 128-byte swizzle;
                        //  five-per-byte: uint8 [N][R], box 208 B x 16 rows, no swizzle)
    CUtensorMap cmap;   // scales fp16 [N][K/128], box 8 x 16, no swizzle
};

struct SParams {
    SMaps m[kMaxPer];
    SDesc d[kMaxPer];
    int cta_tile[kMaxCtas + 1];   // flat tile range [cta_tile[c], cta_tile[c + 1]) of CTA c
    int count;
    int M;                        // token rows of every product (x [M][K], y [M][N])
    unsigned int smem_usable;     // dynamic shared memory past the 1024-byte alignment
    int kmax;
    int skip_loads;               // test only: issue no copies (exercises the timeout path)
    int first;                    // 1 for the first launch of a call, 0 for the later ones
    unsigned long long timeout_ns;
};

// Shared memory layout (bytes from the 128-aligned base).
__host__ __device__ constexpr int bar_off() { return 0; }
// Lanes of a quad that hold distinct tokens after a tile's lane reduction.
__host__ __device__ constexpr int gc_lanes(int mt) { return mt == 8 ? 4 : (mt == 4 ? 2 : 1); }
__host__ __device__ constexpr int rec_off() { return kW * kMaxNS * 8; }  // [kW][2][8][gc_lanes] float4
__host__ __device__ constexpr int rtile_off(int mt) { return rec_off() + kW * 2 * 8 * gc_lanes(mt) * 16; }  // [kW][2] int
__host__ __device__ constexpr int wmax_off(int mt) { return rtile_off(mt) + kW * 2 * 4; }  // [kW] uint
__host__ __device__ constexpr int d1_off(int mt) { return wmax_off(mt) + kW * 4; }
// d1 holds one float per (set, column): kmax / 1024 * mt sets of 8 columns.
// Digit form: one 16-byte record per (set, lane q) -- minus the all-ones sums
// of the lane's two columns and its factor 2^(16 (q & 1) - eC) -- for 4 (MT =
// 1) or 8 (MT = 2) sets per 1024 k, then the exponents eC per (token, group).
__host__ __device__ constexpr int d1_bytes(int kmax, int mt, bool x8) {
    return x8 ? kmax / 4 * mt + ((kmax / 128 * mt + 15) & ~15) : kmax / 32 * mt;
}
__host__ __device__ constexpr int lut_off(int kmax, int mt, bool x8) { return d1_off(mt) + d1_bytes(kmax, mt, x8) + 64; }
__host__ __device__ constexpr int xs_off(int kmax, int mt, int f, bool x8) { return lut_off(kmax, mt, x8) + lut_bytes(f); }
// staged x: MT token rows (M real, the rest zero); fp16 (2 bytes per k and
// row) or four signed digits (4 bytes per k and row)
__host__ __device__ constexpr int xs_bytes(int k, int mt, bool x8) { return k * (x8 ? 4 : 2) * mt; }
__host__ __device__ constexpr int ring_off(int kmax, int mt, int f, bool x8) {
    return (xs_off(kmax, mt, f, x8) + xs_bytes(kmax, mt, x8) + 1023) & ~1023;
}
size_t smem_bytes(int kmax, int mt, int ns, int f, bool x8) {
    return 1024 + static_cast<size_t>(ring_off(kmax, mt, f, x8)) + static_cast<size_t>(kW) * ns * stage_bytes(f);
}

// The 2-bit codes (c = digit, code i at bits 2i) of the five base-3 digits of
// byte v; an invalid byte (243..255) gives code 1 (t = 0) five times.
__device__ __forceinline__ uint32_t t5_codes(uint32_t v) {
    if (v >= 243u) return 0x155u;
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 5; i++) {
        out |= (v % 3u) << (2 * i);
        v /= 3u;
    }
    return out;
}

// Slot words 2q, 2q+1 (codes of the lane's 32 weights) from its 8-byte
// window at p (4-byte aligned, the window starting sh bits in), the table
// entries of this lane at lutl (entry v at lutl[32 v]) and the digit offset
// times two, dd.
__device__ __forceinline__ void t5_words(const uint8_t *p, uint32_t sh, const uint32_t *lutl, uint32_t dd,
                                         uint32_t &lo, uint32_t &hi) {
    const uint32_t w0 = *reinterpret_cast<const uint32_t *>(p);
    const uint32_t w1 = *reinterpret_cast<const uint32_t *>(p + 4);
    const uint32_t w2 = *reinterpret_cast<const uint32_t *>(p + 8);
    const uint32_t b03 = __funnelshift_r(w0, w1, sh), b47 = __funnelshift_r(w1, w2, sh);
    uint32_t l[8];
#pragma unroll
    for (int i = 0; i < 8; i++) l[i] = lutl[32u * __byte_perm(i < 4 ? b03 : b47, 0u, 0x4440u + (i & 3))];
    // the 80-bit string of the eight 10-bit code groups, as three words
    const uint32_t s0 = l[0] + (l[1] << 10) + (l[2] << 20) + (l[3] << 30);
    const uint32_t s1 = (l[3] >> 2) + (l[4] << 8) + (l[5] << 18) + (l[6] << 28);
    const uint32_t s2 = (l[6] >> 4) + (l[7] << 6);
    lo = __funnelshift_r(s0, s1, dd);
    hi = __funnelshift_r(s1, s2, dd);
}

// Digit form: the A registers of mma p of a group from the lane's words wg
// (2-bit slots: fields p of words 2q and 2q + 1 of rows g, g + 8, bytes c *
// 4^p; 1-bit: bits 2p and 2p + 1 of word q of rows g, g + 8, bytes b * 2^bit).
template <int F>
__device__ __forceinline__ void x8_a(const uint32_t *wg, int p, uint32_t &a0, uint32_t &a1, uint32_t &a2,
                                     uint32_t &a3) {
    if constexpr (F == 0) {
        const uint32_t mk = 0x03030303u << (2 * p);
        a0 = wg[0] & mk;
        a1 = wg[1] & mk;
        a2 = wg[2] & mk;
        a3 = wg[3] & mk;
    } else {
        const uint32_t m0 = 0x01010101u << (2 * p), m1 = m0 << 1;
        a0 = wg[0] & m0;
        a1 = wg[1] & m0;
        a2 = wg[0] & m1;
        a3 = wg[1] & m1;
    }
}

// The lane's two digit sums joined, t restored: 2-bit slots d0 + 256 d1
// (the chain started at minus the all-ones sums); 1-bit 2 (d0 + 256 d1) - oc
// with oc the all-ones sums joined the same way.
template <int F>
__device__ __forceinline__ int x8_join(int d0, int d1, int oc) {
    const int j = d0 + d1 * 256;
    return F == 0 ? j : 2 * j - oc;
}

__device__ __forceinline__ bool step_wait(uint64_t *bar, uint32_t parity, unsigned long long deadline) {
    while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
        if (globaltimer() > deadline) {
            atomicExch(&g_tern_gemvstep_status, static_cast<unsigned int>(TERN_ERR_TIMEOUT));
            return false;
        }
    }
    return true;
}

// A warp's position in its own sequence of units: piece = matrix i inside
// this CTA's tile range; the next unit is slice kb of tile `tile`
// (matrix-relative), `left` units of this warp's share remain.  Advanced by
// increments: no division per unit.
struct Cursor {
    int i;          // matrix, or -1 when the sequence is exhausted
    int tile, kb;   // next unit
    int B;          // units per tile (K / 1024)
    int left;       // units left in this piece
};

__device__ __forceinline__ void piece_range(const SDesc &d, int T0, int T1, int warp, int &tbeg, int &U, int &v0,
                                            int &v1) {
    tbeg = max(T0, d.tile0) - d.tile0;
    const int tend = min(T1, d.tile0 + d.ntile) - d.tile0;
    U = (tend - tbeg) * (d.K >> 10);
    v0 = static_cast<int>((static_cast<long long>(U) * warp) / kW);
    v1 = static_cast<int>((static_cast<long long>(U) * (warp + 1)) / kW);
}

// Enter matrix i's piece (and skip pieces where this warp has no unit).
__device__ __forceinline__ void cursor_enter(Cursor &c, const SParams &p, int i, int T0, int T1, int warp) {
    for (c.i = i;; c.i++) {
        if (c.i >= p.count || p.d[c.i].tile0 >= T1) {
            c.i = -1;
            return;
        }
        int tbeg, U, v0, v1;
        piece_range(p.d[c.i], T0, T1, warp, tbeg, U, v0, v1);
        if (v1 > v0) {
            c.B = p.d[c.i].K >> 10;
            c.tile = tbeg + v0 / c.B;
            c.kb = v0 - (v0 / c.B) * c.B;
            c.left = v1 - v0;
            return;
        }
    }
}

__device__ __forceinline__ void cursor_next(Cursor &c, const SParams &p, int T0, int T1, int warp) {
    if (--c.left == 0) {
        cursor_enter(c, p, c.i + 1, T0, T1, warp);
        return;
    }
    if (++c.kb == c.B) {
        c.kb = 0;
        c.tile++;
    }
}

// MT = token rows padded to 1, 2 or 4: the group-per-column form with
// (group, token) pairs in the mma columns (gcm_slice, or b1_slice for F = 1).
// MT = 8 (5..8 token rows; not for F = 1): the eight columns are the eight
// tokens of one group, so a slice is eight sets of one group, each group's
// eight-mma chain (group_mma) taken in turn, group by group.
// X8 (F = 0, MT = 1 or 2): the digit form; for MT = 1 set h of a 1024-k
// unit is groups h and h + 4 (columns 4 (G / 4) + digit), for MT = 2 a set
// is one group (columns 4 token + digit).
template <int MT, int F, bool X8>
__global__ void __launch_bounds__(kThreads, 1) gemv_step_kernel(const __grid_constant__ SParams p) {
    static_assert(!X8 || MT <= 4, "digit form: one to four token rows");
    // digit-form arithmetic: ternary codes (2-bit slots, and five-per-byte
    // bytes once decoded to slot words) or 1-bit weights
    constexpr int FA = F == 1 ? 1 : 0;
    constexpr int GPB = 8 / MT;  // groups per set
    // digit form: sets per 1024-k unit (MT = 4: two column sets per group,
    // tokens 0, 1 and 2, 3)
    constexpr int kSPU = MT == 1 ? 4 : (MT == 2 ? 8 : 16);
    constexpr int kSlotStage = slot_stage(F);
    constexpr int kStageBytes = stage_bytes(F);
    constexpr int kWords = F == 1 ? 2 : 4;  // weight words of a group a lane holds
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(base + bar_off());  // [kW][kMaxNS]
    float *rec = reinterpret_cast<float *>(base + rec_off());
    int *rec_tile = reinterpret_cast<int *>(base + rtile_off(MT));
    unsigned int *wmax = reinterpret_cast<unsigned int *>(base + wmax_off(MT));
    float *d1 = reinterpret_cast<float *>(base + d1_off(MT));
    __half *xs = reinterpret_cast<__half *>(base + xs_off(p.kmax, MT, F, X8));
    uint32_t *lut = reinterpret_cast<uint32_t *>(base + lut_off(p.kmax, MT, X8));
    // digit form: staged digits, (set, q) records, exponents per (token, group)
    uint8_t *xs8 = base + xs_off(p.kmax, MT, F, X8);
    int4 *recs = reinterpret_cast<int4 *>(d1);
    int8_t *egrp = reinterpret_cast<int8_t *>(base + d1_off(MT) + p.kmax / 4 * MT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int row = tile_row(g);
    const float4 qm = make_float4(q == 0 ? 1.f : 0.f, q == 1 ? 1.f : 0.f, q == 2 ? 1.f : 0.f, q == 3 ? 1.f : 0.f);
    const float2 qh = make_float2(q < 2 ? 1.f : 0.f, q < 2 ? 0.f : 1.f);
    // 128-byte-swizzled position of the lane's words of group G in `row`:
    // words 2q, 2q+1 of group G % 4 of box G / 4 (ternary), or word q of
    // group G (1-bit: 16 bytes per group row)
    uint32_t off[F == 1 ? 8 : 4];
    if constexpr (F == 0) {
#pragma unroll
        for (int j = 0; j < 4; j++) off[j] = row * kBox + (((2 * j + (q >> 1)) ^ (row & 7)) << 4) + (q & 1) * 8;
    } else if constexpr (F == 1) {
#pragma unroll
        for (int G8 = 0; G8 < 8; G8++) off[G8] = row * kBox + ((G8 ^ (row & 7)) << 4) + 4 * q;
    } else {
        // five-per-byte: the lane's window in group G of `row` starts at byte
        // 26 G + sq (sq = 0, 6, 12, 19) at digit 0, 2, 4, 1.  off[0] / off[1]:
        // 4-byte-aligned window offsets for even / odd G (add 52 (G / 2));
        // off[2] / off[3]: the matching shifts in bits.
        const int sq = q == 0 ? 0 : (q == 1 ? 6 : (q == 2 ? 12 : 19));
        off[0] = row * kT5Row + (sq & ~3);
        off[1] = row * kT5Row + 26 + sq - ((sq + 2) & 3);
        off[2] = (sq & 3) * 8;
        off[3] = ((sq + 2) & 3) * 8;
    }
    const uint32_t t5dd = 2u * (q == 0 ? 0u : (q == 1 ? 2u : (q == 2 ? 4u : 1u)));
    const uint32_t *lutl = lut + lane;
    const int T0 = p.cta_tile[blockIdx.x], T1 = p.cta_tile[blockIdx.x + 1];
    // first matrix with a tile at or after T0
    int i0 = 0;
    {
        int lo = 0, hi = p.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (p.d[mid].tile0 + p.d[mid].ntile <= T0) lo = mid + 1; else hi = mid;
        }
        i0 = lo;
    }
    // The ring takes what this CTA's largest staged x leaves (2..4 stages).
    int kcta = 1024;
    for (int i = i0; T0 < T1 && i < p.count && p.d[i].tile0 < T1; i++) kcta = max(kcta, p.d[i].K);
    const uint32_t roff =
        (static_cast<uint32_t>(xs_off(p.kmax, MT, F, X8)) + static_cast<uint32_t>(xs_bytes(kcta, MT, X8)) + 1023u) &
        ~1023u;
    const int ns = min(kMaxNS, static_cast<int>((p.smem_usable - roff) / (kW * kStageBytes)));
    const int M = p.M;
    uint8_t *ring = base + roff;

    // one barrier per thread of the first warps (the fence orders this
    // thread's initialisation before the copies that arrive on it)
    static_assert(kW * kMaxNS <= kThreads, "one thread per ring barrier");
    if (threadIdx.x < kW * kMaxNS) {
        mbar_init(&full[threadIdx.x], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if constexpr (F == 2) {
        for (int i = threadIdx.x; i < 256 * 32; i += kThreads) lut[i] = t5_codes(static_cast<uint32_t>(i >> 5));
    }
    __syncthreads();
    // Ordering between launches (programmatic dependent launch).  The inputs
    // of a call may come from the kernel before it, so its first launch waits
    // for that kernel before anything reads x, and only then lets the next
    // launch start.  The later launches of the same call read inputs that were
    // complete before the first launch went past its wait, so they start their
    // successors at once and do not wait before reading; they wait at the end
    // instead, so that every launch still completes after the one before it
    // (a kernel after the call that waits for its last launch sees all outputs).
    if (!p.first) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const unsigned long long deadline = globaltimer() + p.timeout_ns;
    uint64_t *my_full = full + warp * kMaxNS;
    // slot stages (4096 bytes, 1024-aligned: the 128-byte swizzle pattern is
    // tied to the address) for all warps first, then the 256-byte scale stages
    uint8_t *my_ring = ring + warp * ns * kSlotStage;
    uint8_t *my_scl = ring + kW * ns * kSlotStage + warp * ns * kScaleStage;

    // ---- issue side: this warp's units, in order, into its ring ----
    Cursor ic;
    ic.i = -1;
    if (T0 < T1 && !p.skip_loads) cursor_enter(ic, p, i0, T0, T1, warp);
    int issued = 0;
    // Lane 0 issues; all lanes keep the cursor (uniform).  Rows past N are
    // filled with zeros by the copy and never stored.
    auto issue = [&](int st) {
        if (lane == 0) {
            uint8_t *stage = my_ring + st * kSlotStage;
            mbar_expect_tx(&my_full[st], kStageBytes);
            if constexpr (F == 0)
                tma_load_3d(stage, &p.m[ic.i].smap, 0, ic.tile * kRows, ic.kb * 2, &my_full[st]);
            else if constexpr (F == 1)
                tma_load_2d(stage, &p.m[ic.i].smap, ic.kb * kBox, ic.tile * kRows, &my_full[st]);
            else
                tma_load_2d(stage, &p.m[ic.i].smap, ic.kb * kT5Row, ic.tile * kRows, &my_full[st]);
            tma_load_2d(my_scl + st * kScaleStage, &p.m[ic.i].cmap, ic.kb * kSG, ic.tile * kRows, &my_full[st]);
        }
        cursor_next(ic, p, T0, T1, warp);
        issued++;
    };
    // Only the first stage of every ring goes out before the first piece's
    // activations are staged: the staging's small loads of x would otherwise
    // queue in DRAM behind every SM's whole ring (~20 MB, ~3 us); one stage
    // per warp (~10 MB in flight) still covers the staging.  The other stages
    // follow right after it, before any stage is consumed and refilled, so
    // stage st still holds the warp's unit st.
    if (ns > 0 && ic.i >= 0) issue(0);
    bool topped = false;

    if (p.first) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }

    int s = 0;
    uint32_t ph = 0;
    int consumed = 0;
    bool dead = false;
    const int nthr = kThreads;
    for (int i = i0; T0 < T1 && i < p.count && p.d[i].tile0 < T1; i++) {
        const SDesc &d = p.d[i];
        const int K = d.K, N = d.N, B = K >> 10;
        // ---- stage x of matrix i: E from max |x|, pair order, all-ones sums ----
        __syncthreads();  // the previous piece is finished with xs, d1, rec
        const __half *xlane = xs + lane * 8;
        int E = 0;
        if constexpr (X8) {
            // ---- digit form.  Work item (token m, 32-k chunk, field half
            // fp): the 16 x of fields 2fp, 2fp + 1 (2-bit slots: k = 16 r +
            // 4 b + f) or of bits 4fp .. 4fp + 3 (1-bit: k = 8 i + bit) of
            // the chunk, each as four digits, written as one 16-byte B
            // fragment per digit.  The eight items of a 128-k group are eight
            // consecutive lanes.
            if (lane < 2) rec_tile[warp * 2 + lane] = -1;
            const int nit = K >> 4;  // a multiple of 64: every warp runs whole iterations
            for (int idx = threadIdx.x; idx < MT * nit; idx += nthr) {
                const int m = idx / nit, it = idx - m * nit;
                const int c32 = it >> 1, fp = it & 1, base = c32 << 5;
                uint32_t hv[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // element e = half (e & 1) of hv[e >> 1]
                if (m < M && TERN_GUARD(base + 32 <= K, g_tern_gemvstep_guard)) {
                    const __half *src = d.x + static_cast<size_t>(m) * d.xs + base;
                    if constexpr (FA == 0) {
                        uint4 v[4];
#pragma unroll
                        for (int j = 0; j < 4; j++) v[j] = *reinterpret_cast<const uint4 *>(src + 8 * j);
                        // hv[4 r + b] = the pair at k = 16 r + 4 b + 2 fp
#pragma unroll
                        for (int r = 0; r < 2; r++)
#pragma unroll
                            for (int b = 0; b < 4; b++) {
                                const uint4 &vv = v[(8 * r + 2 * b) >> 2];
                                hv[4 * r + b] = (b & 1) ? (fp ? vv.w : vv.z) : (fp ? vv.y : vv.x);
                            }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; i++) {
                            const uint2 v = *reinterpret_cast<const uint2 *>(src + 8 * i + 4 * fp);
                            hv[2 * i] = v.x;
                            hv[2 * i + 1] = v.y;
                        }
                    }
                }
                // largest |x| of the group (inf and NaN clamp to 65504)
                uint32_t mx = 0;
#pragma unroll
                for (int e = 0; e < 8; e++) mx = __vmaxu2(mx, __vminu2(hv[e] & 0x7FFF7FFFu, 0x7BFF7BFFu));
                mx = max(mx & 0xFFFFu, mx >> 16);
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                // eC = 29 - floor(log2 max|x|) (normal or subnormal max); 0 for an all-zero group
                int eC = 0;
                if (mx != 0) eC = 29 - (mx >= 0x400u ? static_cast<int>(mx >> 10) - 15 : (31 - __clz(mx)) - 24);
                const int e0 = 127 + eC - 4 * fp;  // biased exponent of 2^(eC - 4 fp)
                // w[s][j]: fragment word j of digit s.  The four x of one word
                // (2-bit slots: word (e & 1) * 2 + (e >> 3), byte (e >> 1) & 3;
                // 1-bit: word e & 3, byte e >> 2) are converted together: the
                // signed base-256 digits of X are the bytes of
                // (X + 0x80808080) ^ 0x80808080 (exact for |X| < 2^31 - 2^24), and a
                // 4 x 4 byte transpose puts digit s of the four x into word s.
                uint32_t w[4][4];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t D[4];
#pragma unroll
                    for (int b4 = 0; b4 < 4; b4++) {
                        // element e holding byte b4 of word j
                        const int e = FA == 0 ? (j >> 1) + ((j & 1) << 3) + (b4 << 1) : (b4 << 2) + j;
                        const int sh = FA == 0 ? 2 * (e & 1) : (e & 3);
                        const float xv =
                            __half2float(__ushort_as_half(static_cast<unsigned short>(hv[e >> 1] >> (16 * (e & 1)))));
                        const int X = __float2int_rn(xv * __int_as_float((e0 - sh) << 23));
                        D[b4] = (static_cast<uint32_t>(X) + 0x80808080u) ^ 0x80808080u;
                    }
                    const uint32_t t0 = __byte_perm(D[0], D[1], 0x5140), t1 = __byte_perm(D[0], D[1], 0x7362);
                    const uint32_t t2 = __byte_perm(D[2], D[3], 0x5140), t3 = __byte_perm(D[2], D[3], 0x7362);
                    w[0][j] = __byte_perm(t0, t2, 0x5410);
                    w[1][j] = __byte_perm(t0, t2, 0x7632);
                    w[2][j] = __byte_perm(t1, t3, 0x5410);
                    w[3][j] = __byte_perm(t1, t3, 0x7632);
                }
                const int u = base >> 10, G8 = (base >> 7) & 7, qq = (base >> 5) & 3;
                const int set = MT == 1 ? u * 4 + (G8 & 3) : (MT == 2 ? u * 8 + G8 : (u * 8 + G8) * 2 + (m >> 1));
                const int col0 = MT == 1 ? 4 * (G8 >> 2) : (MT == 2 ? 4 * m : 4 * (m & 1));
#pragma unroll
                for (int s2 = 0; s2 < 4; s2++) {
                    const int xo = ((set * 2 + fp) * 32 + 4 * (col0 + s2) + qq) << 4;
                    if (TERN_GUARD(xo + 16 <= xs_bytes(kcta, MT, X8), g_tern_gemvstep_guard))
                        *reinterpret_cast<uint4 *>(xs8 + xo) = make_uint4(w[s2][0], w[s2][1], w[s2][2], w[s2][3]);
                }
                const int eo = m * (K >> 7) + (base >> 7);
                if ((lane & 7) == 0 && TERN_GUARD(eo < MT * (p.kmax >> 7), g_tern_gemvstep_guard))
                    egrp[eo] = static_cast<int8_t>(eC);
            }
            __syncthreads();
            // one all-ones chain per set (A = weight code 1, or bit 1, in every
            // field), and the lane records: for 2-bit slots minus the sums of
            // columns 2q, 2q + 1 (the chains start there), for 1-bit weights
            // their sum O_2q + 256 O_2q+1 (subtracted from twice the chain);
            // then the factor 2^(16 (q & 1) - eC)
            for (int sl = warp; sl < B * kSPU; sl += kW) {
                int c[4] = {0, 0, 0, 0};
#pragma unroll
                for (int fp = 0; fp < 2; fp++) {
                    const uint4 xq = *reinterpret_cast<const uint4 *>(xs8 + (((sl * 2 + fp) * 32 + lane) << 4));
#pragma unroll
                    for (int pp = 0; pp < 2; pp++) {
                        const uint32_t m0 = 0x01010101u << (2 * (2 * fp + pp));
                        const uint32_t m1 = FA == 0 ? m0 : m0 << 1;
                        imma_acc(c, m0, m0, m1, m1, pp ? xq.z : xq.x, pp ? xq.w : xq.y);
                    }
                }
                if (g == 0) {
                    const int u = sl / kSPU, hs = sl - u * kSPU;
                    const int G8 = MT == 1 ? hs + 4 * (q >> 1) : (MT == 2 ? hs : hs >> 1);
                    const int m = MT == 1 ? 0 : (MT == 2 ? (q >> 1) : 2 * (hs & 1) + (q >> 1));
                    const int eC = egrp[m * (K >> 7) + u * 8 + G8];
                    const float fac = __int_as_float((127 + 16 * (q & 1) - eC) << 23);
                    if (TERN_GUARD(sl * 4 + q < p.kmax / 64 * MT, g_tern_gemvstep_guard))
                        recs[sl * 4 + q] = FA == 0 ? make_int4(-c[0], -c[1], __float_as_int(fac), 0)
                                                   : make_int4(c[0] + c[1] * 256, 0, __float_as_int(fac), 0);
                }
            }
            __syncthreads();
        } else {
        // x of token m, elements 8 c8 .. 8 c8 + 7, for the staging items
        // idx0 + u * nthr (u < kLd; idx = m * K / 8 + c8; zeros past tot or for
        // padding tokens m >= M): at eight token rows (ten or more items per
        // thread) loaded four at a time, so that a thread's global loads
        // overlap instead of queueing one round trip per item.
        constexpr int kLd = MT == 8 ? 4 : 1;
        auto load_items = [&](int idx0, int tot, uint4 (&v)[kLd]) {
            const int per_m = K / 8;
#pragma unroll
            for (int u = 0; u < kLd; u++) {
                const int idx = idx0 + u * nthr;
                const int m = idx / per_m, c8 = idx - m * per_m;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (idx < tot && m < M)
                    v[u] = *reinterpret_cast<const uint4 *>(d.x + static_cast<size_t>(m) * d.xs + c8 * 8);
            }
        };
        {
            unsigned int mx = 0;
            const int tot = M * (K / 8);
            for (int idx0 = threadIdx.x; idx0 < tot; idx0 += kLd * nthr) {
                uint4 v[kLd];
                load_items(idx0, tot, v);
#pragma unroll
                for (int u = 0; u < kLd; u++) {
                    const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                    for (int e = 0; e < 4; e++) mx = __vmaxu2(mx, __vminu2(wv[e] & 0x7FFF7FFFu, 0x7BFF7BFFu));
                }
            }
            mx = max(mx & 0xFFFFu, mx >> 16);
            mx = __reduce_max_sync(0xffffffffu, mx);
            if (lane == 0) wmax[warp] = mx;
            if (lane < 2) rec_tile[warp * 2 + lane] = -1;
        }
        __syncthreads();
        unsigned int mx = 0;
#pragma unroll
        for (int w = 0; w < kW; w++) mx = max(mx, wmax[w]);
        const int ex = max(static_cast<int>(mx >> 10), 1) - 15;
        // the largest staged factor is 2^E: x * 2^E stays finite
        E = min(F == 1 ? 7 : 8, 15 - ex);
        if constexpr (F == 1) {
            // factor of bit position p (0..15 in a half) is 2^(E - (p & 7));
            // 8 consecutive x are positions p0 .. p0 + 7, p0 = 0 or 8
            uint32_t fac2[4];
#pragma unroll
            for (int c = 0; c < 4; c++)
                fac2[c] = (static_cast<uint32_t>(15 + E - 2 * c) << 10) |
                          (static_cast<uint32_t>(15 + E - 2 * c - 1) << 26);
            const int per_m = K / 8, tot = MT * per_m;
            for (int idx0 = threadIdx.x; idx0 < tot; idx0 += kLd * nthr) {
                uint4 v[kLd];
                load_items(idx0, tot, v);
#pragma unroll
                for (int u = 0; u < kLd; u++) {
                    const int idx = idx0 + u * nthr;
                    if (idx >= tot) break;
                    const int m = idx / per_m, c8 = idx - m * per_m;
                    const uint32_t pr[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    const int kl = c8 * 8;
                    const int gk = kl >> 7;
                    const int bi = (gk / GPB) * 1024 + b1_xs_index((gk % GPB) * MT + m, kl & 127);
                    unsigned short *dst = reinterpret_cast<unsigned short *>(xs + bi);
                    if (!TERN_GUARD((bi + 263) * 2 <= xs_bytes(kcta, MT, X8), g_tern_gemvstep_guard)) continue;
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        uint32_t h2;
                        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(h2) : "r"(pr[c]), "r"(fac2[c]));
                        dst[(c >> 1) * 256 + (c & 1) * 4] = static_cast<unsigned short>(h2);
                        dst[(c >> 1) * 256 + (c & 1) * 4 + 2] = static_cast<unsigned short>(h2 >> 16);
                    }
                }
            }
        } else {
            uint32_t fac2[4];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const int e0 = E - 2 * (2 * c < 5 ? 2 * c : 2 * c - 5);
                const int e1 = E - 2 * (2 * c + 1 < 5 ? 2 * c + 1 : 2 * c + 1 - 5);
                fac2[c] = (static_cast<uint32_t>(15 + e0) << 10) | (static_cast<uint32_t>(15 + e1) << 26);
            }
            // token m of group G sits in column (G % GPB) * MT + m of set G / GPB
            const int per_m = K / 8, tot = MT * per_m;
            for (int idx0 = threadIdx.x; idx0 < tot; idx0 += kLd * nthr) {
                uint4 v[kLd];
                load_items(idx0, tot, v);
#pragma unroll
                for (int u = 0; u < kLd; u++) {
                    const int idx = idx0 + u * nthr;
                    if (idx >= tot) break;
                    const int m = idx / per_m, c8 = idx - m * per_m;
                    const uint32_t pr[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    const int kl = c8 * 8;
                    const int gk = kl >> 7;
                    const int bi = xs_pair_index<8>((gk % GPB) * MT + m, ((gk / GPB) << 7) | (kl & 127));
                    unsigned short *dst = reinterpret_cast<unsigned short *>(xs + bi);
                    if (!TERN_GUARD((bi + 773) * 2 <= xs_bytes(kcta, MT, X8), g_tern_gemvstep_guard)) continue;
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        uint32_t h2;
                        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(h2) : "r"(pr[c]), "r"(fac2[c]));
                        dst[c * 256] = static_cast<unsigned short>(h2);
                        dst[c * 256 + 4] = static_cast<unsigned short>(h2 >> 16);
                    }
                }
            }
        }
        __syncthreads();
        // one all-ones chain per set: d1[set * 8 + column]
        for (int sl = warp; sl < B * MT; sl += kW) {
            float c[4];
            if constexpr (F != 1)
                group_mma<8>(c, kOnes, kOnes, kOnes, kOnes, xlane + sl * 1024);
            else
                b1_ones_chain(c, xlane + sl * 1024);
            if (g == 0) *reinterpret_cast<float2 *>(d1 + sl * kSG + 2 * q) = make_float2(c[0], c[1]);
        }
        __syncthreads();
        }  // fp16 staging

        if (!topped) {
            for (int st = 1; st < ns && ic.i >= 0; st++) issue(st);
            topped = true;
        }
        // Lanes q < kGcLanes hold complete sums after a tile's lane
        // reduction; lane (g, q) stores v = (row g: tokens t0, t1; row g+8:
        // tokens t0, t1), t0 = 2q, t1 = 2q + 1 (MT = 4), 0, 1 (MT = 2), or
        // token 0 only from v.x, v.z (MT = 1).
        // MT = 8: every lane holds its own tokens 2q, 2q + 1.
        constexpr int kGcLanes = gc_lanes(MT);
        // A K segment after the first adds its sum to the fp16 y of the ones
        // before it (one more rounding of the partial sum).
        const bool accum = d.accum != 0;
        auto put = [&](size_t idx, float v) {
            if (accum) v += __half2float(d.y[idx]);
            d.y[idx] = __float2half_rn(v);
        };
        auto gc_store = [&](int tile, float4 v) {
            if (q >= kGcLanes) return;
            const int n0 = tile * kRows + row, n1 = n0 + 8;
            const int t0 = MT >= 4 ? 2 * q : 0, t1 = t0 + 1;
            if (n0 < N) {
                if (t0 < M) put(static_cast<size_t>(t0) * N + n0, v.x);
                if (MT > 1 && t1 < M) put(static_cast<size_t>(t1) * N + n0, v.y);
            }
            if (n1 < N) {
                if (t0 < M) put(static_cast<size_t>(t0) * N + n1, v.z);
                if (MT > 1 && t1 < M) put(static_cast<size_t>(t1) * N + n1, v.w);
            }
        };

        // ---- this warp's units of the piece ----
        int tbeg, U, v0, v1;
        piece_range(d, T0, T1, warp, tbeg, U, v0, v1);
        // (the staging is done with wmax: it keeps the piece's first tile and
        // unit count for the combine below)
        if (threadIdx.x == 0) {
            wmax[0] = static_cast<unsigned int>(tbeg);
            wmax[1] = static_cast<unsigned int>(U);
        }
        const float post = X8 ? 1.0f : ldexpf(1.0f, 24 - E);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        // (tile, slice) of unit v, by increments
        const int tl_first = v0 / B;
        const bool first_partial = v0 - tl_first * B != 0;
        int tl = tl_first, kb = v0 - tl_first * B;
        int to_end = B - kb;  // units until the current tile (or this warp's range) ends
        if (to_end > v1 - v0) to_end = v1 - v0;
        const uint8_t *stage = my_ring + s * kSlotStage;
        const uint8_t *scs = my_scl + s * kScaleStage;
        for (int v = v0; v < v1; v++) {
            bool ok = !dead;
            if (ok) ok = __all_sync(0xffffffffu, step_wait(&my_full[s], ph, deadline));
            dead = dead || !ok;
            if (ok) {
                uint32_t wd[kSG][kWords];
                // the lane's words of group G8 of the stage
                auto load_wd = [&](int G8) {
                    if constexpr (F == 2) {
                        const uint8_t *pw = stage + off[G8 & 1] + 52 * (G8 >> 1);
                        const uint32_t sh = off[2 + (G8 & 1)];
                        t5_words(pw, sh, lutl, t5dd, wd[G8][0], wd[G8][2]);
                        t5_words(pw + 8 * kT5Row, sh, lutl, t5dd, wd[G8][1], wd[G8][3]);
                    } else if constexpr (F == 0) {
                        const uint8_t *bx = stage + (G8 >> 2) * (kRows * kBox);
                        const uint2 a = *reinterpret_cast<const uint2 *>(bx + off[G8 & 3]);
                        const uint2 b = *reinterpret_cast<const uint2 *>(bx + off[G8 & 3] + 8 * kBox);
                        wd[G8][0] = a.x;
                        wd[G8][1] = b.x;
                        wd[G8][2] = a.y;
                        wd[G8][3] = b.y;
                    } else {
                        wd[G8][0] = *reinterpret_cast<const uint32_t *>(stage + off[G8]);
                        wd[G8][1] = *reinterpret_cast<const uint32_t *>(stage + off[G8] + 8 * kBox);
                    }
                };
                // The digit form at two token rows reads the second half of
                // the stage after the first half's mmas (fewer live registers)
                // and refills the stage only then.
                constexpr bool kLate = X8 && MT == 2;
#pragma unroll
                for (int G8 = 0; G8 < (kLate ? kSG / 2 : kSG); G8++) load_wd(G8);
                // scales of the lane's groups (rows `row`, `row` + 8): MT = 1
                // groups 2q, 2q+1; MT = 2, 4: one group per set h (4h + q, or
                // 2h + q/2); MT = 8: all eight groups of both rows
                __half2 sh[MT == 1 ? 2 : (MT == 8 ? 1 : MT)];
                uint4 s8a, s8b;
                uint2 s4a, s4b;
                if constexpr (X8 && MT == 1) {
                    // digit form, one token: groups 4 (q / 2) + h of set h
                    s4a = *reinterpret_cast<const uint2 *>(scs + row * 16 + 8 * (q >> 1));
                    s4b = *reinterpret_cast<const uint2 *>(scs + (row + 8) * 16 + 8 * (q >> 1));
                } else if constexpr (MT == 8 || X8) {
                    s8a = *reinterpret_cast<const uint4 *>(scs + row * 16);
                    s8b = *reinterpret_cast<const uint4 *>(scs + (row + 8) * 16);
                } else if (MT == 1) {
                    sh[0] = *reinterpret_cast<const __half2 *>(scs + row * 16 + 4 * q);
                    sh[MT == 1 ? 1 : 0] = *reinterpret_cast<const __half2 *>(scs + (row + 8) * 16 + 4 * q);
                } else {
#pragma unroll
                    for (int h = 0; h < MT; h++) {
                        const int grp = MT == 2 ? 4 * h + q : 2 * h + (q >> 1);
                        sh[h] = __halves2half2(*reinterpret_cast<const __half *>(scs + row * 16 + 2 * grp),
                                               *reinterpret_cast<const __half *>(scs + (row + 8) * 16 + 2 * grp));
                    }
                }
                // The stage is in registers: refill it with this warp's next
                // unit (the warp barrier and the proxy fence order the reads
                // before the copy that overwrites it).
                auto refill = [&]() {
                    __syncwarp();
                    consumed++;
                    if (ic.i >= 0) {
                        if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        issue(s);
                    }
                };
                if constexpr (!kLate) refill();
                if constexpr (X8 && MT == 1) {
                    // four sets of two groups (h, h + 4); lanes q < 2 keep
                    // group h, lanes q >= 2 group h + 4.  acc[0] = row g,
                    // acc[2] = row g + 8.
                    int dd[kSG][4];
                    int4 rr[4];
#pragma unroll
                    for (int h = 0; h < 4; h++) rr[h] = recs[(kb * 4 + h) * 4 + q];
#pragma unroll
                    for (int fp = 0; fp < 2; fp++) {
                        uint4 xq[4];
#pragma unroll
                        for (int h = 0; h < 4; h++)
                        {
                            const int xo = (((kb * 4 + h) * 2 + fp) * 32 + lane) << 4;
                            xq[h] = TERN_GUARD(xo + 16 <= xs_bytes(kcta, MT, X8), g_tern_gemvstep_guard)
                                        ? *reinterpret_cast<const uint4 *>(xs8 + xo)
                                        : make_uint4(0u, 0u, 0u, 0u);
                        }
#pragma unroll
                        for (int fi = 0; fi < 2; fi++) {
#pragma unroll
                            for (int G8 = 0; G8 < kSG; G8++) {
                                const uint4 &xv = xq[G8 & 3];
                                const uint32_t b0 = fi ? xv.z : xv.x, b1 = fi ? xv.w : xv.y;
                                uint32_t a0, a1, a2, a3;
                                x8_a<FA>(wd[G8], 2 * fp + fi, a0, a1, a2, a3);
                                if (fp == 0 && fi == 0)
                                    imma_init(dd[G8], a0, a1, a2, a3, b0, b1, FA == 0 ? rr[G8 & 3].x : 0,
                                              FA == 0 ? rr[G8 & 3].y : 0);
                                else
                                    imma_acc(dd[G8], a0, a1, a2, a3, b0, b1);
                            }
                        }
                    }
                    const bool hi = q >= 2;
                    const float2 a01 = __half22float2(*reinterpret_cast<const __half2 *>(&s4a.x));
                    const float2 a23 = __half22float2(*reinterpret_cast<const __half2 *>(&s4a.y));
                    const float2 b01 = __half22float2(*reinterpret_cast<const __half2 *>(&s4b.x));
                    const float2 b23 = __half22float2(*reinterpret_cast<const __half2 *>(&s4b.y));
                    const float sA[4] = {a01.x, a01.y, a23.x, a23.y}, sB[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
                    for (int h = 0; h < 4; h++) {
                        const int oc = rr[h].x;
                        const int ia = x8_join<FA>(dd[h][0], dd[h][1], oc), ib = x8_join<FA>(dd[h + 4][0], dd[h + 4][1], oc);
                        const int ja = x8_join<FA>(dd[h][2], dd[h][3], oc), jb = x8_join<FA>(dd[h + 4][2], dd[h + 4][3], oc);
                        const float fac = __int_as_float(rr[h].z);
                        acc[0] = fmaf(sA[h] * fac, static_cast<float>(hi ? ib : ia), acc[0]);
                        acc[2] = fmaf(sB[h] * fac, static_cast<float>(hi ? jb : ja), acc[2]);
                    }
                } else if constexpr (X8 && MT == 2) {
                    // two tokens: one set per group, lane q holds token q / 2;
                    // four groups at a time.  acc[0] = row g, acc[2] = row g + 8.
                    const uint32_t sw[2][4] = {{s8a.x, s8a.y, s8a.z, s8a.w}, {s8b.x, s8b.y, s8b.z, s8b.w}};
#pragma unroll
                    for (int hf = 0; hf < 2; hf++) {
                        if (hf == 1) {
#pragma unroll
                            for (int G8 = kSG / 2; G8 < kSG; G8++) load_wd(G8);
                            refill();
                        }
                        int dd[4][4];
                        int2 rr[4];
#pragma unroll
                        for (int j = 0; j < 4; j++)
                            rr[j] = *reinterpret_cast<const int2 *>(recs + (kb * 8 + 4 * hf + j) * 4 + q);
#pragma unroll
                        for (int fp = 0; fp < 2; fp++) {
                            uint4 xq[4];
#pragma unroll
                            for (int j = 0; j < 4; j++)
                            {
                                const int xo = (((kb * 8 + 4 * hf + j) * 2 + fp) * 32 + lane) << 4;
                                xq[j] = TERN_GUARD(xo + 16 <= xs_bytes(kcta, MT, X8), g_tern_gemvstep_guard)
                                            ? *reinterpret_cast<const uint4 *>(xs8 + xo)
                                            : make_uint4(0u, 0u, 0u, 0u);
                            }
#pragma unroll
                            for (int fi = 0; fi < 2; fi++) {
#pragma unroll
                                for (int j = 0; j < 4; j++) {
                                    const uint32_t b0 = fi ? xq[j].z : xq[j].x, b1 = fi ? xq[j].w : xq[j].y;
                                    uint32_t a0, a1, a2, a3;
                                    x8_a<FA>(wd[4 * hf + j], 2 * fp + fi, a0, a1, a2, a3);
                                    if (fp == 0 && fi == 0)
                                        imma_init(dd[j], a0, a1, a2, a3, b0, b1, FA == 0 ? rr[j].x : 0,
                                                  FA == 0 ? rr[j].y : 0);
                                    else
                                        imma_acc(dd[j], a0, a1, a2, a3, b0, b1);
                                }
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const int G8 = 4 * hf + j;
                            const float sa = __half2float(__ushort_as_half(
                                static_cast<unsigned short>(sw[0][G8 >> 1] >> (16 * (G8 & 1)))));
                            const float sb = __half2float(__ushort_as_half(
                                static_cast<unsigned short>(sw[1][G8 >> 1] >> (16 * (G8 & 1)))));
                            const float fac = __int_as_float(recs[(kb * 8 + G8) * 4 + q].z);
                            acc[0] = fmaf(sa * fac, static_cast<float>(x8_join<FA>(dd[j][0], dd[j][1], rr[j].x)), acc[0]);
                            acc[2] = fmaf(sb * fac, static_cast<float>(x8_join<FA>(dd[j][2], dd[j][3], rr[j].x)), acc[2]);
                        }
                    }
                } else if constexpr (X8 && MT == 4) {
                    // two column sets per group (tokens 0, 1 and 2, 3), both
                    // fed by the same A registers; two groups at a time.
                    // acc[0] / acc[1] = row g, tokens q/2 and 2 + q/2;
                    // acc[2] / acc[3] = row g + 8.
                    const uint32_t sw[2][4] = {{s8a.x, s8a.y, s8a.z, s8a.w}, {s8b.x, s8b.y, s8b.z, s8b.w}};
#pragma unroll
                    for (int qt = 0; qt < 4; qt++) {
                        int dd[2][2][4];
                        int2 rr[2][2];
#pragma unroll
                        for (int j = 0; j < 2; j++)
#pragma unroll
                            for (int cs = 0; cs < 2; cs++)
                                rr[j][cs] = *reinterpret_cast<const int2 *>(
                                    recs + ((kb * 8 + 2 * qt + j) * 2 + cs) * 4 + q);
#pragma unroll
                        for (int fp = 0; fp < 2; fp++) {
                            uint4 xq[2][2];
#pragma unroll
                            for (int j = 0; j < 2; j++)
#pragma unroll
                                for (int cs = 0; cs < 2; cs++) {
                                    const int xo = ((((kb * 8 + 2 * qt + j) * 2 + cs) * 2 + fp) * 32 + lane) << 4;
                                    xq[j][cs] = TERN_GUARD(xo + 16 <= xs_bytes(kcta, MT, X8), g_tern_gemvstep_guard)
                                                    ? *reinterpret_cast<const uint4 *>(xs8 + xo)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                                }
#pragma unroll
                            for (int fi = 0; fi < 2; fi++) {
#pragma unroll
                                for (int j = 0; j < 2; j++) {
                                    uint32_t a0, a1, a2, a3;
                                    x8_a<FA>(wd[2 * qt + j], 2 * fp + fi, a0, a1, a2, a3);
#pragma unroll
                                    for (int cs = 0; cs < 2; cs++) {
                                        const uint4 &xv = xq[j][cs];
                                        const uint32_t b0 = fi ? xv.z : xv.x, b1 = fi ? xv.w : xv.y;
                                        if (fp == 0 && fi == 0)
                                            imma_init(dd[j][cs], a0, a1, a2, a3, b0, b1, FA == 0 ? rr[j][cs].x : 0,
                                                      FA == 0 ? rr[j][cs].y : 0);
                                        else
                                            imma_acc(dd[j][cs], a0, a1, a2, a3, b0, b1);
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 2; j++) {
                            const int G8 = 2 * qt + j;
                            const float sa = __half2float(__ushort_as_half(
                                static_cast<unsigned short>(sw[0][G8 >> 1] >> (16 * (G8 & 1)))));
                            const float sb = __half2float(__ushort_as_half(
                                static_cast<unsigned short>(sw[1][G8 >> 1] >> (16 * (G8 & 1)))));
#pragma unroll
                            for (int cs = 0; cs < 2; cs++) {
                                const float fac = __int_as_float(recs[((kb * 8 + G8) * 2 + cs) * 4 + q].z);
                                acc[cs] = fmaf(sa * fac,
                                               static_cast<float>(x8_join<FA>(dd[j][cs][0], dd[j][cs][1], rr[j][cs].x)),
                                               acc[cs]);
                                acc[2 + cs] = fmaf(sb * fac,
                                                   static_cast<float>(x8_join<FA>(dd[j][cs][2], dd[j][cs][3], rr[j][cs].x)),
                                                   acc[2 + cs]);
                            }
                        }
                    }
                } else if constexpr (MT == 8) {
                    // group by group: acc[0..1] = row g, tokens 2q, 2q+1;
                    // acc[2..3] = row g+8
                    const uint32_t sw[2][4] = {{s8a.x, s8a.y, s8a.z, s8a.w}, {s8b.x, s8b.y, s8b.z, s8b.w}};
#pragma unroll
                    for (int G8 = 0; G8 < kSG; G8++) {
                        float c[4];
                        group_mma<8>(c, wd[G8][0], wd[G8][2], wd[G8][1], wd[G8][3], xlane + (kb * 8 + G8) * 1024);
                        const float2 on = *reinterpret_cast<const float2 *>(d1 + (kb * 8 + G8) * kSG + 2 * q);
                        const float sa = __half2float(__ushort_as_half(
                            static_cast<unsigned short>(sw[0][G8 >> 1] >> (16 * (G8 & 1)))));
                        const float sb = __half2float(__ushort_as_half(
                            static_cast<unsigned short>(sw[1][G8 >> 1] >> (16 * (G8 & 1)))));
                        acc[0] = fmaf(sa, c[0] - on.x, acc[0]);
                        acc[1] = fmaf(sa, c[1] - on.y, acc[1]);
                        acc[2] = fmaf(sb, c[2] - on.x, acc[2]);
                        acc[3] = fmaf(sb, c[3] - on.y, acc[3]);
                    }
                } else {
                float out[MT][4];
                if constexpr (F != 1)
                    gcm_slice<MT>(wd, xlane + kb * MT * 1024, qm, qh, out);
                else
                    b1_slice<MT>(wd, xlane + kb * MT * 1024, qm, qh, out);
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
                    // t = c - 1 (ternary) or t = 2b - 1 (1-bit)
                    constexpr float kMul = F == 1 ? 2.f : 1.f;
                    acc[0] = fmaf(sa0, fmaf(kMul, out[h][0], -on.x), acc[0]);
                    acc[1] = fmaf(sa1, fmaf(kMul, out[h][1], -on.y), acc[1]);
                    acc[2] = fmaf(sb0, fmaf(kMul, out[h][2], -on.x), acc[2]);
                    acc[3] = fmaf(sb1, fmaf(kMul, out[h][3], -on.y), acc[3]);
                }
                }
            }
            stage += kSlotStage;
            scs += kScaleStage;
            if (++s == ns) {
                s = 0;
                ph ^= 1;
                stage = my_ring;
                scs = my_scl;
            }
            if (--to_end == 0) {
                // ---- this warp's part of a tile is complete: sum the lanes q
                // that hold other groups of the same tokens ----
                if constexpr (X8 && MT == 4) {
                    // lanes q, q ^ 1 hold the two digit pairs of tokens q / 2
                    // (acc[0], acc[2]) and 2 + q / 2 (acc[1], acc[3]); lane 0
                    // ends with tokens 0, 1 and lane 1 with tokens 2, 3 (rows g, g + 8)
                    float o[4];
#pragma unroll
                    for (int c = 0; c < 4; c++) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 1);
#pragma unroll
                    for (int c = 0; c < 4; c++) o[c] = __shfl_xor_sync(0xffffffffu, acc[c], 2);
                    const bool odd = (q & 1) != 0;
                    const float v0 = odd ? acc[1] : acc[0], v2 = odd ? acc[3] : acc[2];
                    acc[0] = v0;
                    acc[1] = odd ? o[1] : o[0];
                    acc[2] = v2;
                    acc[3] = odd ? o[3] : o[2];
                } else if constexpr (X8 && MT == 2) {
                    // lanes q, q ^ 1 hold the two digit pairs of token q / 2:
                    // lane 0 ends with (row g: tokens 0, 1; row g + 8: 0, 1)
                    const float tg = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
                    const float tg8 = acc[2] + __shfl_xor_sync(0xffffffffu, acc[2], 1);
                    acc[1] = __shfl_xor_sync(0xffffffffu, tg, 2);
                    acc[3] = __shfl_xor_sync(0xffffffffu, tg8, 2);
                    acc[0] = tg;
                    acc[2] = tg8;
                } else {
                if (MT == 1) {
                    acc[0] += acc[1];
                    acc[2] += acc[3];
                    acc[1] = acc[3] = 0.f;
                }
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    if (MT <= 2) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 1);
                    if (MT <= 4) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 2);
                }
                }
                const int tile = tbeg + tl;
                const bool whole = kb == B - 1 && (tl != tl_first || !first_partial);
                const float4 vv = make_float4(acc[0] * post, acc[1] * post, acc[2] * post, acc[3] * post);
                if (whole) {
                    if (!dead) gc_store(tile, vv);
                } else {
                    const int slot = (tl == tl_first) ? 0 : 1;
                    if (q < kGcLanes)
                        *reinterpret_cast<float4 *>(rec + (((warp * 2 + slot) * 8 + g) * kGcLanes + q) * 4) = vv;
                    if (lane == 0) rec_tile[warp * 2 + slot] = dead ? -2 : tile;
                }
                acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                to_end = min(B, v1 - v - 1);
            }
            if (++kb == B) {
                kb = 0;
                tl++;
            }
        }
        // ---- tiles of this piece split over several warps: summed in warp
        // order by the first warp that holds a part ----
        // (no partial tile is stored once any warp of the CTA has given up)
        if (__syncthreads_or(dead ? 1 : 0) == 0) {
            // warp w2 holds units [PU w2 / kW, PU (w2 + 1) / kW) of the piece
            // (32-bit: a piece has far fewer than 2^27 units)
            const int pbeg = static_cast<int>(wmax[0]);
            const unsigned int PU = wmax[1], UB = static_cast<unsigned int>(B);
            const unsigned int pv0 = (PU * static_cast<unsigned int>(warp)) / kW;
#pragma unroll 1
            for (int slot = 0; slot < 2; slot++) {
                const int tile = rec_tile[warp * 2 + slot];
                if (tile < 0) continue;
                // The first warp holding a part holds the tile's first unit:
                // slot 1 always, slot 0 when this warp's range starts there.
                if (slot == 0 && pv0 % UB != 0u) continue;
                // The other parts are the slot-0 parts of the following warps
                // whose ranges start inside the tile, up to warp wl (the last
                // with PU w / kW < tend); warps with empty ranges hold none.
                const unsigned int tend = static_cast<unsigned int>(tile - pbeg + 1) * UB;
                const int wl = static_cast<int>(min(static_cast<unsigned int>(kW - 1), (kW * tend - 1u) / PU));
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                if (q < kGcLanes) {
                    sum = *reinterpret_cast<const float4 *>(rec + (((warp * 2 + slot) * 8 + g) * kGcLanes + q) * 4);
                    for (int w2 = warp + 1; w2 <= wl; w2++) {
                        if (PU < kW && (PU * (w2 + 1u)) / kW == (PU * w2) / kW) continue;
                        const float4 o = *reinterpret_cast<const float4 *>(rec + (((w2 * 2) * 8 + g) * kGcLanes + q) * 4);
                        sum.x += o.x;
                        sum.y += o.y;
                        sum.z += o.z;
                        sum.w += o.w;
                    }
                }
                gc_store(tile, sum);
            }
        }
    }
    // A warp that gave up may still have copies of its own in flight: they
    // must land before the CTA exits (bounded).
    if (dead) {
        const unsigned long long dl2 = globaltimer() + p.timeout_ns;
        for (int u = consumed; u < issued; u++) {
            const int st = static_cast<int>(u % ns);
            const uint32_t phs = static_cast<uint32_t>((u / ns) & 1);
            step_wait(&my_full[st], phs, dl2);
        }
    }
    if (!p.first) asm volatile("griddepcontrol.wait;" ::: "memory");
}

bool g_attr_step[64][3][4][2];

using StepKernel = void (*)(SParams);
StepKernel step_kernel(int mt, int f, bool x8) {
    if (x8) {
        if (f == 0)
            return mt == 1 ? gemv_step_kernel<1, 0, true>
                           : (mt == 2 ? gemv_step_kernel<2, 0, true> : (mt == 4 ? gemv_step_kernel<4, 0, true> : nullptr));
        if (f == 1)
            return mt == 1 ? gemv_step_kernel<1, 1, true>
                           : (mt == 2 ? gemv_step_kernel<2, 1, true> : (mt == 4 ? gemv_step_kernel<4, 1, true> : nullptr));
        return mt == 1 ? gemv_step_kernel<1, 2, true>
                       : (mt == 2 ? gemv_step_kernel<2, 2, true> : (mt == 4 ? gemv_step_kernel<4, 2, true> : nullptr));
    }
    if (f == 0)
        return mt == 1 ? gemv_step_kernel<1, 0, false>
                       : (mt == 2 ? gemv_step_kernel<2, 0, false>
                                  : (mt == 4 ? gemv_step_kernel<4, 0, false> : gemv_step_kernel<8, 0, false>));
    if (f == 1)  // no eight-token form for the 1-bit weights
        return mt == 1 ? gemv_step_kernel<1, 1, false>
                       : (mt == 2 ? gemv_step_kernel<2, 1, false> : (mt == 4 ? gemv_step_kernel<4, 1, false> : nullptr));
    return mt == 1 ? gemv_step_kernel<1, 2, false>
                   : (mt == 2 ? gemv_step_kernel<2, 2, false>
                              : (mt == 4 ? gemv_step_kernel<4, 2, false> : gemv_step_kernel<8, 2, false>));
}

int step_mt(int M) { return M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : 8)); }

// What staging one piece's x costs a CTA, in 1024-k units of streaming
// (measured on B200: a piece's staging takes ~1.5-5 us at one token row,
// ~3.5-8.5 us at four and ~5.5-6.5 us at eight, against ~10, ~6.5 and ~6
// units streamed per microsecond and CTA).
int piece_cost(int K, int M) {
    const int B = K / 1024;
    if (M == 1) return 5 + (12 * B) / 5;
    if (M == 2) return 6 + (5 * B) / 2;
    if (M <= 4) return 10 + (13 * B) / 5;
    return 20 + 3 * B;
}

// Greedy cut of the flat tile list into CTA ranges whose units plus piece
// costs stay within C (each range that starts or continues a matrix pays that
// matrix's piece cost).  Returns the number of ranges; with `cut` non-null
// writes their first tiles cut[1..].
int cut_ranges(const SDesc *d, const int *pc, int count, long long C, int *cut) {
    int n = 0;
    long long acc = 0;
    bool open = false;
    for (int i = 0; i < count; i++) {
        const int B = d[i].K / 1024;
        int left = d[i].ntile, t = d[i].tile0;
        while (left > 0) {
            if (open && acc + pc[i] + B > C) {
                n++;
                if (cut) cut[n] = t;
                acc = 0;
            }
            open = true;
            acc += pc[i];
            long long take = (C - acc) / B;
            if (take < 1) take = 1;
            if (take > left) take = left;
            acc += take * B;
            left -= static_cast<int>(take);
            t += static_cast<int>(take);
            if (left > 0) {
                n++;
                if (cut) cut[n] = t;
                acc = 0;
                open = false;
            }
        }
    }
    return open ? n + 1 : n;
}

// Cuts at the multiples of total / grid along the same cost axis (so that
// every CTA gets a range), each range kept within Cmax.  Returns the number
// of ranges (above grid: unusable); writes the first tiles of ranges
// 1 .. grid - 1 to cut[] and the axis length to *end.
int cut_even(const SDesc *d, const int *pc, int count, double total, int grid, long long Cmax, int *cut,
             long long *end) {
    const double target = total / grid;
    int n = 1;
    long long acc = 0, pos = 0;
    for (int i = 0; i < count; i++) {
        const long long B = d[i].K / 1024;
        long long left = d[i].ntile;
        int t = d[i].tile0;
        bool pending = true;  // the range has not paid matrix i's piece cost yet
        while (left > 0) {
            long long add = (pending ? pc[i] : 0) + B;
            if (acc > 0 && (acc + add > Cmax || (n < grid && pos + 0.5 * add > n * target))) {
                if (n < grid) cut[n] = t;
                n++;
                acc = 0;
                add = pc[i] + B;
            }
            pos += add;
            acc += add;
            pending = false;
            t++;
            left--;
            // tiles that can follow before the next cut: within Cmax, and
            // before the axis passes the next multiple of the target
            long long k = std::max<long long>(0, (Cmax - acc) / B);
            if (n < grid) {
                const double r = n * target - static_cast<double>(pos) - 0.5 * static_cast<double>(B);
                k = std::min<long long>(k, r >= 0 ? static_cast<long long>(std::floor(r / static_cast<double>(B))) + 1 : 0);
            }
            k = std::min(k, left);
            pos += k * B;
            acc += k * B;
            t += static_cast<int>(k);
            left -= k;
        }
    }
    *end = pos;
    return n;
}

// Cut the flat tile list of one launch (d[i].tile0, ntile, K; tiles in
// descriptor order) into at most `grid` CTA ranges of about equal cost
// (units plus the staging of each piece): cta_tile[c] .. cta_tile[c + 1] is
// CTA c's range, cta_tile[0] = 0, cta_tile[grid] = all tiles; trailing CTAs
// may get empty ranges.  The smallest bound C whose greedy cut needs no more
// ranges than CTAs is the best possible largest range; cuts at even steps of
// the cost axis within that bound give every CTA a range (the axis length,
// which depends on where the cuts fall, is refined over a few passes); where
// they need more ranges than CTAs, the greedy cut stands.
void plan_ranges(const SDesc *d, int count, int M, int grid, int *cta_tile) {
    int pc[TERN_MAX_STEP];
    long long hi = 0, pcsum = 0, total_units = 0;
    int tiles = 0;
    for (int i = 0; i < count; i++) {
        pc[i] = piece_cost(d[i].K, M);
        pcsum += pc[i];
        total_units += static_cast<long long>(d[i].ntile) * (d[i].K / 1024);
        hi += static_cast<long long>(d[i].ntile) * (d[i].K / 1024) + static_cast<long long>(pc[i]) * d[i].ntile;
        tiles = std::max(tiles, d[i].tile0 + d[i].ntile);
    }
    long long lo = std::max<long long>(1, total_units / grid);
    while (lo < hi) {
        const long long mid = (lo + hi) / 2;
        if (cut_ranges(d, pc, count, mid, nullptr) <= grid) hi = mid; else lo = mid + 1;
    }
    int used = cut_ranges(d, pc, count, lo, cta_tile);
    int cut[kMaxCtas + 1];
    double total = static_cast<double>(total_units + pcsum) + static_cast<double>(grid - 1) * pcsum / count;
    for (int pass = 0; pass < 4; pass++) {
        long long end = 0;
        const int n = cut_even(d, pc, count, total, grid, lo, cut, &end);
        if (n <= grid && n > used) {
            used = n;
            for (int c = 1; c < n; c++) cta_tile[c] = cut[c];
        }
        total = static_cast<double>(end);
    }
    cta_tile[0] = 0;
    for (int c = used; c <= grid; c++) cta_tile[c] = tiles;
}
int mt_index(int mt) { return mt == 1 ? 0 : (mt == 2 ? 1 : (mt == 4 ? 2 : 3)); }

// The digit form serves every weight storage at one and two token rows
// unless the group-per-column fp16 form is asked for (TERN_OPT_STEP_FORM =
// 1); at three and four rows only when asked for (= 2): its 16 bytes of
// staged x per k leave one ring stage per warp at K = 5120 and 6144, and the
// verify step at M = 4 measured 2.25 ms against 1.41 ms in the fp16 form.
bool step_x8(int M, int fmt) { return g_opt.step_form == 1 ? false : M <= (g_opt.step_form == 2 ? 4 : 2); }

}  // namespace

bool gemv_step_digit_form(int M, int fmt) { return step_x8(M, fmt); }

bool gemv_step_fits(int K, int M, int fmt, bool x8) {
    return K % 1024 == 0 && M >= 1 && M <= (fmt == 1 ? 4 : 8) && (!x8 || M <= 4) &&
           smem_bytes(K, step_mt(M), 1, fmt, x8) <= kSmemBudget;
}

bool gemv_step_supports(const MatDesc *md, int count, int M, int fmt, bool x8) {
    if (count < 1 || count > TERN_MAX_STEP || M < 1 || M > (fmt == 1 ? 4 : 8)) return false;
    int kmax = 0;
    for (int i = 0; i < count; i++) {
        if (md[i].K % 1024 != 0) return false;
        kmax = std::max(kmax, md[i].K);
    }
    // one ring stage per warp at least (refilled as soon as it is read)
    return (!x8 || M <= 4) && smem_bytes(kmax, step_mt(M), 1, fmt, x8) <= kSmemBudget;
}

namespace {

// One launch over md[0..count) (count <= kMaxPer).
tern_status launch_chunk(const DeviceInfo &dev, const MatDesc *md, int count, int M, int fmt, bool x8, bool first,
                         cudaStream_t stream) {
    thread_local SParams p;  // large (parameter space); filled on the host for each launch, per host thread
    std::memset(&p, 0, sizeof(p));
    const int mt = step_mt(M);
    int kmax = 0;
    long long total_units = 0;
    int tiles = 0;
    for (int i = 0; i < count; i++) {
        SDesc &d = p.d[i];
        d.x = md[i].x;
        d.y = md[i].y;
        d.N = md[i].N;
        d.K = md[i].K;
        d.tile0 = tiles;
        d.ntile = (md[i].N + kRows - 1) / kRows;
        const int kfull = md[i].kfull > 0 ? md[i].kfull : md[i].K;
        d.xs = kfull;
        d.accum = md[i].accum;
        tiles += d.ntile;
        total_units += static_cast<long long>(d.ntile) * (md[i].K / 1024);
        kmax = std::max(kmax, md[i].K);
        tern_status st;
        if (fmt == 0) {
            // the slot matrix seen as [K/512 chunks][N rows][128 bytes]: one
            // copy brings both 512-k boxes of a unit
            const uint64_t sdims[3] = {static_cast<uint64_t>(kBox), static_cast<uint64_t>(md[i].N),
                                       static_cast<uint64_t>(md[i].K / 512)};
            const uint64_t sstr[2] = {static_cast<uint64_t>(kfull / 4), static_cast<uint64_t>(kBox)};
            const uint32_t sbox[3] = {static_cast<uint32_t>(kBox), static_cast<uint32_t>(kRows), 2};
            st = encode_tiled_3d(&p.m[i].smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots, sdims, sstr, sbox,
                                 CU_TENSOR_MAP_SWIZZLE_128B);
        } else if (fmt == 1) {
            // the bit matrix [N rows][K/8 bytes]: one 128-byte box is a unit's row
            st = encode_tiled_2d(&p.m[i].smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots,
                                 static_cast<uint64_t>(md[i].K / 8), static_cast<uint64_t>(md[i].N),
                                 static_cast<uint64_t>(kfull / 8), kBox, kRows, CU_TENSOR_MAP_SWIZZLE_128B);
        } else {
            // the base-3 bytes [N rows][R bytes], R = 208 K / 1024: one
            // 208-byte box is a unit's row (a multiple of 16 bytes)
            const uint64_t R = static_cast<uint64_t>(md[i].K / 1024) * kT5Row;
            const uint64_t Rfull = static_cast<uint64_t>(kfull / 1024) * kT5Row;
            st = encode_tiled_2d(&p.m[i].smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, md[i].slots, R,
                                 static_cast<uint64_t>(md[i].N), Rfull, kT5Row, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        }
        if (st != TERN_OK) return st;
        const int G = md[i].K / kGroup;
        st = encode_tiled_2d(&p.m[i].cmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, md[i].scales, static_cast<uint64_t>(G),
                             static_cast<uint64_t>(md[i].N), static_cast<uint64_t>(kfull / kGroup) * 2, kSG, kRows,
                             CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != TERN_OK) return st;
    }
    const size_t budget = std::min<size_t>(kSmemBudget, dev.max_smem_optin);
    // The whole budget: every CTA sizes its ring from what its own staged x leaves.
    const size_t smem = std::min(budget, smem_bytes(kmax, mt, kMaxNS, fmt, x8));
    if (smem_bytes(kmax, mt, 1, fmt, x8) > smem)
        return fail(TERN_ERR_SHAPE, "step kernel needs %zu B of shared memory", smem_bytes(kmax, mt, 1, fmt, x8));
    int grid = std::min<int>(std::min(dev.sms, kMaxCtas), tiles);
    if (g_opt.gemv_grid > 0) grid = std::min(grid, g_opt.gemv_grid);
    plan_ranges(p.d, count, M, grid, p.cta_tile);
    p.count = count;
    p.M = M;
    p.smem_usable = static_cast<unsigned int>(smem - 1024);
    p.kmax = kmax;
    p.skip_loads = g_gemm_skip_loads;
    p.first = first ? 1 : 0;
    p.timeout_ns = g_gemm_timeout_ns;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, step_kernel(mt, fmt, x8), p);
    if (e != cudaSuccess) return cuda_fail(e, "gemv step kernel launch");
    return TERN_OK;
}

}  // namespace

tern_status launch_gemv_step(const MatDesc *md, int count, int M, int fmt, bool x8, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    if (fmt < 0 || fmt > 2) return fail(TERN_ERR_INVALID_ARG, "step kernel: unknown weight format %d", fmt);
    if (!gemv_step_supports(md, count, M, fmt, x8) || step_kernel(step_mt(M), fmt, x8) == nullptr)
        return fail(TERN_ERR_SHAPE, "step kernel: unsupported shapes");
    const int mi = mt_index(step_mt(M));
    if (!g_attr_step[dev.device][fmt][mi][x8]) {
        cudaError_t e = cudaFuncSetAttribute(step_kernel(step_mt(M), fmt, x8), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(dev.max_smem_optin));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemv step)");
        g_attr_step[dev.device][fmt][mi][x8] = true;
    }
    // Equal-sized launches of at most kMaxPer matrices each.
    const int launches = (count + kMaxPer - 1) / kMaxPer;
    int done = 0;
    for (int l = 0; l < launches; l++) {
        const int n = (count - done) / (launches - l);
        st = launch_chunk(dev, md + done, n, M, fmt, x8, l == 0, stream);
        if (st != TERN_OK) return st;
        done += n;
    }
    return TERN_OK;
}

tern_status read_gemvstep_guard(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_gemvstep_guard, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device guard count");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_gemvstep_guard, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device guard count");
    }
    *out = v;
    return TERN_OK;
}

tern_status read_gemvstep_status(bool reset, unsigned int *out) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tern_gemvstep_status, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    if (reset && v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tern_gemvstep_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing device status");
    }
    *out = v;
    return TERN_OK;
}

// The CTA ranges one launch of the step kernel would use (see plan_ranges).
tern_status gemv_step_plan(const int64_t *N, const int64_t *K, int count, int M, int grid, int32_t *first_tile) {
    if (!N || !K || !first_tile) return fail(TERN_ERR_INVALID_ARG, "null pointer");
    if (count < 1 || count > kMaxPer) return fail(TERN_ERR_SHAPE, "count must be in [1, %d] (got %d)", kMaxPer, count);
    if (M < 1 || M > 8) return fail(TERN_ERR_SHAPE, "M must be in [1, 8] (got %d)", M);
    if (grid < 1 || grid > kMaxCtas) return fail(TERN_ERR_SHAPE, "grid must be in [1, %d] (got %d)", kMaxCtas, grid);
    SDesc d[kMaxPer];
    int tiles = 0;
    for (int i = 0; i < count; i++) {
        if (N[i] < 1 || N[i] > 0x7FFFFFF0ll || K[i] < 1024 || K[i] % 1024 != 0 || K[i] > (1 << 20))
            return fail(TERN_ERR_SHAPE, "descriptor %d: N >= 1 and K a positive multiple of 1024 required", i);
        std::memset(&d[i], 0, sizeof(SDesc));
        d[i].N = static_cast<int>(N[i]);
        d[i].K = static_cast<int>(K[i]);
        d[i].tile0 = tiles;
        d[i].ntile = static_cast<int>((N[i] + kRows - 1) / kRows);
        if (tiles > 0x7FFFFFFF - d[i].ntile) return fail(TERN_ERR_SHAPE, "too many rows");
        tiles += d[i].ntile;
    }
    const int g = std::min(grid, tiles);
    int cta_tile[kMaxCtas + 1];
    plan_ranges(d, count, M, g, cta_tile);
    for (int c = 0; c <= g; c++) first_tile[c] = cta_tile[c];
    for (int c = g + 1; c <= grid; c++) first_tile[c] = tiles;
    return TERN_OK;
}

}  // namespace tern
