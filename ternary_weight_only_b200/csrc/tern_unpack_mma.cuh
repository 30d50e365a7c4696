// Device helpers shared by the bandwidth kernels that feed mma.sync m16n8k16
// straight from the 2-bit slots (internal header, not installed).
//
// The unpack: a slot word holds 16 codes; its "pair j" is field j of both
// 16-bit halves.  One AND with 0x00030003 << 2j' (j' = j for j < 5, j - 5 on
// the word shifted right by 10 for j >= 5) leaves an fp16 pair whose halves
// are the subnormals c * 4^j' * 2^-24, exactly; the staged activations carry
// the inverse power of four, and t = c - 1 is restored by subtracting the
// same mma chain run on the all-ones word (code 1 everywhere).
#pragma once

#include "tern_internal.cuh"

namespace tern {

constexpr uint32_t kOnes = 0x55555555u;  // every 2-bit field = code 1 (t = 0)

// D = A * B + C and D = A * B, m16n8k16, fp16 in, fp32 accumulate (no side
// effects, so the compiler may interleave the chains of neighbouring groups).
__device__ __forceinline__ void mma_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_zero(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// D = A * B + C and D = A * B + {c0, c1, c0, c1}, m16n8k32, A unsigned 8-bit,
// B signed 8-bit, exact 32-bit integer accumulation.
__device__ __forceinline__ void imma_acc(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void imma_init(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1, int c0, int c1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%10,%11};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c0), "r"(c1));
}

// Index (in halves) of x[m][kl] in this kernel's staging area.  Per group
// of 128 k the B fragments of its eight mmas: chunk i (pairs j = 2i, 2i+1)
// holds, per token m and lane q (words 2q, 2q+1 of the group), 8 halves
// [j & 1][word 2q + wi][half] = x at word position j (lo) and j+8 (hi).
// Layout [group][chunk][m][q][8]: a lane's four 16-byte loads hit distinct
// banks within every quarter warp.
template <int MT>
__device__ __forceinline__ int xs_pair_index(int m, int kl) {
    const int grp = kl >> 7;
    const int word = (kl >> 4) & 7;
    const int hi = (kl >> 3) & 1;
    const int j = kl & 7;
    return (((grp * 4 + (j >> 1)) * MT + m) * 4 + (word >> 1)) * 8 + (j & 1) * 4 + (word & 1) * 2 + hi;
}

// The eight mmas of one 16-row x 128-k group: pair j of the lane's words
// (a = row g, b = row g+8; .x = word 2q, .y = word 2q+1) against the staged x
// of pair j, one accumulation chain (the unrolled groups of a slice give the
// scheduler independent chains).  Shared by the weight path and the all-ones
// pass, so the two round identically.
__device__ __forceinline__ void group_mma_b(float (&c)[4], uint32_t ax, uint32_t ay, uint32_t bx, uint32_t by,
                                            const uint4 &x0, const uint4 &x1, const uint4 &x2, const uint4 &x3) {
    const uint32_t ax5 = ax >> 10, ay5 = ay >> 10, bx5 = bx >> 10, by5 = by >> 10;
    mma_zero(c, ax & 0x00030003u, bx & 0x00030003u, ay & 0x00030003u, by & 0x00030003u, x0.x, x0.y);
    mma_acc(c, ax & 0x000C000Cu, bx & 0x000C000Cu, ay & 0x000C000Cu, by & 0x000C000Cu, x0.z, x0.w);
    mma_acc(c, ax & 0x00300030u, bx & 0x00300030u, ay & 0x00300030u, by & 0x00300030u, x1.x, x1.y);
    mma_acc(c, ax & 0x00C000C0u, bx & 0x00C000C0u, ay & 0x00C000C0u, by & 0x00C000C0u, x1.z, x1.w);
    mma_acc(c, ax & 0x03000300u, bx & 0x03000300u, ay & 0x03000300u, by & 0x03000300u, x2.x, x2.y);
    mma_acc(c, ax5 & 0x00030003u, bx5 & 0x00030003u, ay5 & 0x00030003u, by5 & 0x00030003u, x2.z, x2.w);
    mma_acc(c, ax5 & 0x000C000Cu, bx5 & 0x000C000Cu, ay5 & 0x000C000Cu, by5 & 0x000C000Cu, x3.x, x3.y);
    mma_acc(c, ax5 & 0x00300030u, bx5 & 0x00300030u, ay5 & 0x00300030u, by5 & 0x00300030u, x3.z, x3.w);
}

// The four B-fragment loads of one group (chunks of MT x 32 x 8 halves).
template <int MT>
__device__ __forceinline__ void load_xfrag(const __half *xb, uint4 (&xf)[4]) {
    constexpr int kChunk = MT * 32;
#pragma unroll
    for (int i = 0; i < 4; i++) xf[i] = *reinterpret_cast<const uint4 *>(xb + i * kChunk);
}

template <int MT>
__device__ __forceinline__ void group_mma(float (&c)[4], uint32_t ax, uint32_t ay, uint32_t bx, uint32_t by,
                                          const __half *xb) {
    uint4 xf[4];
    load_xfrag<MT>(xb, xf);
    group_mma_b(c, ax, ay, bx, by, xf[0], xf[1], xf[2], xf[3]);
}

// Lane q's pick among four values (q = 0..3).
__device__ __forceinline__ float sel4(int q, float a, float b, float c, float d) {
    const float lo = (q & 1) ? b : a;
    const float hi = (q & 1) ? d : c;
    return (q & 2) ? hi : lo;
}

// The same pick as a dot product with the one-hot weights m = (q == 0..3),
// on the floating-point pipe instead of the integer one (exact for finite
// values: the other terms are +-0 and adding them changes nothing).
__device__ __forceinline__ float pick4(const float4 &m, float a, float b, float c, float d) {
    return fmaf(m.w, d, fmaf(m.z, c, fmaf(m.y, b, m.x * a)));
}

// Tile row read by mma row g (row g + 8 reads tile row tile_row(g) + 8): the
// rows of one half warp fall on distinct shared-memory banks for 128-byte
// and 272-byte row strides alike.
__device__ __forceinline__ int tile_row(int g) { return g < 4 ? 2 * g : 2 * g - 7; }

// One 16-row x 1024-k slice at M = 1 in the group-per-column form: the eight
// scale groups of the slice sit in the eight B columns (group n = column n, x
// staged by xs_pair_index<8> with the group as the "token"), weight group G
// runs its eight-mma chain into its own accumulator, and only column G of it
// is kept.  wd[G] = {row g word 2q, row g+8 word 2q, row g word 2q+1, row g+8
// word 2q+1} of group G (overwritten).  The mmas go field by field (j outer,
// group inner), so eight independent chains separate two dependent mmas.
// Returns, for lane (g, q): v0 / v2 = group 2q of rows g / g+8, v1 / v3 =
// group 2q+1 of rows g / g+8 (qm = one-hot (q == 0..3) as floats).  The chain per group is the one group_mma_b
// runs, so the all-ones pass through group_mma_b rounds identically.
__device__ __forceinline__ void gc_slice(uint32_t (&wd)[8][4], const uint4 (&xf)[4], const float4 &qm, float &v0,
                                         float &v1, float &v2, float &v3) {
    float dd[8][4];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        if (j == 5) {
#pragma unroll
            for (int G8 = 0; G8 < 8; G8++)
#pragma unroll
                for (int i = 0; i < 4; i++) wd[G8][i] >>= 10;
        }
        const uint32_t m = 0x00030003u << (2 * (j < 5 ? j : j - 5));
        const uint4 &xv = xf[j >> 1];
        const uint32_t b0 = (j & 1) ? xv.z : xv.x, b1 = (j & 1) ? xv.w : xv.y;
#pragma unroll
        for (int G8 = 0; G8 < 8; G8++) {
            if (j == 0)
                mma_zero(dd[G8], wd[G8][0] & m, wd[G8][1] & m, wd[G8][2] & m, wd[G8][3] & m, b0, b1);
            else
                mma_acc(dd[G8], wd[G8][0] & m, wd[G8][1] & m, wd[G8][2] & m, wd[G8][3] & m, b0, b1);
        }
    }
    v0 = pick4(qm, dd[0][0], dd[2][0], dd[4][0], dd[6][0]);
    v1 = pick4(qm, dd[1][1], dd[3][1], dd[5][1], dd[7][1]);
    v2 = pick4(qm, dd[0][2], dd[2][2], dd[4][2], dd[6][2]);
    v3 = pick4(qm, dd[1][3], dd[3][3], dd[5][3], dd[7][3]);
}

// The lane's own columns of the eight per-group accumulators of a
// group-per-column slice (dd[G] = group G's chain; the column map is the one
// gcm_slice describes).
template <int MG>
__device__ __forceinline__ void gc_pick(const float (&dd)[8][4], const float4 &qm, const float2 &qh,
                                        float (&out)[MG][4]) {
    if (MG == 1) {
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const int o = c & 1;  // column 2q + o: group 2q + o
            out[0][c] = pick4(qm, dd[o][c], dd[2 + o][c], dd[4 + o][c], dd[6 + o][c]);
        }
    } else if (MG == 2) {
#pragma unroll
        for (int h = 0; h < MG; h++)
#pragma unroll
            for (int c = 0; c < 4; c++)
                out[h][c] = pick4(qm, dd[4 * h][c], dd[4 * h + 1][c], dd[4 * h + 2][c], dd[4 * h + 3][c]);
    } else {
#pragma unroll
        for (int h = 0; h < MG; h++)
#pragma unroll
            for (int c = 0; c < 4; c++) out[h][c] = fmaf(qh.y, dd[(2 * h + 1) % 8][c], qh.x * dd[(2 * h) % 8][c]);
    }
}

// Group-per-column slice for MG token rows (MG = 1, 2 or 4): the eight B
// columns carry (group, token) pairs, column n = group n / MG of a "set",
// token n % MG; a 1024-k slice has MG sets of 8 / MG groups, staged by
// xs_pair_index<8>(column, set * 128 + k % 128), so `xs` (the lane's
// fragments of the slice's first set) reaches set h at xs + 1024 h.  Weight
// group G (set G / (8/MG)) runs its eight-mma chain into its own accumulator;
// only the columns of its own group are kept.  Lane (g, q) holds columns 2q,
// 2q+1 of every set: out[h][0..1] = row g, out[h][2..3] = row g+8, for
//   MG = 1: groups 2q, 2q+1 (token 0);
//   MG = 2: group 4h + q, tokens 0, 1;
//   MG = 4: group 2h + q/2, tokens 2(q%2), 2(q%2)+1.
// qm = one-hot (q == 0..3), qh = one-hot (q/2 == 0..1), as floats.  The chain
// per group is the one group_mma_b runs (same fragments, same order), so the
// all-ones pass through group_mma_b rounds identically.
template <int MG>
__device__ __forceinline__ void gcm_slice(uint32_t (&wd)[8][4], const __half *xs, const float4 &qm, const float2 &qh,
                                          float (&out)[MG][4]) {
    constexpr int GPB = 8 / MG;  // groups per set
    float dd[8][4];
    uint4 xq[MG];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        if ((j & 1) == 0) {
#pragma unroll
            for (int h = 0; h < MG; h++) xq[h] = *reinterpret_cast<const uint4 *>(xs + h * 1024 + (j >> 1) * 256);
        }
        if (j == 5) {
#pragma unroll
            for (int G8 = 0; G8 < 8; G8++)
#pragma unroll
                for (int i = 0; i < 4; i++) wd[G8][i] >>= 10;
        }
        const uint32_t m = 0x00030003u << (2 * (j < 5 ? j : j - 5));
#pragma unroll
        for (int G8 = 0; G8 < 8; G8++) {
            const uint4 &xv = xq[G8 / GPB];
            const uint32_t b0 = (j & 1) ? xv.z : xv.x, b1 = (j & 1) ? xv.w : xv.y;
            if (j == 0)
                mma_zero(dd[G8], wd[G8][0] & m, wd[G8][1] & m, wd[G8][2] & m, wd[G8][3] & m, b0, b1);
            else
                mma_acc(dd[G8], wd[G8][0] & m, wd[G8][1] & m, wd[G8][2] & m, wd[G8][3] & m, b0, b1);
        }
    }
    gc_pick<MG>(dd, qm, qh, out);
}

// ---- the 1-bit variant: weights in {-1, +1}, one bit b = (t + 1) / 2 each,
// weight k of a row at bit k % 8 of byte k / 8 ("Bonsai 27B ternary / 1-bit
// quantization", ThakiCloud blog, section "What it is") ----
//
// A 32-bit word holds 32 consecutive weights of one row; its "pair p"
// (p = 0..15) is bit p of both 16-bit halves (weights p and p + 16).  One AND
// with 0x00010001 << p' (p' = p for p < 8; the word shifted right by 8 and
// p' = p - 8 otherwise) leaves an fp16 pair whose halves are the subnormals
// b * 2^(p' - 24), exactly.  mma i (0..7) of a 16-row x 128-k group takes
// pairs 2i (A registers a0, a1: rows g, g+8) and 2i + 1 (a2, a3) of the
// lane's word q of rows g and g+8, so one mma sees the factors 2^(2i & 7)
// and 2^((2i+1) & 7); the staged x carries their inverses (b1_xs_index).
// With t = 2b - 1 a group's sum is 2 D(bits) - D(all ones), D(all ones)
// from the very same chain on the all-ones word.

// Index (in halves) of x at k = kl (0..127 inside the group) of column col
// in the 1-bit staging area of one set: per mma pair (chunk c = mmas 2c,
// 2c + 1) and lane (col, q) eight halves [mma & 1][pair & 1][half], so the
// B fragments of two mmas are one 16-byte load, as for the ternary layout.
__device__ __forceinline__ int b1_xs_index(int col, int kl) {
    const int q = (kl >> 5) & 3;
    const int hi = (kl >> 4) & 1;
    const int p = kl & 15;
    return (((p >> 2) * 8 + col) * 4 + q) * 8 + ((p >> 1) & 1) * 4 + (p & 1) * 2 + hi;
}

// The A registers of mma i from the lane's words (w0 = row g, w1 = row g+8),
// already shifted right by 8 for i >= 4.
__device__ __forceinline__ void b1_a_regs(int i, uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
    const uint32_t m0 = 0x00010001u << ((2 * i) & 7), m1 = 0x00010001u << ((2 * i + 1) & 7);
    a[0] = w0 & m0;
    a[1] = w1 & m0;
    a[2] = w0 & m1;
    a[3] = w1 & m1;
}

// D(all ones) of one set's column: the eight-mma chain b1_slice runs for a
// group, on the all-ones word (every A register is its mask), with the B
// fragments at xb (the lane's eight halves of chunk 0; chunk c at + 256 c).
__device__ __forceinline__ void b1_ones_chain(float (&c)[4], const __half *xb) {
    uint4 xf[4];
    load_xfrag<8>(xb, xf);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        uint32_t a[4];
        b1_a_regs(i, 0xFFFFFFFFu, 0xFFFFFFFFu, a);
        const uint4 &xv = xf[i >> 1];
        const uint32_t b0 = (i & 1) ? xv.z : xv.x, b1 = (i & 1) ? xv.w : xv.y;
        if (i == 0)
            mma_zero(c, a[0], a[1], a[2], a[3], b0, b1);
        else
            mma_acc(c, a[0], a[1], a[2], a[3], b0, b1);
    }
}

// The 1-bit group-per-column slice (same columns, sets and outputs as
// gcm_slice): wd[G] = {row g word q, row g+8 word q} of group G
// (overwritten).  The mmas go i outer, group inner: eight independent chains.
template <int MG>
__device__ __forceinline__ void b1_slice(uint32_t (&wd)[8][2], const __half *xs, const float4 &qm, const float2 &qh,
                                         float (&out)[MG][4]) {
    constexpr int GPB = 8 / MG;  // groups per set
    float dd[8][4];
    uint4 xq[MG];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        if ((i & 1) == 0) {
#pragma unroll
            for (int h = 0; h < MG; h++) xq[h] = *reinterpret_cast<const uint4 *>(xs + h * 1024 + (i >> 1) * 256);
        }
        if (i == 4) {
#pragma unroll
            for (int G8 = 0; G8 < 8; G8++) {
                wd[G8][0] >>= 8;
                wd[G8][1] >>= 8;
            }
        }
#pragma unroll
        for (int G8 = 0; G8 < 8; G8++) {
            const uint4 &xv = xq[G8 / GPB];
            const uint32_t b0 = (i & 1) ? xv.z : xv.x, b1 = (i & 1) ? xv.w : xv.y;
            uint32_t a[4];
            b1_a_regs(i, wd[G8][0], wd[G8][1], a);
            if (i == 0)
                mma_zero(dd[G8], a[0], a[1], a[2], a[3], b0, b1);
            else
                mma_acc(dd[G8], a[0], a[1], a[2], a[3], b0, b1);
        }
    }
    gc_pick<MG>(dd, qm, qh, out);
}

}  // namespace tern
