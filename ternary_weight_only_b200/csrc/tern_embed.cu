// Ternary embedding lookup: rows of a ternary-g128 matrix gathered by token
// id and written out as fp16 s * t.
//
// The pages list the embeddings among the ternary matrices (the model keeps
// only normalisation and scale parameters in high precision: "Ternary-Bonsai-
// 27B" model summary, aitrends.kr, section "Differentiators"; "Bonsai 27B
// ternary / 1-bit quantization", ThakiCloud blog, section "What it is"), so a
// token's input vector is one row of such a matrix: out[m][k] = s[id][k/128] *
// t[id][k].  With tied weights the output head's slots and scales serve as
// the table.  s * t is exactly representable in fp16 (t is -1, 0 or +1).
//
// Bandwidth-bound streaming kernel.  A work item is 64 consecutive weights of
// one row; item f of the flat list (row f / (K/64), chunk f % (K/64)) fills
// bytes 128 f .. 128 f + 127 of `out`, so the 32 items of a warp fill one
// contiguous 4 KB stretch even across rows.  A lane loads its item's 16 bytes
// of slots and the row's scale of their group, turns each 16-code word into
// 16 exact fp16 values (LOP3 + HFMA2 per pair, a byte permute into k order,
// one HMUL2 by the scale) and puts its 128 bytes into a warp-private 4 KB of
// shared memory (16-byte slots XOR-swizzled by lane, so that neither
// direction has bank conflicts); the warp then writes the 4 KB with eight
// fully coalesced 512-byte stores.  Per row: K/4 + K/64 bytes read, 2K bytes
// written.
#include <cstring>

#include "tern_internal.cuh"

namespace tern {

namespace {

constexpr int kEmbedThreads = 128;
constexpr int kEmbedWarps = kEmbedThreads / 32;

__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// One slot word (16 codes) -> 16 fp16 values s * t in k order, as 8 pairs.
__device__ __forceinline__ void word_to_f16(uint32_t w, uint32_t s2, uint32_t (&o)[8]) {
    uint32_t p[8];  // p[j] = {t[j], t[j+8]}
    unpack_word(w, p);
#pragma unroll
    for (int c = 0; c < 4; c++) {
        o[c] = hmul2_bits(byte_perm(p[2 * c], p[2 * c + 1], 0x5410u), s2);      // {t[2c],   t[2c+1]}
        o[c + 4] = hmul2_bits(byte_perm(p[2 * c], p[2 * c + 1], 0x7632u), s2);  // {t[2c+8], t[2c+9]}
    }
}

// Grid-stride over warp items of 32 flat items each.
__global__ void __launch_bounds__(kEmbedThreads) embed_kernel(const int32_t *__restrict__ ids, int M,
                                                              const uint8_t *__restrict__ slots,
                                                              const __half *__restrict__ scales, int V, int K,
                                                              __half *__restrict__ out, int32_t *bad_count) {
    __shared__ uint4 stage[kEmbedWarps][32 * 8];  // 4 KB per warp
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint4 *wst = stage[warp];
    const long long nchunk = K / 64;
    const long long items = static_cast<long long>(M) * nchunk;
    const long long groups = (items + 31) / 32;
    for (long long gi = static_cast<long long>(blockIdx.x) * kEmbedWarps + warp; gi < groups;
         gi += static_cast<long long>(gridDim.x) * kEmbedWarps) {
        const long long f = gi * 32 + lane;
        uint32_t o[32];
        if (f < items) {
            const int m = static_cast<int>(f / nchunk);
            const int chunk = static_cast<int>(f - static_cast<long long>(m) * nchunk);
            const int id = __ldg(ids + m);
            const bool valid = id >= 0 && id < V;
            if (!valid && bad_count && chunk == 0) atomicAdd(bad_count, 1);
            if (valid) {
                const uint4 w = __ldg(reinterpret_cast<const uint4 *>(slots + static_cast<size_t>(id) * (K / 4)) + chunk);
                // 64 weights = half a group: one scale
                const uint16_t sb = __ldg(reinterpret_cast<const unsigned short *>(scales) +
                                          static_cast<size_t>(id) * (K / 128) + chunk / 2);
                const uint32_t s2 = static_cast<uint32_t>(sb) | (static_cast<uint32_t>(sb) << 16);
                const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 4; i++) word_to_f16(wv[i], s2, *reinterpret_cast<uint32_t(*)[8]>(o + 8 * i));
            } else {
#pragma unroll
                for (int i = 0; i < 32; i++) o[i] = 0u;
            }
        }
        // lane's 16-byte piece c (0..7) goes to slot c ^ (lane & 7) of its 128 bytes
        __syncwarp();
        if (f < items) {
#pragma unroll
            for (int c = 0; c < 8; c++)
                wst[lane * 8 + (c ^ (lane & 7))] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
        __syncwarp();
        // store j covers bytes 512 j .. 512 j + 511 of the warp's 4 KB: lane
        // takes 16-byte piece 32 j + lane, made by lane p = 4 j + lane / 8
        uint4 *dst = reinterpret_cast<uint4 *>(out) + gi * 256;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int piece = 32 * j + lane;
            const int p = piece >> 3, c = piece & 7;
            if (gi * 32 + p < items) dst[piece] = wst[p * 8 + (c ^ (p & 7))];
        }
    }
}

}  // namespace

tern_status launch_embed(const int32_t *ids, int64_t M, const uint8_t *slots, const uint16_t *scales, int64_t V,
                         int64_t K, uint16_t *out, int32_t *bad_count, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    const long long groups = (M * (K / 64) + 31) / 32;
    const long long want = (groups + kEmbedWarps - 1) / kEmbedWarps;
    const long long cap = static_cast<long long>(dev.sms) * 16;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    embed_kernel<<<grid, kEmbedThreads, 0, stream>>>(ids, static_cast<int>(M), slots,
                                                     reinterpret_cast<const __half *>(scales),
                                                     static_cast<int>(V), static_cast<int>(K),
                                                     reinterpret_cast<__half *>(out), bad_count);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "embed kernel launch");
    return TERN_OK;
}

}  // namespace tern
