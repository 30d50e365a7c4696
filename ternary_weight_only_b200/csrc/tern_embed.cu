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
// Bandwidth-bound streaming kernel: a thread takes 64 consecutive weights of
// one row (one 16-byte load of slots, the row's scale of their group), turns
// each 16-code word into 16 exact fp16 values (LOP3 + HFMA2 per pair, a byte
// permute into k order, one HMUL2 by the scale) and writes 128 bytes.  Per
// row: K/4 + K/64 bytes read, 2K bytes written.
#include <cstring>

#include "tern_internal.cuh"

namespace tern {

namespace {

constexpr int kEmbedThreads = 128;

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

// grid = (ceil(K / 64 / kEmbedThreads), min(M, 65535)): block (bx, by) writes
// chunk bx of rows by, by + gridDim.y, ...
__global__ void __launch_bounds__(kEmbedThreads) embed_kernel(const int32_t *__restrict__ ids, int M,
                                                              const uint8_t *__restrict__ slots,
                                                              const __half *__restrict__ scales, int V, int K,
                                                              __half *__restrict__ out, int32_t *bad_count) {
    const int chunk = blockIdx.x * kEmbedThreads + threadIdx.x;  // 64 weights each
    const int nchunk = K / 64;
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
        const int id = ids[m];
        const bool valid = id >= 0 && id < V;
        if (!valid && bad_count && blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(bad_count, 1);
        if (chunk >= nchunk) continue;
        uint4 *dst = reinterpret_cast<uint4 *>(out + static_cast<size_t>(m) * K + static_cast<size_t>(chunk) * 64);
        if (!valid) {
#pragma unroll
            for (int i = 0; i < 8; i++) dst[i] = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(slots + static_cast<size_t>(id) * (K / 4)) + chunk);
        // 64 weights = half a group: one scale
        const uint16_t sb = __ldg(reinterpret_cast<const unsigned short *>(scales) +
                                  static_cast<size_t>(id) * (K / 128) + chunk / 2);
        const uint32_t s2 = static_cast<uint32_t>(sb) | (static_cast<uint32_t>(sb) << 16);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            uint32_t o[8];
            word_to_f16(wv[i], s2, o);
            dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
    }
}

}  // namespace

tern_status launch_embed(const int32_t *ids, int64_t M, const uint8_t *slots, const uint16_t *scales, int64_t V,
                         int64_t K, uint16_t *out, int32_t *bad_count, cudaStream_t stream) {
    const int nchunk = static_cast<int>(K / 64);
    dim3 grid(static_cast<unsigned>((nchunk + kEmbedThreads - 1) / kEmbedThreads),
              static_cast<unsigned>(M < 65535 ? M : 65535));
    embed_kernel<<<grid, kEmbedThreads, 0, stream>>>(ids, static_cast<int>(M), slots,
                                                     reinterpret_cast<const __half *>(scales),
                                                     static_cast<int>(V), static_cast<int>(K),
                                                     reinterpret_cast<__half *>(out), bad_count);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "embed kernel launch");
    return TERN_OK;
}

}  // namespace tern
