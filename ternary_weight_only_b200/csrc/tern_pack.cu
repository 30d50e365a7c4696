// Slot packing and unpacking for the ternary-g128 format.
//
// The format: t in {-1,0,+1} per weight and one fp16 scale per 128 weights
// along K ("Bonsai 27B ternary / 1-bit quantization", ThakiCloud blog,
// section "How compression works"), stored in 2-bit slots ("Ternary
// quantization: 27B in 7 GB", devnsb blog, section "Limits").  The byte
// layout (code c = t + 1, four codes per byte, least significant pair first)
// is the one documented in tern.h.
//
// Both kernels are plain streaming kernels: every thread turns 16 consecutive
// int8 codes (one 16-byte load) into one 32-bit slot word, so code j of the
// chunk lands at bit 2j of the word -- byte j/4, bit pair j%4.
//
// The 1-bit variant (weights in {-1, +1} with the same fp16 scale per 128
// weights: "Bonsai 27B ternary / 1-bit quantization", ThakiCloud blog,
// sections "What it is" and "How compression works") packs one bit
// b = (t + 1) / 2 per weight, weight k of a row at bit k % 8 of byte k / 8:
// a thread turns 32 codes (two 16-byte loads) into one 32-bit word, code j
// at bit j.
//
// The five-per-byte packing (the denser "native ternary" storage the pages
// expect: "Ternary-Bonsai-27B" model summary, aitrends.kr, sections "TL;DR"
// and "Technical features"; "Ternary quantization: 27B in 7 GB", devnsb blog,
// section "Limits") is documented in tern.h: base-3 digits c = t + 1, five
// per byte, 26 bytes per 128-weight group, rows padded to 16 bytes.  A
// thread packs or unpacks one group of one row.
#include "tern_internal.cuh"

namespace tern {
namespace {

constexpr int kPackThreads = 256;

__device__ __forceinline__ uint32_t code_of(int t, int &bad) {
    // t in {-1,0,1} -> t + 1; anything else -> 3 (invalid)
    const bool ok = (t >= -1) && (t <= 1);
    bad += ok ? 0 : 1;
    return ok ? static_cast<uint32_t>(t + 1) : 3u;
}

__global__ void __launch_bounds__(kPackThreads) pack_kernel(const int4 *__restrict__ codes,
                                                            uint32_t *__restrict__ slots,
                                                            int64_t nchunks,
                                                            const uint16_t *__restrict__ sc_in,
                                                            uint16_t *__restrict__ sc_out,
                                                            int64_t nscales,
                                                            int32_t *invalid_count) {
    int bad = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nchunks;
         i += stride) {
        const int4 v = codes[i];
        const uint32_t w4[4] = {static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y),
                                static_cast<uint32_t>(v.z), static_cast<uint32_t>(v.w)};
        uint32_t out = 0;
#pragma unroll
        for (int b = 0; b < 4; b++) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int t = static_cast<int8_t>((w4[b] >> (8 * j)) & 0xFF);
                out |= code_of(t, bad) << (2 * (4 * b + j));
            }
        }
        slots[i] = out;
    }
    if (sc_out != nullptr) {
        for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nscales;
             i += stride)
            sc_out[i] = sc_in[i];
    }
    if (invalid_count != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
        if ((threadIdx.x & 31) == 0 && bad != 0) atomicAdd(invalid_count, bad);
    }
}

__global__ void __launch_bounds__(kPackThreads) unpack_kernel(const uint32_t *__restrict__ slots,
                                                              int4 *__restrict__ codes,
                                                              int64_t nchunks) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nchunks;
         i += stride) {
        const uint32_t w = slots[i];
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; b++) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t c = (w >> (2 * (4 * b + j))) & 3u;
                // c - 1 for c in {0,1,2}; the sentinel 2 for the invalid code 3
                const int t = (c == 3u) ? 2 : static_cast<int>(c) - 1;
                word |= (static_cast<uint32_t>(t) & 0xFFu) << (8 * j);
            }
            o[b] = word;
        }
        codes[i] = make_int4(static_cast<int>(o[0]), static_cast<int>(o[1]),
                             static_cast<int>(o[2]), static_cast<int>(o[3]));
    }
}

__global__ void __launch_bounds__(kPackThreads) pack_b1_kernel(const int4 *__restrict__ codes,
                                                               uint32_t *__restrict__ bits, int64_t nwords,
                                                               const uint16_t *__restrict__ sc_in,
                                                               uint16_t *__restrict__ sc_out, int64_t nscales,
                                                               int32_t *invalid_count) {
    int bad = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords; i += stride) {
        const int4 v0 = codes[2 * i], v1 = codes[2 * i + 1];
        const uint32_t w8[8] = {static_cast<uint32_t>(v0.x), static_cast<uint32_t>(v0.y),
                                static_cast<uint32_t>(v0.z), static_cast<uint32_t>(v0.w),
                                static_cast<uint32_t>(v1.x), static_cast<uint32_t>(v1.y),
                                static_cast<uint32_t>(v1.z), static_cast<uint32_t>(v1.w)};
        uint32_t out = 0;
#pragma unroll
        for (int b = 0; b < 8; b++) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int t = static_cast<int8_t>((w8[b] >> (8 * j)) & 0xFF);
                // +1 -> bit 1; -1 -> bit 0; anything else -> bit 0, counted
                bad += (t == 1 || t == -1) ? 0 : 1;
                out |= static_cast<uint32_t>(t == 1) << (4 * b + j);
            }
        }
        bits[i] = out;
    }
    if (sc_out != nullptr) {
        for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nscales; i += stride)
            sc_out[i] = sc_in[i];
    }
    if (invalid_count != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
        if ((threadIdx.x & 31) == 0 && bad != 0) atomicAdd(invalid_count, bad);
    }
}

__global__ void __launch_bounds__(kPackThreads) unpack_b1_kernel(const uint32_t *__restrict__ bits,
                                                                 int4 *__restrict__ codes, int64_t nwords) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords; i += stride) {
        const uint32_t w = bits[i];
        uint32_t o[8];
#pragma unroll
        for (int b = 0; b < 8; b++) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t t = ((w >> (4 * b + j)) & 1u) ? 0x01u : 0xFFu;  // +1 or -1 as int8
                word |= t << (8 * j);
            }
            o[b] = word;
        }
        codes[2 * i] = make_int4(static_cast<int>(o[0]), static_cast<int>(o[1]), static_cast<int>(o[2]),
                                 static_cast<int>(o[3]));
        codes[2 * i + 1] = make_int4(static_cast<int>(o[4]), static_cast<int>(o[5]), static_cast<int>(o[6]),
                                     static_cast<int>(o[7]));
    }
}

constexpr int kT5Bytes = 26;  // bytes per 128-weight group

__global__ void __launch_bounds__(kPackThreads) pack_t5_kernel(const int8_t *__restrict__ codes, uint8_t *__restrict__ out,
                                                               int64_t N, int64_t K, int64_t R,
                                                               const uint16_t *__restrict__ sc_in,
                                                               uint16_t *__restrict__ sc_out, int32_t *invalid_count) {
    const int64_t G = K / kGroup;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int bad = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N * G; i += stride) {
        const int64_t n = i / G, g = i - n * G;
        const int4 *src = reinterpret_cast<const int4 *>(codes + n * K + g * kGroup);
        uint8_t c[kGroup];
#pragma unroll
        for (int v = 0; v < 8; v++) {
            const int4 w = src[v];
            const uint32_t w4[4] = {static_cast<uint32_t>(w.x), static_cast<uint32_t>(w.y),
                                    static_cast<uint32_t>(w.z), static_cast<uint32_t>(w.w)};
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int t = static_cast<int8_t>((w4[b >> 2] >> (8 * (b & 3))) & 0xFF);
                const bool ok = t >= -1 && t <= 1;
                bad += ok ? 0 : 1;
                c[v * 16 + b] = static_cast<uint8_t>(ok ? t + 1 : 1);  // an invalid code is stored as t = 0
            }
        }
        uint16_t *dst = reinterpret_cast<uint16_t *>(out + n * R + g * kT5Bytes);  // 2-byte aligned
#pragma unroll
        for (int h = 0; h < kT5Bytes / 2; h++) {
            uint32_t v2[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int j = 2 * h + e;  // byte j of the group: weights 5j .. 5j+4 (125..127 for j = 25)
                uint32_t v = 0;
#pragma unroll
                for (int d = 4; d >= 0; d--)
                    if (5 * j + d < kGroup) v = 3 * v + c[5 * j + d];
                    else v = 3 * v;
                v2[e] = v;
            }
            dst[h] = static_cast<uint16_t>(v2[0] | (v2[1] << 8));
        }
        if (g == G - 1)
            for (int64_t b = G * kT5Bytes; b < R; b++) out[n * R + b] = 0;  // row padding
    }
    if (sc_out != nullptr) {
        for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N * G; i += stride)
            sc_out[i] = sc_in[i];
    }
    if (invalid_count != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
        if ((threadIdx.x & 31) == 0 && bad != 0) atomicAdd(invalid_count, bad);
    }
}

__global__ void __launch_bounds__(kPackThreads) unpack_t5_kernel(const uint8_t *__restrict__ in, int8_t *__restrict__ codes,
                                                                 int64_t N, int64_t K, int64_t R) {
    const int64_t G = K / kGroup;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N * G; i += stride) {
        const int64_t n = i / G, g = i - n * G;
        const uint16_t *src = reinterpret_cast<const uint16_t *>(in + n * R + g * kT5Bytes);
        uint32_t t4[kGroup / 4];
#pragma unroll
        for (int w = 0; w < kGroup / 4; w++) t4[w] = 0;
#pragma unroll
        for (int h = 0; h < kT5Bytes / 2; h++) {
            const uint32_t pair = src[h];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int j = 2 * h + e;
                uint32_t v = (pair >> (8 * e)) & 0xFF;
                const bool ok = v < 243;
#pragma unroll
                for (int d = 0; d < 5; d++) {
                    const int k = 5 * j + d;
                    const uint32_t t = ok ? (v % 3) - 1 : 2;  // t = c - 1, or the sentinel 2
                    v /= 3;
                    if (k < kGroup) t4[k >> 2] |= (t & 0xFFu) << (8 * (k & 3));
                }
            }
        }
        int4 *dst = reinterpret_cast<int4 *>(codes + n * K + g * kGroup);
#pragma unroll
        for (int v = 0; v < 8; v++)
            dst[v] = make_int4(static_cast<int>(t4[4 * v]), static_cast<int>(t4[4 * v + 1]),
                               static_cast<int>(t4[4 * v + 2]), static_cast<int>(t4[4 * v + 3]));
    }
}

int grid_for(int64_t work, int sms) {
    const int64_t want = (work + kPackThreads - 1) / kPackThreads;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace

tern_status launch_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K,
                        uint8_t *slots, uint16_t *scales_out, int32_t *invalid_count,
                        cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    const int64_t nchunks = N * K / 16;
    const int64_t nscales = N * (K / kGroup);
    const uint16_t *sin = scales_in;
    uint16_t *sout = (scales_in == scales_out) ? nullptr : scales_out;
    pack_kernel<<<grid_for(nchunks, dev.sms), kPackThreads, 0, stream>>>(
        reinterpret_cast<const int4 *>(codes), reinterpret_cast<uint32_t *>(slots), nchunks, sin,
        sout, nscales, invalid_count);
    return cuda_fail(cudaGetLastError(), "pack kernel launch");
}

tern_status launch_unpack(const uint8_t *slots, int64_t N, int64_t K, int8_t *codes,
                          cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    const int64_t nchunks = N * K / 16;
    unpack_kernel<<<grid_for(nchunks, dev.sms), kPackThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(slots), reinterpret_cast<int4 *>(codes), nchunks);
    return cuda_fail(cudaGetLastError(), "unpack kernel launch");
}

tern_status launch_pack_b1(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bits,
                           uint16_t *scales_out, int32_t *invalid_count, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    const int64_t nwords = N * K / 32;
    const int64_t nscales = N * (K / kGroup);
    uint16_t *sout = (scales_in == scales_out) ? nullptr : scales_out;
    pack_b1_kernel<<<grid_for(nwords, dev.sms), kPackThreads, 0, stream>>>(
        reinterpret_cast<const int4 *>(codes), reinterpret_cast<uint32_t *>(bits), nwords, scales_in, sout, nscales,
        invalid_count);
    return cuda_fail(cudaGetLastError(), "1-bit pack kernel launch");
}

tern_status launch_unpack_b1(const uint8_t *bits, int64_t N, int64_t K, int8_t *codes, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    const int64_t nwords = N * K / 32;
    unpack_b1_kernel<<<grid_for(nwords, dev.sms), kPackThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t *>(bits), reinterpret_cast<int4 *>(codes), nwords);
    return cuda_fail(cudaGetLastError(), "1-bit unpack kernel launch");
}

int64_t t5_row_bytes(int64_t K) { return (K / kGroup * kT5Bytes + 15) / 16 * 16; }

tern_status launch_pack_t5(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *out,
                           uint16_t *scales_out, int32_t *invalid_count, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    uint16_t *sout = (scales_in == scales_out) ? nullptr : scales_out;
    pack_t5_kernel<<<grid_for(N * (K / kGroup), dev.sms), kPackThreads, 0, stream>>>(
        codes, out, N, K, t5_row_bytes(K), scales_in, sout, invalid_count);
    return cuda_fail(cudaGetLastError(), "five-per-byte pack kernel launch");
}

tern_status launch_unpack_t5(const uint8_t *in, int64_t N, int64_t K, int8_t *codes, cudaStream_t stream) {
    DeviceInfo dev;
    tern_status st = current_device(&dev);
    if (st != TERN_OK) return st;
    unpack_t5_kernel<<<grid_for(N * (K / kGroup), dev.sms), kPackThreads, 0, stream>>>(in, codes, N, K,
                                                                                       t5_row_bytes(K));
    return cuda_fail(cudaGetLastError(), "five-per-byte unpack kernel launch");
}

}  // namespace tern
