// Internal declarations shared by the CUDA sources of libtern (not installed).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tern.h"

namespace tern {

constexpr int kGroup = 128;  // weights per fp16 scale along K

// ---- host-side error reporting (thread-local message) ----------------------
tern_status fail(tern_status st, const char *fmt, ...);
tern_status cuda_fail(cudaError_t e, const char *what);
void clear_error();

struct DeviceInfo {
    int device = -1;
    int sms = 0;
    int major = 0, minor = 0;
    size_t max_smem_optin = 0;
};
// Properties of the current device (cached per device).
tern_status current_device(DeviceInfo *out);

// Process-wide knobs (tern_set_option).
struct Options {
    int gemv_ksplit = 0;
    int gemv_cluster = 0;
    int gemv_ctas = 0;
    int gemm_path = 0;
};
extern Options g_opt;

// ---- launchers (defined in the kernel sources) ----------------------------
tern_status launch_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K,
                        uint8_t *slots, uint16_t *scales_out, int32_t *invalid_count,
                        cudaStream_t stream);
tern_status launch_unpack(const uint8_t *slots, int64_t N, int64_t K, int8_t *codes,
                          cudaStream_t stream);

struct MatDesc {
    const __half *x;
    const uint8_t *slots;
    const __half *scales;
    __half *y;
    int N, K;
};
// Bandwidth-bound product for M in [1,8] over `count` matrices in one launch.
tern_status launch_gemv_mma(const MatDesc *d, int count, int M, cudaStream_t stream);

// ---- device helpers -------------------------------------------------------
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
    // (a & b) | c
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// D = A * B + C, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float4 ld_shared_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint2 ldg_nc_u2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

}  // namespace tern
