// Internal declarations shared by the CUDA sources of libtern (not installed).
#pragma once

#include <cuda.h>
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
    int gemm_min_m = 0;
    int gemv_variant = 0;
    int gemv_grid = 0;
    int gemv_prefetch = 0;
    int step_form = 0;
};
extern Options g_opt;

// ---- launchers (defined in the kernel sources) ----------------------------
tern_status launch_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K,
                        uint8_t *slots, uint16_t *scales_out, int32_t *invalid_count,
                        cudaStream_t stream);
tern_status launch_unpack(const uint8_t *slots, int64_t N, int64_t K, int8_t *codes,
                          cudaStream_t stream);
// the 1-bit variant: bits uint8 [N][K/8], weight k at bit k % 8 of byte k / 8
tern_status launch_pack_b1(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bits,
                           uint16_t *scales_out, int32_t *invalid_count, cudaStream_t stream);
tern_status launch_unpack_b1(const uint8_t *bits, int64_t N, int64_t K, int8_t *codes, cudaStream_t stream);
// five trits per byte: uint8 [N][t5_row_bytes(K)], 26 bytes per 128-weight group
int64_t t5_row_bytes(int64_t K);
tern_status launch_pack_t5(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *out,
                           uint16_t *scales_out, int32_t *invalid_count, cudaStream_t stream);
tern_status launch_unpack_t5(const uint8_t *in, int64_t N, int64_t K, int8_t *codes, cudaStream_t stream);

struct MatDesc {
    const __half *x;
    const uint8_t *slots;
    const __half *scales;
    __half *y;
    int N, K;
    // Step kernel only: the full row length of x, slots and scales when the
    // product covers a K segment of a wider matrix (0: K), and whether the
    // result is added to y instead of written.
    int kfull = 0;
    int accum = 0;
};
// Bandwidth-bound product for M in [1,8] over `count` matrices in one launch:
// TMA-staged kernel (default) and the register-ring kernel (variant 1).
tern_status launch_gemv_tma(const MatDesc *d, int count, int M, cudaStream_t stream);
// Producer/consumer form of the same kernel (K a multiple of 1024, x small).
bool gemv_pc_supports(const MatDesc *d, int count, int M, bool token_columns);
// M = 1 uses the group-per-column form unless token_columns is set.
tern_status launch_gemv_pc(const MatDesc *d, int count, int M, bool token_columns, cudaStream_t stream);
// Tensor-core (tcgen05) bandwidth kernel for M in [1,4]; splits tiles along K
// when a large enough zero-initialised workspace is given.
tern_status launch_gemv_tc(const MatDesc *d, int count, int M, void *workspace, size_t ws_bytes,
                           cudaStream_t stream);
size_t gemv_tc_workspace_bytes(const MatDesc *d, int count, int M, int sms);
// M = 1 product of the tcgen05 kernel with its scratch in a static device area.
tern_status gemv_noalloc(const MatDesc &d, cudaStream_t stream);
// Partition of a grouped bandwidth launch: for each matrix i with ntile[i]
// 16-row tiles and between nbmin[i] and nbc[i] k-slices per CTA, choose
// Pout[i] warps per tile (power of two, <= nbmin[i]) and cl_out[i] CTAs (or
// clusters) within `cap` in total (see tern_gemv_tma.cu).
tern_status plan_partition(const int *ntile, const int *nbc, const int *nbmin, int count, int warps,
                           long long cap, int forced_P, int *Pout, long long *cl_out);
// 2-D tiled tensor map (row-major: `inner` contiguous elements per row, `outer`
// rows `row_bytes` apart) for TMA loads of `box_inner` x `box_outer` boxes.
tern_status encode_tiled_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                            uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                            CUtensorMapSwizzle swizzle);
// Rank-3 tiled map: dims[0] innermost (elements), strides[] in bytes for
// dims 1 and 2 (multiples of 16), box[] in elements.
tern_status encode_tiled_3d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, const uint64_t dims[3],
                            const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle);
// Tensor-core prefill product (any M; meant for large M).
tern_status launch_gemm_tc(const MatDesc &d, int M, cudaStream_t stream);
// Device-side status words written by bounded waits that gave up (one per
// kernel source file; read and optionally cleared).
tern_status read_gemm_status(bool reset, unsigned int *out);
tern_status read_gemv_status(bool reset, unsigned int *out);
tern_status read_gemvtc_status(bool reset, unsigned int *out);
tern_status read_gemvpc_status(bool reset, unsigned int *out);
// Ternary embedding rows gathered by id, written as fp16 s * t.
tern_status launch_embed(const int32_t *ids, int64_t M, const uint8_t *slots, const uint16_t *scales, int64_t V,
                         int64_t K, uint16_t *out, int32_t *bad_count, cudaStream_t stream);
// Persistent launch over many matrices (M = 1..8, 1..4 for fmt 1; K multiples of 1024); fmt 0
// = ternary slots, 1 = the 1-bit variant (MatDesc::slots holds the bits), 2 =
// five trits per byte (MatDesc::slots holds the base-3 bytes).
// x8: the digit form (M <= 4) or the fp16 group-per-column form.
bool gemv_step_supports(const MatDesc *d, int count, int M, int fmt, bool x8);
// whether one product of depth K at M token rows fits the step kernel
bool gemv_step_fits(int K, int M, int fmt, bool x8);
// the form the step kernels use by default for M token rows (TERN_OPT_STEP_FORM)
bool gemv_step_digit_form(int M, int fmt);
tern_status launch_gemv_step(const MatDesc *d, int count, int M, int fmt, bool x8, cudaStream_t stream);
// The CTA ranges one launch of the step kernel uses for these shapes on
// `grid` CTAs: first_tile[0..grid] (host only).
tern_status gemv_step_plan(const int64_t *N, const int64_t *K, int count, int M, int grid, int32_t *first_tile);
tern_status read_gemvstep_status(bool reset, unsigned int *out);
extern unsigned long long g_gemm_timeout_ns;
extern int g_gemm_skip_loads;

// ---- debug build: in-kernel index checks -----------------------------------
// Compiled with -DTERN_DEBUG_GUARDS, TERN_GUARD(ok, counter) counts a failed
// check in the device word `counter` and yields false, so that the access it
// protects is skipped (no trap, the context stays usable); in the normal
// build it is the constant true and costs nothing.
#ifdef TERN_DEBUG_GUARDS
#define TERN_GUARD(ok, counter) (tern::guard_check((ok), &(counter)))
#else
#define TERN_GUARD(ok, counter) true
#endif
__device__ __forceinline__ bool guard_check(bool ok, unsigned int *counter) {
    if (!ok) atomicAdd(counter, 1u);
    return ok;
}
// Failed index checks of the step kernel since the last read (0 in the normal build).
tern_status read_gemvstep_guard(bool reset, unsigned int *out);

// ---- device helpers -------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}


// As mbar_try_wait, but the thread may sleep in hardware up to `hint_ns`
// nanoseconds while the phase is incomplete (it wakes when the phase
// completes), so a waiting warp does not spin through issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Bring a tile of a tensor into L2 only (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int c0, int c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map), "r"(c0), "r"(c1),
                 "r"(c2)
                 : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

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

// D = A * B (C = 0), m16n8k16, fp16 inputs, fp32 result: the zero
// accumulator is an immediate operand, so no registers are cleared for it.
__device__ __forceinline__ void mma_16816_zc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
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


// Two fp16 codes -> exact fp16 ternary pair.  One LOP3 places the 2-bit code c
// of two weights into the mantissas of an fp16 pair whose exponent field makes
// each half 1024 + c*4^j (j = bit pair inside the half); one HFMA2 with the
// constants (4^-j, -(1024*4^-j + 1)) gives c - 1 = t exactly, because every
// intermediate is an exactly representable fp16 value.  Pair j of a 32-bit
// slot word holds weights j (low half) and j+8 (high half).  Code 3 (invalid)
// gives 2, a finite value.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t (&t)[8]) {
    constexpr uint32_t kExp = 0x64006400u;  // fp16 1024.0 in both halves
    const uint32_t w10 = w >> 10;
    t[0] = hfma2_u32(lop3_and_or(w, 0x00030003u, kExp), 0x3C003C00u, 0xE401E401u);  // *1     -1025
    t[1] = hfma2_u32(lop3_and_or(w, 0x000C000Cu, kExp), 0x34003400u, 0xDC04DC04u);  // *1/4   -257
    t[2] = hfma2_u32(lop3_and_or(w, 0x00300030u, kExp), 0x2C002C00u, 0xD410D410u);  // *1/16  -65
    t[3] = hfma2_u32(lop3_and_or(w, 0x00C000C0u, kExp), 0x24002400u, 0xCC40CC40u);  // *1/64  -17
    t[4] = hfma2_u32(lop3_and_or(w, 0x03000300u, kExp), 0x1C001C00u, 0xC500C500u);  // *1/256 -5
    t[5] = hfma2_u32(lop3_and_or(w10, 0x00030003u, kExp), 0x3C003C00u, 0xE401E401u);
    t[6] = hfma2_u32(lop3_and_or(w10, 0x000C000Cu, kExp), 0x34003400u, 0xDC04DC04u);
    t[7] = hfma2_u32(lop3_and_or(w10, 0x00300030u, kExp), 0x2C002C00u, 0xD410D410u);
}

// Index (in halves) of x[m][kl] in the "fragment order" staging area of the
// bandwidth kernels.  Unit = 4 halves {x[b+2r], x[b+2r+8], x[b+2r+1], x[b+2r+9]}
// with b the start of a 16-weight slot word, so that unit r is exactly the B
// fragment of the mma that consumes pairs 2r and 2r+1 of that word; units are
// laid out [group][word][m][lane q][r] so that a warp's fragment loads are
// contiguous (no bank conflicts).
__device__ __forceinline__ int xs_index(int m, int kl, int M) {
    const int grp = kl >> 7;
    const int kk = kl & 127;
    const int q = kk >> 5;
    const int wi = (kk >> 4) & 1;
    const int hi = (kk >> 3) & 1;
    const int j = kk & 7;
    const int unit = (((grp * 2 + wi) * M + m) * 4 + q) * 4 + (j >> 1);
    return unit * 4 + (j & 1) * 2 + hi;
}

__device__ __forceinline__ uint2 ldg_nc_u2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

}  // namespace tern
