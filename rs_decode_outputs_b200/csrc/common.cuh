// Device-side helpers shared by the ReplaySSM kernels: kernel parameters,
// element conversions, 16-byte chunk loads, 1-D bulk copies into shared memory
// completed on an mbarrier, bounded waits, and warp reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rs.h"

namespace rs {

// Everything a kernel needs to find a handle's data.  Built on the host from the
// workspace layout; passed by value.
struct Params {
    int kind, B, H, R, CC, G, cap, cap_mask, heads_per_group, capd;
    int in_dtype, out_dtype, copy_dtype, shared_lowp;
    float gdn_scale;
    size_t blk_r, blk_c;   // ring block strides in bytes: R-wide rows (x, v), CC-wide rows (q, k, B, C)
    float *master;       // fp32 [B][H][R][CC] (NULL with shared_lowp)
    void *copy;          // copy_dtype [B][H][R][CC] (NULL with RS_NONE)
    float *scale;        // fp32 [B][H] (E4M3)
    void *ra, *rb, *rc, *rd, *re;   // ring regions (see rs_layout)
    int32_t *head, *tail;
    uint32_t *err, *arrive;
    const float *A, *D;  // Mamba-2 [H]
    float *rec;          // scratch: Mamba-2 group records, then one replay record per (b, h) tile
    size_t rec_tile_off; // floats from rec to the first tile record
};

// Threads of the CTAs that hold a state tile in registers.
constexpr int kTileThreads = 256;

// Upper bound on a spin on an mbarrier, in SM clock cycles (about a second).
constexpr long long kWaitLimitCycles = 2000000000LL;

// ---------------------------------------------------------------- elements --

__device__ __forceinline__ float ld_in(const void *p, size_t i, int dtype) {
    if (dtype == RS_BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    return static_cast<const float *>(p)[i];
}

__device__ __forceinline__ void st_out(void *p, size_t i, float v, int dtype) {
    if (dtype == RS_BF16) static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
    else static_cast<float *>(p)[i] = v;
}

// Element `i` of a shared-memory array of the input dtype, as float.
__device__ __forceinline__ float lds_in(const void *smem_ptr, size_t i, int dtype) {
    if (dtype == RS_BF16)
        return __uint_as_float(static_cast<uint32_t>(static_cast<const unsigned short *>(smem_ptr)[i]) << 16);
    return static_cast<const float *>(smem_ptr)[i];
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Storage types of a state tile.
struct StF32 { static constexpr int bytes = 4; };
struct StBF16 { static constexpr int bytes = 2; };
struct StE4M3 { static constexpr int bytes = 1; };

// Expand one 16-byte chunk into 16 / bytes floats.
template <typename TS> struct Chunk;
template <> struct Chunk<StF32> {
    static constexpr int n = 4;
    __device__ __forceinline__ static void expand(const uint4 &c, float *o) {
        o[0] = __uint_as_float(c.x); o[1] = __uint_as_float(c.y);
        o[2] = __uint_as_float(c.z); o[3] = __uint_as_float(c.w);
    }
};
template <> struct Chunk<StBF16> {
    static constexpr int n = 8;
    __device__ __forceinline__ static void expand(const uint4 &c, float *o) {
        o[0] = bf16_lo(c.x); o[1] = bf16_hi(c.x); o[2] = bf16_lo(c.y); o[3] = bf16_hi(c.y);
        o[4] = bf16_lo(c.z); o[5] = bf16_hi(c.z); o[6] = bf16_lo(c.w); o[7] = bf16_hi(c.w);
    }
};
template <> struct Chunk<StE4M3> {
    static constexpr int n = 16;
    __device__ __forceinline__ static void expand2(uint32_t w, float *o) {
        __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xffffu), __NV_E4M3);
        __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
        float2 a = __half22float2(*reinterpret_cast<__half2 *>(&lo));
        float2 b = __half22float2(*reinterpret_cast<__half2 *>(&hi));
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    }
    __device__ __forceinline__ static void expand(const uint4 &c, float *o) {
        expand2(c.x, o); expand2(c.y, o + 4); expand2(c.z, o + 8); expand2(c.w, o + 12);
    }
};

// Round-to-nearest-even fp32 -> bf16 bits, and fp32 pair -> E4M3 pair (satfinite).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_e4m3x2(float a, float b) {
    // element a in the low byte
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// ------------------------------------------------------ geometry of a tile --
//
// A state tile is R rows of CC contiguous elements.  It is read in 16-byte
// chunks; TPR threads share a row, each taking CPT chunks of it, strided by TPR
// so that TPR neighbouring threads cover TPR * 16 contiguous bytes.
template <int CC, int EB, int TPR_MAX = 8>
struct Geom {
    static constexpr int VEC = 16 / EB;          // elements per chunk
    static constexpr int CHUNKS = CC / VEC;      // chunks per row
    static constexpr int TPR = CHUNKS < TPR_MAX ? CHUNKS : TPR_MAX;
    static constexpr int CPT = CHUNKS / TPR;     // chunks per thread per row
    static_assert(CC * EB >= 16, "row must hold at least one 16-byte chunk");
    static_assert(CHUNKS % TPR == 0, "chunks must split evenly");
};

// Two fp32 fused multiply-adds in one packed instruction: a * b + c elementwise.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long x, y, z, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(z) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(x), "l"(y), "l"(z));
    float2 o;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
    return o;
}

// Two fp32 products in one packed instruction: a * b elementwise.
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    unsigned long long x, y, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(x), "l"(y));
    float2 o;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
    return o;
}

// Sum over the TPR lanes that share a row (TPR a power of two <= 8, aligned).
template <int TPR>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ------------------------------------------- bulk copy + mbarrier (sm_90+) --

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
    // make the initialised barrier visible to the async (bulk-copy) proxy
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// One bounded test of a barrier phase.  The thread may sleep in the hardware
// for up to the hinted time (nanoseconds) while the phase is incomplete, so a
// waiting warp does not keep re-issuing the test.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the barrier to complete, for at most
// kWaitLimitCycles.  Returns false if the wait gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long limit = kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return false;
    }
    return true;
}

// 1-D bulk copy global -> shared of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing on `bar`.  No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Asynchronous 16-byte global -> shared copy through the L1 path (both
// addresses 16-byte aligned); completion by cp_async_wait_all.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
// Four 8x8 b16 matrices from shared memory: lanes 8 q .. 8 q + 7 address the
// eight 16-byte rows of matrix q; lane l receives row l / 4, elements
// 2 (l % 4) and 2 (l % 4) + 1 of each (the mma.sync fragment layout).
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&a)[4], const void *smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(smem_u32(smem_row)));
}

// The same for two matrices (lanes 0 .. 15 address them).
__device__ __forceinline__ void ldmatrix_x2(uint32_t (&a)[2], const void *smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(a[0]), "=r"(a[1])
                 : "r"(smem_u32(smem_row)));
}

// D += A B for one m16n8k16 bf16 tile with fp32 accumulation.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// L2 policy for data streamed once per step (the checkpoints): evict first, so
// that the small, re-read ring entries stay resident.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

}  // namespace rs
