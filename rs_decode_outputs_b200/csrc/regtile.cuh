// A (sequence, head) state tile held in fp32 registers by a 256-thread CTA.
//
// Used by the kernels that rewrite state (commit, eager baseline, checkpoint
// load).  Thread geometry: TPR threads share a row; each holds CPT chunks of 4
// consecutive columns of that row (chunk c at columns (lane + c*TPR)*4), for
// NPASS rows spaced RPB = 256 / TPR apart.  Loads and stores move whole chunks,
// so a row is touched by TPR neighbouring threads in contiguous pieces.
#pragma once

#include "common.cuh"

namespace rs {

template <int CC, int NPASS>
struct RegTile {
    static constexpr int CHUNKS = CC / 4;
    static constexpr int TPR = CHUNKS < 8 ? CHUNKS : 8;
    static constexpr int CPT = CHUNKS / TPR;
    static constexpr int RPB = kTileThreads / TPR;
    static constexpr int NE = CPT * 4;  // elements per thread per row
    static_assert(CC % 4 == 0 && CHUNKS % TPR == 0, "bad tile width");

    float s[NPASS][NE];
    int lane, row0, R;

    __device__ __forceinline__ void init(int rows) {
        lane = threadIdx.x % TPR;
        row0 = threadIdx.x / TPR;
        R = rows;
    }
    __device__ __forceinline__ int row(int k) const { return row0 + k * RPB; }
    __device__ __forceinline__ bool valid(int k) const { return row(k) < R; }
    __device__ __forceinline__ int col(int c) const { return (lane + c * TPR) * 4; }
    __device__ __forceinline__ size_t idx(int k, int c) const {
        return static_cast<size_t>(row(k)) * CC + col(c);
    }

    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int e = 0; e < NE; ++e) s[k][e] = 0.f;
    }

    // ---- loads (tile = base of this (b, h) tile) ----
    __device__ __forceinline__ void load_f32(const float *tile) {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (valid(k)) v = *reinterpret_cast<const float4 *>(tile + idx(k, c));
                s[k][c * 4 + 0] = v.x; s[k][c * 4 + 1] = v.y;
                s[k][c * 4 + 2] = v.z; s[k][c * 4 + 3] = v.w;
            }
    }
    __device__ __forceinline__ void load_bf16(const __nv_bfloat16 *tile) {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                uint2 v = make_uint2(0u, 0u);
                if (valid(k)) v = *reinterpret_cast<const uint2 *>(tile + idx(k, c));
                s[k][c * 4 + 0] = bf16_lo(v.x); s[k][c * 4 + 1] = bf16_hi(v.x);
                s[k][c * 4 + 2] = bf16_lo(v.y); s[k][c * 4 + 3] = bf16_hi(v.y);
            }
    }
    __device__ __forceinline__ void load_e4m3(const uint8_t *tile, float scale) {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                uint32_t v = 0u;
                if (valid(k)) v = *reinterpret_cast<const uint32_t *>(tile + idx(k, c));
                float f[4];
                Chunk<StE4M3>::expand2(v, f);
#pragma unroll
                for (int e = 0; e < 4; ++e) s[k][c * 4 + e] = f[e] * scale;
            }
    }

    // ---- stores ----
    __device__ __forceinline__ void store_f32(float *tile) const {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c)
                if (valid(k))
                    *reinterpret_cast<float4 *>(tile + idx(k, c)) =
                        make_float4(s[k][c * 4], s[k][c * 4 + 1], s[k][c * 4 + 2], s[k][c * 4 + 3]);
    }
    __device__ __forceinline__ void store_bf16(__nv_bfloat16 *tile) const {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c)
                if (valid(k))
                    *reinterpret_cast<uint2 *>(tile + idx(k, c)) =
                        make_uint2(pack_bf16x2(s[k][c * 4], s[k][c * 4 + 1]),
                                   pack_bf16x2(s[k][c * 4 + 2], s[k][c * 4 + 3]));
    }
    // Round every element to bf16 in place (a bf16-state step keeps only bf16).
    __device__ __forceinline__ void round_bf16() {
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int e = 0; e < NE; ++e) s[k][e] = __bfloat162float(__float2bfloat16_rn(s[k][e]));
    }

    // Largest |element| over the tile (whole CTA; all threads get the result).
    __device__ __forceinline__ float absmax(float *red /* smem [kTileThreads/32] */) const {
        float m = 0.f;
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
            if (valid(k))
#pragma unroll
                for (int e = 0; e < NE; ++e) m = fmaxf(m, fabsf(s[k][e]));
        m = warp_max(m);
        __syncthreads();
        if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = m;
        __syncthreads();
        float r = red[0];
#pragma unroll
        for (int w = 1; w < kTileThreads / 32; ++w) r = fmaxf(r, red[w]);
        return r;
    }

    // E4M3 copy: scale = absmax / 448 (1 for an all-zero tile), code =
    // RNE_satfinite(s / scale) with an IEEE division.  Returns the scale.
    __device__ __forceinline__ float store_e4m3(uint8_t *tile, float *red) const {
        const float amax = absmax(red);
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
        for (int k = 0; k < NPASS; ++k)
#pragma unroll
            for (int c = 0; c < CPT; ++c)
                if (valid(k)) {
                    uint32_t lo = pack_e4m3x2(__fdiv_rn(s[k][c * 4], scale), __fdiv_rn(s[k][c * 4 + 1], scale));
                    uint32_t hi = pack_e4m3x2(__fdiv_rn(s[k][c * 4 + 2], scale), __fdiv_rn(s[k][c * 4 + 3], scale));
                    *reinterpret_cast<uint32_t *>(tile + idx(k, c)) = (lo & 0xffffu) | (hi << 16);
                }
        return scale;
    }
};

// Load a tile of the given storage into fp32 registers.
template <int CC, int NPASS>
__device__ __forceinline__ void load_tile(RegTile<CC, NPASS> &t, const void *base, size_t tile,
                                          int dtype, const float *scales) {
    const size_t n = static_cast<size_t>(t.R) * CC;
    if (dtype == RS_F32) t.load_f32(static_cast<const float *>(base) + tile * n);
    else if (dtype == RS_BF16) t.load_bf16(static_cast<const __nv_bfloat16 *>(base) + tile * n);
    else t.load_e4m3(static_cast<const uint8_t *>(base) + tile * n, scales[tile]);
}

// Store the registers as the given storage (E4M3 also writes scales[tile]).
template <int CC, int NPASS>
__device__ __forceinline__ void store_tile(const RegTile<CC, NPASS> &t, void *base, size_t tile,
                                           int dtype, float *scales, float *red) {
    const size_t n = static_cast<size_t>(t.R) * CC;
    if (dtype == RS_F32) t.store_f32(static_cast<float *>(base) + tile * n);
    else if (dtype == RS_BF16) t.store_bf16(static_cast<__nv_bfloat16 *>(base) + tile * n);
    else {
        float sc = t.store_e4m3(static_cast<uint8_t *>(base) + tile * n, red);
        if (threadIdx.x == 0) scales[tile] = sc;
    }
}

}  // namespace rs
