// The streaming half of the output-only kernels: every (sequence, head) tile of
// the checkpoint is contracted with up to NP vectors (Mamba-2: the C_t of the
// output positions; GDN: the transformed queries), in one pass over the tile,
// which sits in shared memory after a 1-D bulk copy.
#pragma once

#include "common.cuh"

namespace rs {

constexpr int kOutThreads = 128;

// Dynamic shared memory: the tile first (128-byte aligned), then a prologue area.
__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// y[j][r] = mul[j] * (tile[r, :] . vec[j]) + z[j][r]   for j < npos, r < R.
// y element (j, r) lives at y_off + j * y_pos_stride + r.
template <int CC, typename TS, int NP>
__device__ __forceinline__ void tile_matvec(const unsigned char *s_tile, int R,
                                            const float *s_vec, int npos, const float *s_mul,
                                            const float *s_z, void *y, size_t y_pos_stride,
                                            size_t y_off, int out_dtype) {
    using G = Geom<CC, TS::bytes>;
    constexpr int VEC = G::VEC, TPR = G::TPR, CPT = G::CPT, RPB = kOutThreads / TPR;
    const int lane = threadIdx.x % TPR, row0 = threadIdx.x / TPR;

    float vec[NP][CPT * VEC];
#pragma unroll
    for (int j = 0; j < NP; ++j)
#pragma unroll
        for (int c = 0; c < CPT; ++c)
#pragma unroll
            for (int v = 0; v < VEC; ++v)
                vec[j][c * VEC + v] = j < npos ? s_vec[j * CC + (lane + c * TPR) * VEC + v] : 0.f;

    const int npass = (R + RPB - 1) / RPB;
    for (int k = 0; k < npass; ++k) {
        const int r = row0 + k * RPB;
        const bool ok = r < R;
        float acc[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[j] = 0.f;
        if (ok) {
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(
                    s_tile + (static_cast<size_t>(r) * CC + (lane + c * TPR) * VEC) * TS::bytes);
                float f[VEC];
                Chunk<TS>::expand(raw, f);
#pragma unroll
                for (int v = 0; v < VEC; ++v)
#pragma unroll
                    for (int j = 0; j < NP; ++j) acc[j] = fmaf(f[v], vec[j][c * VEC + v], acc[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[j] = row_sum<TPR>(acc[j]);
        if (ok && lane == 0) {
#pragma unroll
            for (int j = 0; j < NP; ++j)
                if (j < npos)
                    st_out(y, y_off + j * y_pos_stride + r, fmaf(s_mul[j], acc[j], s_z[j * R + r]),
                           out_dtype);
        }
    }
}

// Zero outputs of one tile (a sequence whose buffer cannot serve the request).
__device__ __forceinline__ void zero_outputs(int R, int npos, void *y, size_t y_pos_stride,
                                             size_t y_off, int out_dtype) {
    for (int e = threadIdx.x; e < npos * R; e += blockDim.x)
        st_out(y, y_off + (e / R) * y_pos_stride + (e % R), 0.f, out_dtype);
}

// Copy `n` contiguous elements of `ebytes` bytes from global to shared memory
// with 16-byte moves when both ends allow it (cooperative over the CTA).
__device__ __forceinline__ void copy_g2s(void *dst, const void *src, int nbytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src);
    if ((a & 15) == 0 && (nbytes & 15) == 0) {
        for (int i = threadIdx.x; i < nbytes / 16; i += blockDim.x)
            static_cast<uint4 *>(dst)[i] = static_cast<const uint4 *>(src)[i];
    } else if ((a & 3) == 0 && (nbytes & 3) == 0) {
        for (int i = threadIdx.x; i < nbytes / 4; i += blockDim.x)
            static_cast<uint32_t *>(dst)[i] = static_cast<const uint32_t *>(src)[i];
    } else {
        for (int i = threadIdx.x; i < nbytes / 2; i += blockDim.x)
            static_cast<uint16_t *>(dst)[i] = static_cast<const uint16_t *>(src)[i];
    }
}

}  // namespace rs
