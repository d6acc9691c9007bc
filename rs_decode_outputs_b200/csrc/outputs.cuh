// Sizes shared by the two halves of the output-only path: the prep kernel
// writes one record per (sequence, head) tile into the workspace scratch
// region, the streaming kernel reads it next to the checkpoint tile.
//
// Tile record:    mul [8] | z [NP][R]            (Mamba-2)
//                 mul [8] | z [NP][R] | vec [NP][CC]   (GDN: vec = transformed queries)
// Group record:   vec [NP][CC]                   (Mamba-2: C of the output positions,
//                                                 one per (sequence, group))
// All fp32, each record padded to 16 bytes.  NP is the number of output
// positions the kernels are compiled for: npos rounded up to 1, 2, 5 or 8.
#pragma once

#include "common.cuh"

namespace rs {

__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline int prep_np(int npos) {
    return npos <= 1 ? 1 : npos <= 2 ? 2 : npos <= 5 ? 5 : 8;
}

// Floats per tile record for NPr compiled positions.
__host__ __device__ inline size_t tile_rec_floats(int kind, int NPr, int R, int CC) {
    return align_up(8 + (size_t)NPr * R + (kind == RS_GDN ? (size_t)NPr * CC : 0), 4);
}

// Floats per group record (Mamba-2 only).
__host__ __device__ inline size_t group_rec_floats(int NPr, int CC) { return align_up((size_t)NPr * CC, 4); }

// Floats of scratch a handle needs for calls with up to npos_max positions.
__host__ __device__ inline size_t scratch_floats(int kind, int B, int H, int G, int npos_max, int R, int CC) {
    const int NPr = prep_np(npos_max);
    return (size_t)B * H * tile_rec_floats(kind, NPr, R, CC) +
           (kind == RS_MAMBA2 ? (size_t)B * G * group_rec_floats(NPr, CC) : 0);
}

}  // namespace rs
