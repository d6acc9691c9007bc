// Sizes shared by the two halves of the output-only path: the prep kernel
// writes one record per (sequence, head) tile into the workspace scratch
// region, the streaming kernel reads it next to the checkpoint tile and the
// tile's ring block.
//
// With e_j = L - npos + j the buffer index of output position j (0-based, L
// buffered entries, entry i in ring slot (head + i) mod cap), every output is
//     y_j[r] = mul_j (S0[r, :] . vec_j) + sum_{i<=e_j} coef_j[i] w_i[r]
// where w_i is the tile's ring row of entry i (Mamba-2 x_i, GDN v_i).
//
// Tile record:   hdr [16] | coef [NP][coef_stride(cap)] | vec [NP][CC] (GDN only)
//                hdr[0..7] = mul_j, hdr[8] = head slot, hdr[9] = L (int bits)
// Group record:  vec [NP][CC]   (Mamba-2: C_{e_j}, one per (sequence, group))
// All fp32, each record padded to 16 bytes.  NP is the number of output
// positions the kernels are compiled for: npos rounded up to 1, 2, 5 or 8.
#pragma once

#include "common.cuh"

namespace rs {

__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr int kRecHdr = 16;     // floats of the tile-record header
constexpr int kRecHeadSlot = 8; // header word: ring slot of buffer entry 0
constexpr int kRecLen = 9;      // header word: buffered entries L

__host__ __device__ inline int prep_np(int npos) {
    return npos <= 1 ? 1 : npos <= 2 ? 2 : npos <= 5 ? 5 : 8;
}

// Row stride (floats) of coef [NP][.] in a tile record: cap rounded up to 4,
// plus 4, so that the rows of different positions start in different
// shared-memory banks (they are read 8 rows at a time by the tensor-core path).
__host__ __device__ inline int coef_stride(int cap) { return (cap + 3) / 4 * 4 + 4; }

// Floats per tile record for NPr compiled positions.
__host__ __device__ inline size_t tile_rec_floats(int kind, int NPr, int cap, int CC) {
    return align_up(kRecHdr + (size_t)NPr * coef_stride(cap) + (kind == RS_GDN ? (size_t)NPr * CC : 0), 4);
}

// Floats per group record (Mamba-2 only).
__host__ __device__ inline size_t group_rec_floats(int NPr, int CC) { return align_up((size_t)NPr * CC, 4); }

// Floats of scratch a handle needs for calls with up to npos_max positions.
__host__ __device__ inline size_t scratch_floats(int kind, int B, int H, int G, int npos_max, int cap, int CC) {
    const int NPr = prep_np(npos_max);
    return (size_t)B * H * tile_rec_floats(kind, NPr, cap, CC) +
           (kind == RS_MAMBA2 ? (size_t)B * G * group_rec_floats(NPr, CC) : 0);
}

}  // namespace rs
