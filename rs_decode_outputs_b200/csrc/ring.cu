// Ring-buffer and checkpoint kernels shared by both layer kinds: append,
// pointer-only rollback, checkpoint load (master + derived copy), workspace
// initialisation and the eager baseline's slot selection.
#include "regtile.cuh"
#include "launch.h"

namespace rs {

// Copy one row of nbytes (a multiple of 2) with the 32 lanes of a warp, in the
// widest pieces both ends allow.
__device__ __forceinline__ void warp_copy(void *dst, const void *src, size_t nbytes, int lane) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | nbytes;
    if ((a & 15) == 0) {
        for (size_t i = lane; i < nbytes / 16; i += 32)
            static_cast<uint4 *>(dst)[i] = static_cast<const uint4 *>(src)[i];
    } else if ((a & 3) == 0) {
        for (size_t i = lane; i < nbytes / 4; i += 32)
            static_cast<uint32_t *>(dst)[i] = static_cast<const uint32_t *>(src)[i];
    } else {
        for (size_t i = lane; i < nbytes / 2; i += 32)
            static_cast<uint16_t *>(dst)[i] = static_cast<const uint16_t *>(src)[i];
    }
}

// ----------------------------------------------------------------- append --
// One CTA per sequence ("ReplaySSM for hybrid SSM-Transformer stacks", How
// ReplaySSM works, step 2: append the step's SSM input to the buffer).  Writes
// slots tail .. tail+T-1 (mod cap), then advances tail.  Refuses, with a sticky
// error bit, when the buffer would hold more than cap entries.
__global__ void __launch_bounds__(256) append_kernel(const Params p, rs_inputs in, int T, int kind) {
    const int b = blockIdx.x;
    const int head = p.head[b], tail = p.tail[b];
    if (tail - head + T > p.cap || tail - head < 0) {
        if (threadIdx.x == 0) atomicOr(&p.err[b], RS_SEQ_ERR_OVERFLOW);
        return;
    }
    const int H = p.H, R = p.R, CC = p.CC, Bn = p.B;
    const size_t ib = p.in_dtype == RS_BF16 ? 2 : 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const size_t rrow = (size_t)R * ib, crow = (size_t)CC * ib;   // bytes of one ring row
    for (int t = 0; t < T; ++t) {
        const int slot = (tail + t) & p.cap_mask;
        const size_t src = (size_t)t * Bn + b;   // input row [t][b]
        // per-head rows (one warp per row) and per-head scalars
        for (int h = warp; h < H; h += nw) {
            const size_t bh = (size_t)b * H + h;
            if (kind == RS_MAMBA2) {
                warp_copy(static_cast<char *>(p.ra) + bh * p.blk_r + slot * rrow,
                          static_cast<const char *>(in.x) + (src * H + h) * rrow, rrow, lane);
            } else {
                warp_copy(static_cast<char *>(p.ra) + bh * p.blk_c + slot * crow,
                          static_cast<const char *>(in.q) + (src * H + h) * crow, crow, lane);
                warp_copy(static_cast<char *>(p.rb) + bh * p.blk_c + slot * crow,
                          static_cast<const char *>(in.k) + (src * H + h) * crow, crow, lane);
                warp_copy(static_cast<char *>(p.rc) + bh * p.blk_r + slot * rrow,
                          static_cast<const char *>(in.v) + (src * H + h) * rrow, rrow, lane);
            }
        }
        for (int h = threadIdx.x; h < H; h += blockDim.x) {
            const size_t at = ((size_t)b * H + h) * p.capd + slot;
            if (kind == RS_MAMBA2) {
                static_cast<float *>(p.rb)[at] = in.dt[src * H + h];
            } else {
                static_cast<float *>(p.rd)[at] = in.alpha[src * H + h];
                static_cast<float *>(p.re)[at] = in.beta[src * H + h];
            }
        }
        if (kind == RS_MAMBA2) {   // per-group rows of B and C
            for (int g = warp; g < p.G; g += nw) {
                const size_t bg = (size_t)b * p.G + g;
                warp_copy(static_cast<char *>(p.rc) + bg * p.blk_c + slot * crow,
                          static_cast<const char *>(in.B) + (src * p.G + g) * crow, crow, lane);
                warp_copy(static_cast<char *>(p.rd) + bg * p.blk_c + slot * crow,
                          static_cast<const char *>(in.C) + (src * p.G + g) * crow, crow, lane);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) p.tail[b] = tail + T;
}

cudaError_t launch_append(const Params &p, const rs_inputs &in, int T, cudaStream_t st) {
    append_kernel<<<p.B, 256, 0, st>>>(p, in, T, p.kind);
    return cudaGetLastError();
}

// --------------------------------------------------------------- rollback --
// How ReplaySSM works, step 4: rejecting the last k tokens moves the tail back
// by k; the checkpoint is not touched.  Integer-only, one thread per sequence.
__global__ void rollback_kernel(const Params p, const int32_t *__restrict__ k) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= p.B) return;
    const int kb = k[b];
    const int len = p.tail[b] - p.head[b];
    if (kb < 0 || kb > len) atomicOr(&p.err[b], RS_SEQ_ERR_ROLLBACK);
    else p.tail[b] -= kb;
}

cudaError_t launch_rollback(const Params &p, const int32_t *k, cudaStream_t st) {
    rollback_kernel<<<(p.B + 255) / 256, 256, 0, st>>>(p, k);
    return cudaGetLastError();
}

// Eager baseline's "rollback": the state after keep[b] accepted positions
// becomes current, by index.
__global__ void eager_accept_kernel(const Params p, int32_t *cur, const int32_t *__restrict__ keep,
                                    int nslots) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= p.B) return;
    const int kb = keep[b];
    if (kb < 0 || kb > nslots - 1) atomicOr(&p.err[b], RS_SEQ_ERR_ROLLBACK);
    else cur[b] = (cur[b] + kb) % nslots;
}

cudaError_t launch_eager_accept(const Params &p, int32_t *cur, const int32_t *keep, int nslots,
                                cudaStream_t st) {
    eager_accept_kernel<<<(p.B + 255) / 256, 256, 0, st>>>(p, cur, keep, nslots);
    return cudaGetLastError();
}

// --------------------------------------------------------- load checkpoint --
// Replace the checkpoint by an fp32 state: write the master and derive the
// copy from it (How ReplaySSM works, step 5: the copy is always derived from
// the high-precision checkpoint); the buffer becomes empty.
template <int CC, int NPASS>
__global__ void __launch_bounds__(kTileThreads) load_checkpoint_kernel(const Params p, const float *state) {
    __shared__ float red[kTileThreads / 32];
    const int tile = blockIdx.x;
    RegTile<CC, NPASS> t;
    t.init(p.R);
    t.load_f32(state + (size_t)tile * p.R * CC);
    if (!p.shared_lowp) t.store_f32(p.master + (size_t)tile * p.R * CC);
    if (p.copy_dtype != RS_NONE) store_tile(t, p.copy, tile, p.copy_dtype, p.scale, red);
    if (tile % p.H == 0 && threadIdx.x == 0) {
        const int b = tile / p.H;
        p.head[b] = 0;
        p.tail[b] = 0;
        p.err[b] = 0u;
        p.arrive[b] = 0u;
    }
}

template <int CC, int NPASS>
static cudaError_t launch_load_t(const Params &p, const float *state, cudaStream_t st) {
    load_checkpoint_kernel<CC, NPASS><<<p.B * p.H, kTileThreads, 0, st>>>(p, state);
    return cudaGetLastError();
}

template <int CC>
static cudaError_t launch_load_cc(const Params &p, const float *state, cudaStream_t st) {
    RS_DISPATCH_NPASS(CC, p.R, return launch_load_t, (p, state, st));
    return cudaErrorInvalidValue;
}

cudaError_t launch_load_checkpoint(const Params &p, const float *state, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_load_cc, (p, state, st));
    return cudaErrorInvalidValue;
}

// -------------------------------------------------------------------- init --
// After the host zeroes the workspace: E4M3 scales start at 1 (an all-zero tile).
__global__ void fill_kernel(float *x, size_t n, float v) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        x[i] = v;
}

cudaError_t launch_init(const Params &p, cudaStream_t st) {
    if (p.copy_dtype == RS_E4M3) {
        const size_t n = (size_t)p.B * p.H;
        fill_kernel<<<(unsigned)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024), 256, 0, st>>>(p.scale, n, 1.f);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

// ------------------------------------------------------ wait self-test ----
// One thread waits, through the same bounded wait the streaming kernel uses,
// on a barrier phase that nothing completes; it gives up after `limit` cycles
// and records RS_SEQ_ERR_TIMEOUT and the cycles it waited.
__global__ void wait_selftest_kernel(uint32_t *out, long long limit) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    const long long t0 = clock64();
    const bool done = mbar_wait_bounded(&bar, 0, limit);
    const long long waited = clock64() - t0;
    out[0] = done ? 0u : static_cast<uint32_t>(RS_SEQ_ERR_TIMEOUT);
    out[1] = static_cast<uint32_t>(waited & 0xffffffffLL);
    out[2] = static_cast<uint32_t>(waited >> 32);
}

cudaError_t launch_wait_selftest(uint32_t *out, long long limit, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(out, limit);
    return cudaGetLastError();
}

}  // namespace rs
