// Mamba-2 kernels of the ReplaySSM decode path.
//
// Recurrence (one (sequence, head), state h in R^{P x N}; head h reads group
// g = h / (H / G) of B and C):
//     h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,      y_t = h_t C_t + D x_t
//
// Replay ("ReplaySSM: Cache SSM Inputs, Not State", Abstract; "ReplaySSM for
// hybrid SSM-Transformer stacks", How ReplaySSM works, steps 2-4).  With the
// checkpoint S0 and the L buffered entries 1..L since it, the output at
// buffered position e is
//     y_e = exp(A sum_{m<=e} dt_m) (S0 C_e)
//           + sum_{i<=e} exp(A sum_{i<m<=e} dt_m) dt_i (B_i . C_e) x_i  +  D x_e
// (unrolling the recurrence; no intermediate state is formed), and the state a
// commit writes is
//     S_L = exp(A sum_m dt_m) S0 + sum_i exp(A sum_{m>i} dt_m) dt_i x_i B_i^T.
#include "outputs.cuh"
#include "regtile.cuh"
#include "launch.h"

namespace rs {

// -------------------------------------------------------------- commit ----
// One CTA (256 threads) per (sequence, head) tile of a sequence being
// committed; the tile lives in fp32 registers.  The buffer is folded with the
// closed form of S_L above; the master is rewritten, then the copy is derived
// from it.  The last CTA of a sequence to finish moves head to tail.

template <int CC, int NPASS>
__global__ void __launch_bounds__(kTileThreads)
m2_commit_kernel(const Params p, int min_len, const int32_t *__restrict__ mask) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kTileThreads / 32];
    const int R = p.R, H = p.H, cap = p.cap;
    const int tile = blockIdx.x;
    const int b = tile / H, h = tile % H, g = h / p.heads_per_group;
    const int head = p.head[b];
    const int L = p.tail[b] - head;
    if (L < (min_len > 1 ? min_len : 1) || L > cap || (mask && mask[b] == 0)) return;

    const int in_bytes = p.in_dtype == RS_BF16 ? 2 : 4;
    float *s_dt = reinterpret_cast<float *>(smem);
    float *s_w = s_dt + cap;
    float *s_x = s_w + cap;  // [cap][R]
    unsigned char *s_B = smem + align_up(4 * (2 * (size_t)cap + (size_t)cap * R), 16);  // [cap][CC]
    const int tid = threadIdx.x;
    // this head's ring blocks (x, dt) and this group's B block
    const unsigned char *xblk = static_cast<const unsigned char *>(p.ra) + ((size_t)b * H + h) * p.blk_r;
    const float *dtblk = static_cast<const float *>(p.rb) + ((size_t)b * H + h) * p.capd;
    const unsigned char *bblk = static_cast<const unsigned char *>(p.rc) + ((size_t)b * p.G + g) * p.blk_c;

    RegTile<CC, NPASS> t;
    t.init(R);
    if (p.shared_lowp) load_tile(t, p.copy, tile, p.copy_dtype, p.scale);
    else t.load_f32(p.master + (size_t)tile * R * CC);

    for (int i = tid; i < L; i += kTileThreads) s_dt[i] = dtblk[(head + i) & p.cap_mask];
    const int bshift = __ffs(CC * in_bytes / 16) - 1;   // 16-byte pieces per row, log2
    for (int q = tid; q < (L << bshift); q += kTileThreads) {
        const int i = q >> bshift, w = q & ((1 << bshift) - 1);
        const unsigned char *src = bblk + (size_t)((head + i) & p.cap_mask) * CC * in_bytes;
        reinterpret_cast<uint4 *>(s_B + (size_t)i * CC * in_bytes)[w] = reinterpret_cast<const uint4 *>(src)[w];
    }
    for (int i = tid >> 5; i < L; i += kTileThreads / 32) {
        const unsigned char *row = xblk + (size_t)((head + i) & p.cap_mask) * R * in_bytes;
        for (int r = tid & 31; r < R; r += 32) s_x[i * R + r] = ld_in(row, r, p.in_dtype);
    }
    __syncthreads();
    const float A = p.A[h];
    // w_i = exp(A sum_{m>i} dt_m) dt_i
    for (int i = tid; i < L; i += kTileThreads) {
        float after = 0.f;
        for (int m = i + 1; m < L; ++m) after += s_dt[m];
        s_w[i] = expf(A * after) * s_dt[i];
    }
    float tot = 0.f;
    for (int m = 0; m < L; ++m) tot += s_dt[m];
    const float decay = expf(A * tot);
    __syncthreads();

#pragma unroll
    for (int k = 0; k < NPASS; ++k)
#pragma unroll
        for (int e = 0; e < RegTile<CC, NPASS>::NE; ++e) t.s[k][e] *= decay;
    for (int i = 0; i < L; ++i) {
        float Bf[RegTile<CC, NPASS>::NE];
#pragma unroll
        for (int c = 0; c < RegTile<CC, NPASS>::CPT; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) Bf[c * 4 + e] = ld_in(s_B, (size_t)i * CC + t.col(c) + e, p.in_dtype);
        const float wi = s_w[i];
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            const float u = t.valid(k) ? wi * s_x[(size_t)i * R + t.row(k)] : 0.f;
#pragma unroll
            for (int e = 0; e < RegTile<CC, NPASS>::NE; ++e) t.s[k][e] = fmaf(u, Bf[e], t.s[k][e]);
        }
    }

    if (!p.shared_lowp) t.store_f32(p.master + (size_t)tile * R * CC);
    if (p.copy_dtype != RS_NONE) store_tile(t, p.copy, tile, p.copy_dtype, p.scale, red);

    __syncthreads();
    if (tid == 0) {   // no fence: nothing in this kernel reads head after the CTAs' reads at entry
        if (atomicAdd(&p.arrive[b], 1u) == static_cast<unsigned>(H - 1)) {
            p.arrive[b] = 0u;
            p.head[b] = head + L;
        }
    }
}

size_t m2_commit_smem(const Params &p) {
    const int in_bytes = p.in_dtype == RS_BF16 ? 2 : 4;
    return align_up(4 * (2 * (size_t)p.cap + (size_t)p.cap * p.R), 16) +
           (size_t)in_bytes * p.cap * p.CC;
}

template <int CC, int NPASS>
static cudaError_t launch_m2_commit_t(const Params &p, int min_len, const int32_t *mask,
                                      cudaStream_t st) {
    const size_t smem = m2_commit_smem(p);
    auto k = m2_commit_kernel<CC, NPASS>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<p.B * p.H, kTileThreads, smem, st>>>(p, min_len, mask);
    return cudaGetLastError();
}

template <int CC>
static cudaError_t launch_m2_commit_cc(const Params &p, int min_len, const int32_t *mask,
                                       cudaStream_t st) {
    RS_DISPATCH_NPASS(CC, p.R, return launch_m2_commit_t, (p, min_len, mask, st));
    return cudaErrorInvalidValue;
}

cudaError_t launch_m2_commit(const Params &p, int min_len, const int32_t *mask, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_m2_commit_cc, (p, min_len, mask, st));
    return cudaErrorInvalidValue;
}

// --------------------------------------------------------------- eager ----
// Baseline: read the state tile, apply T recurrence steps, write it back (or,
// in slot mode, write every intermediate state to its own slot), output y at
// every step.  Inputs are read straight from the caller's [T][B][...] arrays.

template <int CC, int NPASS>
__global__ void __launch_bounds__(kTileThreads)
m2_eager_kernel(const Params p, void *state, int sdt, rs_inputs in, int T, void *y,
                const int32_t *__restrict__ cur, int nslots) {
    __shared__ float red[kTileThreads / 32];
    const int R = p.R, H = p.H, Bn = p.B;
    const int tile = blockIdx.x;
    const int b = tile / H, h = tile % H, g = h / p.heads_per_group;
    const size_t n_tile = (size_t)R * CC;
    const size_t n_all = (size_t)Bn * H;
    RegTile<CC, NPASS> t;
    t.init(R);

    int c0 = 0;
    if (cur) {
        c0 = cur[b];
        if (c0 < 0 || c0 >= nslots) {
            for (int e = threadIdx.x; e < T * R; e += blockDim.x)
                st_out(y, ((size_t)(e / R) * n_all + tile) * R + e % R, 0.f, p.out_dtype);
            if (threadIdx.x == 0) atomicOr(&p.err[b], RS_SEQ_ERR_ROLLBACK);
            return;
        }
    }
    load_tile(t, state, (size_t)c0 * n_all + tile, sdt, nullptr);
    const float A = p.A[h];
    const float Dh = p.D ? p.D[h] : 0.f;
    constexpr int NE = RegTile<CC, NPASS>::NE, CPT = RegTile<CC, NPASS>::CPT, TPR = RegTile<CC, NPASS>::TPR;

    for (int ts = 0; ts < T; ++ts) {
        const size_t bh = (size_t)ts * n_all + tile;
        const float dt = in.dt[bh];
        const size_t bg = ((size_t)ts * Bn + b) * p.G + g;
        float Bf[NE], Cf[NE];
#pragma unroll
        for (int c = 0; c < CPT; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                Bf[c * 4 + e] = ld_in(in.B, bg * CC + t.col(c) + e, p.in_dtype);
                Cf[c * 4 + e] = ld_in(in.C, bg * CC + t.col(c) + e, p.in_dtype);
            }
        const float decay = expf(dt * A);
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            const float xr = t.valid(k) ? ld_in(in.x, bh * R + t.row(k), p.in_dtype) : 0.f;
            const float u = dt * xr;
#pragma unroll
            for (int e = 0; e < NE; ++e) t.s[k][e] = fmaf(decay, t.s[k][e], u * Bf[e]);
        }
        if (sdt == RS_BF16) t.round_bf16();
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < NE; ++e) acc = fmaf(t.s[k][e], Cf[e], acc);
            acc = row_sum<TPR>(acc);
            if (t.valid(k) && t.lane == 0) {
                const float xr = ld_in(in.x, bh * R + t.row(k), p.in_dtype);
                st_out(y, bh * R + t.row(k), fmaf(Dh, xr, acc), p.out_dtype);
            }
        }
        if (cur) store_tile(t, state, (size_t)((c0 + 1 + ts) % nslots) * n_all + tile, sdt, nullptr, red);
    }
    if (!cur) store_tile(t, state, tile, sdt, nullptr, red);
}

template <int CC, int NPASS>
static cudaError_t launch_m2_eager_t(const Params &p, void *state, int sdt, const rs_inputs &in,
                                     int T, void *y, const int32_t *cur, int nslots,
                                     cudaStream_t st) {
    m2_eager_kernel<CC, NPASS><<<p.B * p.H, kTileThreads, 0, st>>>(p, state, sdt, in, T, y, cur,
                                                                 nslots);
    return cudaGetLastError();
}

template <int CC>
static cudaError_t launch_m2_eager_cc(const Params &p, void *state, int sdt, const rs_inputs &in,
                                      int T, void *y, const int32_t *cur, int nslots,
                                      cudaStream_t st) {
    RS_DISPATCH_NPASS(CC, p.R, return launch_m2_eager_t, (p, state, sdt, in, T, y, cur, nslots, st));
    return cudaErrorInvalidValue;
}

cudaError_t launch_m2_eager(const Params &p, void *state, int sdt, const rs_inputs &in, int T,
                            void *y, const int32_t *cur, int nslots, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_m2_eager_cc, (p, state, sdt, in, T, y, cur, nslots, st));
    return cudaErrorInvalidValue;
}

}  // namespace rs
