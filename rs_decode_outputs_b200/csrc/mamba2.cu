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

// ------------------------------------------------------------- outputs ----
// One CTA per (sequence, head) tile.  Thread 0 starts the bulk copy of the
// checkpoint tile at entry; while it is in flight the CTA stages the buffered
// inputs it needs and forms the per-entry coefficients; then it waits for the
// tile and streams it once against the NP C vectors.

struct M2OutSmem {
    size_t dt, C, coef, mul, z, Braw, xraw, total;
};

__host__ __device__ inline M2OutSmem m2_out_smem(size_t tile_bytes, int cap, int CC, int R,
                                                 int NP, int in_bytes) {
    M2OutSmem s;
    size_t o = align_up(tile_bytes, 128);
    s.dt = o;   o = align_up(o + 4 * cap, 16);
    s.C = o;    o = align_up(o + 4 * (size_t)NP * CC, 16);
    s.coef = o; o = align_up(o + 4 * (size_t)NP * cap, 16);
    s.mul = o;  o = align_up(o + 4 * (size_t)NP, 16);
    s.z = o;    o = align_up(o + 4 * (size_t)NP * R, 16);
    s.Braw = o; o = align_up(o + (size_t)in_bytes * cap * CC, 16);
    s.xraw = o; o = align_up(o + (size_t)in_bytes * cap * R, 16);
    s.total = o;
    return s;
}

template <int CC, typename TS, int NP>
__global__ void __launch_bounds__(kOutThreads)
m2_outputs_kernel(const Params p, const void *__restrict__ state, int npos, void *y) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t bar;

    const int R = p.R, H = p.H, cap = p.cap;
    const int tile = blockIdx.x;
    const int b = tile / H, h = tile % H, g = h / p.heads_per_group;
    const int in_bytes = p.in_dtype == RS_BF16 ? 2 : 4;
    const uint32_t tile_bytes = static_cast<uint32_t>(R) * CC * TS::bytes;
    const M2OutSmem L_ = m2_out_smem(tile_bytes, cap, CC, R, NP, in_bytes);
    float *s_dt = reinterpret_cast<float *>(smem + L_.dt);
    float *s_C = reinterpret_cast<float *>(smem + L_.C);
    float *s_coef = reinterpret_cast<float *>(smem + L_.coef);
    float *s_mul = reinterpret_cast<float *>(smem + L_.mul);
    float *s_z = reinterpret_cast<float *>(smem + L_.z);
    unsigned char *s_B = smem + L_.Braw;
    unsigned char *s_x = smem + L_.xraw;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    constexpr int nwarps = kOutThreads / 32;

    if (tid == 0) {
        mbar_init(&bar, 1);
        bulk_tile_g2s(smem, static_cast<const unsigned char *>(state) + (size_t)tile * tile_bytes,
                      tile_bytes, &bar, policy_evict_first());
    }

    const int head = p.head[b];
    const int L = p.tail[b] - head;
    const bool ok = npos >= 1 && L >= npos && L <= cap;
    const size_t ring_bh = (size_t)b * cap;   // first slot row of sequence b

    if (ok) {
        // ---- stage the buffered entries (all loads independent) ----
        for (int i = tid; i < L; i += kOutThreads) {
            const int slot = (head + i) & p.cap_mask;
            s_dt[i] = static_cast<const float *>(p.rb)[(ring_bh + slot) * H + h];
        }
        const int bchunks = CC * in_bytes / 16;   // 16-byte pieces per B row
        for (int q = tid; q < L * bchunks; q += kOutThreads) {
            const int i = q / bchunks, w = q % bchunks;
            const int slot = (head + i) & p.cap_mask;
            const unsigned char *src = static_cast<const unsigned char *>(p.rc) +
                                       (((ring_bh + slot) * p.G + g) * CC) * in_bytes;
            reinterpret_cast<uint4 *>(s_B + (size_t)i * CC * in_bytes)[w] =
                reinterpret_cast<const uint4 *>(src)[w];
        }
        for (int q = tid; q < L * R; q += kOutThreads) {
            const int i = q / R, r = q % R;
            const int slot = (head + i) & p.cap_mask;
            const size_t src = ((ring_bh + slot) * H + h) * R + r;
            if (in_bytes == 2)
                reinterpret_cast<uint16_t *>(s_x)[q] = static_cast<const uint16_t *>(p.ra)[src];
            else
                reinterpret_cast<float *>(s_x)[q] = static_cast<const float *>(p.ra)[src];
        }
        for (int q = tid; q < npos * CC; q += kOutThreads) {
            const int j = q / CC, n = q % CC;
            const int slot = (head + L - npos + j) & p.cap_mask;
            s_C[q] = ld_in(p.rd, ((ring_bh + slot) * p.G + g) * CC + n, p.in_dtype);
        }
    }
    __syncthreads();   // staged inputs; barrier initialisation visible to all

    if (ok) {
        const float A = p.A[h];
        // coef[j][i] = exp(A sum_{i<m<=e_j} dt_m) dt_i (B_i . C_{e_j}) for i <= e_j
        for (int w = warp; w < npos * L; w += nwarps) {
            const int j = w / L, i = w % L, e = L - npos + j;
            if (i > e) continue;
            float d = 0.f;
            for (int n = lane; n < CC; n += 32) d = fmaf(ld_in(s_B, (size_t)i * CC + n, p.in_dtype), s_C[j * CC + n], d);
            d = warp_sum(d);
            if (lane == 0) {
                float after = 0.f;
                for (int m = i + 1; m <= e; ++m) after += s_dt[m];
                s_coef[j * cap + i] = expf(A * after) * s_dt[i] * d;
            }
        }
        if (tid < npos) {
            const int e = L - npos + tid;
            float tot = 0.f;
            for (int m = 0; m <= e; ++m) tot += s_dt[m];
            const float tile_scale = p.copy_dtype == RS_E4M3 ? p.scale[tile] : 1.f;
            s_mul[tid] = expf(A * tot) * tile_scale;
        }
    }
    __syncthreads();

    if (ok) {
        // z[j][r] = sum_{i<=e_j} coef[j][i] x_i[r] + D x_{e_j}[r]
        const float Dh = p.D ? p.D[h] : 0.f;
        for (int q = tid; q < npos * R; q += kOutThreads) {
            const int j = q / R, r = q % R, e = L - npos + j;
            float acc = 0.f;
            for (int i = 0; i <= e; ++i) acc = fmaf(s_coef[j * cap + i], ld_in(s_x, (size_t)i * R + r, p.in_dtype), acc);
            s_z[q] = fmaf(Dh, ld_in(s_x, (size_t)e * R + r, p.in_dtype), acc);
        }
    }

    // Every thread waits for the tile, so that no copy is in flight at exit.
    const bool arrived = mbar_wait_bounded(&bar, 0);
    __syncthreads();
    const size_t y_pos_stride = (size_t)p.B * H * R;
    const size_t y_off = (size_t)tile * R;
    if (!ok || !arrived) {
        zero_outputs(R, npos, y, y_pos_stride, y_off, p.out_dtype);
        if (tid == 0) atomicOr(&p.err[b], !arrived ? RS_SEQ_ERR_TIMEOUT : RS_SEQ_ERR_EMPTY);
        return;
    }
    tile_matvec<CC, TS, NP>(smem, R, s_C, npos, s_mul, s_z, y, y_pos_stride, y_off, p.out_dtype);
}

size_t m2_outputs_smem(const Params &p, int NP) {
    const int eb = p.copy_dtype == RS_BF16 ? 2 : p.copy_dtype == RS_E4M3 ? 1 : 4;
    return m2_out_smem((size_t)p.R * p.CC * eb, p.cap, p.CC, p.R, NP,
                       p.in_dtype == RS_BF16 ? 2 : 4).total;
}

template <int CC, typename TS, int NP>
static cudaError_t launch_m2_out_t(const Params &p, int npos, void *y, cudaStream_t st) {
    const void *state = p.copy_dtype == RS_NONE ? static_cast<const void *>(p.master) : p.copy;
    const size_t smem = m2_outputs_smem(p, NP);
    auto k = m2_outputs_kernel<CC, TS, NP>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<p.B * p.H, kOutThreads, smem, st>>>(p, state, npos, y);
    return cudaGetLastError();
}

template <int CC, typename TS>
static cudaError_t launch_m2_out_np(const Params &p, int npos, void *y, cudaStream_t st) {
    if (npos <= 1) return launch_m2_out_t<CC, TS, 1>(p, npos, y, st);
    if (npos <= 2) return launch_m2_out_t<CC, TS, 2>(p, npos, y, st);
    if (npos <= 4) return launch_m2_out_t<CC, TS, 4>(p, npos, y, st);
    return launch_m2_out_t<CC, TS, 8>(p, npos, y, st);
}

template <int CC>
static cudaError_t launch_m2_out_cc(const Params &p, int npos, void *y, cudaStream_t st) {
    switch (p.copy_dtype) {
        case RS_BF16: return launch_m2_out_np<CC, StBF16>(p, npos, y, st);
        case RS_E4M3: return launch_m2_out_np<CC, StE4M3>(p, npos, y, st);
        default: return launch_m2_out_np<CC, StF32>(p, npos, y, st);
    }
}

cudaError_t launch_m2_outputs(const Params &p, int npos, void *y, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_m2_out_cc, (p, npos, y, st));
    return cudaErrorInvalidValue;
}

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
    const size_t ring_bh = (size_t)b * cap;
    const int tid = threadIdx.x;

    RegTile<CC, NPASS> t;
    t.init(R);
    if (p.shared_lowp) load_tile(t, p.copy, tile, p.copy_dtype, p.scale);
    else t.load_f32(p.master + (size_t)tile * R * CC);

    for (int i = tid; i < L; i += kTileThreads)
        s_dt[i] = static_cast<const float *>(p.rb)[(ring_bh + ((head + i) & p.cap_mask)) * H + h];
    const int bchunks = CC * in_bytes / 16;
    for (int q = tid; q < L * bchunks; q += kTileThreads) {
        const int i = q / bchunks, w = q % bchunks;
        const int slot = (head + i) & p.cap_mask;
        const unsigned char *src = static_cast<const unsigned char *>(p.rc) +
                                   (((ring_bh + slot) * p.G + g) * CC) * in_bytes;
        reinterpret_cast<uint4 *>(s_B + (size_t)i * CC * in_bytes)[w] = reinterpret_cast<const uint4 *>(src)[w];
    }
    for (int q = tid; q < L * R; q += kTileThreads) {
        const int i = q / R, r = q % R;
        const int slot = (head + i) & p.cap_mask;
        s_x[q] = ld_in(p.ra, ((ring_bh + slot) * H + h) * R + r, p.in_dtype);
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
    if (tid == 0) {
        __threadfence();
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
