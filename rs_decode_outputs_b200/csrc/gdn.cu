// Gated DeltaNet kernels of the ReplaySSM decode path.
//
// Recurrence (one (sequence, head), state S in R^{dv x dk}):
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = scale S_t q_t
// Row r of the update:  s_r <- alpha (s_r - beta (s_r . k) k) + beta v[r] k.
//
// Replay ("ReplaySSM: Cache SSM Inputs, Not State", Abstract; "ReplaySSM for
// hybrid SSM-Transformer stacks", How ReplaySSM works, steps 2-4).  With
// M_j = alpha_j (I - beta_j k_j k_j^T), the state after buffered entries 1..e is
// S0 M_1..M_e + sum_{i<=e} beta_i v_i k_i^T M_{i+1}..M_e, so the output at
// position e is
//     o_e = scale ( S0 qt + sum_{i<=e} c_i v_i ),   qt = M_1..M_e q_e,
//     c_i = beta_i k_i^T (M_{i+1}..M_e q_e),
// and qt, c are formed by one backward sweep over the buffer per output position:
//     u <- q_e;  for i = e..1:  c_i = beta_i (k_i . u);  u <- alpha_i (u - beta_i (k_i . u) k_i)
// The checkpoint is then read once, as a matrix-vector product with qt.
#include "outputs.cuh"
#include "regtile.cuh"
#include "launch.h"

namespace rs {

struct GdnOutSmem {
    size_t alpha, beta, q, coef, mul, z, kraw, vraw, total;
};

__host__ __device__ inline GdnOutSmem gdn_out_smem(size_t tile_bytes, int cap, int CC, int R,
                                                   int NP, int in_bytes) {
    GdnOutSmem s;
    size_t o = align_up(tile_bytes, 128);
    s.alpha = o; o = align_up(o + 4 * (size_t)cap, 16);
    s.beta = o;  o = align_up(o + 4 * (size_t)cap, 16);
    s.q = o;     o = align_up(o + 4 * (size_t)NP * CC, 16);
    s.coef = o;  o = align_up(o + 4 * (size_t)NP * cap, 16);
    s.mul = o;   o = align_up(o + 4 * (size_t)NP, 16);
    s.z = o;     o = align_up(o + 4 * (size_t)NP * R, 16);
    s.kraw = o;  o = align_up(o + (size_t)in_bytes * cap * CC, 16);
    s.vraw = o;  o = align_up(o + (size_t)in_bytes * cap * R, 16);
    s.total = o;
    return s;
}

// ------------------------------------------------------------- outputs ----

template <int CC, typename TS, int NP>
__global__ void __launch_bounds__(kOutThreads)
gdn_outputs_kernel(const Params p, const void *__restrict__ state, int npos, void *y) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t bar;

    const int R = p.R, H = p.H, cap = p.cap;
    const int tile = blockIdx.x;
    const int b = tile / H, h = tile % H;
    const int in_bytes = p.in_dtype == RS_BF16 ? 2 : 4;
    const uint32_t tile_bytes = static_cast<uint32_t>(R) * CC * TS::bytes;
    const GdnOutSmem L_ = gdn_out_smem(tile_bytes, cap, CC, R, NP, in_bytes);
    float *s_alpha = reinterpret_cast<float *>(smem + L_.alpha);
    float *s_beta = reinterpret_cast<float *>(smem + L_.beta);
    float *s_q = reinterpret_cast<float *>(smem + L_.q);
    float *s_coef = reinterpret_cast<float *>(smem + L_.coef);
    float *s_mul = reinterpret_cast<float *>(smem + L_.mul);
    float *s_z = reinterpret_cast<float *>(smem + L_.z);
    unsigned char *s_k = smem + L_.kraw;
    unsigned char *s_v = smem + L_.vraw;

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
    const size_t ring_bh = (size_t)b * cap;

    if (ok) {
        for (int i = tid; i < L; i += kOutThreads) {
            const size_t at = (ring_bh + ((head + i) & p.cap_mask)) * H + h;
            s_alpha[i] = static_cast<const float *>(p.rd)[at];
            s_beta[i] = static_cast<const float *>(p.re)[at];
        }
        const int kchunks = CC * in_bytes / 16;
        for (int q = tid; q < L * kchunks; q += kOutThreads) {
            const int i = q / kchunks, w = q % kchunks;
            const size_t at = ((ring_bh + ((head + i) & p.cap_mask)) * H + h) * CC;
            reinterpret_cast<uint4 *>(s_k + (size_t)i * CC * in_bytes)[w] =
                reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.rb) + at * in_bytes)[w];
        }
        for (int q = tid; q < L * R; q += kOutThreads) {
            const int i = q / R, r = q % R;
            const size_t src = ((ring_bh + ((head + i) & p.cap_mask)) * H + h) * R + r;
            if (in_bytes == 2)
                reinterpret_cast<uint16_t *>(s_v)[q] = static_cast<const uint16_t *>(p.rc)[src];
            else
                reinterpret_cast<float *>(s_v)[q] = static_cast<const float *>(p.rc)[src];
        }
        for (int q = tid; q < npos * CC; q += kOutThreads) {
            const int j = q / CC, c = q % CC;
            const int slot = (head + L - npos + j) & p.cap_mask;
            s_q[q] = ld_in(p.ra, ((ring_bh + slot) * H + h) * CC + c, p.in_dtype);
        }
    }
    __syncthreads();

    if (ok) {
        // Backward sweep for each output position (one warp per position).
        constexpr int UPL = (CC + 31) / 32;
        for (int j = warp; j < npos; j += nwarps) {
            const int e = L - npos + j;
            float u[UPL];
#pragma unroll
            for (int m = 0; m < UPL; ++m) {
                const int c = lane + 32 * m;
                u[m] = c < CC ? s_q[j * CC + c] : 0.f;
            }
            for (int i = e; i >= 0; --i) {
                float kr[UPL];
                float ku = 0.f;
#pragma unroll
                for (int m = 0; m < UPL; ++m) {
                    const int c = lane + 32 * m;
                    kr[m] = c < CC ? ld_in(s_k, (size_t)i * CC + c, p.in_dtype) : 0.f;
                    ku = fmaf(kr[m], u[m], ku);
                }
                ku = warp_sum(ku);
                const float a = s_alpha[i], f = s_beta[i] * ku;
                if (lane == 0) s_coef[j * cap + i] = f;
#pragma unroll
                for (int m = 0; m < UPL; ++m) u[m] = a * fmaf(-f, kr[m], u[m]);
            }
            __syncwarp();
#pragma unroll
            for (int m = 0; m < UPL; ++m) {
                const int c = lane + 32 * m;
                if (c < CC) s_q[j * CC + c] = u[m];
            }
        }
        const float sc = p.gdn_scale;
        if (tid < npos) s_mul[tid] = sc * (p.copy_dtype == RS_E4M3 ? p.scale[tile] : 1.f);
    }
    __syncthreads();

    if (ok) {
        const float sc = p.gdn_scale;
        for (int q = tid; q < npos * R; q += kOutThreads) {
            const int j = q / R, r = q % R, e = L - npos + j;
            float acc = 0.f;
            for (int i = 0; i <= e; ++i) acc = fmaf(s_coef[j * cap + i], ld_in(s_v, (size_t)i * R + r, p.in_dtype), acc);
            s_z[q] = sc * acc;
        }
    }

    const bool arrived = mbar_wait_bounded(&bar, 0);
    __syncthreads();
    const size_t y_pos_stride = (size_t)p.B * H * R;
    const size_t y_off = (size_t)tile * R;
    if (!ok || !arrived) {
        zero_outputs(R, npos, y, y_pos_stride, y_off, p.out_dtype);
        if (tid == 0) atomicOr(&p.err[b], !arrived ? RS_SEQ_ERR_TIMEOUT : RS_SEQ_ERR_EMPTY);
        return;
    }
    tile_matvec<CC, TS, NP>(smem, R, s_q, npos, s_mul, s_z, y, y_pos_stride, y_off, p.out_dtype);
}

size_t gdn_outputs_smem(const Params &p, int NP) {
    const int eb = p.copy_dtype == RS_BF16 ? 2 : p.copy_dtype == RS_E4M3 ? 1 : 4;
    return gdn_out_smem((size_t)p.R * p.CC * eb, p.cap, p.CC, p.R, NP,
                        p.in_dtype == RS_BF16 ? 2 : 4).total;
}

template <int CC, typename TS, int NP>
static cudaError_t launch_gdn_out_t(const Params &p, int npos, void *y, cudaStream_t st) {
    const void *state = p.copy_dtype == RS_NONE ? static_cast<const void *>(p.master) : p.copy;
    const size_t smem = gdn_outputs_smem(p, NP);
    auto k = gdn_outputs_kernel<CC, TS, NP>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<p.B * p.H, kOutThreads, smem, st>>>(p, state, npos, y);
    return cudaGetLastError();
}

template <int CC, typename TS>
static cudaError_t launch_gdn_out_np(const Params &p, int npos, void *y, cudaStream_t st) {
    if (npos <= 1) return launch_gdn_out_t<CC, TS, 1>(p, npos, y, st);
    if (npos <= 2) return launch_gdn_out_t<CC, TS, 2>(p, npos, y, st);
    if (npos <= 4) return launch_gdn_out_t<CC, TS, 4>(p, npos, y, st);
    return launch_gdn_out_t<CC, TS, 8>(p, npos, y, st);
}

template <int CC>
static cudaError_t launch_gdn_out_cc(const Params &p, int npos, void *y, cudaStream_t st) {
    switch (p.copy_dtype) {
        case RS_BF16: return launch_gdn_out_np<CC, StBF16>(p, npos, y, st);
        case RS_E4M3: return launch_gdn_out_np<CC, StE4M3>(p, npos, y, st);
        default: return launch_gdn_out_np<CC, StF32>(p, npos, y, st);
    }
}

cudaError_t launch_gdn_outputs(const Params &p, int npos, void *y, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_gdn_out_cc, (p, npos, y, st));
    return cudaErrorInvalidValue;
}

// -------------------------------------------------------------- commit ----
// Fold the buffer into the fp32 master row by row, in buffer order, with the
// tile in registers; rewrite master and copy; the last CTA of a sequence moves
// head to tail.

template <int CC, int NPASS>
__global__ void __launch_bounds__(kTileThreads)
gdn_commit_kernel(const Params p, int min_len, const int32_t *__restrict__ mask) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kTileThreads / 32];
    using T = RegTile<CC, NPASS>;
    const int R = p.R, H = p.H, cap = p.cap;
    const int tile = blockIdx.x;
    const int b = tile / H, h = tile % H;
    const int head = p.head[b];
    const int L = p.tail[b] - head;
    if (L < (min_len > 1 ? min_len : 1) || L > cap || (mask && mask[b] == 0)) return;

    const int in_bytes = p.in_dtype == RS_BF16 ? 2 : 4;
    float *s_alpha = reinterpret_cast<float *>(smem);
    float *s_beta = s_alpha + cap;
    float *s_v = s_beta + cap;  // [cap][R]
    unsigned char *s_k = smem + align_up(4 * (2 * (size_t)cap + (size_t)cap * R), 16);  // [cap][CC]
    const size_t ring_bh = (size_t)b * cap;
    const int tid = threadIdx.x;

    T t;
    t.init(R);
    if (p.shared_lowp) load_tile(t, p.copy, tile, p.copy_dtype, p.scale);
    else t.load_f32(p.master + (size_t)tile * R * CC);

    for (int i = tid; i < L; i += kTileThreads) {
        const size_t at = (ring_bh + ((head + i) & p.cap_mask)) * H + h;
        s_alpha[i] = static_cast<const float *>(p.rd)[at];
        s_beta[i] = static_cast<const float *>(p.re)[at];
    }
    const int kchunks = CC * in_bytes / 16;
    for (int q = tid; q < L * kchunks; q += kTileThreads) {
        const int i = q / kchunks, w = q % kchunks;
        const size_t at = ((ring_bh + ((head + i) & p.cap_mask)) * H + h) * CC;
        reinterpret_cast<uint4 *>(s_k + (size_t)i * CC * in_bytes)[w] =
            reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.rb) + at * in_bytes)[w];
    }
    for (int q = tid; q < L * R; q += kTileThreads) {
        const int i = q / R, r = q % R;
        s_v[q] = ld_in(p.rc, ((ring_bh + ((head + i) & p.cap_mask)) * H + h) * R + r, p.in_dtype);
    }
    __syncthreads();

    for (int i = 0; i < L; ++i) {
        float kf[T::NE];
#pragma unroll
        for (int c = 0; c < T::CPT; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) kf[c * 4 + e] = ld_in(s_k, (size_t)i * CC + t.col(c) + e, p.in_dtype);
        const float a = s_alpha[i], bt = s_beta[i];
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < T::NE; ++e) d = fmaf(t.s[k][e], kf[e], d);
            d = row_sum<T::TPR>(d);
            const float vr = t.valid(k) ? s_v[(size_t)i * R + t.row(k)] : 0.f;
            const float m = bt * fmaf(-a, d, vr);   // beta v[r] - alpha beta (s . k)
#pragma unroll
            for (int e = 0; e < T::NE; ++e) t.s[k][e] = fmaf(a, t.s[k][e], m * kf[e]);
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

size_t gdn_commit_smem(const Params &p) {
    const int in_bytes = p.in_dtype == RS_BF16 ? 2 : 4;
    return align_up(4 * (2 * (size_t)p.cap + (size_t)p.cap * p.R), 16) +
           (size_t)in_bytes * p.cap * p.CC;
}

template <int CC, int NPASS>
static cudaError_t launch_gdn_commit_t(const Params &p, int min_len, const int32_t *mask,
                                       cudaStream_t st) {
    const size_t smem = gdn_commit_smem(p);
    auto k = gdn_commit_kernel<CC, NPASS>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<p.B * p.H, kTileThreads, smem, st>>>(p, min_len, mask);
    return cudaGetLastError();
}

template <int CC>
static cudaError_t launch_gdn_commit_cc(const Params &p, int min_len, const int32_t *mask,
                                        cudaStream_t st) {
    RS_DISPATCH_NPASS(CC, p.R, return launch_gdn_commit_t, (p, min_len, mask, st));
    return cudaErrorInvalidValue;
}

cudaError_t launch_gdn_commit(const Params &p, int min_len, const int32_t *mask, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_gdn_commit_cc, (p, min_len, mask, st));
    return cudaErrorInvalidValue;
}

// --------------------------------------------------------------- eager ----

template <int CC, int NPASS>
__global__ void __launch_bounds__(kTileThreads)
gdn_eager_kernel(const Params p, void *state, int sdt, rs_inputs in, int T, void *y,
                 const int32_t *__restrict__ cur, int nslots) {
    __shared__ float red[kTileThreads / 32];
    using RT = RegTile<CC, NPASS>;
    const int R = p.R, H = p.H;
    const int tile = blockIdx.x;
    const int b = tile / H;
    const size_t n_all = (size_t)p.B * H;
    RT t;
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
    const float sc = p.gdn_scale;

    for (int ts = 0; ts < T; ++ts) {
        const size_t bh = (size_t)ts * n_all + tile;
        const float a = in.alpha[bh], bt = in.beta[bh];
        float kf[RT::NE], qf[RT::NE];
#pragma unroll
        for (int c = 0; c < RT::CPT; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kf[c * 4 + e] = ld_in(in.k, bh * CC + t.col(c) + e, p.in_dtype);
                qf[c * 4 + e] = ld_in(in.q, bh * CC + t.col(c) + e, p.in_dtype);
            }
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < RT::NE; ++e) d = fmaf(t.s[k][e], kf[e], d);
            d = row_sum<RT::TPR>(d);
            const float vr = t.valid(k) ? ld_in(in.v, bh * R + t.row(k), p.in_dtype) : 0.f;
            const float m = bt * fmaf(-a, d, vr);
#pragma unroll
            for (int e = 0; e < RT::NE; ++e) t.s[k][e] = fmaf(a, t.s[k][e], m * kf[e]);
        }
        if (sdt == RS_BF16) t.round_bf16();
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            float o = 0.f;
#pragma unroll
            for (int e = 0; e < RT::NE; ++e) o = fmaf(t.s[k][e], qf[e], o);
            o = row_sum<RT::TPR>(o);
            if (t.valid(k) && t.lane == 0) st_out(y, bh * R + t.row(k), sc * o, p.out_dtype);
        }
        if (cur) store_tile(t, state, (size_t)((c0 + 1 + ts) % nslots) * n_all + tile, sdt, nullptr, red);
    }
    if (!cur) store_tile(t, state, tile, sdt, nullptr, red);
}

template <int CC, int NPASS>
static cudaError_t launch_gdn_eager_t(const Params &p, void *state, int sdt, const rs_inputs &in,
                                      int T, void *y, const int32_t *cur, int nslots,
                                      cudaStream_t st) {
    gdn_eager_kernel<CC, NPASS><<<p.B * p.H, kTileThreads, 0, st>>>(p, state, sdt, in, T, y, cur,
                                                                  nslots);
    return cudaGetLastError();
}

template <int CC>
static cudaError_t launch_gdn_eager_cc(const Params &p, void *state, int sdt, const rs_inputs &in,
                                       int T, void *y, const int32_t *cur, int nslots,
                                       cudaStream_t st) {
    RS_DISPATCH_NPASS(CC, p.R, return launch_gdn_eager_t, (p, state, sdt, in, T, y, cur, nslots, st));
    return cudaErrorInvalidValue;
}

cudaError_t launch_gdn_eager(const Params &p, void *state, int sdt, const rs_inputs &in, int T,
                             void *y, const int32_t *cur, int nslots, cudaStream_t st) {
    RS_DISPATCH_CC(p.CC, return launch_gdn_eager_cc, (p, state, sdt, in, T, y, cur, nslots, st));
    return cudaErrorInvalidValue;
}

}  // namespace rs
