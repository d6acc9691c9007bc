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
    float *s_v = s_beta + cap;  // [cap][R] fp32
    float *s_k = reinterpret_cast<float *>(smem + align_up(4 * (2 * (size_t)cap + (size_t)cap * R), 16));  // [cap][CC] fp32
    const int tid = threadIdx.x;
    // this head's ring blocks
    const size_t bh = (size_t)b * H + h;
    const unsigned char *kblk = static_cast<const unsigned char *>(p.rb) + bh * p.blk_c;
    const unsigned char *vblk = static_cast<const unsigned char *>(p.rc) + bh * p.blk_r;
    const float *ablk = static_cast<const float *>(p.rd) + bh * p.capd;
    const float *bblk = static_cast<const float *>(p.re) + bh * p.capd;

    T t;
    t.init(R);
    if (p.shared_lowp) load_tile(t, p.copy, tile, p.copy_dtype, p.scale);
    else t.load_f32(p.master + (size_t)tile * R * CC);

    for (int i = tid; i < L; i += kTileThreads) {
        const int slot = (head + i) & p.cap_mask;
        s_alpha[i] = ablk[slot];
        s_beta[i] = bblk[slot];
    }
    // k rows as fp32, 16 input bytes per thread and step
    const int kshift = __ffs(CC * in_bytes / 16) - 1;   // 16-byte pieces per row, log2
    for (int q = tid; q < (L << kshift); q += kTileThreads) {
        const int i = q >> kshift, w = q & ((1 << kshift) - 1);
        const uint4 v = reinterpret_cast<const uint4 *>(kblk + (size_t)((head + i) & p.cap_mask) * CC * in_bytes)[w];
        float *dst = s_k + (size_t)i * CC + w * (16 / in_bytes);
        if (in_bytes == 2) {
            reinterpret_cast<float4 *>(dst)[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
            reinterpret_cast<float4 *>(dst)[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
        } else {
            *reinterpret_cast<uint4 *>(dst) = v;
        }
    }
    for (int i = tid >> 5; i < L; i += kTileThreads / 32) {
        const unsigned char *row = vblk + (size_t)((head + i) & p.cap_mask) * R * in_bytes;
        for (int r = tid & 31; r < R; r += 32) s_v[i * R + r] = ld_in(row, r, p.in_dtype);
    }
    __syncthreads();

    for (int i = 0; i < L; ++i) {
        float kf[T::NE];
#pragma unroll
        for (int c = 0; c < T::CPT; ++c) {
            const float4 f = *reinterpret_cast<const float4 *>(s_k + (size_t)i * CC + t.col(c));
            kf[c * 4] = f.x;
            kf[c * 4 + 1] = f.y;
            kf[c * 4 + 2] = f.z;
            kf[c * 4 + 3] = f.w;
        }
        const float a = s_alpha[i], bt = s_beta[i];
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
            float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < T::NE; e += 2)
                d2 = ffma2(make_float2(t.s[k][e], t.s[k][e + 1]), make_float2(kf[e], kf[e + 1]), d2);
            const float d = row_sum<T::TPR>(d2.x + d2.y);
            const float vr = t.valid(k) ? s_v[(size_t)i * R + t.row(k)] : 0.f;
            const float m = bt * fmaf(-a, d, vr);   // beta v[r] - alpha beta (s . k)
#pragma unroll
            for (int e = 0; e < T::NE; e += 2) {   // s <- alpha s + m k
                const float2 r = ffma2(make_float2(a, a), make_float2(t.s[k][e], t.s[k][e + 1]),
                                       fmul2(make_float2(m, m), make_float2(kf[e], kf[e + 1])));
                t.s[k][e] = r.x;
                t.s[k][e + 1] = r.y;
            }
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

size_t gdn_commit_smem(const Params &p) {
    return align_up(4 * (2 * (size_t)p.cap + (size_t)p.cap * p.R), 16) + 4 * (size_t)p.cap * p.CC;
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
