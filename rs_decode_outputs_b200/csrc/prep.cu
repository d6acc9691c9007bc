// Replay prologue ("prep") kernels, optionally fused with the append of the
// step's inputs.
//
// For every (sequence, head) they reduce the buffered inputs to the few
// numbers the output-only pass needs at NP output positions (e_j = L - npos + j,
// 0-based buffer index), so that  y_j[r] = mul_j (S0[r, :] . vec_j) + z_j[r]:
// Mamba-2 ("ReplaySSM for hybrid SSM-Transformer stacks", How ReplaySSM works,
// step 2: the output is a function of the checkpoint and the recent inputs):
//   vec_j = C_{e_j},  mul_j = exp(A sum_{m<=e_j} dt_m) (x the fp8 tile scale),
//   z_j = sum_{i<=e_j} exp(A sum_{i<m<=e_j} dt_m) dt_i (B_i . C_{e_j}) x_i + D x_{e_j}
// GDN:  vec_j = M_1..M_{e_j} q_{e_j}  (M_i = alpha_i (I - beta_i k_i k_i^T)), by the
//   backward sweep  u <- q_{e_j};  for i = e_j..1: c_i = beta_i (k_i . u);
//   u <- alpha_i (u - c_i k_i);  mul_j = scale (x tile scale),  z_j = scale sum_i c_i v_i.
//
// With T > 0 the kernel also appends the T step inputs (step 2: append the new
// SSM input to the buffer): the new entries are read straight from the inputs,
// written into their ring slots, and the last CTA of a sequence to finish
// advances its tail by T (per-sequence arrival counter).  A sequence whose
// buffer would overflow is left unchanged and flagged.
//
// Both kernels are short latency-bound chains; they read the pointers once,
// stage exactly the buffered rows they need into shared memory with one round
// of asynchronous copies, and compute from shared memory.
#include "outputs.cuh"
#include "launch.h"

namespace rs {

constexpr int kPrepWarps = 8;   // warps per CTA, one head per warp

__device__ __forceinline__ float warp_incl_scan(float v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Asynchronous copy of one row of `bytes` from global to shared memory with
// threads t, t + nthr, ...: 16-byte pieces when both ends and the size allow,
// else 4-byte pieces, else 2-byte plain loads (synchronous).
__device__ __forceinline__ void stage_row(void *dst, const void *src, int bytes, int t, int nthr) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | (uintptr_t)bytes;
    if ((a & 15) == 0) {
        for (int q = t; q < bytes / 16; q += nthr)
            cp_async16(static_cast<char *>(dst) + 16 * q, static_cast<const char *>(src) + 16 * q);
    } else if ((a & 3) == 0) {
        for (int q = t; q < bytes / 4; q += nthr)
            cp_async4(static_cast<char *>(dst) + 4 * q, static_cast<const char *>(src) + 4 * q);
    } else {
        for (int q = t; q < bytes / 2; q += nthr)
            static_cast<uint16_t *>(dst)[q] = static_cast<const uint16_t *>(src)[q];
    }
}

// Plain copy of one row (shared or global source, global destination).
__device__ __forceinline__ void copy_row(void *dst, const void *src, int bytes, int t, int nthr) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | (uintptr_t)bytes;
    if ((a & 15) == 0) {
        for (int q = t; q < bytes / 16; q += nthr) static_cast<uint4 *>(dst)[q] = static_cast<const uint4 *>(src)[q];
    } else if ((a & 3) == 0) {
        for (int q = t; q < bytes / 4; q += nthr) static_cast<uint32_t *>(dst)[q] = static_cast<const uint32_t *>(src)[q];
    } else {
        for (int q = t; q < bytes / 2; q += nthr) static_cast<uint16_t *>(dst)[q] = static_cast<const uint16_t *>(src)[q];
    }
}

// Last arrival of the CTAs of sequence b advances its tail by T.
__device__ __forceinline__ void arrive_and_advance(const Params &p, int b, int tail, int T, int ctas) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&p.arrive[b], 1u) == static_cast<unsigned>(ctas - 1)) {
            p.arrive[b] = 0u;
            p.tail[b] = tail + T;
        }
    }
}

// ---------------------------------------------------------------- Mamba-2 --
// One CTA per (sequence, group, chunk of kPrepWarps heads).  Buffered entries
// are staged compactly, buffer index i at row i.  Shared memory:
//   braw [cap][CC] | craw [NP][CC] | Cf [NP][CC] | bc [NP][cap] |
//   per warp: xraw [cap][R] | dt [cap] | cum [cap] | coef [NP][cap]
struct M2PrepSmem {
    size_t braw, craw, cf, bc, warps, per_warp, x, dt, cum, coef, total;
};

__host__ __device__ inline M2PrepSmem m2_prep_smem(int cap, int R, int CC, int NP, int ib) {
    M2PrepSmem s;
    size_t o = 0;
    s.braw = o; o = align_up(o + (size_t)cap * CC * ib, 16);
    s.craw = o; o = align_up(o + (size_t)NP * CC * ib, 16);
    s.cf = o;   o = align_up(o + 4 * (size_t)NP * CC, 16);
    s.bc = o;   o = align_up(o + 4 * (size_t)NP * cap, 16);
    s.warps = o;
    size_t w = 0;
    s.x = w;    w = align_up(w + (size_t)cap * R * ib, 16);
    s.dt = w;   w = align_up(w + 4 * (size_t)cap, 16);
    s.cum = w;  w = align_up(w + 4 * (size_t)cap, 16);
    s.coef = w; w = align_up(w + 4 * (size_t)NP * cap, 16);
    s.per_warp = w;
    s.total = o + kPrepWarps * w;
    return s;
}

template <int CC, int NP>
__global__ void __launch_bounds__(32 * kPrepWarps)
m2_prep_kernel(const Params p, int npos, int T, rs_inputs in) {
    extern __shared__ __align__(16) unsigned char psm[];
    __shared__ int s_head, s_tail;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int Bn = p.B, H = p.H, R = p.R, cap = p.cap, ib = p.in_dtype == RS_BF16 ? 2 : 4;
    const int hpg = p.heads_per_group;
    const int g = blockIdx.y, b = blockIdx.z;
    const int hl = blockIdx.x * kPrepWarps + warp;   // head within the group
    const bool has_head = hl < hpg;
    const int h = g * hpg + hl;
    const int tile = b * H + h;
    const M2PrepSmem S = m2_prep_smem(cap, R, CC, NP, ib);
    unsigned char *braw = psm + S.braw, *craw = psm + S.craw;
    float *Cf = reinterpret_cast<float *>(psm + S.cf), *bc = reinterpret_cast<float *>(psm + S.bc);
    unsigned char *wsm = psm + S.warps + (size_t)warp * S.per_warp;
    unsigned char *xraw = wsm + S.x;
    float *dt = reinterpret_cast<float *>(wsm + S.dt), *cum = reinterpret_cast<float *>(wsm + S.cum);
    float *coef = reinterpret_cast<float *>(wsm + S.coef);
    const size_t trf = tile_rec_floats(RS_MAMBA2, NP, R, CC);
    float *trec = p.rec + p.rec_tile_off + (size_t)tile * trf;
    float *grec = p.rec + ((size_t)b * p.G + g) * group_rec_floats(NP, CC);
    const size_t rowB = (size_t)CC * ib, rowX = (size_t)R * ib;

    if (threadIdx.x == 0) {
        s_head = p.head[b];
        s_tail = p.tail[b];
    }
    __syncthreads();
    const int head = s_head, tail = s_tail, L_old = tail - head, L = L_old + T;
    if (L_old < 0 || L > cap) {   // corrupt pointers or ring overflow: nothing is appended
        if (has_head)
            for (size_t i = lane; i < trf; i += 32) trec[i] = 0.f;
        if (blockIdx.x == 0)
            for (size_t i = threadIdx.x; i < (size_t)NP * CC; i += blockDim.x) grec[i] = 0.f;
        if (threadIdx.x == 0) atomicOr(&p.err[b], T > 0 ? RS_SEQ_ERR_OVERFLOW : RS_SEQ_ERR_EMPTY);
        return;
    }
    const bool ok = npos >= 1 && L >= npos;
    const unsigned char *bblk = static_cast<const unsigned char *>(p.rc) + ((size_t)b * p.G + g) * p.blk_c;
    const unsigned char *cblk = static_cast<const unsigned char *>(p.rd) + ((size_t)b * p.G + g) * p.blk_c;
    const unsigned char *xblk = static_cast<const unsigned char *>(p.ra) + (size_t)tile * p.blk_r;
    const float *dtblk = static_cast<const float *>(p.rb) + (size_t)tile * p.capd;
    // source row of buffer entry i: ring slot for the entries already buffered, the step inputs for the new ones
    auto b_src = [&](int i) -> const void * {
        return i < L_old ? static_cast<const void *>(bblk + (size_t)((head + i) & p.cap_mask) * rowB)
                         : static_cast<const void *>(static_cast<const unsigned char *>(in.B) +
                                                     (((size_t)(i - L_old) * Bn + b) * p.G + g) * rowB);
    };
    auto c_src = [&](int i) -> const void * {
        return i < L_old ? static_cast<const void *>(cblk + (size_t)((head + i) & p.cap_mask) * rowB)
                         : static_cast<const void *>(static_cast<const unsigned char *>(in.C) +
                                                     (((size_t)(i - L_old) * Bn + b) * p.G + g) * rowB);
    };
    // ---- one round of asynchronous copies
    if (ok) {
        for (int i = warp; i < L; i += kPrepWarps) stage_row(braw + (size_t)i * rowB, b_src(i), (int)rowB, lane, 32);
        for (int j = warp; j < npos; j += kPrepWarps)
            stage_row(craw + (size_t)j * rowB, c_src(L - npos + j), (int)rowB, lane, 32);
    }
    if (has_head) {
        for (int i = 0; i < L; ++i) {
            const void *src = i < L_old ? static_cast<const void *>(xblk + (size_t)((head + i) & p.cap_mask) * rowX)
                                        : static_cast<const void *>(static_cast<const unsigned char *>(in.x) +
                                                                    (((size_t)(i - L_old) * Bn + b) * H + h) * rowX);
            stage_row(xraw + (size_t)i * rowX, src, (int)rowX, lane, 32);
        }
        for (int i = lane; i < L; i += 32)
            cp_async4(dt + i, i < L_old ? dtblk + ((head + i) & p.cap_mask) : in.dt + ((size_t)(i - L_old) * Bn + b) * H + h);
    }
    cp_async_wait_all();
    __syncthreads();

    if (ok) {
        // ---- C of the output positions as fp32, and B_i . C_{e_j} (shared by the CTA's heads)
        for (int q = threadIdx.x; q < npos * CC; q += blockDim.x) Cf[q] = lds_in(craw, q, p.in_dtype);
        __syncthreads();
        if (blockIdx.x == 0)
            for (int q = threadIdx.x; q < npos * CC; q += blockDim.x) grec[q] = Cf[q];
        for (int w = warp; w < npos * L; w += kPrepWarps) {
            const int j = w / L, i = w - (w / L) * L;
            if (i > L - npos + j) continue;
            float d = 0.f;
            for (int n = lane; n < CC; n += 32) d = fmaf(lds_in(braw, (size_t)i * CC + n, p.in_dtype), Cf[j * CC + n], d);
            d = warp_sum(d);
            if (lane == 0) bc[j * cap + i] = d;
        }
        __syncthreads();
        if (has_head) {
            // ---- per head: prefix sums of dt, coefficients, z
            float *mul = trec, *z = trec + 8;
            const float A = p.A[h];
            const float Dh = p.D ? p.D[h] : 0.f;
            const float tscale = p.copy_dtype == RS_E4M3 ? p.scale[tile] : 1.f;
            float carry = 0.f;
            for (int i0 = 0; i0 < L; i0 += 32) {
                const int i = i0 + lane;
                const float d = i < L ? dt[i] : 0.f;
                const float c = warp_incl_scan(d, lane) + carry;
                if (i < L) cum[i] = c;
                carry = __shfl_sync(0xffffffffu, c, 31);
            }
            __syncwarp();
            for (int j = 0; j < npos; ++j) {
                const int e = L - npos + j;
                const float ce = cum[e];
                if (lane == 0) mul[j] = expf(A * ce) * tscale;
                for (int i = lane; i <= e; i += 32) coef[j * cap + i] = expf(A * (ce - cum[i])) * dt[i] * bc[j * cap + i];
            }
            __syncwarp();
            constexpr int RL = 8;   // rows per lane, R <= 256
            float acc[NP][RL];
#pragma unroll
            for (int j = 0; j < NP; ++j)
#pragma unroll
                for (int m = 0; m < RL; ++m) acc[j][m] = 0.f;
            for (int i = 0; i < L; ++i) {
                float cf[NP];
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const int e = L - npos + j;
                    cf[j] = (j < npos && i <= e) ? coef[j * cap + i] : 0.f;
                    if (j < npos && i == e) cf[j] += Dh;
                }
#pragma unroll
                for (int m = 0; m < RL; ++m) {
                    const int r = lane + 32 * m;
                    if (r >= R) break;
                    const float xv = lds_in(xraw, (size_t)i * R + r, p.in_dtype);
#pragma unroll
                    for (int j = 0; j < NP; ++j) acc[j][m] = fmaf(cf[j], xv, acc[j][m]);
                }
            }
#pragma unroll
            for (int m = 0; m < RL; ++m) {
                const int r = lane + 32 * m;
                if (r >= R) break;
#pragma unroll
                for (int j = 0; j < NP; ++j)
                    if (j < npos) z[j * R + r] = acc[j][m];
            }
        }
    } else {
        if (has_head)
            for (size_t i = lane; i < trf; i += 32) trec[i] = 0.f;
        if (blockIdx.x == 0)
            for (size_t i = threadIdx.x; i < (size_t)NP * CC; i += blockDim.x) grec[i] = 0.f;
        if (threadIdx.x == 0 && T == 0) atomicOr(&p.err[b], RS_SEQ_ERR_EMPTY);
    }

    if (T > 0) {
        // ---- append: the new entries into their ring slots
        if (has_head) {
            for (int t = 0; t < T; ++t) {
                const int slot = (tail + t) & p.cap_mask;
                copy_row(const_cast<unsigned char *>(xblk) + (size_t)slot * rowX, xraw + (size_t)(L_old + t) * rowX,
                         (int)rowX, lane, 32);
            }
            for (int t = lane; t < T; t += 32)
                const_cast<float *>(dtblk)[(tail + t) & p.cap_mask] = dt[L_old + t];
        }
        if (blockIdx.x == 0)
            for (int t = warp; t < T; t += kPrepWarps) {
                const int slot = (tail + t) & p.cap_mask;
                copy_row(const_cast<unsigned char *>(bblk) + (size_t)slot * rowB,
                         static_cast<const unsigned char *>(in.B) + (((size_t)t * Bn + b) * p.G + g) * rowB, (int)rowB, lane, 32);
                copy_row(const_cast<unsigned char *>(cblk) + (size_t)slot * rowB,
                         static_cast<const unsigned char *>(in.C) + (((size_t)t * Bn + b) * p.G + g) * rowB, (int)rowB, lane, 32);
            }
        arrive_and_advance(p, b, tail, T, gridDim.x * gridDim.y);
        if (threadIdx.x == 0 && !ok) atomicOr(&p.err[b], RS_SEQ_ERR_EMPTY);
    }
}

// -------------------------------------------------------------------- GDN --
// One warp per (sequence, head); a CTA holds kPrepWarps heads of one sequence.
// Per-warp shared memory (entries compact, buffer index i at row i):
//   kraw [cap][CC] | vraw [cap][R] | qraw [NP][CC] | alpha [cap] | beta [cap] | coef [NP][cap]
struct GdnPrepSmem {
    size_t k, v, q, alpha, beta, coef, per_warp;
};

__host__ __device__ inline GdnPrepSmem gdn_prep_smem(int cap, int R, int CC, int NP, int ib) {
    GdnPrepSmem s;
    size_t w = 0;
    s.k = w;     w = align_up(w + (size_t)cap * CC * ib, 16);
    s.v = w;     w = align_up(w + (size_t)cap * R * ib, 16);
    s.q = w;     w = align_up(w + (size_t)NP * CC * ib, 16);
    s.alpha = w; w = align_up(w + 4 * (size_t)cap, 16);
    s.beta = w;  w = align_up(w + 4 * (size_t)cap, 16);
    s.coef = w;  w = align_up(w + 4 * (size_t)NP * cap, 16);
    s.per_warp = w;
    return s;
}

template <int CC, int NP>
__global__ void __launch_bounds__(32 * kPrepWarps)
gdn_prep_kernel(const Params p, int npos, int T, rs_inputs in) {
    extern __shared__ __align__(16) unsigned char psm[];
    __shared__ int s_head, s_tail;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int Bn = p.B, H = p.H, R = p.R, cap = p.cap, ib = p.in_dtype == RS_BF16 ? 2 : 4;
    const int b = blockIdx.y;
    const int h = blockIdx.x * kPrepWarps + warp;
    const bool has_head = h < H;
    const int tile = b * H + h;
    const GdnPrepSmem S = gdn_prep_smem(cap, R, CC, NP, ib);
    unsigned char *wsm = psm + (size_t)warp * S.per_warp;
    unsigned char *kraw = wsm + S.k, *vraw = wsm + S.v, *qraw = wsm + S.q;
    float *alpha = reinterpret_cast<float *>(wsm + S.alpha), *beta = reinterpret_cast<float *>(wsm + S.beta);
    float *coef = reinterpret_cast<float *>(wsm + S.coef);
    const size_t trf = tile_rec_floats(RS_GDN, NP, R, CC);
    float *trec = p.rec + p.rec_tile_off + (size_t)tile * trf;
    const size_t rowC = (size_t)CC * ib, rowR = (size_t)R * ib;

    if (threadIdx.x == 0) {
        s_head = p.head[b];
        s_tail = p.tail[b];
    }
    __syncthreads();
    const int head = s_head, tail = s_tail, L_old = tail - head, L = L_old + T;
    if (L_old < 0 || L > cap) {
        if (has_head)
            for (size_t i = lane; i < trf; i += 32) trec[i] = 0.f;
        if (threadIdx.x == 0) atomicOr(&p.err[b], T > 0 ? RS_SEQ_ERR_OVERFLOW : RS_SEQ_ERR_EMPTY);
        return;
    }
    const bool ok = npos >= 1 && L >= npos;
    const size_t bh = has_head ? (size_t)tile : 0;
    unsigned char *qblk = static_cast<unsigned char *>(p.ra) + bh * p.blk_c;
    unsigned char *kblk = static_cast<unsigned char *>(p.rb) + bh * p.blk_c;
    unsigned char *vblk = static_cast<unsigned char *>(p.rc) + bh * p.blk_r;
    float *ablk = static_cast<float *>(p.rd) + bh * p.capd;
    float *bblk = static_cast<float *>(p.re) + bh * p.capd;
    auto src_row = [&](const unsigned char *blk, const void *inp, size_t row, int i) -> const void * {
        return i < L_old ? static_cast<const void *>(blk + (size_t)((head + i) & p.cap_mask) * row)
                         : static_cast<const void *>(static_cast<const unsigned char *>(inp) +
                                                     (((size_t)(i - L_old) * Bn + b) * H + h) * row);
    };
    if (has_head) {
        // ---- one round of asynchronous copies
        for (int i = 0; i < L; ++i) {
            stage_row(kraw + (size_t)i * rowC, src_row(kblk, in.k, rowC, i), (int)rowC, lane, 32);
            if (ok) stage_row(vraw + (size_t)i * rowR, src_row(vblk, in.v, rowR, i), (int)rowR, lane, 32);
        }
        if (ok)
            for (int j = 0; j < npos; ++j)
                stage_row(qraw + (size_t)j * rowC, src_row(qblk, in.q, rowC, L - npos + j), (int)rowC, lane, 32);
        for (int i = lane; i < L; i += 32) {
            const size_t at = ((size_t)(i - L_old) * Bn + b) * H + h;
            cp_async4(alpha + i, i < L_old ? ablk + ((head + i) & p.cap_mask) : in.alpha + at);
            cp_async4(beta + i, i < L_old ? bblk + ((head + i) & p.cap_mask) : in.beta + at);
        }
        cp_async_wait_all();
        __syncwarp();

        if (ok) {
            float *mul = trec, *z = trec + 8, *vec = z + (size_t)NP * R;
            const float sc = p.gdn_scale;
            const float tscale = p.copy_dtype == RS_E4M3 ? p.scale[tile] : 1.f;
            constexpr int UPL = (CC + 31) / 32;
            float u[NP][UPL];
#pragma unroll
            for (int j = 0; j < NP; ++j)
#pragma unroll
                for (int m = 0; m < UPL; ++m) {
                    const int c = lane + 32 * m;
                    u[j][m] = (j < npos && c < CC) ? lds_in(qraw, (size_t)j * CC + c, p.in_dtype) : 0.f;
                }
            // lockstep backward sweep of all output positions
            for (int i = L - 1; i >= 0; --i) {
                float kr[UPL];
#pragma unroll
                for (int m = 0; m < UPL; ++m) {
                    const int c = lane + 32 * m;
                    kr[m] = c < CC ? lds_in(kraw, (size_t)i * CC + c, p.in_dtype) : 0.f;
                }
                const float a = alpha[i], bt = beta[i];
                float d[NP];
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    d[j] = 0.f;
#pragma unroll
                    for (int m = 0; m < UPL; ++m) d[j] = fmaf(kr[m], u[j][m], d[j]);
                }
#pragma unroll
                for (int j = 0; j < NP; ++j)
                    if (j < npos) d[j] = warp_sum(d[j]);
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    if (j < npos && i <= L - npos + j) {
                        const float f = bt * d[j];
                        if (lane == 0) coef[j * cap + i] = f;
#pragma unroll
                        for (int m = 0; m < UPL; ++m) u[j][m] = a * fmaf(-f, kr[m], u[j][m]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                if (j < npos) {
#pragma unroll
                    for (int m = 0; m < UPL; ++m) {
                        const int c = lane + 32 * m;
                        if (c < CC) vec[j * CC + c] = u[j][m];
                    }
                    if (lane == 0) mul[j] = sc * tscale;
                }
            }
            __syncwarp();
            constexpr int RL = 8;   // rows per lane, R <= 256
            float acc[NP][RL];
#pragma unroll
            for (int j = 0; j < NP; ++j)
#pragma unroll
                for (int m = 0; m < RL; ++m) acc[j][m] = 0.f;
            for (int i = 0; i < L; ++i) {
                float cf[NP];
#pragma unroll
                for (int j = 0; j < NP; ++j) cf[j] = (j < npos && i <= L - npos + j) ? coef[j * cap + i] : 0.f;
#pragma unroll
                for (int m = 0; m < RL; ++m) {
                    const int r = lane + 32 * m;
                    if (r >= R) break;
                    const float vv = lds_in(vraw, (size_t)i * R + r, p.in_dtype);
#pragma unroll
                    for (int j = 0; j < NP; ++j) acc[j][m] = fmaf(cf[j], vv, acc[j][m]);
                }
            }
#pragma unroll
            for (int m = 0; m < RL; ++m) {
                const int r = lane + 32 * m;
                if (r >= R) break;
#pragma unroll
                for (int j = 0; j < NP; ++j)
                    if (j < npos) z[j * R + r] = sc * acc[j][m];
            }
        } else {
            for (size_t i = lane; i < trf; i += 32) trec[i] = 0.f;
        }

        if (T > 0) {   // ---- append: the new entries into their ring slots
            for (int t = 0; t < T; ++t) {
                const int slot = (tail + t) & p.cap_mask;
                const size_t at = ((size_t)t * Bn + b) * H + h;
                copy_row(kblk + (size_t)slot * rowC, kraw + (size_t)(L_old + t) * rowC, (int)rowC, lane, 32);
                copy_row(qblk + (size_t)slot * rowC, static_cast<const unsigned char *>(in.q) + at * rowC, (int)rowC, lane, 32);
                copy_row(vblk + (size_t)slot * rowR, static_cast<const unsigned char *>(in.v) + at * rowR, (int)rowR, lane, 32);
            }
            for (int t = lane; t < T; t += 32) {
                ablk[(tail + t) & p.cap_mask] = alpha[L_old + t];
                bblk[(tail + t) & p.cap_mask] = beta[L_old + t];
            }
        }
    }
    if (T > 0) arrive_and_advance(p, b, tail, T, gridDim.x);
    if (threadIdx.x == 0 && !ok) atomicOr(&p.err[b], RS_SEQ_ERR_EMPTY);
}

size_t prep_smem(const Params &p, int NP) {
    const int ib = p.in_dtype == RS_BF16 ? 2 : 4;
    if (p.kind == RS_MAMBA2) return m2_prep_smem(p.cap, p.R, p.CC, NP, ib).total;
    return kPrepWarps * gdn_prep_smem(p.cap, p.R, p.CC, NP, ib).per_warp;
}

template <int KIND, int CC, int NP>
static cudaError_t launch_prep_t(const Params &p, int npos, int T, const rs_inputs &in, cudaStream_t st) {
    const size_t smem = prep_smem(p, NP);
    if (KIND == RS_MAMBA2) {
        auto k = m2_prep_kernel<CC, NP>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const dim3 grid((p.heads_per_group + kPrepWarps - 1) / kPrepWarps, p.G, p.B);
        k<<<grid, 32 * kPrepWarps, smem, st>>>(p, npos, T, in);
    } else {
        auto k = gdn_prep_kernel<CC, NP>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const dim3 grid((p.H + kPrepWarps - 1) / kPrepWarps, p.B);
        k<<<grid, 32 * kPrepWarps, smem, st>>>(p, npos, T, in);
    }
    return cudaGetLastError();
}

template <int KIND>
struct PrepCC {
    template <int CC>
    static cudaError_t go(const Params &p, int npos, int T, const rs_inputs &in, cudaStream_t st) {
        switch (prep_np(npos)) {
            case 1: return launch_prep_t<KIND, CC, 1>(p, npos, T, in, st);
            case 2: return launch_prep_t<KIND, CC, 2>(p, npos, T, in, st);
            case 5: return launch_prep_t<KIND, CC, 5>(p, npos, T, in, st);
            default: return launch_prep_t<KIND, CC, 8>(p, npos, T, in, st);
        }
    }
};

cudaError_t launch_prep(const Params &p, int npos, int T, const rs_inputs &in, cudaStream_t st) {
    if (p.kind == RS_MAMBA2) {
        RS_DISPATCH_CC(p.CC, return PrepCC<RS_MAMBA2>::go, (p, npos, T, in, st));
    } else {
        RS_DISPATCH_CC(p.CC, return PrepCC<RS_GDN>::go, (p, npos, T, in, st));
    }
    return cudaErrorInvalidValue;
}

}  // namespace rs
