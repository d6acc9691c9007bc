// Replay prologue ("prep") kernels, optionally fused with the append of the
// step's inputs.
//
// For every (sequence, head) they reduce the buffer to the few numbers the
// streaming pass needs at NP output positions e_j = L - npos + j (0-based
// buffer index), so that
//     y_j[r] = mul_j (S0[r, :] . vec_j) + sum_{i<=e_j} coef_j[i] w_i[r]
// with w_i the head's ring row of entry i, which the streaming pass reads
// together with the checkpoint tile.
// Mamba-2 ("ReplaySSM for hybrid SSM-Transformer stacks", How ReplaySSM works,
// step 2: the output is a function of the checkpoint and the recent inputs):
//   vec_j = C_{e_j},  mul_j = exp(A sum_{m<=e_j} dt_m) (x the fp8 tile scale),
//   coef_j[i] = exp(A sum_{i<m<=e_j} dt_m) dt_i (B_i . C_{e_j})  (+ D at i = e_j),
//   w_i = x_i.
// GDN:  vec_j = M_1..M_{e_j} q_{e_j}  (M_i = alpha_i (I - beta_i k_i k_i^T)), by the
//   backward sweep  u <- q_{e_j};  for i = e_j..1: c_i = beta_i (k_i . u);
//   u <- alpha_i (u - c_i k_i);  mul_j = scale (x tile scale),
//   coef_j[i] = scale c_i,  w_i = v_i.  Several positions over bf16 inputs take
//   an equivalent Gram form of the sweep (gdn_gram_records).
//
// With T > 0 the kernel also appends the T step inputs (step 2: append the new
// SSM input to the buffer): the new entries are read straight from the inputs
// and written into their ring slots, and the last CTA of a sequence to finish
// advances its tail by T (per-sequence arrival counter; every CTA has read the
// pointers before it arrives).  A sequence whose buffer would overflow is left
// unchanged and flagged.
#include "outputs.cuh"
#include "launch.h"

namespace rs {

constexpr int kPrepWarps = 8;   // warps per CTA

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

// Last arrival of the `ctas` CTAs of sequence b advances its tail by T.  No
// fence: every CTA has read the pointers before it arrives, nothing in this
// kernel reads the tail or the ring slots it writes, and the next kernel on
// the stream sees all of this kernel's writes.
__device__ __forceinline__ void arrive_and_advance(const Params &p, int b, int tail, int T, int ctas) {
    __syncthreads();
    if (threadIdx.x == 0) {
        if (atomicAdd(&p.arrive[b], 1u) == static_cast<unsigned>(ctas - 1)) {
            p.arrive[b] = 0u;
            p.tail[b] = tail + T;
        }
    }
}

// Let the streaming kernel queued behind this one start launching now (it
// waits for this grid's results itself before it reads them).
__device__ __forceinline__ void allow_dependent_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void write_header(float *trec, int head, int L, int cap_mask) {
    trec[kRecHeadSlot] = __int_as_float(head & cap_mask);
    trec[kRecLen] = __int_as_float(L);
}

// Sum of the elementwise products of two 16-byte chunks of bf16 or fp32.
__device__ __forceinline__ float chunk_dot(const uint4 &a, const uint4 &c, int ib) {
    if (ib == 2) {
        float d = bf16_lo(a.x) * bf16_lo(c.x);
        d = fmaf(bf16_hi(a.x), bf16_hi(c.x), d);
        d = fmaf(bf16_lo(a.y), bf16_lo(c.y), d);
        d = fmaf(bf16_hi(a.y), bf16_hi(c.y), d);
        d = fmaf(bf16_lo(a.z), bf16_lo(c.z), d);
        d = fmaf(bf16_hi(a.z), bf16_hi(c.z), d);
        d = fmaf(bf16_lo(a.w), bf16_lo(c.w), d);
        return fmaf(bf16_hi(a.w), bf16_hi(c.w), d);
    }
    float d = __uint_as_float(a.x) * __uint_as_float(c.x);
    d = fmaf(__uint_as_float(a.y), __uint_as_float(c.y), d);
    d = fmaf(__uint_as_float(a.z), __uint_as_float(c.z), d);
    return fmaf(__uint_as_float(a.w), __uint_as_float(c.w), d);
}

// ---------------------------------------------------------------- Mamba-2 --
// One CTA per (sequence, group), built as a few rounds of independent global
// reads with the arithmetic in between:
//   1. reads that need no pointer: the first round of the new x rows (for the
//      append) and A, D, the fp8 scales of the heads;
//   2. the pointers;
//   3. dt of every (head, entry), C_{e_j} and the B rows; the group's
//      B_i . C_{e_j} (lane groups of TPRB lanes per B row, rows spread over the
//      warps);
//   4. per head (several heads per warp when L <= 16, one lane segment each):
//      prefix sums of dt by segmented shuffles, multipliers, coefficients;
//   5. the append stores and the tail.
// Heads are taken in chunks of up to kM2HeadChunk per round of 3-4.
// Shared memory: bc [NP][cap] | dt [HC][cap] | A, D, scale [HC] | per warp: cum [cap].
constexpr int kM2StageFloats = 4096;   // dt floats staged per chunk

__host__ __device__ inline int m2_head_chunk(int hpg, int cap) {
    const int hc = kM2StageFloats / cap;
    return hc < 1 ? 1 : hc < hpg ? hc : hpg;
}

__host__ __device__ inline size_t m2_prep_floats(int cap, int NP, int hpg) {
    const size_t hc = m2_head_chunk(hpg, cap);
    return (size_t)NP * cap + hc * cap + 3 * hc + (size_t)kPrepWarps * cap;
}

// A CTA-wide copy of `rows` rows of `row_bytes` bytes from a contiguous source
// to dst0 + r * dst_stride, in 16-, 4- or 2-byte units as the addresses allow;
// unit k of the copy is handled by thread k mod blockDim.
struct RowCopy {
    const unsigned char *src;
    unsigned char *dst0;
    size_t dst_stride;
    int unit, upr, total;
    static constexpr int U = 4;   // units a thread moves per round

    __device__ void init(unsigned char *d0, size_t stride, const unsigned char *s, int rows, int row_bytes) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(d0) | (uintptr_t)stride |
                            reinterpret_cast<uintptr_t>(s) | (uintptr_t)row_bytes;
        src = s;
        dst0 = d0;
        dst_stride = stride;
        unit = (a & 15) == 0 ? 16 : (a & 3) == 0 ? 4 : 2;
        upr = row_bytes / unit;
        total = rows * upr;
    }
    __device__ void load(uint4 (&v)[U], int k0) const {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = k0 + u * (int)blockDim.x;
            if (k >= total) break;
            const unsigned char *s = src + (size_t)k * unit;
            if (unit == 16) v[u] = *reinterpret_cast<const uint4 *>(s);
            else if (unit == 4) v[u].x = *reinterpret_cast<const uint32_t *>(s);
            else v[u].x = *reinterpret_cast<const uint16_t *>(s);
        }
    }
    __device__ void store(const uint4 (&v)[U], int k0, size_t dst_off) const {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = k0 + u * (int)blockDim.x;
            if (k >= total) break;
            const int r = k / upr, w = k - (k / upr) * upr;
            unsigned char *d = dst0 + dst_off + (size_t)r * dst_stride + (size_t)w * unit;
            if (unit == 16) *reinterpret_cast<uint4 *>(d) = v[u];
            else if (unit == 4) *reinterpret_cast<uint32_t *>(d) = v[u].x;
            else *reinterpret_cast<uint16_t *>(d) = static_cast<uint16_t>(v[u].x);
        }
    }
    // rounds from unit k_begin + threadIdx.x on: loads, then stores
    __device__ void run(int k_begin, size_t dst_off) const {
        for (int k0 = k_begin + threadIdx.x; k0 < total; k0 += U * blockDim.x) {
            uint4 v[U];
            load(v, k0);
            store(v, k0, dst_off);
        }
    }
};

template <int CC, int NP>
__global__ void __launch_bounds__(32 * kPrepWarps, (NP <= 2 ? 3 : 2))
m2_prep_kernel(const Params p, int npos, int T, rs_inputs in) {
    extern __shared__ __align__(16) float psm[];
    allow_dependent_launch();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int Bn = p.B, H = p.H, R = p.R, cap = p.cap, G = p.G, hpg = p.heads_per_group;
    const int ib = p.in_dtype == RS_BF16 ? 2 : 4;
    const int b = blockIdx.x / G, g = blockIdx.x - (blockIdx.x / G) * G;
    const int h0 = g * hpg;   // first head of the group
    const int HC = m2_head_chunk(hpg, cap);
    float *bc = psm;
    float *sdt = bc + (size_t)NP * cap;
    float *sA = sdt + (size_t)HC * cap, *sD = sA + HC, *sS = sD + HC;
    float *cum = sS + HC + (size_t)warp * cap;
    const size_t trf = tile_rec_floats(RS_MAMBA2, NP, cap, CC);
    const int cstr = coef_stride(cap);
    float *grec = p.rec + ((size_t)b * G + g) * group_rec_floats(NP, CC);
    float *trec0 = p.rec + p.rec_tile_off + ((size_t)b * H + h0) * trf;   // the group's heads
    const size_t rowB = (size_t)CC * ib, rowX = (size_t)R * ib;
    const bool tscale_on = p.copy_dtype == RS_E4M3;

    // ---- 1. reads that need no pointer
    RowCopy xcopy;   // the new x rows of step 0 of the append, heads h0 .. h0 + hpg - 1
    uint4 xfirst[RowCopy::U];
    if (T > 0) {
        xcopy.init(static_cast<unsigned char *>(p.ra) + ((size_t)b * H + h0) * p.blk_r, p.blk_r,
                   static_cast<const unsigned char *>(in.x) + ((size_t)b * H + h0) * rowX, hpg, (int)rowX);
        xcopy.load(xfirst, threadIdx.x);
    }
    auto stage_params = [&](int c0, int nh) {
        for (int k = threadIdx.x; k < nh; k += blockDim.x) {
            const int h = h0 + c0 + k;
            sA[k] = p.A[h];
            sD[k] = p.D ? p.D[h] : 0.f;
            sS[k] = tscale_on ? p.scale[(size_t)b * H + h] : 1.f;
        }
    };
    stage_params(0, hpg < HC ? hpg : HC);

    // ---- 2. the pointers
    const int head = p.head[b], tail = p.tail[b];
    const int L_old = tail - head, L = L_old + T;
    if (L_old < 0 || L > cap) {   // corrupt pointers or ring overflow: nothing is appended
        for (size_t i = threadIdx.x; i < (size_t)hpg * trf; i += blockDim.x) trec0[i] = 0.f;
        for (int i = threadIdx.x; i < NP * CC; i += blockDim.x) grec[i] = 0.f;
        if (g == 0 && threadIdx.x == 0) atomicOr(&p.err[b], T > 0 ? RS_SEQ_ERR_OVERFLOW : RS_SEQ_ERR_EMPTY);
        return;
    }
    unsigned char *bblk = static_cast<unsigned char *>(p.rc) + ((size_t)b * G + g) * p.blk_c;
    unsigned char *cblk = static_cast<unsigned char *>(p.rd) + ((size_t)b * G + g) * p.blk_c;
    const float *dtring = static_cast<const float *>(p.rb) + ((size_t)b * H + h0) * p.capd;   // [hpg][capd]
    // row of buffer entry i: its ring slot for the entries already buffered, the step inputs for the new ones
    auto b_row = [&](int i) -> const unsigned char * {
        return i < L_old ? bblk + (size_t)((head + i) & p.cap_mask) * rowB
                         : static_cast<const unsigned char *>(in.B) + (((size_t)(i - L_old) * Bn + b) * G + g) * rowB;
    };
    auto c_row = [&](int i) -> const unsigned char * {
        return i < L_old ? cblk + (size_t)((head + i) & p.cap_mask) * rowB
                         : static_cast<const unsigned char *>(in.C) + (((size_t)(i - L_old) * Bn + b) * G + g) * rowB;
    };
    auto dt_at = [&](int hl, int i) -> float {
        return i < L_old ? dtring[(size_t)hl * p.capd + ((head + i) & p.cap_mask)]
                         : in.dt[((size_t)(i - L_old) * Bn + b) * H + h0 + hl];
    };
    auto stage_dt = [&](int c0, int nh) {
        for (int k = threadIdx.x; k < nh * L; k += blockDim.x) {
            const int hl = k / L, i = k - (k / L) * L;
            sdt[hl * cap + i] = dt_at(c0 + hl, i);
        }
    };

    const bool ok = npos >= 1 && L >= npos;
    if (ok) {
        // ---- 3. dt, then B_i . C_{e_j} for i < L (and the group record: C_{e_j} in fp32)
        stage_dt(0, hpg < HC ? hpg : HC);
        const int nch = CC * ib / 16;
        const int TPRB = nch < 32 ? nch : 32, CPLB = nch / TPRB, RPI = 32 / TPRB;
        const int q = lane % TPRB, sub = lane / TPRB;
        uint4 cch[NP][2];
#pragma unroll
        for (int j = 0; j < NP; ++j)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                cch[j][c] = make_uint4(0u, 0u, 0u, 0u);
                if (j < npos && c < CPLB)
                    cch[j][c] = reinterpret_cast<const uint4 *>(c_row(L - npos + j))[q + c * TPRB];
            }
        for (int i0 = warp * RPI; i0 < L; i0 += kPrepWarps * RPI) {
            const int i = i0 + sub;
            uint4 bch[2];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                bch[c] = make_uint4(0u, 0u, 0u, 0u);
                if (i < L && c < CPLB) bch[c] = reinterpret_cast<const uint4 *>(b_row(i))[q + c * TPRB];
            }
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                if (j >= npos) break;
                float d = chunk_dot(bch[0], cch[j][0], ib);
                if (CPLB > 1) d += chunk_dot(bch[1], cch[j][1], ib);
                for (int o = TPRB / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                if (q == 0 && i < L) bc[j * cap + i] = d;
            }
        }
        if (warp == kPrepWarps - 1 && sub == 0) {
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                if (j >= npos) break;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if (c >= CPLB) break;
                    const int col = (q + c * TPRB) * (16 / ib);
                    const uint4 w = cch[j][c];
                    if (ib == 2) {
                        float4 *dst = reinterpret_cast<float4 *>(grec + j * CC + col);
                        dst[0] = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
                        dst[1] = make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
                    } else {
                        *reinterpret_cast<uint4 *>(grec + j * CC + col) = w;
                    }
                }
            }
        }
        __syncthreads();
        // ---- 4. per head: prefix sums of dt, multipliers, coefficients
        const int SW = L <= 1 ? 1 : L <= 2 ? 2 : L <= 4 ? 4 : L <= 8 ? 8 : L <= 16 ? 16 : 32;
        for (int c0 = 0; c0 < hpg; c0 += HC) {
            const int nh = hpg - c0 < HC ? hpg - c0 : HC;
            if (c0 > 0) {   // next chunk of heads
                __syncthreads();
                stage_params(c0, nh);
                stage_dt(c0, nh);
                __syncthreads();
            }
            if (L <= 32) {
                // lane segments of SW lanes, one head each, entry i = lane within the segment
                const int nseg = 32 / SW, seg = lane / SW, i = lane - seg * SW;
                for (int hb = warp * nseg; hb < nh; hb += kPrepWarps * nseg) {
                    const int hc = hb + seg;
                    const bool hv = hc < nh;
                    const float dv = hv && i < L ? sdt[hc * cap + i] : 0.f;
                    float c = dv;
                    for (int o = 1; o < SW; o <<= 1) {
                        const float t = __shfl_up_sync(0xffffffffu, c, o, SW);
                        if (i >= o) c += t;
                    }
                    const float A = hv ? sA[hc] : 0.f, Dh = hv ? sD[hc] : 0.f, tsc = hv ? sS[hc] : 0.f;
                    float *trec = trec0 + (size_t)(c0 + (hv ? hc : 0)) * trf;
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        if (j >= npos) break;
                        const int e = L - npos + j;
                        const float ce = __shfl_sync(0xffffffffu, c, e, SW);
                        if (hv && i == 0) trec[j] = expf(A * ce) * tsc;
                        if (hv && i < L)
                            trec[kRecHdr + j * cstr + i] =
                                i <= e ? fmaf(expf(A * (ce - c)) * dv, bc[j * cap + i], i == e ? Dh : 0.f) : 0.f;
                    }
                    if (hv && i == 0) write_header(trec, head, L, p.cap_mask);
                }
            } else {
                for (int hc = warp; hc < nh; hc += kPrepWarps) {
                    const float *dts = sdt + (size_t)hc * cap;
                    float *trec = trec0 + (size_t)(c0 + hc) * trf;
                    float carry = 0.f;
                    for (int i0 = 0; i0 < L; i0 += 32) {
                        const int i = i0 + lane;
                        const float c = warp_incl_scan(i < L ? dts[i] : 0.f, lane) + carry;
                        if (i < L) cum[i] = c;
                        carry = __shfl_sync(0xffffffffu, c, 31);
                    }
                    __syncwarp();
                    const float A = sA[hc], Dh = sD[hc], tsc = sS[hc];
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        if (j >= npos) break;
                        const int e = L - npos + j;
                        const float ce = cum[e];
                        if (lane == 0) trec[j] = expf(A * ce) * tsc;
                        for (int i = lane; i < L; i += 32)
                            trec[kRecHdr + j * cstr + i] =
                                i <= e ? fmaf(expf(A * (ce - cum[i])) * dts[i], bc[j * cap + i], i == e ? Dh : 0.f)
                                       : 0.f;
                    }
                    if (lane == 0) write_header(trec, head, L, p.cap_mask);
                    __syncwarp();   // cum is reused by the warp's next head
                }
            }
        }
    } else {
        for (size_t i = threadIdx.x; i < (size_t)hpg * trf; i += blockDim.x) trec0[i] = 0.f;
        for (int i = threadIdx.x; i < NP * CC; i += blockDim.x) grec[i] = 0.f;
        if (T == 0 && g == 0 && threadIdx.x == 0) atomicOr(&p.err[b], RS_SEQ_ERR_EMPTY);
    }

    if (T > 0) {
        // ---- 5. append: the new entries of the group's heads and the group's B, C rows
        xcopy.store(xfirst, threadIdx.x, (size_t)(tail & p.cap_mask) * rowX);
        xcopy.run(RowCopy::U * blockDim.x, (size_t)(tail & p.cap_mask) * rowX);   // units past the first round
        for (int t = 1; t < T; ++t) {
            RowCopy xc;
            xc.init(static_cast<unsigned char *>(p.ra) + ((size_t)b * H + h0) * p.blk_r, p.blk_r,
                    static_cast<const unsigned char *>(in.x) + (((size_t)t * Bn + b) * H + h0) * rowX, hpg, (int)rowX);
            xc.run(0, (size_t)((tail + t) & p.cap_mask) * rowX);
        }
        for (int w = threadIdx.x; w < hpg * T; w += blockDim.x) {
            const int hl = w / T, t = w - (w / T) * T;
            static_cast<float *>(p.rb)[((size_t)b * H + h0 + hl) * p.capd + ((tail + t) & p.cap_mask)] =
                in.dt[((size_t)t * Bn + b) * H + h0 + hl];
        }
        for (int t = warp; t < T; t += kPrepWarps) {
            const int slot = (tail + t) & p.cap_mask;
            copy_row(bblk + (size_t)slot * rowB, b_row(L_old + t), (int)rowB, lane, 32);
            copy_row(cblk + (size_t)slot * rowB, c_row(L_old + t), (int)rowB, lane, 32);
        }
        arrive_and_advance(p, b, tail, T, G);
    }
}

// -------------------------------------------------------------------- GDN --
// One warp per (sequence, head); a CTA holds kPrepWarps heads of one sequence.
// Per-warp shared memory (entries compact, buffer index i at row i; rows of
// CC inputs at a pitch of kpitch bytes):
//   kraw [cap][kpitch] | qraw [NP][kpitch] | alpha [cap] | beta [cap]
//   (Gram form only:) G, upper triangle by columns [cap (cap - 1) / 2] | P [NP][32]
struct GdnPrepSmem {
    size_t k, q, alpha, beta, g, pc, per_warp, kpitch;
};

// Several positions over bf16 inputs with at most 32 buffered entries take
// the Gram form of the backward sweep (gdn_gram_records).
__host__ __device__ inline bool gdn_gram(int cap, int CC, int NP, int ib) {
    return NP >= 2 && ib == 2 && cap <= 32 && CC % 16 == 0;
}

__host__ __device__ inline GdnPrepSmem gdn_prep_smem(int cap, int CC, int NP, int ib) {
    GdnPrepSmem s;
    // the Gram form reads 8 rows at one column with ldmatrix: rows 16 bytes
    // apart in the bank pattern (a pitch of 16 mod 128) keep those reads free
    // of bank conflicts
    s.kpitch = (size_t)CC * ib + (gdn_gram(cap, CC, NP, ib) ? 16 : 0);
    size_t w = 0;
    s.k = w;     w = align_up(w + (size_t)cap * s.kpitch, 16);
    s.q = w;     w = align_up(w + (size_t)NP * s.kpitch, 16);
    s.alpha = w; w = align_up(w + 4 * (size_t)cap, 16);
    s.beta = w;  w = align_up(w + 4 * (size_t)cap, 16);
    s.g = s.pc = w;
    if (gdn_gram(cap, CC, NP, ib)) {
        w = align_up(w + 4 * (size_t)(cap * (cap - 1) / 2), 16);
        s.pc = w;
        w = align_up(w + 4 * (size_t)NP * 32, 16);
    }
    s.per_warp = w;
    return s;
}

// The backward sweep of one head in Gram form.  Write E_j(l) for the product
// alpha_l ... alpha_{e_j} (1 for l > e_j).  By induction down from u = q_j, the
// sweep's vector before step i is
//     u = E_j(i + 1) (q_j - sum_{i<m<=e_j} h_m k_m),   h_m = c_m / E_j(m + 1),
// so c_i = beta_i (k_i . u) gives
//     h_i = beta_i (k_i . q_j - sum_{i<m<=e_j} h_m (k_i . k_m)):
// the decay factors out of the recurrence.  Hence:
//   1. the dot products first, as two small products on the tensor cores,
//      G = K K^T (strict upper triangle) and P = K Q^T (bf16 operands staged
//      in shared memory, fp32 accumulation);
//   2. the triangular recurrence for h with one lane per entry, all positions
//      in lockstep (one broadcast per position and step);
//   3. E_j(l) by a suffix-product scan over the lanes, then
//      coef_j[i] = scale h_i E_j(i + 1)  and  vec_j = E_j(0) (q_j - sum_m h_m k_m).
// Requires L <= 32, CC a multiple of 16, 1 <= npos <= NP <= 8, npos <= L;
// kraw and qraw rows (bf16) kp bytes apart, kp a multiple of 16.
template <int CC, int NP>
__device__ __forceinline__ void gdn_gram_records(const unsigned char *kraw, const unsigned char *qraw, size_t kp,
                                                 const float *alpha, const float *beta, float *gs, float *ps,
                                                 int L, int npos, int lane, float sc, float *coef, int cstr,
                                                 float *vec) {
    constexpr int KS = CC / 16;
    constexpr unsigned FULL = 0xffffffffu;
    const int MT = (L + 15) >> 4, NTL = (L + 7) >> 3;   // 16-row and 8-column blocks of G
    // ---- 1. G and P.  Rows past L repeat row L - 1 (and positions past npos
    // repeat npos - 1); their results are not stored.
    float gacc[2][4][4], pacc[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int f = 0; f < 4; ++f) {
            pacc[mt][f] = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) gacc[mt][nt][f] = 0.f;
        }
    }
    const unsigned char *arow[2] = {kraw + (size_t)min(lane & 15, L - 1) * kp,
                                    kraw + (size_t)min(16 + (lane & 15), L - 1) * kp};
    const unsigned char *qrow = qraw + (size_t)min(lane & 7, npos - 1) * kp;
    const int acol = (lane >> 4) * 16, qcol = ((lane >> 3) & 1) * 16;   // bytes
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[2][4];
        ldmatrix_x4(a[0], arow[0] + ks * 32 + acol);
        if (MT > 1) {
            ldmatrix_x4(a[1], arow[1] + ks * 32 + acol);
        } else {
#pragma unroll
            for (int f = 0; f < 4; ++f) a[1][f] = a[0][f];
        }
        uint32_t bq[2];
        ldmatrix_x2(bq, qrow + ks * 32 + qcol);
        // B of G's column block nt = rows 8 nt .. 8 nt + 7 of K: fragments 0 and 2
        // (nt even) or 1 and 3 (nt odd) of the A operand of row block nt / 2
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 2 * mt; nt < 4; ++nt)
                if (mt < MT && nt < NTL)
                    mma_bf16(gacc[mt][nt], a[mt], a[nt >> 1][nt & 1], a[nt >> 1][2 + (nt & 1)]);
        mma_bf16(pacc[0], a[0], bq[0], bq[1]);
        if (MT > 1) mma_bf16(pacc[1], a[1], bq[0], bq[1]);
    }
    // accumulator f of lane (g, t): row g + 8 (f / 2), column 2 t + f % 2 of the block
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        if (mt >= MT) break;
#pragma unroll
        for (int f = 0; f < 4; ++f) {
            const int i = 16 * mt + g + 8 * (f >> 1), j = 2 * t + (f & 1);
            if (i < L && j < npos) ps[j * 32 + i] = pacc[mt][f];
        }
#pragma unroll
        for (int nt = 2 * mt; nt < 4; ++nt) {
            if (nt >= NTL) break;
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const int i = 16 * mt + g + 8 * (f >> 1), m = 8 * nt + 2 * t + (f & 1);
                if (i < m && m < L) gs[m * (m - 1) / 2 + i] = gacc[mt][nt][f];
            }
        }
    }
    __syncwarp();
    // ---- 2. h_i = beta_i (P[j][i] - acc_i), acc_i = sum of h_m G[i][m] over the
    // entries m > i done so far; lane i owns entry i
    const float bl = lane < L ? beta[lane] : 0.f;
    float pj[NP], acc[NP], hv[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        pj[j] = (j < npos && lane < L) ? ps[j * 32 + lane] : 0.f;
        acc[j] = 0.f;
        hv[j] = 0.f;
    }
    for (int i = L - 1; i >= 0; --i) {
        const float gi = lane < i ? gs[i * (i - 1) / 2 + lane] : 0.f;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            if (j < npos && i <= L - npos + j) {
                const float hi = __shfl_sync(FULL, bl * (pj[j] - acc[j]), i);
                acc[j] = fmaf(hi, gi, acc[j]);
                if (lane == i) hv[j] = hi;
            }
        }
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < NP; ++j)
        if (j < npos) ps[j * 32 + lane] = hv[j];   // h of position j, 0 past e_j
    // ---- 3. decay products and coefficients
    float e0[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        e0[j] = 0.f;
        if (j >= npos) continue;
        const int e = L - npos + j;
        float v = 1.f;
        if (lane <= e) v = alpha[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {   // inclusive suffix product: E_j(lane)
            const float w = __shfl_down_sync(FULL, v, o);
            if (lane + o < 32) v *= w;
        }
        float nxt = __shfl_down_sync(FULL, v, 1);   // E_j(lane + 1)
        if (lane == 31) nxt = 1.f;
        e0[j] = __shfl_sync(FULL, v, 0);
        if (lane < L) coef[j * cstr + lane] = lane <= e ? sc * hv[j] * nxt : 0.f;
    }
    __syncwarp();
    // vec_j = E_j(0) (q_j - sum_m h_m k_m), lanes over columns
    constexpr int UPL = (CC + 31) / 32;
    float va[NP][UPL];
#pragma unroll
    for (int j = 0; j < NP; ++j)
#pragma unroll
        for (int u = 0; u < UPL; ++u) {
            const int c = lane + 32 * u;
            va[j][u] = (j < npos && c < CC) ? lds_in(qraw + (size_t)j * kp, c, RS_BF16) : 0.f;
        }
    for (int m = 0; m < L; ++m) {
        float kr[UPL];
#pragma unroll
        for (int u = 0; u < UPL; ++u) {
            const int c = lane + 32 * u;
            kr[u] = c < CC ? lds_in(kraw + (size_t)m * kp, c, RS_BF16) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            if (j >= npos) continue;
            const float hm = ps[j * 32 + m];
#pragma unroll
            for (int u = 0; u < UPL; ++u) va[j][u] = fmaf(-hm, kr[u], va[j][u]);
        }
    }
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        if (j >= npos) continue;
#pragma unroll
        for (int u = 0; u < UPL; ++u) {
            const int c = lane + 32 * u;
            if (c < CC) vec[j * CC + c] = e0[j] * va[j][u];
        }
    }
}

template <int CC, int NP>
__global__ void __launch_bounds__(32 * kPrepWarps, (NP == 1 ? 5 : NP == 2 ? 3 : 2))
gdn_prep_kernel(const Params p, int npos, int T, rs_inputs in) {
    extern __shared__ __align__(16) unsigned char psm_g[];
    allow_dependent_launch();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int Bn = p.B, H = p.H, R = p.R, cap = p.cap, ib = p.in_dtype == RS_BF16 ? 2 : 4;
    const int cps = (H + kPrepWarps - 1) / kPrepWarps;   // CTAs per sequence
    const int b = blockIdx.x / cps, hc = blockIdx.x - (blockIdx.x / cps) * cps;
    const int h = hc * kPrepWarps + warp;
    const bool has_head = h < H;
    const size_t tile = (size_t)b * H + h;
    const GdnPrepSmem S = gdn_prep_smem(cap, CC, NP, ib);
    unsigned char *wsm = psm_g + (size_t)warp * S.per_warp;
    unsigned char *kraw = wsm + S.k, *qraw = wsm + S.q;
    float *alpha = reinterpret_cast<float *>(wsm + S.alpha), *beta = reinterpret_cast<float *>(wsm + S.beta);
    const size_t trf = tile_rec_floats(RS_GDN, NP, cap, CC);
    float *trec = p.rec + p.rec_tile_off + tile * trf;
    const size_t rowC = (size_t)CC * ib, rowR = (size_t)R * ib;

    const int head = p.head[b], tail = p.tail[b];
    const int L_old = tail - head, L = L_old + T;
    if (L_old < 0 || L > cap) {
        if (has_head)
            for (size_t i = lane; i < trf; i += 32) trec[i] = 0.f;
        if (hc == 0 && threadIdx.x == 0) atomicOr(&p.err[b], T > 0 ? RS_SEQ_ERR_OVERFLOW : RS_SEQ_ERR_EMPTY);
        return;
    }
    const bool ok = npos >= 1 && L >= npos;
    const size_t bh = has_head ? tile : 0;
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
    // A decode step's new q and v rows, read now so that the append below does
    // not wait for them: 8-byte pieces, up to 4 per lane (rows of <= 1 KB).
    const bool pre_qv = T == 1 && has_head && rowC % 256 == 0 && rowR % 256 == 0 && rowC <= 1024 &&
                        rowR <= 1024 && ((reinterpret_cast<uintptr_t>(in.q) | reinterpret_cast<uintptr_t>(in.v)) & 7) == 0;
    // The v rows of the T <= NP new entries of a verification step, read now
    // too: rows of <= 256 bytes, one 8-byte piece per lane and row.
    const bool pre_v = NP >= 2 && !pre_qv && T > 1 && T <= NP && has_head && rowR <= 256 && rowR % 8 == 0 &&
                       (reinterpret_cast<uintptr_t>(in.v) & 7) == 0;
    uint2 vpre[NP];
    if (pre_v) {
#pragma unroll
        for (int t = 0; t < NP; ++t)
            if (t < T && lane * 8 < (int)rowR)
                vpre[t] = reinterpret_cast<const uint2 *>(static_cast<const unsigned char *>(in.v) +
                                                          (((size_t)t * Bn + b) * H + h) * rowR)[lane];
    }
    uint2 qv[2][4];
    if (pre_qv) {
        const size_t at = (size_t)b * H + h;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u * 256 < (int)rowC)
                qv[0][u] = reinterpret_cast<const uint2 *>(static_cast<const unsigned char *>(in.q) + at * rowC)[lane + 32 * u];
            if (u * 256 < (int)rowR)
                qv[1][u] = reinterpret_cast<const uint2 *>(static_cast<const unsigned char *>(in.v) + at * rowR)[lane + 32 * u];
        }
    }
    if (has_head) {
        // ---- one round of asynchronous copies
        for (int i = 0; i < L; ++i) stage_row(kraw + i * S.kpitch, src_row(kblk, in.k, rowC, i), (int)rowC, lane, 32);
        if (ok)
            for (int j = 0; j < npos; ++j)
                stage_row(qraw + j * S.kpitch, src_row(qblk, in.q, rowC, L - npos + j), (int)rowC, lane, 32);
        for (int i = lane; i < L; i += 32) {
            const size_t at = ((size_t)(i - L_old) * Bn + b) * H + h;
            cp_async4(alpha + i, i < L_old ? ablk + ((head + i) & p.cap_mask) : in.alpha + at);
            cp_async4(beta + i, i < L_old ? bblk + ((head + i) & p.cap_mask) : in.beta + at);
        }
        cp_async_wait_all();
        __syncwarp();

        if (ok && gdn_gram(cap, CC, NP, ib)) {
            const int cstr = coef_stride(cap);
            float *coef = trec + kRecHdr;
            const float sc = p.gdn_scale;
            const float tscale = p.copy_dtype == RS_E4M3 ? p.scale[tile] : 1.f;
            if constexpr (NP >= 2 && CC % 16 == 0)
                gdn_gram_records<CC, NP>(kraw, qraw, S.kpitch, alpha, beta, reinterpret_cast<float *>(wsm + S.g),
                                         reinterpret_cast<float *>(wsm + S.pc), L, npos, lane, sc, coef, cstr,
                                         coef + (size_t)NP * cstr);
            if (lane < npos) trec[lane] = sc * tscale;
            if (lane == 0) write_header(trec, head, L, p.cap_mask);
        } else if (ok) {
            const int cstr = coef_stride(cap);
            float *coef = trec + kRecHdr, *vec = coef + (size_t)NP * cstr;
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
                    if (j >= npos) continue;
                    if (i <= L - npos + j) {
                        const float f = bt * d[j];
                        if (lane == 0) coef[j * cstr + i] = sc * f;
#pragma unroll
                        for (int m = 0; m < UPL; ++m) u[j][m] = a * fmaf(-f, kr[m], u[j][m]);
                    } else if (lane == 0) {
                        coef[j * cstr + i] = 0.f;
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
                    if (lane == 0) trec[j] = sc * tscale;
                }
            }
            if (lane == 0) write_header(trec, head, L, p.cap_mask);
        } else {
            for (size_t i = lane; i < trf; i += 32) trec[i] = 0.f;
        }

        if (T > 0) {   // ---- append: the new entries into their ring slots
            for (int t = 0; t < T; ++t) {
                const int slot = (tail + t) & p.cap_mask;
                const size_t at = ((size_t)t * Bn + b) * H + h;
                copy_row(kblk + (size_t)slot * rowC, kraw + (L_old + t) * S.kpitch, (int)rowC, lane, 32);
                if (pre_qv) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (u * 256 < (int)rowC) reinterpret_cast<uint2 *>(qblk + (size_t)slot * rowC)[lane + 32 * u] = qv[0][u];
                        if (u * 256 < (int)rowR) reinterpret_cast<uint2 *>(vblk + (size_t)slot * rowR)[lane + 32 * u] = qv[1][u];
                    }
                } else {
                    // q: the staged row when the outputs covered this entry (T <= npos)
                    const unsigned char *qsrc = ok && T <= npos
                                                    ? qraw + (npos - T + t) * S.kpitch
                                                    : static_cast<const unsigned char *>(in.q) + at * rowC;
                    copy_row(qblk + (size_t)slot * rowC, qsrc, (int)rowC, lane, 32);
                    if (!pre_v)
                        copy_row(vblk + (size_t)slot * rowR, static_cast<const unsigned char *>(in.v) + at * rowR, (int)rowR, lane, 32);
                }
            }
            if (pre_v) {
#pragma unroll
                for (int t = 0; t < NP; ++t)
                    if (t < T && lane * 8 < (int)rowR)
                        reinterpret_cast<uint2 *>(vblk + (size_t)((tail + t) & p.cap_mask) * rowR)[lane] = vpre[t];
            }
            for (int t = lane; t < T; t += 32) {
                ablk[(tail + t) & p.cap_mask] = alpha[L_old + t];
                bblk[(tail + t) & p.cap_mask] = beta[L_old + t];
            }
            // the last of the sequence's H warps to get here advances the tail
            // (every warp has read the pointers before it arrives; no fence, as
            // in arrive_and_advance)
            __syncwarp();
            if (lane == 0) {
                if (atomicAdd(&p.arrive[b], 1u) == static_cast<unsigned>(H - 1)) {
                    p.arrive[b] = 0u;
                    p.tail[b] = tail + T;
                }
            }
        }
    }
    if (!ok && T == 0 && hc == 0 && threadIdx.x == 0) atomicOr(&p.err[b], RS_SEQ_ERR_EMPTY);
}

size_t prep_smem(const Params &p, int NP) {
    const int ib = p.in_dtype == RS_BF16 ? 2 : 4;
    if (p.kind == RS_MAMBA2) return 4 * m2_prep_floats(p.cap, NP, p.heads_per_group);
    return kPrepWarps * gdn_prep_smem(p.cap, p.CC, NP, ib).per_warp;
}

template <int KIND, int CC, int NP>
static cudaError_t launch_prep_t(const Params &p, int npos, int T, const rs_inputs &in, cudaStream_t st) {
    const size_t smem = prep_smem(p, NP);
    if (KIND == RS_MAMBA2) {
        auto k = m2_prep_kernel<CC, NP>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<(unsigned)((size_t)p.B * p.G), 32 * kPrepWarps, smem, st>>>(p, npos, T, in);
    } else {
        auto k = gdn_prep_kernel<CC, NP>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const size_t cps = (p.H + kPrepWarps - 1) / kPrepWarps;
        k<<<(unsigned)(cps * p.B), 32 * kPrepWarps, smem, st>>>(p, npos, T, in);
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
