// The streaming half of the output-only kernels (decode and multi-position
// verification), for both layer kinds.
//
// ReplaySSM computes every output from the read-only checkpoint and the
// buffered inputs ("ReplaySSM: Cache SSM Inputs, Not State", Abstract; "ReplaySSM
// for hybrid SSM-Transformer stacks", How ReplaySSM works, steps 2 and 4).  The
// prep kernel reduces each (sequence, head)'s buffer to a record
// (mul_j, coef_j, vec_j); this kernel makes the one pass over the checkpoint
// tile and the head's ring block of rows w_i (Mamba-2 x_i, GDN v_i):
//     y_j[r] = mul_j (S0[r, :] . vec_j) + sum_{i<=e_j} coef_j[i] w_i[r],   j < npos, r < R.
//
// The pass is bound by HBM bandwidth.  One CTA per SM runs over a contiguous
// range of tiles with a shared-memory ring of stages.  A stage holds TT
// consecutive tiles (about 32 KB, so that each bulk copy moves enough bytes
// to keep the copy engine's per-operation cost small), their TT ring blocks
// and their TT records: three 1-D bulk copies per stage, issued by one
// producer thread in tile order (transaction-counted "full" barrier,
// checkpoint evict-first in L2).  NT
// teams of four consumer warps take the stages in turn (stage k goes to team
// k mod NT); each team owns SPT stages of the ring, which it uses in order,
// and frees a stage ("empty" barrier) once it has contracted all its tiles.
// Every barrier therefore sees each of its uses waited for in order by the
// same waiters, so a phase-parity wait never aliases an older phase.  Every
// wait is bounded: one that gives up sets RS_SEQ_ERR_TIMEOUT and the role stops.
//
// Mamba-2's contraction vector C_{e_j} is one per (sequence, group) and is the
// same for all heads of the group: the consumers keep it in registers and
// reload it (plain cached loads, issued before the stage wait) only when the
// group changes.
#include "outputs.cuh"
#include "launch.h"

namespace rs {

constexpr int kTeamWarps = 4;                   // consumer warps per team (one tile at a time)
constexpr int kTeamThreads = 32 * kTeamWarps;
constexpr size_t kStreamSmemBudget = 224 * 1024;
constexpr size_t kStageTarget = 32 * 1024;      // checkpoint bytes a stage aims for
constexpr int kMaxTilesPerStage = 8;

template <int NP>
struct Roles {
    static constexpr int NT = NP <= 2 ? 3 : 2;        // consumer teams
    static constexpr int NCW = NT * kTeamWarps;       // consumer warps
    static constexpr int THREADS = 32 * (NCW + 1);    // + the producer warp
};

struct StreamLayout {
    size_t blk_off, rec_off, stage_bytes, bars, total;
    int TT;       // tiles per stage
    int S, SPT;   // stages in all, stages per team
};

// Stage: TT tiles (padded to 128 bytes) | TT ring blocks | TT tile records.
__host__ __device__ inline StreamLayout stream_layout(size_t tile_bytes, size_t blk_bytes, size_t rec_bytes,
                                                      int nt) {
    StreamLayout l;
    size_t tt = kStageTarget / tile_bytes;
    tt = tt < 1 ? 1 : tt > (size_t)kMaxTilesPerStage ? (size_t)kMaxTilesPerStage : tt;
    l.TT = (int)tt;
    l.blk_off = align_up(tt * tile_bytes, 128);
    l.rec_off = align_up(l.blk_off + tt * blk_bytes, 16);
    l.stage_bytes = align_up(l.rec_off + tt * rec_bytes, 128);
    size_t spt = (kStreamSmemBudget - 1024) / (l.stage_bytes + 16) / nt;
    spt = spt < 1 ? 1 : spt > 8 ? 8 : spt;
    l.S = (int)(spt * nt);
    l.SPT = (int)spt;
    l.bars = (size_t)l.S * l.stage_bytes;
    l.total = l.bars + align_up(16 * (size_t)l.S, 128);
    return l;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 1-D bulk copy without its own expect_tx (the caller sets the total).
__device__ __forceinline__ void bulk_pieces(void *dst, const void *src, uint32_t bytes,
                                            uint64_t *bar, uint64_t policy) {
    uint32_t off = 0;
    while (off < bytes) {
        const uint32_t n = bytes - off < 32768u ? bytes - off : 32768u;
        bulk_g2s(static_cast<char *>(dst) + off, static_cast<const char *>(src) + off, n, bar, policy);
        off += n;
    }
}

// Programmatic dependent launch: wait until the grid this one depends on (the
// prep kernel before it in the stream) has completed and its writes are
// visible; a no-op when the launch has no such dependency.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// The contraction vectors a consumer thread needs: vec_j at its CPT chunks.
template <int NP, int CPT, int VEC, int TPR>
__device__ __forceinline__ void load_vec_global(float (&v)[NP][CPT * VEC], const float *__restrict__ vec,
                                                int CC, int npos, int tl) {
#pragma unroll
    for (int j = 0; j < NP; ++j)
#pragma unroll
        for (int c = 0; c < CPT; ++c)
#pragma unroll
            for (int e = 0; e < VEC; e += 4) {
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                if (j < npos) f = *reinterpret_cast<const float4 *>(vec + j * CC + (tl + c * TPR) * VEC + e);
                v[j][c * VEC + e] = f.x;
                v[j][c * VEC + e + 1] = f.y;
                v[j][c * VEC + e + 2] = f.z;
                v[j][c * VEC + e + 3] = f.w;
            }
}

template <int KIND, int CC, typename TS, int NP>
__global__ void __launch_bounds__(Roles<NP>::THREADS, 1)
stream_outputs_kernel(const Params p, const void *__restrict__ state, int npos, void *y) {
    using RL = Roles<NP>;
    extern __shared__ __align__(128) unsigned char smem[];
    const int R = p.R, H = p.H;
    const uint32_t tile_bytes = static_cast<uint32_t>(R) * CC * TS::bytes;
    const int cap = p.cap;
    const size_t rfl = tile_rec_floats(KIND, NP, cap, CC);
    const uint32_t rec_bytes = static_cast<uint32_t>(4 * rfl);
    const uint32_t blk_bytes = static_cast<uint32_t>(p.blk_r);
    const float *trec = p.rec + p.rec_tile_off;
    // ring rows the outputs sum over: Mamba-2 x, GDN v ([B][H][cap][R] blocks)
    const unsigned char *wring = static_cast<const unsigned char *>(KIND == RS_MAMBA2 ? p.ra : p.rc);
    const StreamLayout lay = stream_layout(tile_bytes, blk_bytes, rec_bytes, RL::NT);
    const int S = lay.S, SPT = lay.SPT, TT = lay.TT;
    // stage k of this CTA -> team k % NT, the team's m-th stage (m = k / NT),
    // ring slot (k % NT) * SPT + m % SPT, use m / SPT of that slot
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bars);
    uint64_t *empty = full + S;

    const int ntiles_all = p.B * H;
    const int per = ntiles_all / gridDim.x, extra = ntiles_all % gridDim.x;
    const int t0 = blockIdx.x * per + (blockIdx.x < extra ? blockIdx.x : extra);
    const int nt = per + (blockIdx.x < extra ? 1 : 0);
    const int nst = (nt + TT - 1) / TT;   // stages this CTA streams
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, kTeamWarps);
        }
    }
    __syncthreads();

    auto stage = [&](int s) { return smem + (size_t)s * lay.stage_bytes; };

    if (warp == RL::NCW) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_state = policy_evict_first();
            const uint64_t pol_rec = policy_evict_last();
            // The checkpoint does not depend on the prep kernel that precedes
            // this one in the stream, so the first ring's worth of checkpoint
            // copies starts at once; the records and ring blocks the prep
            // kernel writes are copied after griddepcontrol.wait (the prep
            // grid has finished and its writes are visible).
            const int pre = nst < S ? nst : S;
            for (int k = 0; k < pre; ++k) {   // stage k < S: slot k % NT * SPT + k / NT, first use
                const int s = (k % RL::NT) * SPT + k / RL::NT;
                const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
                mbar_expect_tx(full + s, cnt * (tile_bytes + blk_bytes + rec_bytes));
                bulk_pieces(stage(s), static_cast<const unsigned char *>(state) + (size_t)first * tile_bytes,
                            cnt * tile_bytes, full + s, pol_state);
            }
            grid_dependency_wait();
            for (int k = 0; k < pre; ++k) {
                const int s = (k % RL::NT) * SPT + k / RL::NT;
                const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
                unsigned char *st = stage(s);
                bulk_pieces(st + lay.rec_off, trec + (size_t)first * rfl, cnt * rec_bytes, full + s, pol_rec);
                bulk_pieces(st + lay.blk_off, wring + (size_t)first * blk_bytes, cnt * blk_bytes, full + s, pol_rec);
            }
            int team = 0, ms = 0, u = 1;   // stage S: team 0, m = SPT -> m % SPT = 0, m / SPT = 1
            for (int k = pre; k < nst; ++k) {
                const int s = team * SPT + ms;
                const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
                if (!mbar_wait_bounded(empty + s, (u - 1) & 1)) {
                    atomicOr(&p.err[first / H], RS_SEQ_ERR_TIMEOUT);
                    break;
                }
                unsigned char *st = stage(s);
                mbar_expect_tx(full + s, cnt * (tile_bytes + blk_bytes + rec_bytes));
                bulk_pieces(st + lay.rec_off, trec + (size_t)first * rfl, cnt * rec_bytes, full + s, pol_rec);
                bulk_pieces(st + lay.blk_off, wring + (size_t)first * blk_bytes, cnt * blk_bytes, full + s, pol_rec);
                bulk_pieces(st, static_cast<const unsigned char *>(state) + (size_t)first * tile_bytes,
                            cnt * tile_bytes, full + s, pol_state);
                if (++team == RL::NT) {
                    team = 0;
                    if (++ms == SPT) {
                        ms = 0;
                        ++u;
                    }
                }
            }
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    // Team `team` (four warps) contracts stages team, team + NT, ...
    using G = Geom<CC, TS::bytes>;
    constexpr int VEC = G::VEC, TPR = G::TPR, CPT = G::CPT;
    const int team = warp / kTeamWarps;
    const int ttid = threadIdx.x % kTeamThreads;
    const int tl = ttid % TPR, row0 = ttid / TPR;
    const size_t y_pos_stride = (size_t)p.B * H * R;
    const int hpg = p.heads_per_group;
    const size_t gfl = group_rec_floats(NP, CC);
    // A lane group (TPR lanes) covers RG rows per iteration: all RG x CPT chunks
    // are loaded first, each row's partial dot goes to its own accumulator, and
    // the RG partials are reduced across the group by a reduce-scatter, after
    // which lane pair (2m, 2m+1) of the group holds the full sum of row m.
    constexpr int RG = TPR == 8 ? 4 : 1;
    constexpr int GROUPS = kTeamThreads / TPR;   // lane groups per team
    const int niter = (R + GROUPS * RG - 1) / (GROUPS * RG);
    float v[NP][CPT * VEC];
    int cur_bg = -1;   // (sequence, group) whose C vectors v holds (Mamba-2)
    grid_dependency_wait();   // the group records are the prep kernel's output
    for (int m = 0; m * RL::NT + team < nst; ++m) {
        const int k = m * RL::NT + team, s = team * SPT + m % SPT, u = m / SPT;
        const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
        if (KIND == RS_MAMBA2) {   // issued before the wait, so the load overlaps it
            const int b = first / H, bg = b * p.G + (first - b * H) / hpg;
            if (bg != cur_bg) {
                load_vec_global<NP, CPT, VEC, TPR>(v, p.rec + (size_t)bg * gfl, CC, npos, tl);
                cur_bg = bg;
            }
        }
        if (!mbar_wait_bounded(full + s, u & 1)) {
            if (lane == 0) atomicOr(&p.err[first / H], RS_SEQ_ERR_TIMEOUT);
            break;
        }
        const unsigned char *st = stage(s);
        for (int i = 0; i < cnt; ++i) {
            const int tile = first + i;
            const unsigned char *tl_data = st + (size_t)i * tile_bytes;
            const unsigned char *wblk = st + lay.blk_off + (size_t)i * blk_bytes;
            const float *mul = reinterpret_cast<const float *>(st + lay.rec_off + (size_t)i * rec_bytes);
            const int hs = __float_as_int(mul[kRecHeadSlot]);
            const int Lr = min(max(__float_as_int(mul[kRecLen]), 0), cap);
            const float *coef = mul + kRecHdr;
            if (KIND == RS_MAMBA2) {
                const int b = tile / H, bg = b * p.G + (tile - b * H) / hpg;
                if (bg != cur_bg) {
                    load_vec_global<NP, CPT, VEC, TPR>(v, p.rec + (size_t)bg * gfl, CC, npos, tl);
                    cur_bg = bg;
                }
            } else {
                const float *vec = coef + (size_t)NP * cap;
#pragma unroll
                for (int j = 0; j < NP; ++j)
#pragma unroll
                    for (int c = 0; c < CPT; ++c)
#pragma unroll
                        for (int e = 0; e < VEC; ++e)
                            v[j][c * VEC + e] = j < npos ? vec[j * CC + (tl + c * TPR) * VEC + e] : 0.f;
            }
            float mj[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) mj[j] = j < npos ? mul[j] : 0.f;
            const size_t y_off = (size_t)tile * R;
            for (int it = 0; it < niter; ++it) {
                const int rbase = (it * GROUPS + row0) * RG;   // first row of this group
                uint4 raw[RG][CPT];
#pragma unroll
                for (int r = 0; r < RG; ++r)
#pragma unroll
                    for (int c = 0; c < CPT; ++c) {
                        raw[r][c] = make_uint4(0u, 0u, 0u, 0u);
                        if (rbase + r < R)
                            raw[r][c] = *reinterpret_cast<const uint4 *>(
                                tl_data + ((size_t)(rbase + r) * CC + (tl + c * TPR) * VEC) * TS::bytes);
                    }
                // even / odd columns accumulate in the two halves of packed fp32 FMAs
                float2 acc2[NP][RG];
#pragma unroll
                for (int j = 0; j < NP; ++j)
#pragma unroll
                    for (int r = 0; r < RG; ++r) acc2[j][r] = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < RG; ++r)
#pragma unroll
                    for (int c = 0; c < CPT; ++c) {
                        float f[VEC];
                        Chunk<TS>::expand(raw[r][c], f);
#pragma unroll
                        for (int e = 0; e < VEC; e += 2)
#pragma unroll
                            for (int j = 0; j < NP; ++j)
                                acc2[j][r] = ffma2(make_float2(f[e], f[e + 1]),
                                                   make_float2(v[j][c * VEC + e], v[j][c * VEC + e + 1]), acc2[j][r]);
                    }
                float acc[NP][RG];
#pragma unroll
                for (int j = 0; j < NP; ++j)
#pragma unroll
                    for (int r = 0; r < RG; ++r) acc[j][r] = acc2[j][r].x + acc2[j][r].y;
                if constexpr (RG == 4) {
                    const bool hi = tl & 4, b1 = tl & 2;
                    const int row = rbase + (hi ? 2 : 0) + (b1 ? 1 : 0);
                    // buffer terms of the row, entries split between the lane pair
                    float zr[NP];
#pragma unroll
                    for (int j = 0; j < NP; ++j) zr[j] = 0.f;
                    if (row < R)
                        for (int e = tl & 1; e < Lr; e += 2) {
                            const float w = lds_in(wblk, (size_t)((hs + e) & p.cap_mask) * R + row, p.in_dtype);
#pragma unroll
                            for (int j = 0; j < NP; ++j)
                                if (j < npos) zr[j] = fmaf(coef[j * cap + e], w, zr[j]);
                        }
#pragma unroll
                    for (int j = 0; j < NP; ++j) zr[j] += __shfl_xor_sync(0xffffffffu, zr[j], 1);
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        // xor 4: keep rows {0,1} (hi = 0) or {2,3} (hi = 1)
                        const float k0 = (hi ? acc[j][2] : acc[j][0]) + __shfl_xor_sync(0xffffffffu, hi ? acc[j][0] : acc[j][2], 4);
                        const float k1 = (hi ? acc[j][3] : acc[j][1]) + __shfl_xor_sync(0xffffffffu, hi ? acc[j][1] : acc[j][3], 4);
                        // xor 2: keep the first (b1 = 0) or second (b1 = 1) of the pair
                        float t = (b1 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);
                        t += __shfl_xor_sync(0xffffffffu, t, 1);
                        if ((tl & 1) == 0 && row < R && j < npos)
                            st_out(y, y_off + j * y_pos_stride + row, fmaf(mj[j], t, zr[j]), p.out_dtype);
                    }
                } else {
                    // buffer terms of row rbase, entries split over the row's TPR lanes
                    float zr[NP];
#pragma unroll
                    for (int j = 0; j < NP; ++j) zr[j] = 0.f;
                    if (rbase < R)
                        for (int e = tl; e < Lr; e += TPR) {
                            const float w = lds_in(wblk, (size_t)((hs + e) & p.cap_mask) * R + rbase, p.in_dtype);
#pragma unroll
                            for (int j = 0; j < NP; ++j)
                                if (j < npos) zr[j] = fmaf(coef[j * cap + e], w, zr[j]);
                        }
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        const float t = row_sum<TPR>(acc[j][0]);
                        const float zz = row_sum<TPR>(zr[j]);
                        if (tl == 0 && rbase < R && j < npos)
                            st_out(y, y_off + j * y_pos_stride + rbase, fmaf(mj[j], t, zz), p.out_dtype);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
    }
}

static int g_num_sms[64];

static int num_sms() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!g_num_sms[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_num_sms[dev] = n > 0 ? n : 148;
    }
    return g_num_sms[dev];
}

static StreamLayout layout_for(const Params &p, int npos) {
    const int eb = p.copy_dtype == RS_BF16 ? 2 : p.copy_dtype == RS_E4M3 ? 1 : 4;
    const int NPr = prep_np(npos);
    const int nt = NPr <= 2 ? Roles<1>::NT : Roles<8>::NT;
    return stream_layout((size_t)p.R * p.CC * eb, p.blk_r, 4 * tile_rec_floats(p.kind, NPr, p.cap, p.CC), nt);
}

size_t stream_outputs_smem(const Params &p, int npos) { return layout_for(p, npos).total; }

template <int KIND, int CC, typename TS, int NP>
static cudaError_t launch_stream_t(const Params &p, int npos, void *y, cudaStream_t st) {
    const void *state = p.copy_dtype == RS_NONE ? static_cast<const void *>(p.master) : p.copy;
    const StreamLayout lay = layout_for(p, npos);
    auto k = stream_outputs_kernel<KIND, CC, TS, NP>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total);
    if (e != cudaSuccess) return e;
    const int tiles = p.B * p.H;
    int grid = num_sms();
    if (grid > tiles) grid = tiles;
    // may start while the prep kernel before it is still running (see grid_dependency_wait)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Roles<NP>::THREADS);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, p, state, npos, y);
}

template <int KIND, int CC, typename TS>
static cudaError_t launch_stream_np(const Params &p, int npos, void *y, cudaStream_t st) {
    switch (prep_np(npos)) {
        case 1: return launch_stream_t<KIND, CC, TS, 1>(p, npos, y, st);
        case 2: return launch_stream_t<KIND, CC, TS, 2>(p, npos, y, st);
        case 5: return launch_stream_t<KIND, CC, TS, 5>(p, npos, y, st);
        default: return launch_stream_t<KIND, CC, TS, 8>(p, npos, y, st);
    }
}

template <int KIND>
struct StreamCC {
    template <int CC>
    static cudaError_t go(const Params &p, int npos, void *y, cudaStream_t st) {
        switch (p.copy_dtype) {
            case RS_BF16: return launch_stream_np<KIND, CC, StBF16>(p, npos, y, st);
            case RS_E4M3: return launch_stream_np<KIND, CC, StE4M3>(p, npos, y, st);
            default: return launch_stream_np<KIND, CC, StF32>(p, npos, y, st);
        }
    }
};

// Output-only replay / verification, optionally preceded by the append of T
// step inputs: the prep kernel (which also performs the append) writes the
// records, then the streaming pass reads each checkpoint tile once.
cudaError_t launch_outputs(const Params &p, int npos, int T, const rs_inputs &in, void *y, cudaStream_t st,
                           cudaEvent_t *ev) {
    cudaError_t e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    e = launch_prep(p, npos, T, in, st);
    if (e != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    e = cudaErrorInvalidValue;
    if (p.kind == RS_MAMBA2) {
        RS_DISPATCH_CC(p.CC, e = StreamCC<RS_MAMBA2>::go, (p, npos, y, st));
    } else {
        RS_DISPATCH_CC(p.CC, e = StreamCC<RS_GDN>::go, (p, npos, y, st));
    }
    if (e != cudaSuccess) return e;
    if (ev) e = cudaEventRecord(ev[2], st);
    return e;
}

}  // namespace rs
