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
// consecutive tiles (about 32 KB, so that each copy moves enough bytes to keep
// the copy engine's per-operation cost small), their TT ring blocks and their
// TT records.  The tiles come in by 2-D tensor-map copies of boxes of up to 128
// bytes of each row, swizzled in shared memory (16-byte chunk c of row r at
// chunk c ^ (r mod 8) for 128-byte boxes) so that the tensor-core fragment
// loads of the verification path are free of bank conflicts; the blocks and
// records by 1-D bulk copies.  One producer thread issues them in tile order
// (transaction-counted "full" barrier, checkpoint evict-first in L2).  NT
// teams of four consumer warps take the stages in turn (stage k goes to team
// k mod NT); each team owns SPT stages of the ring, which it uses in order,
// and frees a stage ("empty" barrier) once it has contracted all its tiles.
// Every barrier therefore sees each of its uses waited for in order by the
// same waiters, so a phase-parity wait never aliases an older phase.  Every
// wait is bounded: one that gives up sets RS_SEQ_ERR_TIMEOUT and the role stops.
//
// Contraction.  Several positions over a bf16 copy (verification): bf16
// tensor-core MMAs (m16n8k16, fp32 accumulation) of 16-row blocks of the tile
// against the position vectors (up to 8 columns), each vector split into a
// bf16 high part and a bf16 remainder (two MMAs per k-step), which keeps
// about 16 significant bits; per element this costs far fewer instructions
// than unpacking and FMAs.  One position (decode), or an fp32 / fp8 copy:
// CUDA cores, each lane group of TPR lanes owning RG rows at a time, fp32
// FMAs (for one position the MMA's 8 columns would be 7/8 idle, and the
// measured CUDA-core pass is faster).
//
// Mamba-2's contraction vector C_{e_j} is one per (sequence, group) and is the
// same for all heads of the group: the consumers keep it in registers and
// reload it only when the group changes.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "outputs.cuh"
#include "launch.h"

namespace rs {

constexpr int kTeamWarps = 4;                   // consumer warps per team (one tile at a time)
constexpr int kTeamThreads = 32 * kTeamWarps;
constexpr size_t kStreamSmemMax = 227 * 1024;     // opt-in shared memory of one CTA
constexpr size_t kStreamSmemReserve = 1024 + 512; // base alignment slack + barriers
constexpr size_t kStageTarget = 32 * 1024;      // checkpoint bytes a stage aims for
constexpr int kMaxTilesPerStage = 8;
constexpr int kMaxBoxRows = 256;                // tensor-map box height limit

// Consumer teams: 3; 2 for the CUDA-core contraction of many positions (its
// register tile needs more than the 128 registers three teams allow); 4 for
// the tensor-core path up to 5 positions and rows of up to 128 columns, whose
// warps wait mostly on instruction latency (a fourth team measured 5 to 8 %
// faster than three at 5 positions, with the 96 registers 17 warps allow; 8
// positions or 256 columns keep three teams and 128 registers).
__host__ __device__ constexpr bool use_mma(int state_bytes, int NP) { return state_bytes == 2 && NP >= 2; }
__host__ __device__ constexpr int consumer_teams(int NP, bool mma, int CC) {
    return (mma && NP <= 5 && CC <= 128) ? 4 : (NP <= 2 || mma) ? 3 : 2;
}

template <int NP, bool MMA, int CC>
struct Roles {
    static constexpr int NT = consumer_teams(NP, MMA, CC);   // consumer teams
    static constexpr int NCW = NT * kTeamWarps;          // consumer warps
    static constexpr int THREADS = 32 * (NCW + 1);       // + the producer warp
};

// Width of the boxes a checkpoint row is copied in, and the matching swizzle:
// 16-byte chunk bits [4, 4 + log2(BOXB / 16)) of a shared-memory offset are
// XORed with the bits from 7 up (the hardware's 32/64/128-byte swizzles).
__host__ __device__ constexpr int box_bytes_for(int row_bytes) { return row_bytes < 128 ? row_bytes : 128; }
__host__ __device__ constexpr uint32_t swizzle_mask_for(int box_bytes) {
    return box_bytes == 128 ? 7u : box_bytes == 64 ? 3u : box_bytes == 32 ? 1u : 0u;
}

// Tiles per stage: about kStageTarget bytes of checkpoint, tiles plus ring
// blocks within kStageCap bytes, at most kMaxTilesPerStage, and no more rows
// than one box may have.
constexpr size_t kStageCap = 36 * 1024;
__host__ __device__ inline int stage_tiles(int R, size_t row_bytes, size_t blk_bytes) {
    const size_t tile = (size_t)R * row_bytes;
    size_t tt = kStageTarget / tile;
    const size_t by_cap = kStageCap / (tile + blk_bytes), by_rows = (size_t)kMaxBoxRows / (size_t)R;
    tt = tt < by_cap ? tt : by_cap;
    tt = tt < by_rows ? tt : by_rows;
    tt = tt > (size_t)kMaxTilesPerStage ? (size_t)kMaxTilesPerStage : tt;
    return (int)(tt < 1 ? 1 : tt);
}

struct StreamLayout {
    size_t box_region, blk_off, rec_off, stage_bytes, bars, total;
    int TT;         // tiles per stage
    int box_rows;   // rows of every box copy (TT R)
    int S, SPT;     // stages in all, stages per team
    int NT;         // consumer teams in use
};

// Stage (1024-byte aligned): nbox boxes of TT R rows | TT ring blocks | TT records.
__host__ __device__ inline StreamLayout stream_layout(int R, size_t row_bytes, size_t blk_bytes, size_t rec_bytes,
                                                      int nt) {
    StreamLayout l;
    l.TT = stage_tiles(R, row_bytes, blk_bytes);
    l.box_rows = l.TT * R;
    const size_t boxb = (size_t)box_bytes_for((int)row_bytes), nbox = row_bytes / boxb;
    l.box_region = align_up((size_t)l.box_rows * boxb, 1024);
    l.blk_off = nbox * l.box_region;
    l.rec_off = align_up(l.blk_off + (size_t)l.TT * blk_bytes, 16);
    l.stage_bytes = align_up(l.rec_off + (size_t)l.TT * rec_bytes, 1024);
    const size_t fit = (kStreamSmemMax - kStreamSmemReserve) / l.stage_bytes;   // stages that fit
    // four teams (the tensor-core path) only where each gets a stage; else three
    l.NT = (nt == 4 && fit < 4) ? 3 : nt;
    size_t spt = fit / l.NT;
    spt = spt < 1 ? 1 : spt > 8 ? 8 : spt;
    l.S = (int)(spt * l.NT);
    l.SPT = (int)spt;
    l.bars = (size_t)l.S * l.stage_bytes;
    l.total = l.bars + align_up(16 * (size_t)l.S, 128) + 1024;   // + slack to align the base to 1024
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

// 2-D tensor-map copy of one box at element column x, row y (no multicast).
__device__ __forceinline__ void tma_box_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar,
                                           uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
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

// The same from a k-major store: each lane addresses one 16-byte row of a
// transposed 8x8 block, and receives the fragment of the transpose.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&a)[4], const void *smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(smem_u32(smem_row)));
}

// bf16 pair (first value in the low half) rounded to nearest even, and the
// pair of the remainders: hi + lo hold each fp32 value to about 16 bits.
__device__ __forceinline__ void split_bf16x2(float v0, float v1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
    const __nv_bfloat16 l0 = __float2bfloat16_rn(v0 - __bfloat162float(h0));
    const __nv_bfloat16 l1 = __float2bfloat16_rn(v1 - __bfloat162float(h1));
    hi = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
    lo = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
}

// The contraction vectors a CUDA-core consumer thread needs: vec_j at its CPT chunks.
template <int NP, int CPT, int VEC, int TPR>
__device__ __forceinline__ void load_vec(float (&v)[NP][CPT * VEC], const float *vec, int CC, int npos, int tl) {
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

// The B fragments of the MMA path: vec_n (n = lane / 4 < npos, else 0) at
// k = 16 ks + 2 (lane % 4) + {0, 1} and + 8, split into bf16 high and low parts.
template <int KS>
__device__ __forceinline__ void load_vec_frag(uint32_t (&bh)[KS][2], uint32_t (&bl)[KS][2], const float *vec,
                                              int CC, int npos, int lane) {
    const int n = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 f = make_float2(0.f, 0.f);
            if (n < npos) f = *reinterpret_cast<const float2 *>(vec + n * CC + ks * 16 + 2 * t + 8 * h);
            split_bf16x2(f.x, f.y, bh[ks][h], bl[ks][h]);
        }
}

template <int KIND, int CC, typename TS, int NP>
__global__ void __launch_bounds__((Roles<NP, use_mma(TS::bytes, NP), CC>::THREADS), 1)
stream_outputs_kernel(const Params p, const __grid_constant__ CUtensorMap smap, int npos, void *y) {
    using RL = Roles<NP, use_mma(TS::bytes, NP), CC>;
    constexpr int ROWB = CC * TS::bytes, BOXB = box_bytes_for(ROWB), NBOX = ROWB / BOXB, CPB = BOXB / 16;
    constexpr uint32_t SWM = swizzle_mask_for(BOXB);
    constexpr bool USE_MMA = use_mma(TS::bytes, NP);   // bf16 copy, several positions: tensor cores
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int R = p.R, H = p.H, cap = p.cap, cstr = coef_stride(cap);
    const size_t rfl = tile_rec_floats(KIND, NP, cap, CC);
    const uint32_t rec_bytes = static_cast<uint32_t>(4 * rfl);
    const uint32_t blk_bytes = static_cast<uint32_t>(p.blk_r);
    const float *trec = p.rec + p.rec_tile_off;
    // ring rows the outputs sum over: Mamba-2 x, GDN v ([B][H][cap][R] blocks)
    const unsigned char *wring = static_cast<const unsigned char *>(KIND == RS_MAMBA2 ? p.ra : p.rc);
    const StreamLayout lay = stream_layout(R, ROWB, blk_bytes, rec_bytes, RL::NT);
    const int S = lay.S, SPT = lay.SPT, TT = lay.TT, NTU = lay.NT;   // NTU <= RL::NT teams in use
    const uint32_t stage_tx_tiles = static_cast<uint32_t>(NBOX * lay.box_rows * BOXB);
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
            auto copy_tiles = [&](unsigned char *st, int first, uint64_t *bar) {
                // a partial last stage still moves whole boxes (rows past the end read as zeros)
#pragma unroll
                for (int bx = 0; bx < NBOX; ++bx)
                    tma_box_2d(st + bx * lay.box_region, &smap, bx * (BOXB / TS::bytes), first * R, bar, pol_state);
            };
            auto copy_side = [&](unsigned char *st, int first, int cnt, uint64_t *bar) {
                bulk_pieces(st + lay.rec_off, trec + (size_t)first * rfl, cnt * rec_bytes, bar, pol_rec);
                bulk_pieces(st + lay.blk_off, wring + (size_t)first * blk_bytes, cnt * blk_bytes, bar, pol_rec);
            };
            // The checkpoint does not depend on the prep kernel that precedes
            // this one in the stream, so the first ring's worth of checkpoint
            // copies starts at once; the records and ring blocks the prep
            // kernel writes are copied after griddepcontrol.wait (the prep
            // grid has finished and its writes are visible).
            const int pre = nst < S ? nst : S;
            for (int k = 0; k < pre; ++k) {   // stage k < S: slot k % NT * SPT + k / NT, first use
                const int s = (k % NTU) * SPT + k / NTU;
                const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
                mbar_expect_tx(full + s, stage_tx_tiles + cnt * (blk_bytes + rec_bytes));
                copy_tiles(stage(s), first, full + s);
            }
            grid_dependency_wait();
            for (int k = 0; k < pre; ++k) {
                const int s = (k % NTU) * SPT + k / NTU;
                const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
                copy_side(stage(s), first, cnt, full + s);
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
                mbar_expect_tx(full + s, stage_tx_tiles + cnt * (blk_bytes + rec_bytes));
                copy_side(st, first, cnt, full + s);
                copy_tiles(st, first, full + s);
                if (++team == NTU) {
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
    const int team = warp / kTeamWarps;
    if (team >= NTU) return;   // a team the layout has no stages for (see stream_layout)
    const size_t y_pos_stride = (size_t)p.B * H * R;
    const int hpg = p.heads_per_group;
    const size_t gfl = group_rec_floats(NP, CC);
    // byte address of 16-byte chunk q of stage row rr (the swizzled box layout)
    auto chunk_at = [&](const unsigned char *st, int rr, int q) -> const unsigned char * {
        const int bx = q / CPB, c = q - bx * CPB;
        const uint32_t o = static_cast<uint32_t>(rr) * BOXB + static_cast<uint32_t>(c) * 16u;
        return st + (size_t)bx * lay.box_region + (o ^ (((o >> 7) & SWM) << 4));
    };
    grid_dependency_wait();   // the group records are the prep kernel's output

    if constexpr (USE_MMA) {
        // ----------------------------------------------- tensor-core path
        constexpr int KS = CC / 16;
        const int wt = warp % kTeamWarps;   // warp within the team
        const int MB = (R + 15) / 16;       // 16-row blocks of a tile
        uint32_t bh[KS][2], bl[KS][2];
        int cur_bg = -1;
        // The buffer terms sum_i coef_j[i] w_i[r] are a product too: rows r of
        // the ring block (k = ring slot) times the coefficients moved to slot
        // order, in up to two more k-steps with their own accumulators (the
        // multiplier mul_j scales only the checkpoint part).  bf16 rings of up
        // to 32 slots with R a multiple of 8; otherwise summed per lane below.
        const bool zmma = p.in_dtype == RS_BF16 && cap <= 32 && (R & 7) == 0;
        const int KE = (cap + 15) / 16;
        for (int m = 0; m * NTU + team < nst; ++m) {
            const int k = m * NTU + team, s = team * SPT + m % SPT, u = m / SPT;
            const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
            // (sequence, group) of the stage's first tile and its head within the
            // group; consecutive tiles advance the head, and the group index
            // b G + g by one whenever the head wraps
            int bg = 0, hl = 0;
            if (KIND == RS_MAMBA2) {   // issued before the wait, so the loads overlap it
                const int b = first / H, h = first - b * H, g = h / hpg;
                bg = b * p.G + g;
                hl = h - g * hpg;
                if (bg != cur_bg) {
                    load_vec_frag<KS>(bh, bl, p.rec + (size_t)bg * gfl, CC, npos, lane);
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
                const unsigned char *wblk = st + lay.blk_off + (size_t)i * blk_bytes;
                const float *mul = reinterpret_cast<const float *>(st + lay.rec_off + (size_t)i * rec_bytes);
                const int hs = __float_as_int(mul[kRecHeadSlot]);
                const int Lr = min(max(__float_as_int(mul[kRecLen]), 0), cap);
                const float *coef = mul + kRecHdr;
                if (KIND == RS_MAMBA2) {
                    if (i > 0 && ++hl == hpg) {
                        hl = 0;
                        ++bg;
                    }
                    if (bg != cur_bg) {
                        load_vec_frag<KS>(bh, bl, p.rec + (size_t)bg * gfl, CC, npos, lane);
                        cur_bg = bg;
                    }
                } else {
                    load_vec_frag<KS>(bh, bl, coef + (size_t)NP * cstr, CC, npos, lane);
                }
                const size_t y_off = (size_t)tile * R;
                const int g = lane >> 2, t = lane & 3;
                // B fragments of the buffer terms: coef_n[e(s)] at slots s = 16 kse + 2t + {0, 1} (+ 8),
                // e(s) = (s - head slot) mod cap, zero where e(s) >= L, s >= cap or n >= npos
                uint32_t zh[2][2], zl[2][2];
                if (zmma) {
#pragma unroll
                    for (int kse = 0; kse < 2; ++kse)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float cv[2];
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const int sl = kse * 16 + 2 * t + 8 * hh + q;
                                const int e = (sl - hs) & p.cap_mask;
                                cv[q] = (g < npos && sl < cap && e < Lr) ? coef[g * cstr + e] : 0.f;
                            }
                            split_bf16x2(cv[0], cv[1], zh[kse][hh], zl[kse][hh]);
                        }
                }
                for (int mb = wt; mb < MB; mb += kTeamWarps) {
                    // ldmatrix rows: lane l addresses row (l & 7) + 8 ((l >> 3) & 1) of the block, chunk l >> 4
                    int lr = mb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                    lr = lr < R ? lr : R - 1;   // rows past the tile repeat its last row; their results are dropped
                    const int rr = i * R + lr;
                    uint32_t a[KS][4];
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) ldmatrix_x4(a[ks], chunk_at(st, rr, ks * 2 + (lane >> 4)));
                    // four independent accumulation chains: (k-step parity) x (high, low part)
                    float d[4][4];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int f = 0; f < 4; ++f) d[c][f] = 0.f;
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        mma_bf16(d[(ks & 1) * 2], a[ks], bh[ks][0], bh[ks][1]);
                        mma_bf16(d[(ks & 1) * 2 + 1], a[ks], bl[ks][0], bl[ks][1]);
                    }
                    const int row0 = mb * 16 + g, row1 = row0 + 8;
                    float dz[4] = {0.f, 0.f, 0.f, 0.f};   // buffer terms, fragment layout (zmma)
                    if (zmma) {
                        float d2[2][4];
#pragma unroll
                        for (int c = 0; c < 2; ++c)
#pragma unroll
                            for (int f = 0; f < 4; ++f) d2[c][f] = 0.f;
                        // transposed 8x8 blocks of the ring block: lane l reads slot 8 ((l >> 4) & 1) + (l & 7)
                        // of the k-step, rows r0 .. r0 + 7 with r0 = 16 mb + 8 ((l >> 3) & 1)
                        int r0 = mb * 16 + ((lane >> 3) & 1) * 8;
                        r0 = r0 + 8 <= R ? r0 : R - 8;   // stays inside the block; rows >= R are dropped
#pragma unroll
                        for (int kse = 0; kse < 2; ++kse) {
                            if (kse >= KE) break;
                            int sl = kse * 16 + ((lane >> 4) & 1) * 8 + (lane & 7);
                            sl = sl < cap ? sl : 0;   // padding slots read row 0; their coefficients are 0
                            uint32_t a[4];
                            ldmatrix_x4_trans(a, wblk + ((size_t)sl * R + r0) * 2);
                            mma_bf16(d2[0], a, zh[kse][0], zh[kse][1]);
                            mma_bf16(d2[1], a, zl[kse][0], zl[kse][1]);
                        }
#pragma unroll
                        for (int f = 0; f < 4; ++f) dz[f] = d2[0][f] + d2[1][f];
                    }
                    // otherwise: buffer terms of rows g and g + 8, entries split over the lane quad
                    float zq[2][NP];
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr)
#pragma unroll
                        for (int j = 0; j < NP; ++j) zq[hr][j] = 0.f;
                    for (int e = zmma ? Lr : t; e < Lr; e += 4) {
                        const size_t wrow = (size_t)((hs + e) & p.cap_mask) * R;
                        const float w0 = row0 < R ? lds_in(wblk, wrow + row0, p.in_dtype) : 0.f;
                        const float w1 = row1 < R ? lds_in(wblk, wrow + row1, p.in_dtype) : 0.f;
#pragma unroll
                        for (int j = 0; j < NP; ++j) {
                            if (j >= npos) break;
                            const float c = coef[j * cstr + e];
                            zq[0][j] = fmaf(c, w0, zq[0][j]);
                            zq[1][j] = fmaf(c, w1, zq[1][j]);
                        }
                    }
                    if (!zmma) {   // (with zmma the sums above are empty)
#pragma unroll
                        for (int hr = 0; hr < 2; ++hr)
#pragma unroll
                            for (int j = 0; j < NP; ++j) {
                                zq[hr][j] += __shfl_xor_sync(0xffffffffu, zq[hr][j], 1);
                                zq[hr][j] += __shfl_xor_sync(0xffffffffu, zq[hr][j], 2);
                            }
                    }
                    // fragment f = 2 hr + hc: row g + 8 hr, position 2t + hc
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int row = hr ? row1 : row0;
                        if (row >= R) continue;
#pragma unroll
                        for (int hc = 0; hc < 2; ++hc) {
                            const int j = 2 * t + hc;
                            if (j >= npos) continue;
                            const int f = 2 * hr + hc;
                            float z = dz[f];
#pragma unroll
                            for (int jj = 0; jj < NP; ++jj)
                                if (jj == j) z += zq[hr][jj];
                            const float dot = (d[0][f] + d[2][f]) + (d[1][f] + d[3][f]);
                            st_out(y, y_off + j * y_pos_stride + row, fmaf(mul[j], dot, z), p.out_dtype);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);
        }
    } else {
        // ------------------------------------------------ CUDA-core path
        // 8 lanes per row; 16 when many positions are contracted, so that each
        // thread holds fewer columns of the NP vectors
        using G = Geom<CC, TS::bytes, (NP >= 5 ? 16 : 8)>;
        constexpr int VEC = G::VEC, TPR = G::TPR, CPT = G::CPT;
        const int ttid = threadIdx.x % kTeamThreads;
        const int tl = ttid % TPR, row0 = ttid / TPR;
        // A lane group (TPR lanes) covers RG rows per iteration: all RG x CPT chunks
        // are loaded first, each row's partial dot goes to its own accumulator, and
        // the RG partials are reduced across the group by a reduce-scatter (TPR 8:
        // lane pair (2m, 2m+1) of the group ends with row m; TPR 16: lanes 0-7 with
        // row 0, lanes 8-15 with row 1).
        constexpr int RG = TPR == 8 ? 4 : TPR == 16 ? 2 : 1;
        constexpr int GROUPS = kTeamThreads / TPR;   // lane groups per team
        const int niter = (R + GROUPS * RG - 1) / (GROUPS * RG);
        float v[NP][CPT * VEC];
        int cur_bg = -1;   // (sequence, group) whose C vectors v holds (Mamba-2)
        // With R a multiple of 8 the swizzle of a row depends only on the row
        // within its tile, so a thread's chunk offsets are the same in every
        // tile of a single-iteration pass: computed once.
        const bool fixed_offs = (R & 7) == 0 && niter == 1;
        uint32_t offs[RG][CPT];
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int c = 0; c < CPT; ++c)
                offs[r][c] = static_cast<uint32_t>(chunk_at(smem, row0 * RG + r, tl + c * TPR) - smem);
        for (int m = 0; m * NTU + team < nst; ++m) {
            const int k = m * NTU + team, s = team * SPT + m % SPT, u = m / SPT;
            const int first = t0 + k * TT, cnt = nt - k * TT < TT ? nt - k * TT : TT;
            int bg = 0, hl = 0;   // as in the tensor-core path
            if (KIND == RS_MAMBA2) {   // issued before the wait, so the load overlaps it
                const int b = first / H, h = first - b * H, g = h / hpg;
                bg = b * p.G + g;
                hl = h - g * hpg;
                if (bg != cur_bg) {
                    load_vec<NP, CPT, VEC, TPR>(v, p.rec + (size_t)bg * gfl, CC, npos, tl);
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
                const unsigned char *wblk = st + lay.blk_off + (size_t)i * blk_bytes;
                const float *mul = reinterpret_cast<const float *>(st + lay.rec_off + (size_t)i * rec_bytes);
                const int hs = __float_as_int(mul[kRecHeadSlot]);
                const int Lr = min(max(__float_as_int(mul[kRecLen]), 0), cap);
                const float *coef = mul + kRecHdr;
                if (KIND == RS_MAMBA2) {
                    if (i > 0 && ++hl == hpg) {
                        hl = 0;
                        ++bg;
                    }
                    if (bg != cur_bg) {
                        load_vec<NP, CPT, VEC, TPR>(v, p.rec + (size_t)bg * gfl, CC, npos, tl);
                        cur_bg = bg;
                    }
                } else {
                    load_vec<NP, CPT, VEC, TPR>(v, coef + (size_t)NP * cstr, CC, npos, tl);
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
                                    fixed_offs ? st + (size_t)i * R * BOXB + offs[r][c]
                                               : chunk_at(st, i * R + rbase + r, tl + c * TPR));
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
                                    if (j < npos) zr[j] = fmaf(coef[j * cstr + e], w, zr[j]);
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
                    } else if constexpr (RG == 2) {
                        // buffer terms of both rows, entries split over the group's 16 lanes
                        float zr[2][NP];
#pragma unroll
                        for (int r = 0; r < 2; ++r)
#pragma unroll
                            for (int j = 0; j < NP; ++j) zr[r][j] = 0.f;
                        for (int e = tl; e < Lr; e += TPR) {
                            const size_t wrow = (size_t)((hs + e) & p.cap_mask) * R;
#pragma unroll
                            for (int r = 0; r < 2; ++r) {
                                const float w = rbase + r < R ? lds_in(wblk, wrow + rbase + r, p.in_dtype) : 0.f;
#pragma unroll
                                for (int j = 0; j < NP; ++j)
                                    if (j < npos) zr[r][j] = fmaf(coef[j * cstr + e], w, zr[r][j]);
                            }
                        }
                        const bool hi = tl & 8;
                        const int row = rbase + (hi ? 1 : 0);
#pragma unroll
                        for (int j = 0; j < NP; ++j) {
                            // each lane's share of both rows' outputs, then xor 8 keeps row 0 (hi = 0) or row 1
                            const float o0 = fmaf(mj[j], acc[j][0], zr[0][j]), o1 = fmaf(mj[j], acc[j][1], zr[1][j]);
                            float t = (hi ? o1 : o0) + __shfl_xor_sync(0xffffffffu, hi ? o0 : o1, 8);
                            t += __shfl_xor_sync(0xffffffffu, t, 4);
                            t += __shfl_xor_sync(0xffffffffu, t, 2);
                            t += __shfl_xor_sync(0xffffffffu, t, 1);
                            if ((tl & 7) == 0 && row < R && j < npos)
                                st_out(y, y_off + j * y_pos_stride + row, t, p.out_dtype);
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
                                    if (j < npos) zr[j] = fmaf(coef[j * cstr + e], w, zr[j]);
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

static int state_bytes(const Params &p) { return p.copy_dtype == RS_BF16 ? 2 : p.copy_dtype == RS_E4M3 ? 1 : 4; }

static StreamLayout layout_for(const Params &p, int npos) {
    const int NPr = prep_np(npos);
    const bool mma = use_mma(state_bytes(p), NPr);
    const int nt = consumer_teams(NPr, mma, p.CC);   // the kernel's Roles<NP, MMA, CC>::NT
    return stream_layout(p.R, (size_t)p.CC * state_bytes(p), p.blk_r, 4 * tile_rec_floats(p.kind, NPr, p.cap, p.CC), nt);
}

size_t stream_outputs_smem(const Params &p, int npos) { return layout_for(p, npos).total; }

cudaError_t make_state_map(const Params &p, void *map_out) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const int eb = state_bytes(p);
    const size_t row_bytes = (size_t)p.CC * eb;
    const int boxb = box_bytes_for((int)row_bytes);
    void *base = p.copy_dtype == RS_NONE ? static_cast<void *>(p.master) : p.copy;
    const CUtensorMapDataType dt = eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const cuuint64_t dims[2] = {(cuuint64_t)p.CC, (cuuint64_t)p.B * p.H * p.R};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(boxb / eb), (cuuint32_t)(stage_tiles(p.R, row_bytes, p.blk_r) * p.R)};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = boxb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : boxb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : boxb == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
    const CUresult r = encode(static_cast<CUtensorMap *>(map_out), dt, 2, base, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int KIND, int CC, typename TS, int NP>
static cudaError_t launch_stream_t(const Params &p, const CUtensorMap &smap, int npos, void *y, cudaStream_t st) {
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
    cfg.blockDim = dim3(Roles<NP, use_mma(TS::bytes, NP), CC>::THREADS);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, p, smap, npos, y);
}

template <int KIND, int CC, typename TS>
static cudaError_t launch_stream_np(const Params &p, const CUtensorMap &smap, int npos, void *y, cudaStream_t st) {
    switch (prep_np(npos)) {
        case 1: return launch_stream_t<KIND, CC, TS, 1>(p, smap, npos, y, st);
        case 2: return launch_stream_t<KIND, CC, TS, 2>(p, smap, npos, y, st);
        case 5: return launch_stream_t<KIND, CC, TS, 5>(p, smap, npos, y, st);
        default: return launch_stream_t<KIND, CC, TS, 8>(p, smap, npos, y, st);
    }
}

template <int KIND>
struct StreamCC {
    template <int CC>
    static cudaError_t go(const Params &p, const CUtensorMap &smap, int npos, void *y, cudaStream_t st) {
        switch (p.copy_dtype) {
            case RS_BF16: return launch_stream_np<KIND, CC, StBF16>(p, smap, npos, y, st);
            case RS_E4M3: return launch_stream_np<KIND, CC, StE4M3>(p, smap, npos, y, st);
            default: return launch_stream_np<KIND, CC, StF32>(p, smap, npos, y, st);
        }
    }
};

// Output-only replay / verification, optionally preceded by the append of T
// step inputs: the prep kernel writes the per-tile records (and appends), then
// the streaming pass reads each checkpoint tile once.
cudaError_t launch_outputs(const Params &p, const void *state_map, int npos, int T, const rs_inputs &in, void *y,
                           cudaStream_t st, cudaEvent_t *ev) {
    const CUtensorMap &smap = *static_cast<const CUtensorMap *>(state_map);
    cudaError_t e;
    if (ev && (e = cudaEventRecord(ev[0], st)) != cudaSuccess) return e;
    e = launch_prep(p, npos, T, in, st);
    if (e != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[1], st)) != cudaSuccess) return e;
    e = cudaErrorInvalidValue;
    if (p.kind == RS_MAMBA2) {
        RS_DISPATCH_CC(p.CC, e = StreamCC<RS_MAMBA2>::go, (p, smap, npos, y, st));
    } else {
        RS_DISPATCH_CC(p.CC, e = StreamCC<RS_GDN>::go, (p, smap, npos, y, st));
    }
    if (e != cudaSuccess) return e;
    if (ev) e = cudaEventRecord(ev[2], st);
    return e;
}

}  // namespace rs
