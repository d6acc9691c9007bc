// Host-side launchers of the ReplaySSM kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

// Instantiate a launcher for each supported tile width (columns of a state
// tile).  RET_FN is either `return f` or an assignment `e = f`; each case ends
// with a break, so exactly one instantiation runs.
#define RS_DISPATCH_CC(cc, RET_FN, ARGS)        \
    switch (cc) {                               \
        case 16: { RET_FN<16> ARGS; } break;    \
        case 32: { RET_FN<32> ARGS; } break;    \
        case 64: { RET_FN<64> ARGS; } break;    \
        case 128: { RET_FN<128> ARGS; } break;  \
        case 256: { RET_FN<256> ARGS; } break;  \
        default: break;                         \
    }

// Rows of a register-resident tile each thread holds: ceil(R / rows-per-pass),
// rounded up to 1, 2, 4 or 8.  Rows per pass = 256 / (threads sharing a row).
#define RS_DISPATCH_NPASS(CC, R, RET_FN, ARGS)                               \
    {                                                                        \
        constexpr int tpr_ = (CC / 4) < 8 ? (CC / 4) : 8;                    \
        constexpr int rpb_ = ::rs::kTileThreads / tpr_;                      \
        const int np_ = ((R) + rpb_ - 1) / rpb_;                            \
        if (np_ <= 1) { RET_FN<CC, 1> ARGS; }                                \
        else if (np_ <= 2) { RET_FN<CC, 2> ARGS; }                           \
        else if constexpr ((CC) <= 128) {                                    \
            if (np_ <= 4) { RET_FN<CC, 4> ARGS; }                            \
            else if constexpr ((CC) <= 64) {                                 \
                if (np_ <= 8) { RET_FN<CC, 8> ARGS; }                        \
            }                                                                \
        }                                                                    \
    }

namespace rs {

// Output-only replay / verification (both kinds): the prep kernel writes one
// record per tile into p.rec, then the streaming pass reads every checkpoint
// tile once.  launch_outputs does both.
cudaError_t launch_prep(const Params &p, int npos, int T, const rs_inputs &in, cudaStream_t st);
// state_map: the CUtensorMap (host memory) of the checkpoint the outputs read,
// from make_state_map.  ev (may be NULL): three events recorded before the
// prep kernel, between the two kernels and after the streaming kernel.
cudaError_t launch_outputs(const Params &p, const void *state_map, int npos, int T, const rs_inputs &in, void *y,
                           cudaStream_t st, cudaEvent_t *ev = nullptr);
// Encode the tensor map of the checkpoint the outputs read (the copy, or the
// master without one) into map_out (a CUtensorMap, 64-byte aligned).
cudaError_t make_state_map(const Params &p, void *map_out);
size_t prep_smem(const Params &p, int NP);
size_t stream_outputs_smem(const Params &p, int npos);

// Mamba-2
cudaError_t launch_m2_commit(const Params &p, int min_len, const int32_t *mask, cudaStream_t st);
cudaError_t launch_m2_eager(const Params &p, void *state, int sdt, const rs_inputs &in, int T,
                            void *y, const int32_t *cur, int nslots, cudaStream_t st);
size_t m2_commit_smem(const Params &p);

// Gated DeltaNet
cudaError_t launch_gdn_commit(const Params &p, int min_len, const int32_t *mask, cudaStream_t st);
cudaError_t launch_gdn_eager(const Params &p, void *state, int sdt, const rs_inputs &in, int T,
                             void *y, const int32_t *cur, int nslots, cudaStream_t st);
size_t gdn_commit_smem(const Params &p);

// Ring / pointers / checkpoints (both kinds)
cudaError_t launch_append(const Params &p, const rs_inputs &in, int T, cudaStream_t st);
cudaError_t launch_rollback(const Params &p, const int32_t *k, cudaStream_t st);
cudaError_t launch_load_checkpoint(const Params &p, const float *state, cudaStream_t st);
cudaError_t launch_init(const Params &p, cudaStream_t st);
cudaError_t launch_eager_accept(const Params &p, int32_t *cur, const int32_t *keep, int nslots,
                                cudaStream_t st);
cudaError_t launch_wait_selftest(uint32_t *out, long long limit, cudaStream_t st);

}  // namespace rs
