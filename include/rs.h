/*
 * rs.h -- C interface of the ReplaySSM decode library (librs_b200.so).
 *
 * ReplaySSM ("ReplaySSM: Cache SSM Inputs, Not State", Abstract) represents the
 * recurrent state of each sequence of a Mamba-2 or Gated DeltaNet layer as a
 * read-only checkpoint plus a buffer of the SSM inputs seen since that
 * checkpoint.  Each decode step's output is computed from the checkpoint and
 * the buffer without writing state; the checkpoint is rewritten only when the
 * caller commits; speculative tokens are rejected by moving the buffer's tail
 * pointer; a high-precision master checkpoint serves the updates while a
 * low-precision copy serves the outputs.
 *
 * Recurrences (the pages give none; the standard published forms are used):
 *   Mamba-2:  h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D x_t
 *             state tile per (sequence, head): [P][N], row p, column n
 *   GDN:      S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *             o_t = gdn_scale * S_t q_t
 *             state tile per (sequence, head): [dv][dk], row r, column c
 *
 * Conventions for every call
 *   - All data pointers are DEVICE pointers unless a parameter says "host".
 *   - Every call is asynchronous on the given stream (a cudaStream_t passed as
 *     void*; NULL means the legacy default stream) unless it says "synchronises".
 *   - The library never allocates device memory.  The caller allocates one
 *     workspace of rs_workspace_size() bytes (256-byte aligned) that holds the
 *     checkpoints, the input ring and the pointers; it must outlive the handle.
 *   - Host-checkable problems (NULL pointers, bad shapes, T > cap, npos out of
 *     range) return an error and launch nothing.  Data-dependent problems found
 *     on the device (ring overflow, rollback past the checkpoint, too few
 *     buffered entries) leave that sequence's pointers unchanged, write zeros for
 *     its outputs and set a sticky bit in its error word (rs_get_error).  No call
 *     traps or spins without a bound on the device.
 *   - Dense layouts, row-major, no padding:  B = batch, H = nheads,
 *     R = rows of a state tile (Mamba-2 P = headdim, GDN dv = headdim),
 *     Cc = columns (Mamba-2 N = dstate, GDN dk = dstate), G = ngroups.
 */
#ifndef RS_H
#define RS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct rs_ctx *rs_handle;
typedef void *rs_stream; /* cudaStream_t */

typedef enum {
    RS_OK = 0,
    RS_ERR_ARG = -1,          /* invalid argument or configuration */
    RS_ERR_CAPACITY = -2,     /* T or npos larger than the ring allows */
    RS_ERR_CUDA = -4,         /* a CUDA runtime call failed (rs_last_cuda_error) */
    RS_ERR_WORKSPACE = -5,    /* workspace NULL, misaligned or too small */
    RS_ERR_DEVICE_FLAG = -6,  /* rs_get_error: some sequence has a sticky error bit */
    RS_ERR_UNSUPPORTED = -8   /* valid but unsupported shape / dtype combination */
} rs_status;

typedef enum { RS_MAMBA2 = 0, RS_GDN = 1 } rs_kind;

typedef enum {
    RS_NONE = 0,  /* no low-precision copy: outputs read the fp32 master */
    RS_F32 = 1,
    RS_BF16 = 2,  /* bfloat16, round to nearest even */
    RS_E4M3 = 3   /* OCP FP8 E4M3 (fn), RNE, satfinite, one fp32 scale per tile */
} rs_dtype;

/* Per-sequence sticky device error bits (rs_get_error). */
enum {
    RS_SEQ_ERR_OVERFLOW = 1u,  /* rs_append: len + T > cap; nothing written      */
    RS_SEQ_ERR_ROLLBACK = 2u,  /* rs_rollback / rs_eager_accept: k outside range */
    RS_SEQ_ERR_EMPTY = 4u,     /* outputs asked for with len < npos (or len 0)   */
    RS_SEQ_ERR_TIMEOUT = 8u    /* a bounded on-device wait gave up               */
};

typedef struct {
    int32_t kind;        /* rs_kind */
    int32_t batch;       /* B >= 1 sequences */
    int32_t nheads;      /* H >= 1 */
    int32_t headdim;     /* R: Mamba-2 P, GDN dv; 1..256 */
    int32_t dstate;      /* Cc: Mamba-2 N, GDN dk; one of 16, 32, 64, 128, 256 */
    int32_t ngroups;     /* Mamba-2 G, divides H (head h uses group h / (H/G)); GDN: 1 */
    int32_t cap;         /* ring slots per sequence: power of two, 1..256 */
    int32_t npos_max;    /* largest npos of rs_verify_outputs / rs_eager_verify: 1..8 */
    int32_t in_dtype;    /* RS_F32 or RS_BF16: x, B, C (Mamba-2) / q, k, v (GDN) */
    int32_t copy_dtype;  /* RS_NONE, RS_BF16 or RS_E4M3: the output copy */
    int32_t out_dtype;   /* RS_F32 or RS_BF16: y / o */
    int32_t shared_lowp; /* 1: no fp32 master; the low-precision copy serves both
                            outputs and updates (the comparison arm of step 5) */
    float gdn_scale;     /* GDN output scale; 0 is taken as 1 */
} rs_config;

/* Step inputs.  Mamba-2 uses x, dt, B, C; GDN uses q, k, v, alpha, beta.
 * dt, alpha, beta are fp32; the others are in_dtype.  Shapes for T steps:
 *   x [T][B][H][P]   dt [T][B][H]   B, C [T][B][G][N]      (dt after softplus)
 *   q, k [T][B][H][dk]   v [T][B][H][dv]   alpha, beta [T][B][H]
 * Device memory, contiguous, naturally aligned (fp32 arrays to 4 bytes, bf16 to
 * 2); Mamba-2's B and C must be 16-byte aligned.  A missing or misaligned
 * pointer makes the call return RS_ERR_ARG.                                   */
typedef struct {
    const void *x;
    const float *dt;
    const void *B;
    const void *C;
    const void *q;
    const void *k;
    const void *v;
    const float *alpha;
    const float *beta;
} rs_inputs;

/* Byte offsets of the regions of a workspace (each 256-byte aligned; a region a
 * configuration does not use has size 0).  Tests and tools use this to view the
 * checkpoints and pointers; kernels get the same offsets.
 *
 * The input ring keeps, per (sequence, head) or (sequence, group), one block of
 * cap slots; the entry at logical position t sits in slot t mod cap.  Blocks
 * are contiguous so that a whole block moves in one bulk copy; a block's stride
 * is its size rounded up to 16 bytes.  capd = max(cap, 4). */
typedef struct {
    size_t master, master_bytes;   /* fp32 [B][H][R][Cc]          (not with shared_lowp) */
    size_t copy, copy_bytes;       /* copy_dtype [B][H][R][Cc]    (not with RS_NONE)     */
    size_t scale, scale_bytes;     /* fp32 [B][H]                 (RS_E4M3 only)         */
    size_t ring_a, ring_a_bytes;   /* Mamba-2 x [B][H][cap][P]     | GDN q [B][H][cap][dk] */
    size_t ring_b, ring_b_bytes;   /* Mamba-2 dt [B][H][capd] f32  | GDN k [B][H][cap][dk] */
    size_t ring_c, ring_c_bytes;   /* Mamba-2 B [B][G][cap][N]     | GDN v [B][H][cap][dv] */
    size_t ring_d, ring_d_bytes;   /* Mamba-2 C [B][G][cap][N]     | GDN alpha [B][H][capd] */
    size_t ring_e, ring_e_bytes;   /* (unused for Mamba-2)         | GDN beta [B][H][capd]  */
    size_t head, tail, err, arrive;/* int32 / int32 / uint32 / uint32, each [B]            */
    size_t scratch, scratch_bytes; /* fp32 replay records, written and read inside one
                                      output call (NP = npos_max rounded up to 1, 2, 5, 8):
                                      Mamba-2: [B][G][NP Cc] group records, then
                                      [B][H][16 + NP cs] tile records; GDN: [B][H][16 +
                                      NP (cs + Cc)], cs = cap rounded up to 4, plus 4;
                                      each record rounded up to 16 bytes                  */
    size_t total;
} rs_layout;

/* Workspace size and layout for a configuration.  Pure host computation; needs
 * no GPU.  Returns RS_ERR_ARG / RS_ERR_UNSUPPORTED for a bad configuration. */
rs_status rs_workspace_size(const rs_config *cfg, size_t *bytes);
rs_status rs_workspace_layout(const rs_config *cfg, rs_layout *layout);

/* Create a handle over a caller-allocated workspace.  A and D (Mamba-2 only,
 * fp32 [H], device; D may be NULL for 0) are copied into the handle's view by
 * pointer: they must stay valid for the handle's lifetime.  Zeroes the
 * workspace on `stream` (checkpoint = 0, head = tail = 0, no errors, fp8
 * scales = 1).  The handle itself is host memory owned by the library. */
rs_status rs_create(const rs_config *cfg, void *workspace, size_t workspace_bytes,
                    const float *A, const float *D, rs_stream stream, rs_handle *out);
rs_status rs_destroy(rs_handle h);

/* Replace every checkpoint by `state` (fp32 [B][H][R][Cc], device) -- e.g. the
 * state after a prompt -- derive the low-precision copy from it, and empty the
 * buffer (head = tail = 0); error words are cleared.  With shared_lowp the
 * state is quantised straight into the copy. */
rs_status rs_load_checkpoint(rs_handle h, const float *state, rs_stream stream);

/* Append T >= 1 inputs per sequence at the tail of its ring ("ReplaySSM for
 * hybrid SSM-Transformer stacks", How ReplaySSM works, step 2: append the new
 * SSM input to the buffer).  A sequence whose len + T would exceed cap gets
 * RS_SEQ_ERR_OVERFLOW and is left unchanged.  T > cap returns RS_ERR_CAPACITY. */
rs_status rs_append(rs_handle h, const rs_inputs *in, int T, rs_stream stream);

/* Output of the newest buffered input of every sequence, computed from the
 * checkpoint and the buffer without writing any state (Abstract: output
 * computation separated from checkpoint updates; How ReplaySSM works, step 2:
 * no intermediate states are materialised).  Reads the low-precision copy
 * (the fp32 master when copy_dtype is RS_NONE).  y: out_dtype [B][H][R].
 * A sequence with an empty buffer gets zeros and RS_SEQ_ERR_EMPTY. */
rs_status rs_decode_outputs(rs_handle h, void *y, rs_stream stream);

/* One decode step in two kernels: append T >= 1 inputs per sequence (as
 * rs_append) and compute the outputs at those T newest positions (as
 * rs_verify_outputs with npos = T); T <= npos_max.  T = 1 is a plain decode
 * step, y: out_dtype [B][H][R]; T > 1 verifies T speculative positions,
 * y: [T][B][H][R].  The new inputs are read once, straight from `in`, and
 * written into the ring by the same kernel that prepares the replay.  A
 * sequence whose buffer would overflow is left unchanged, gets zeros and
 * RS_SEQ_ERR_OVERFLOW. */
rs_status rs_decode_step(rs_handle h, const rs_inputs *in, int T, void *y, rs_stream stream);

/* Commit (How ReplaySSM works, step 3): for every sequence with
 * len >= max(min_len, 1) and, when mask is not NULL, mask[b] != 0 (int32 [B],
 * device), apply the recurrence from the fp32 master across the buffered
 * inputs, write the new master and re-derive the copy from it (step 5: the
 * master is never derived from the copy), then empty the buffer (head = tail).
 * With shared_lowp the fold starts from the dequantised copy instead. */
rs_status rs_commit(rs_handle h, int min_len, const int32_t *mask, rs_stream stream);

/* Output-only verification (Abstract; How ReplaySSM works, step 4): outputs at
 * the newest npos buffered positions of every sequence from one pass over the
 * checkpoint, without materialising intermediate states.  1 <= npos <= npos_max.
 * y: out_dtype [npos][B][H][R], position 0 the oldest of the npos.  A sequence
 * with len < npos gets zeros and RS_SEQ_ERR_EMPTY. */
rs_status rs_verify_outputs(rs_handle h, int npos, void *y, rs_stream stream);

/* Pointer-only rollback (How ReplaySSM works, step 4: move the buffer tail back
 * by k entries; the checkpoint never changes).  k: int32 [B], device.  A
 * sequence with k outside [0, len] gets RS_SEQ_ERR_ROLLBACK and is unchanged. */
rs_status rs_rollback(rs_handle h, const int32_t *k, rs_stream stream);

/* Eager read-modify-write baseline ("What ReplaySSM is solving": read the whole
 * state, update it, write it back, every step).  Applies T >= 1 steps of the
 * recurrence to `state` (state_dtype RS_F32 or RS_BF16, [B][H][R][Cc], device,
 * caller-owned, independent of the handle's checkpoints) and writes the output
 * of every step, y: out_dtype [T][B][H][R].  Uses the handle's shapes, A, D,
 * gdn_scale.  Also serves as the prompt (prefill) pass before rs_load_checkpoint. */
rs_status rs_eager_step(rs_handle h, void *state, int state_dtype, const rs_inputs *in, int T,
                        void *y, rs_stream stream);

/* Eager speculative baseline: for npos positions, read the state once from
 * slot cur[b] of `slots` (state_dtype [npos_max + 1][B][H][R][Cc]), apply the
 * npos updates in order, write each intermediate state to slot
 * (cur[b] + 1 + p) mod (npos_max + 1) and each output to y [npos][B][H][R].
 * rs_eager_accept then makes the state after keep[b] positions current:
 * cur[b] = (cur[b] + keep[b]) mod (npos_max + 1); keep outside [0, npos_max]
 * sets RS_SEQ_ERR_ROLLBACK.  cur, keep: int32 [B], device. */
rs_status rs_eager_verify(rs_handle h, void *slots, int state_dtype, const int32_t *cur,
                          const rs_inputs *in, int npos, void *y, rs_stream stream);
rs_status rs_eager_accept(rs_handle h, int32_t *cur, const int32_t *keep, rs_stream stream);

/* Synchronises `stream`, then copies the per-sequence error words to
 * seq_flags_host (uint32 [B], host, may be NULL) and their OR to *any_host
 * (may be NULL).  Returns RS_ERR_DEVICE_FLAG when any bit is set. */
rs_status rs_get_error(rs_handle h, uint32_t *seq_flags_host, uint32_t *any_host,
                       rs_stream stream);
rs_status rs_clear_error(rs_handle h, rs_stream stream);

/* Synchronises `stream`, then copies head / tail (int32 [B] each, host; either
 * may be NULL).  head is the position of the checkpoint, tail one past the
 * newest buffered input; both only grow except that rollback lowers tail. */
rs_status rs_read_ptrs(rs_handle h, int32_t *head_host, int32_t *tail_host, rs_stream stream);

/* Diagnostics. */
const char *rs_status_string(int status);
const char *rs_last_cuda_error(void);     /* text of the last failing CUDA call */
uint64_t rs_launch_count(void);           /* kernels launched by this library so far */

/* Failure-detection check, no handle needed: one device thread waits, with
 * the bounded wait every on-device wait of the library uses, on a barrier
 * phase that nothing completes, gives up after limit_cycles (1 .. the
 * library's own limit, 2e9 cycles) and writes, into result (device, uint32
 * [3]): RS_SEQ_ERR_TIMEOUT, then the cycles it waited (low, high words).  The
 * context stays usable.  RS_ERR_ARG for a NULL result or a limit out of range. */
rs_status rs_selftest_bounded_wait(uint32_t *result, long long limit_cycles, rs_stream stream);

/* Kernel timing of the output calls (rs_decode_outputs, rs_verify_outputs,
 * rs_decode_step), which each run a small prep kernel and one streaming
 * kernel.  rs_profile_start creates CUDA events for the next `max_calls`
 * output calls of this handle (1..2^20; later calls are not timed);
 * rs_profile_stop waits for them and returns the number of timed calls and
 * the summed device time (ms) of the prep kernels and of the streaming
 * kernels, then frees the events.  Either output pointer may be NULL.  Not
 * thread-safe with concurrent calls on the same handle. */
rs_status rs_profile_start(rs_handle h, int max_calls);
rs_status rs_profile_stop(rs_handle h, int *calls, float *prep_ms, float *stream_ms);

/* rs_decode_outputs with its replay records kept in a fixed library-owned
 * device array instead of the workspace's scratch region.  The pages have no
 * counterpart to this call: it exists for callers that must not size or
 * provide scratch memory.  The array holds RS_STATIC_SCRATCH_BYTES; a handle
 * whose records need more (rs_layout.scratch_bytes) gets RS_ERR_CAPACITY and
 * nothing is launched.  No device memory is allocated or freed.  The array is
 * shared by every handle of the process on a device, so calls that may overlap
 * in time (other streams, other host threads) race; calls ordered on one
 * stream do not.  Results equal rs_decode_outputs bit for bit. */
#define RS_STATIC_SCRATCH_BYTES (16u << 20)
rs_status rs_decode_outputs_static_scratch(rs_handle h, void *y, rs_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* RS_H */
