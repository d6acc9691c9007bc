// C interface of the ReplaySSM decode library: configuration checks, workspace
// layout, handle bookkeeping and kernel dispatch.  See include/rs.h for the
// contract of every entry point.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include <cuda.h>

#include "launch.h"
#include "outputs.cuh"
#include "regtile.cuh"

namespace {

std::atomic<uint64_t> g_launches{0};
thread_local char g_cuda_err[256] = "";

rs_status cuda_fail(cudaError_t e, const char *where) {
    std::snprintf(g_cuda_err, sizeof g_cuda_err, "%s: %s", where, cudaGetErrorString(e));
    return RS_ERR_CUDA;
}

rs_status launched(cudaError_t e, const char *where, int n = 1) {
    if (e != cudaSuccess) return cuda_fail(e, where);
    g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed);
    return RS_OK;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

int elem_bytes(int dt) { return dt == RS_BF16 ? 2 : dt == RS_E4M3 ? 1 : 4; }

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Largest per-thread register tile the state-rewriting kernels hold: rows per
// pass is 256 / min(8, CC / 4); each thread keeps ceil(R / rows-per-pass) rows
// of 4 * (CC / 4 / min(8, CC / 4)) floats.
bool regtile_fits(int R, int CC) {
    const int tpr = (CC / 4) < 8 ? CC / 4 : 8;
    const int rpb = rs::kTileThreads / tpr;
    const int np = (R + rpb - 1) / rpb;
    const int ne = CC / tpr;
    if (np > 8) return false;
    const int npr = np <= 1 ? 1 : np <= 2 ? 2 : np <= 4 ? 4 : 8;
    if (npr == 4 && CC > 128) return false;
    if (npr == 8 && CC > 64) return false;
    return npr * ne <= 64;
}

rs_status check_config(const rs_config *c) {
    if (!c) return RS_ERR_ARG;
    if (c->kind != RS_MAMBA2 && c->kind != RS_GDN) return RS_ERR_ARG;
    if (c->batch < 1 || c->nheads < 1 || c->headdim < 1 || c->headdim > 256) return RS_ERR_ARG;
    if (c->dstate != 16 && c->dstate != 32 && c->dstate != 64 && c->dstate != 128 && c->dstate != 256)
        return RS_ERR_ARG;
    if (c->kind == RS_MAMBA2 && (c->ngroups < 1 || c->nheads % c->ngroups != 0)) return RS_ERR_ARG;
    if (c->kind == RS_GDN && c->ngroups != 1) return RS_ERR_ARG;
    if (!pow2(c->cap) || c->cap > 256) return RS_ERR_ARG;
    if (c->npos_max < 1 || c->npos_max > 8 || c->npos_max > c->cap) return RS_ERR_ARG;
    if (c->in_dtype != RS_F32 && c->in_dtype != RS_BF16) return RS_ERR_ARG;
    if (c->copy_dtype != RS_NONE && c->copy_dtype != RS_BF16 && c->copy_dtype != RS_E4M3) return RS_ERR_ARG;
    if (c->out_dtype != RS_F32 && c->out_dtype != RS_BF16) return RS_ERR_ARG;
    if (c->shared_lowp != 0 && c->shared_lowp != 1) return RS_ERR_ARG;
    if (c->shared_lowp && c->copy_dtype == RS_NONE) return RS_ERR_ARG;
    if (c->gdn_scale < 0.f || c->gdn_scale != c->gdn_scale) return RS_ERR_ARG;
    if (!regtile_fits(c->headdim, c->dstate)) return RS_ERR_UNSUPPORTED;
    if ((size_t)c->batch * c->nheads > 0x7fffffffull) return RS_ERR_UNSUPPORTED;
    return RS_OK;
}

rs_status make_layout(const rs_config *c, rs_layout *L) {
    rs_status s = check_config(c);
    if (s != RS_OK) return s;
    std::memset(L, 0, sizeof *L);
    const size_t B = c->batch, H = c->nheads, R = c->headdim, CC = c->dstate, G = c->ngroups;
    const size_t cap = c->cap, E = B * H * R * CC, ib = elem_bytes(c->in_dtype);
    size_t o = 0;
    auto put = [&](size_t &off, size_t &sz, size_t bytes) {
        off = o;
        sz = bytes;
        o = align256(o + bytes);
    };
    put(L->master, L->master_bytes, c->shared_lowp ? 0 : 4 * E);
    put(L->copy, L->copy_bytes, c->copy_dtype == RS_NONE ? 0 : E * elem_bytes(c->copy_dtype));
    put(L->scale, L->scale_bytes, c->copy_dtype == RS_E4M3 ? 4 * B * H : 0);
    const size_t capd = cap < 4 ? 4 : cap;
    const size_t blk_r = (cap * R * ib + 15) / 16 * 16;   // x / v block per (b, h)
    const size_t blk_c = cap * CC * ib;                   // q / k block per (b, h), B / C per (b, g)
    if (c->kind == RS_MAMBA2) {
        put(L->ring_a, L->ring_a_bytes, B * H * blk_r);
        put(L->ring_b, L->ring_b_bytes, 4 * B * H * capd);
        put(L->ring_c, L->ring_c_bytes, B * G * blk_c);
        put(L->ring_d, L->ring_d_bytes, B * G * blk_c);
        put(L->ring_e, L->ring_e_bytes, 0);
    } else {
        put(L->ring_a, L->ring_a_bytes, B * H * blk_c);
        put(L->ring_b, L->ring_b_bytes, B * H * blk_c);
        put(L->ring_c, L->ring_c_bytes, B * H * blk_r);
        put(L->ring_d, L->ring_d_bytes, 4 * B * H * capd);
        put(L->ring_e, L->ring_e_bytes, 4 * B * H * capd);
    }
    size_t dummy;
    put(L->head, dummy, 4 * B);
    put(L->tail, dummy, 4 * B);
    put(L->err, dummy, 4 * B);
    put(L->arrive, dummy, 4 * B);
    put(L->scratch, L->scratch_bytes,
        4 * rs::scratch_floats(c->kind, c->batch, c->nheads, c->ngroups, c->npos_max, c->cap, c->dstate));
    L->total = o;
    return RS_OK;
}

bool aligned(const void *ptr, uintptr_t n) { return (reinterpret_cast<uintptr_t>(ptr) & (n - 1)) == 0; }

// All inputs of the layer kind present and aligned: fp32 arrays to 4 bytes,
// activations to their element size, and Mamba-2's B and C to 16 bytes (their
// rows are read in 16-byte pieces).
bool has_inputs(int kind, int in_dtype, const rs_inputs *in) {
    if (!in) return false;
    const uintptr_t eb = in_dtype == RS_BF16 ? 2 : 4;
    if (kind == RS_MAMBA2)
        return in->x && in->dt && in->B && in->C && aligned(in->x, eb) && aligned(in->dt, 4) &&
               aligned(in->B, 16) && aligned(in->C, 16);
    return in->q && in->k && in->v && in->alpha && in->beta && aligned(in->q, eb) && aligned(in->k, eb) &&
           aligned(in->v, eb) && aligned(in->alpha, 4) && aligned(in->beta, 4);
}

}  // namespace

struct rs_ctx {
    alignas(64) unsigned char state_map[128];   // CUtensorMap of the checkpoint the outputs read
    rs_config cfg;
    rs_layout lay;
    rs::Params p;
    int device;
    // profiling: three events (before prep, between prep and stream, after stream) per output call
    std::vector<cudaEvent_t> prof;
    int prof_max = 0, prof_n = 0;
};

namespace {

cudaEvent_t *prof_slot(rs_ctx *h) {
    if (h->prof_n < h->prof_max) return &h->prof[3 * (h->prof_n++)];
    return nullptr;
}

void prof_release(rs_ctx *h) {
    for (cudaEvent_t e : h->prof) cudaEventDestroy(e);
    h->prof.clear();
    h->prof_max = h->prof_n = 0;
}

}  // namespace

extern "C" {

rs_status rs_workspace_layout(const rs_config *cfg, rs_layout *layout) {
    if (!layout) return RS_ERR_ARG;
    return make_layout(cfg, layout);
}

rs_status rs_workspace_size(const rs_config *cfg, size_t *bytes) {
    if (!bytes) return RS_ERR_ARG;
    rs_layout L;
    rs_status s = make_layout(cfg, &L);
    if (s == RS_OK) *bytes = L.total;
    return s;
}

rs_status rs_create(const rs_config *cfg, void *workspace, size_t workspace_bytes, const float *A,
                    const float *D, rs_stream stream, rs_handle *out) {
    if (!out) return RS_ERR_ARG;
    *out = nullptr;
    rs_layout L;
    rs_status s = make_layout(cfg, &L);
    if (s != RS_OK) return s;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || workspace_bytes < L.total)
        return RS_ERR_WORKSPACE;
    if (cfg->kind == RS_MAMBA2 && !A) return RS_ERR_ARG;

    rs_ctx *h = new (std::nothrow) rs_ctx;
    if (!h) return RS_ERR_ARG;
    h->cfg = *cfg;
    if (h->cfg.gdn_scale == 0.f) h->cfg.gdn_scale = 1.f;
    h->lay = L;
    char *ws = static_cast<char *>(workspace);
    rs::Params &p = h->p;
    std::memset(&p, 0, sizeof p);
    p.kind = cfg->kind;
    p.B = cfg->batch;
    p.H = cfg->nheads;
    p.R = cfg->headdim;
    p.CC = cfg->dstate;
    p.G = cfg->kind == RS_MAMBA2 ? cfg->ngroups : 1;
    p.heads_per_group = p.H / p.G;
    p.cap = cfg->cap;
    p.cap_mask = cfg->cap - 1;
    p.capd = cfg->cap < 4 ? 4 : cfg->cap;
    {
        const int ib = elem_bytes(cfg->in_dtype);
        p.blk_r = ((size_t)cfg->cap * cfg->headdim * ib + 15) / 16 * 16;
        p.blk_c = (size_t)cfg->cap * cfg->dstate * ib;
    }
    p.in_dtype = cfg->in_dtype;
    p.out_dtype = cfg->out_dtype;
    p.copy_dtype = cfg->copy_dtype;
    p.shared_lowp = cfg->shared_lowp;
    p.gdn_scale = h->cfg.gdn_scale;
    p.master = L.master_bytes ? reinterpret_cast<float *>(ws + L.master) : nullptr;
    p.copy = L.copy_bytes ? ws + L.copy : nullptr;
    p.scale = L.scale_bytes ? reinterpret_cast<float *>(ws + L.scale) : nullptr;
    p.ra = ws + L.ring_a;
    p.rb = ws + L.ring_b;
    p.rc = ws + L.ring_c;
    p.rd = ws + L.ring_d;
    p.re = L.ring_e_bytes ? ws + L.ring_e : nullptr;
    p.head = reinterpret_cast<int32_t *>(ws + L.head);
    p.tail = reinterpret_cast<int32_t *>(ws + L.tail);
    p.err = reinterpret_cast<uint32_t *>(ws + L.err);
    p.arrive = reinterpret_cast<uint32_t *>(ws + L.arrive);
    p.A = A;
    p.D = D;
    p.rec = reinterpret_cast<float *>(ws + L.scratch);
    p.rec_tile_off = cfg->kind == RS_MAMBA2
                         ? (size_t)p.B * p.G * rs::group_rec_floats(rs::prep_np(cfg->npos_max), p.CC)
                         : 0;

    cudaError_t e = cudaGetDevice(&h->device);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "cudaGetDevice"); }
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "cudaDeviceGetAttribute"); }
    size_t need = cfg->kind == RS_MAMBA2 ? rs::m2_commit_smem(p) : rs::gdn_commit_smem(p);
    for (int np = 1; np <= cfg->npos_max; ++np) {   // every output-position count a call may use
        const size_t a = rs::stream_outputs_smem(p, np), b = rs::prep_smem(p, rs::prep_np(np));
        need = a > need ? a : need;
        need = b > need ? b : need;
    }
    if (need > (size_t)optin) {
        delete h;
        return RS_ERR_UNSUPPORTED;
    }
    static_assert(sizeof(CUtensorMap) == sizeof(h->state_map), "tensor map storage");
    e = rs::make_state_map(p, h->state_map);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "cuTensorMapEncodeTiled"); }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = cudaMemsetAsync(workspace, 0, L.total, st);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "cudaMemsetAsync"); }
    if (p.copy_dtype == RS_E4M3) {
        s = launched(rs::launch_init(p, st), "init");
        if (s != RS_OK) { delete h; return s; }
    }
    *out = h;
    return RS_OK;
}

rs_status rs_destroy(rs_handle h) {
    if (h) prof_release(h);
    delete h;
    return RS_OK;
}

rs_status rs_profile_start(rs_handle h, int max_calls) {
    if (!h || max_calls < 1 || max_calls > (1 << 20)) return RS_ERR_ARG;
    prof_release(h);
    h->prof.resize(3 * (size_t)max_calls);
    for (size_t i = 0; i < h->prof.size(); ++i) {
        cudaError_t e = cudaEventCreate(&h->prof[i]);
        if (e != cudaSuccess) {
            h->prof.resize(i);
            prof_release(h);
            return cuda_fail(e, "cudaEventCreate");
        }
    }
    h->prof_max = max_calls;
    h->prof_n = 0;
    return RS_OK;
}

rs_status rs_profile_stop(rs_handle h, int *calls, float *prep_ms, float *stream_ms) {
    if (!h) return RS_ERR_ARG;
    float tp = 0.f, ts = 0.f;
    for (int c = 0; c < h->prof_n; ++c) {
        cudaEvent_t *ev = &h->prof[3 * (size_t)c];
        cudaError_t e = cudaEventSynchronize(ev[2]);
        float a = 0.f, b = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&a, ev[0], ev[1]);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&b, ev[1], ev[2]);
        if (e != cudaSuccess) {
            prof_release(h);
            return cuda_fail(e, "profile events");
        }
        tp += a;
        ts += b;
    }
    if (calls) *calls = h->prof_n;
    if (prep_ms) *prep_ms = tp;
    if (stream_ms) *stream_ms = ts;
    prof_release(h);
    return RS_OK;
}

rs_status rs_load_checkpoint(rs_handle h, const float *state, rs_stream stream) {
    if (!h || !state) return RS_ERR_ARG;
    return launched(rs::launch_load_checkpoint(h->p, state, static_cast<cudaStream_t>(stream)),
                    "load_checkpoint");
}

rs_status rs_append(rs_handle h, const rs_inputs *in, int T, rs_stream stream) {
    if (!h || !has_inputs(h->cfg.kind, h->cfg.in_dtype, in)) return RS_ERR_ARG;
    if (T < 1) return RS_ERR_ARG;
    if (T > h->cfg.cap) return RS_ERR_CAPACITY;
    return launched(rs::launch_append(h->p, *in, T, static_cast<cudaStream_t>(stream)), "append");
}

static rs_status outputs(rs_handle h, int npos, void *y, rs_stream stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const rs_inputs none{};
    return launched(rs::launch_outputs(h->p, h->state_map, npos, 0, none, y, st, prof_slot(h)), "outputs", 2);
}

rs_status rs_decode_outputs(rs_handle h, void *y, rs_stream stream) {
    if (!h || !y) return RS_ERR_ARG;
    return outputs(h, 1, y, stream);
}

rs_status rs_decode_step(rs_handle h, const rs_inputs *in, int T, void *y, rs_stream stream) {
    if (!h || !y || !has_inputs(h->cfg.kind, h->cfg.in_dtype, in)) return RS_ERR_ARG;
    if (T < 1) return RS_ERR_ARG;
    if (T > h->cfg.npos_max || T > h->cfg.cap) return RS_ERR_CAPACITY;
    return launched(rs::launch_outputs(h->p, h->state_map, T, T, *in, y, static_cast<cudaStream_t>(stream), prof_slot(h)),
                    "decode_step", 2);
}

namespace {

// Replay records of rs_decode_outputs_static_scratch: a fixed device array, its
// address looked up once per device.
__device__ __align__(256) float g_static_scratch[RS_STATIC_SCRATCH_BYTES / sizeof(float)];
std::atomic<float *> g_static_scratch_ptr[64];

}  // namespace

rs_status rs_decode_outputs_static_scratch(rs_handle h, void *y, rs_stream stream) {
    if (!h || !y) return RS_ERR_ARG;
    if (h->lay.scratch_bytes > RS_STATIC_SCRATCH_BYTES) return RS_ERR_CAPACITY;
    if (h->device < 0 || h->device >= 64) return RS_ERR_UNSUPPORTED;
    int cur = -1;
    const cudaError_t ce = cudaGetDevice(&cur);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
    if (cur != h->device) return RS_ERR_ARG;   // the array's address is per device
    float *rec = g_static_scratch_ptr[h->device].load();
    if (!rec) {
        void *addr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&addr, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        rec = static_cast<float *>(addr);
        g_static_scratch_ptr[h->device].store(rec);
    }
    rs::Params p = h->p;   // the handle's parameters with the records moved
    p.rec = rec;
    const rs_inputs none{};
    return launched(rs::launch_outputs(p, h->state_map, 1, 0, none, y, static_cast<cudaStream_t>(stream)),
                    "outputs_static_scratch", 2);
}

rs_status rs_selftest_bounded_wait(uint32_t *result, long long limit_cycles, rs_stream stream) {
    if (!result || limit_cycles < 1 || limit_cycles > rs::kWaitLimitCycles) return RS_ERR_ARG;
    return launched(rs::launch_wait_selftest(result, limit_cycles, static_cast<cudaStream_t>(stream)),
                    "selftest_bounded_wait");
}

rs_status rs_verify_outputs(rs_handle h, int npos, void *y, rs_stream stream) {
    if (!h || !y) return RS_ERR_ARG;
    if (npos < 1 || npos > h->cfg.npos_max) return RS_ERR_CAPACITY;
    return outputs(h, npos, y, stream);
}

rs_status rs_commit(rs_handle h, int min_len, const int32_t *mask, rs_stream stream) {
    if (!h) return RS_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h->cfg.kind == RS_MAMBA2) return launched(rs::launch_m2_commit(h->p, min_len, mask, st), "m2_commit");
    return launched(rs::launch_gdn_commit(h->p, min_len, mask, st), "gdn_commit");
}

rs_status rs_rollback(rs_handle h, const int32_t *k, rs_stream stream) {
    if (!h || !k) return RS_ERR_ARG;
    return launched(rs::launch_rollback(h->p, k, static_cast<cudaStream_t>(stream)), "rollback");
}

static rs_status eager(rs_handle h, void *state, int sdt, const rs_inputs *in, int T, void *y,
                       const int32_t *cur, int nslots, rs_stream stream) {
    if (!h || !state || !y || !has_inputs(h->cfg.kind, h->cfg.in_dtype, in) || T < 1) return RS_ERR_ARG;
    if (sdt != RS_F32 && sdt != RS_BF16) return RS_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h->cfg.kind == RS_MAMBA2)
        return launched(rs::launch_m2_eager(h->p, state, sdt, *in, T, y, cur, nslots, st), "m2_eager");
    return launched(rs::launch_gdn_eager(h->p, state, sdt, *in, T, y, cur, nslots, st), "gdn_eager");
}

rs_status rs_eager_step(rs_handle h, void *state, int state_dtype, const rs_inputs *in, int T,
                        void *y, rs_stream stream) {
    return eager(h, state, state_dtype, in, T, y, nullptr, 1, stream);
}

rs_status rs_eager_verify(rs_handle h, void *slots, int state_dtype, const int32_t *cur,
                          const rs_inputs *in, int npos, void *y, rs_stream stream) {
    if (!h || !cur) return RS_ERR_ARG;
    if (npos < 1 || npos > h->cfg.npos_max) return RS_ERR_CAPACITY;
    return eager(h, slots, state_dtype, in, npos, y, cur, h->cfg.npos_max + 1, stream);
}

rs_status rs_eager_accept(rs_handle h, int32_t *cur, const int32_t *keep, rs_stream stream) {
    if (!h || !cur || !keep) return RS_ERR_ARG;
    return launched(rs::launch_eager_accept(h->p, cur, keep, h->cfg.npos_max + 1,
                                            static_cast<cudaStream_t>(stream)),
                    "eager_accept");
}

rs_status rs_get_error(rs_handle h, uint32_t *seq_flags_host, uint32_t *any_host, rs_stream stream) {
    if (!h) return RS_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::vector<uint32_t> tmp;
    uint32_t *dst = seq_flags_host;
    if (!dst) {
        tmp.resize(h->p.B);
        dst = tmp.data();
    }
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    e = cudaMemcpy(dst, h->p.err, sizeof(uint32_t) * h->p.B, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
    uint32_t any = 0;
    for (int b = 0; b < h->p.B; ++b) any |= dst[b];
    if (any_host) *any_host = any;
    return any ? RS_ERR_DEVICE_FLAG : RS_OK;
}

rs_status rs_clear_error(rs_handle h, rs_stream stream) {
    if (!h) return RS_ERR_ARG;
    cudaError_t e = cudaMemsetAsync(h->p.err, 0, sizeof(uint32_t) * h->p.B, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RS_OK : cuda_fail(e, "cudaMemsetAsync");
}

rs_status rs_read_ptrs(rs_handle h, int32_t *head_host, int32_t *tail_host, rs_stream stream) {
    if (!h) return RS_ERR_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    if (head_host) {
        e = cudaMemcpy(head_host, h->p.head, sizeof(int32_t) * h->p.B, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
    }
    if (tail_host) {
        e = cudaMemcpy(tail_host, h->p.tail, sizeof(int32_t) * h->p.B, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
    }
    return RS_OK;
}

const char *rs_status_string(int status) {
    switch (status) {
        case RS_OK: return "ok";
        case RS_ERR_ARG: return "invalid argument";
        case RS_ERR_CAPACITY: return "exceeds ring capacity";
        case RS_ERR_CUDA: return "CUDA error";
        case RS_ERR_WORKSPACE: return "bad workspace";
        case RS_ERR_DEVICE_FLAG: return "a sequence has a sticky device error";
        case RS_ERR_UNSUPPORTED: return "unsupported configuration";
        default: return "unknown status";
    }
}

const char *rs_last_cuda_error(void) { return g_cuda_err; }

uint64_t rs_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
