// The whole layer as one object: the call sequence of stages 1-7 over buffers
// carved from one caller-owned arena, and a step that takes host buffers.
//
// The stages are the Prism path in order (Portuguese reading guide, "Método"
// 1-3; news page, "工作原理" step 4: the sparse kernel runs over the permuted
// blocks and the original layout is restored afterwards):
//   forward:  zone indicator (V, hhat) -> shapes + permutation -> permute Q, K, V
//             -> pooled block probabilities -> hybrid selection -> sparse
//             attention -> unpermute O
//   backward: permute dO -> sparse attention backward -> unpermute dQ, dK, dV
// prism_layer_step_host adds the host copies, one cudaMemcpyAsync per tensor,
// on two copy streams: V and hhat first (the indicator needs only them), then
// Q and K, then dO, whose upload overlaps the forward; O downloads while the
// backward runs.  Across calls, the next step's uploads wait only for this
// step's last read of the raster inputs (two events kept in L->io_events), so in
// the blocked layout they overlap this step's attention and its downloads
// (opposite PCIe directions).
#include <math.h>
#include <string.h>

#include "common.cuh"

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t b) { return (b + kAlign - 1) & ~(kAlign - 1); }

// One pass over the buffer list: with base == nullptr it only sums sizes.
size_t carve(prism_layer_t* L, uint8_t* base) {
    prism_sizes_t s;
    prism_query_sizes(&L->prob, &s);
    const int64_t N = s.n_tokens, Z = s.n_zones, MB = s.max_blocks, SW = s.sel_words;
    const int64_t h = L->prob.heads, d = L->prob.head_dim;
    const size_t esz = L->prob.dtype == PRISM_BF16 ? 2 : 4;
    const int64_t pb = L->p_blocks > 0 ? L->p_blocks : MB;
    const bool bwd = L->with_backward != 0, io = L->with_io != 0;
    const bool blocked = !L->raster;                          // raster: no blocked Q, K, V, O
    size_t off = 0;
    auto take = [&](size_t bytes) -> void* {
        void* p = base ? base + off : nullptr;
        off += up(bytes > 0 ? bytes : 1);
        return p;
    };
    const size_t tok = (size_t)N * h * d * esz;          // one token tensor
    L->g = (float*)take(Z * 3 * 4);
    L->rho = (float*)take(Z * 4);
    L->abar = (float*)take(Z * 4);
    L->zone_stats = (float*)take(Z * 8 * 4);
    L->ws_ind_bytes = s.ws_indicator;
    L->ws_ind = take(s.ws_indicator);
    L->shape_id = (uint8_t*)take(Z);
    L->perm = (int32_t*)take(N * 4);
    L->blk_start = (int32_t*)take((MB + 1) * 4);
    L->gran_blk = (int32_t*)take(MB * 4);
    L->n_blk = (int32_t*)take(4);
    L->margin_shape = (float*)take(Z * 2 * 4);
    L->Qp = blocked ? take(tok) : nullptr;
    L->Kp = blocked ? take(tok) : nullptr;
    L->Vp = blocked ? take(tok) : nullptr;
    L->Qbar = (float*)take(h * MB * d * 4);
    L->Kbar = (float*)take(h * MB * d * 4);
    L->P = (float*)take((size_t)h * pb * pb * 4);
    L->sel = (uint32_t*)take(h * MB * SW * 4);
    L->gsel = (uint32_t*)take(h * MB * SW * 4);
    L->gselT = bwd ? (uint32_t*)take(h * MB * SW * 4) : nullptr;
    L->sel_count = (int32_t*)take(h * MB * 4);
    L->margin_sel = (float*)take(h * MB * 4);
    L->dev_status = (uint32_t*)take(4);
    L->Op = blocked ? take(tok) : nullptr;
    L->Of32 = (bwd && L->prob.dtype == PRISM_BF16) ? (float*)take((size_t)N * h * d * 4) : nullptr;
    L->lse = bwd ? (float*)take(N * h * 4) : nullptr;
    L->ws_fwd_bytes = s.ws_attn_fwd;
    L->ws_fwd = take(s.ws_attn_fwd);
    L->dOp = (bwd && blocked) ? take(tok) : nullptr;
    L->dQp = (bwd && blocked) ? take(tok) : nullptr;
    L->dKp = (bwd && blocked) ? take(tok) : nullptr;
    L->dVp = (bwd && blocked) ? take(tok) : nullptr;
    L->ws_bwd_bytes = bwd ? s.ws_attn_bwd : 0;
    L->ws_bwd = bwd ? take(s.ws_attn_bwd) : nullptr;
    const size_t hh_bytes = (size_t)N * L->prob.audio_dim * esz;
    L->Q = io ? take(tok) : nullptr;
    L->K = io ? take(tok) : nullptr;
    L->V = io ? take(tok) : nullptr;
    L->hhat = io ? take(hh_bytes) : nullptr;
    L->O = io ? take(tok) : nullptr;
    L->dO = (io && bwd) ? take(tok) : nullptr;
    L->dQ = (io && bwd) ? take(tok) : nullptr;
    L->dK = (io && bwd) ? take(tok) : nullptr;
    L->dV = (io && bwd) ? take(tok) : nullptr;
    return off;
}

bool params_ok(const prism_layer_t* L) {
    return L->top_k >= 0 && L->top_p > 0.f && isfinite(L->top_p) && L->eps > 0.f && isfinite(L->eps) &&
           L->scale > 0.f && isfinite(L->scale) && L->fixed_shape >= -1 && L->fixed_shape < 16 &&
           L->p_blocks >= 0 && (L->raster == 0 || (L->raster == 1 && L->prob.dtype == PRISM_BF16));
}

#define PRISM_TRY(x)                          \
    do {                                      \
        prism_status_t st_ = (x);             \
        if (st_ != PRISM_OK) return st_;      \
    } while (0)

// inputs_read (nullable): recorded once the raster Q, K, V and hhat have been read
// for the last time in the forward (blocked layout: after the permutes; the
// raster-layout attention reads them until the end of the backward, so then it
// is not recorded here)
prism_status_t run_forward(const prism_layer_t* L, const void* Q, const void* K, const void* V, const void* hhat,
                           void* O, cudaStream_t s, cudaEvent_t qk_ready, cudaEvent_t out_free,
                           cudaEvent_t inputs_read = nullptr) {
    const prism_problem_t* p = &L->prob;
    PRISM_TRY(prism_zone_indicator_ex(p, V, hhat, L->eps, L->guidance, L->g, L->rho, L->abar, L->zone_stats,
                                      L->ws_ind, L->ws_ind_bytes, s));
    PRISM_TRY(prism_assign_shapes_ex(p, L->g, L->rho, L->tau128, L->tau256, L->fixed_shape, L->shape_id, L->perm,
                                     nullptr, L->blk_start, L->gran_blk, L->n_blk, L->margin_shape, s));
    if (L->raster) {
        // the permutation is applied inside the loads and stores: no blocked copies
        if (qk_ready && cudaStreamWaitEvent(s, qk_ready, 0) != cudaSuccess) return PRISM_ERR_CUDA;
        PRISM_TRY(prism_block_pool_score_raster(p, Q, K, L->perm, L->blk_start, L->n_blk, L->scale, L->Qbar, L->Kbar,
                                                L->P, s));
        PRISM_TRY(prism_block_select(p, L->P, L->blk_start, L->gran_blk, L->n_blk, L->top_k, L->top_p, L->sel,
                                     L->sel_count, L->gsel, L->gselT, L->margin_sel, L->dev_status, s));
        if (out_free && cudaStreamWaitEvent(s, out_free, 0) != cudaSuccess) return PRISM_ERR_CUDA;
        return prism_sparse_attn_fwd_raster(p, Q, K, V, L->perm, L->shape_id, L->gsel, L->scale, O, L->lse, L->Of32,
                                            L->dev_status, L->ws_fwd, L->ws_fwd_bytes, s);
    }
    PRISM_TRY(prism_permute(p, V, L->perm, L->Vp, s));
    if (qk_ready && cudaStreamWaitEvent(s, qk_ready, 0) != cudaSuccess) return PRISM_ERR_CUDA;
    PRISM_TRY(prism_permute(p, Q, L->perm, L->Qp, s));
    PRISM_TRY(prism_permute(p, K, L->perm, L->Kp, s));
    if (inputs_read && cudaEventRecord(inputs_read, s) != cudaSuccess) return PRISM_ERR_CUDA;
    PRISM_TRY(prism_block_pool_score(p, L->Qp, L->Kp, L->blk_start, L->n_blk, L->scale, L->Qbar, L->Kbar, L->P, s));
    PRISM_TRY(prism_block_select(p, L->P, L->blk_start, L->gran_blk, L->n_blk, L->top_k, L->top_p, L->sel,
                                 L->sel_count, L->gsel, L->gselT, L->margin_sel, L->dev_status, s));
    PRISM_TRY(prism_sparse_attn_fwd(p, L->Qp, L->Kp, L->Vp, L->gsel, L->scale, L->Op, L->lse, L->Of32,
                                    L->dev_status, L->ws_fwd, L->ws_fwd_bytes, s));
    if (out_free && cudaStreamWaitEvent(s, out_free, 0) != cudaSuccess) return PRISM_ERR_CUDA;
    return prism_unpermute(p, L->Op, L->perm, O, s);
}

// do_read (nullable): recorded once the raster dO has been read for the last time
// (blocked layout: after its permute; raster layout: not recorded here)
prism_status_t run_backward(const prism_layer_t* L, const void* Q, const void* K, const void* V, const void* dO,
                            void* dQ, void* dK, void* dV, cudaStream_t s,
                            cudaEvent_t* done /* [3] nullable: after dQ, dK, dV */, cudaEvent_t do_read = nullptr) {
    const prism_problem_t* p = &L->prob;
    if (L->raster) {
        PRISM_TRY(prism_sparse_attn_bwd_raster(p, Q, K, V, L->Of32, dO, L->lse, L->perm, L->shape_id, L->gsel,
                                               L->gselT, L->scale, dQ, dK, dV, L->dev_status, L->ws_bwd,
                                               L->ws_bwd_bytes, s));
        if (done)
            for (int i = 0; i < 3; ++i)
                if (cudaEventRecord(done[i], s) != cudaSuccess) return PRISM_ERR_CUDA;
        return PRISM_OK;
    }
    PRISM_TRY(prism_permute(p, dO, L->perm, L->dOp, s));
    if (do_read && cudaEventRecord(do_read, s) != cudaSuccess) return PRISM_ERR_CUDA;
    PRISM_TRY(prism_sparse_attn_bwd(p, L->Qp, L->Kp, L->Vp, L->Op, L->Of32, L->dOp, L->lse, L->gsel, L->gselT,
                                    L->scale, L->dQp, L->dKp, L->dVp, L->dev_status, L->ws_bwd, L->ws_bwd_bytes,
                                    s));
    void* outs[3] = {dQ, dK, dV};
    void* srcs[3] = {L->dQp, L->dKp, L->dVp};
    for (int i = 0; i < 3; ++i) {
        PRISM_TRY(prism_unpermute(p, srcs[i], L->perm, outs[i], s));
        if (done && cudaEventRecord(done[i], s) != cudaSuccess) return PRISM_ERR_CUDA;
    }
    return PRISM_OK;
}

}  // namespace

extern "C" prism_status_t prism_layer_init(prism_layer_t* L, const prism_problem_t* prob) {
    if (!L || !prob) return PRISM_ERR_INVALID_ARG;
    prism_sizes_t s;
    PRISM_TRY(prism_query_sizes(prob, &s));
    memset(L, 0, sizeof(*L));
    L->prob = *prob;
    L->top_k = 8;
    L->top_p = 0.9f;
    L->eps = 1e-6f;
    L->tau128 = 0.5f;
    L->tau256 = 0.25f;
    L->scale = 1.f / sqrtf((float)prob->head_dim);
    L->guidance = PRISM_GUIDE_JOINT;
    L->fixed_shape = -1;
    L->with_backward = 1;
    L->with_io = 0;
    L->raster = 0;
    L->p_blocks = 0;
    return PRISM_OK;
}

extern "C" prism_status_t prism_layer_arena_bytes(const prism_layer_t* L, size_t* bytes) {
    if (!L || !bytes) return PRISM_ERR_INVALID_ARG;
    prism_sizes_t s;
    PRISM_TRY(prism_query_sizes(&L->prob, &s));
    if (!params_ok(L) || L->p_blocks > s.max_blocks) return PRISM_ERR_INVALID_ARG;
    prism_layer_t tmp = *L;
    *bytes = carve(&tmp, nullptr);
    return PRISM_OK;
}

extern "C" prism_status_t prism_layer_bind(prism_layer_t* L, void* arena, size_t bytes) {
    size_t need = 0;
    PRISM_TRY(prism_layer_arena_bytes(L, &need));
    if (!arena || (reinterpret_cast<uintptr_t>(arena) & (kAlign - 1))) return PRISM_ERR_INVALID_ARG;
    if (bytes < need) return PRISM_ERR_WORKSPACE;
    carve(L, static_cast<uint8_t*>(arena));
    return PRISM_OK;
}

extern "C" prism_status_t prism_layer_forward(const prism_layer_t* L, const void* Q, const void* K, const void* V,
                                              const void* hhat, void* O, cudaStream_t stream) {
    if (!L || !params_ok(L)) return PRISM_ERR_INVALID_ARG;
    return run_forward(L, Q, K, V, hhat, O, stream, nullptr, nullptr);
}

extern "C" prism_status_t prism_layer_backward(const prism_layer_t* L, const void* Q, const void* K, const void* V,
                                               const void* dO, void* dQ, void* dK, void* dV, cudaStream_t stream) {
    if (!L || !params_ok(L)) return PRISM_ERR_INVALID_ARG;
    if (!L->with_backward) return PRISM_ERR_UNSUPPORTED;
    return run_backward(L, Q, K, V, dO, dQ, dK, dV, stream, nullptr);
}

namespace {
struct Events {
    cudaEvent_t e[10] = {};
    int n = 0;
    ~Events() {
        // destroying an event that is still pending is allowed: it is released once it completes
        for (int i = 0; i < n; ++i) cudaEventDestroy(e[i]);
    }
    bool make(int count) {
        for (; n < count; ++n)
            if (cudaEventCreateWithFlags(&e[n], cudaEventDisableTiming) != cudaSuccess) return false;
        return true;
    }
};

prism_status_t copy(void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, cudaStream_t s) {
    return cudaMemcpyAsync(dst, src, bytes, kind, s) == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}
}  // namespace

namespace {
// The events that carry "the raster inputs have been read" from one host-buffer
// step to the next; created by the first step, kept in L->io_events.
struct IoEvents {
    cudaEvent_t inputs_read = nullptr;   // Q, K, V, hhat
    cudaEvent_t do_read = nullptr;       // dO
};
}  // namespace

extern "C" prism_status_t prism_layer_release(prism_layer_t* L) {
    if (!L) return PRISM_ERR_INVALID_ARG;
    IoEvents* io = static_cast<IoEvents*>(L->io_events);
    if (!io) return PRISM_OK;
    const bool ok = cudaEventDestroy(io->inputs_read) == cudaSuccess && cudaEventDestroy(io->do_read) == cudaSuccess;
    delete io;
    L->io_events = nullptr;
    return ok ? PRISM_OK : PRISM_ERR_CUDA;
}

extern "C" prism_status_t prism_layer_step_host(prism_layer_t* L, const void* hQ, const void* hK,
                                                const void* hV, const void* hhhat, const void* hdO, void* hO,
                                                void* hdQ, void* hdK, void* hdV, cudaStream_t compute,
                                                cudaStream_t h2d, cudaStream_t d2h) {
    if (!L || !params_ok(L) || !L->with_io || !L->Q) return PRISM_ERR_INVALID_ARG;
    const bool bwd = L->with_backward != 0;
    if (!hQ || !hK || !hV || !hhhat || !hO || (bwd && (!hdO || !hdQ || !hdK || !hdV))) return PRISM_ERR_INVALID_ARG;
    if (h2d == compute || d2h == compute || h2d == d2h) return PRISM_ERR_INVALID_ARG;
    prism_sizes_t s;
    PRISM_TRY(prism_query_sizes(&L->prob, &s));
    const size_t esz = L->prob.dtype == PRISM_BF16 ? 2 : 4;
    const size_t tok = (size_t)s.n_tokens * L->prob.heads * L->prob.head_dim * esz;
    const size_t hhb = (size_t)s.n_tokens * L->prob.audio_dim * esz;
    if (!L->io_events) {
        IoEvents* fresh = new IoEvents;
        if (cudaEventCreateWithFlags(&fresh->inputs_read, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&fresh->do_read, cudaEventDisableTiming) != cudaSuccess) {
            if (fresh->inputs_read) cudaEventDestroy(fresh->inputs_read);
            delete fresh;
            return PRISM_ERR_CUDA;
        }
        L->io_events = fresh;
    }
    IoEvents* io = static_cast<IoEvents*>(L->io_events);
    enum { kPrevD2H, kVH, kQK, kDO, kO, kDQ, kDK, kDV, kCount };
    Events ev;
    if (!ev.make(kCount)) return PRISM_ERR_CUDA;
    const cudaMemcpyKind H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;
    // The previous step may still read the raster inputs, and its downloads still
    // read the raster outputs.  Uploads of Q, K, V, hhat wait for its last read of
    // them, the upload of dO for its last read of dO (events the previous call
    // recorded; a never-recorded event counts as complete), and writes of O, dQ,
    // dK, dV wait for its downloads.
    if (cudaEventRecord(ev.e[kPrevD2H], d2h) != cudaSuccess ||
        cudaStreamWaitEvent(h2d, io->inputs_read, 0) != cudaSuccess)
        return PRISM_ERR_CUDA;
    PRISM_TRY(copy(L->V, hV, tok, H2D, h2d));
    PRISM_TRY(copy(L->hhat, hhhat, hhb, H2D, h2d));
    if (cudaEventRecord(ev.e[kVH], h2d) != cudaSuccess) return PRISM_ERR_CUDA;
    PRISM_TRY(copy(L->Q, hQ, tok, H2D, h2d));
    PRISM_TRY(copy(L->K, hK, tok, H2D, h2d));
    if (cudaEventRecord(ev.e[kQK], h2d) != cudaSuccess) return PRISM_ERR_CUDA;
    if (bwd) {
        if (cudaStreamWaitEvent(h2d, io->do_read, 0) != cudaSuccess) return PRISM_ERR_CUDA;
        PRISM_TRY(copy(L->dO, hdO, tok, H2D, h2d));
        if (cudaEventRecord(ev.e[kDO], h2d) != cudaSuccess) return PRISM_ERR_CUDA;
    }
    if (cudaStreamWaitEvent(compute, ev.e[kVH], 0) != cudaSuccess) return PRISM_ERR_CUDA;
    const bool early = !L->raster;             // blocked layout: inputs read by the permutes only
    PRISM_TRY(run_forward(L, L->Q, L->K, L->V, L->hhat, L->O, compute, ev.e[kQK], ev.e[kPrevD2H],
                          early ? io->inputs_read : nullptr));
    if (cudaEventRecord(ev.e[kO], compute) != cudaSuccess || cudaStreamWaitEvent(d2h, ev.e[kO], 0) != cudaSuccess)
        return PRISM_ERR_CUDA;
    PRISM_TRY(copy(hO, L->O, tok, D2H, d2h));
    if (bwd) {
        if (cudaStreamWaitEvent(compute, ev.e[kDO], 0) != cudaSuccess) return PRISM_ERR_CUDA;
        cudaEvent_t done[3] = {ev.e[kDQ], ev.e[kDK], ev.e[kDV]};
        PRISM_TRY(run_backward(L, L->Q, L->K, L->V, L->dO, L->dQ, L->dK, L->dV, compute, done,
                               early ? io->do_read : nullptr));
        void* hs[3] = {hdQ, hdK, hdV};
        void* ds[3] = {L->dQ, L->dK, L->dV};
        for (int i = 0; i < 3; ++i) {
            if (cudaStreamWaitEvent(d2h, done[i], 0) != cudaSuccess) return PRISM_ERR_CUDA;
            PRISM_TRY(copy(hs[i], ds[i], tok, D2H, d2h));
        }
    }
    // raster layout: the inputs are read until the step's compute ends
    if (!early && (cudaEventRecord(io->inputs_read, compute) != cudaSuccess ||
                   cudaEventRecord(io->do_read, compute) != cudaSuccess))
        return PRISM_ERR_CUDA;
    // no join here: all of the step's device work precedes its last download, so
    // the d2h stream marks completion, and the next step's uploads can overlap
    // this step's downloads
    return PRISM_OK;
}

extern "C" size_t prism_layer_sizeof(void) { return sizeof(prism_layer_t); }
