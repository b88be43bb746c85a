// Host side of the C ABI: buffer sizes, argument checks and the attention
// entry points (stages 6-7), which pick the kernel family for the dtype.
#include <atomic>

#include "common.cuh"
#include "ds_handoff.cuh"

namespace prism {
size_t zone_indicator_ws_bytes(const Dims& d);
prism_status_t attn_fwd_sm100(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const uint32_t* gsel,
                              float scale, void* Op, float* lse, float* o_f32, uint32_t* dev_status, void* ws,
                              cudaStream_t s);
size_t attn_fwd_sm100_ws_bytes(const Dims& d);
size_t attn_fwd_raster_ws_bytes(const Dims& d);
prism_status_t attn_fwd_raster(const Dims& d, const void* Q, const void* K, const void* V, const int32_t* perm,
                               const uint8_t* shape_id, const uint32_t* gsel, float scale, void* O, float* lse,
                               float* o_f32, uint32_t* dev_status, void* ws, cudaStream_t s);
prism_status_t attn_bwd_sm100(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* Op,
                              const float* o_f32, const void* dOp, const float* lse, const uint32_t* gsel,
                              const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp,
                              uint32_t* dev_status, void* ws, cudaStream_t s, void* ds, size_t ds_bytes);
size_t attn_bwd_sm100_ws_bytes(const Dims& d);
size_t attn_bwd_ds_bytes(const Dims& d, int64_t pieces);
prism_status_t attn_bwd_raster(const Dims& d, const void* Q, const void* K, const void* V, const float* o_f32,
                               const void* dO, const float* lse, const int32_t* perm, const uint8_t* shape_id,
                               const uint32_t* gsel, const uint32_t* gselT, float scale, void* dQ, void* dK, void* dV,
                               uint32_t* dev_status, void* ws, cudaStream_t s, void* ds, size_t ds_bytes);
prism_status_t attn_fwd_simt(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const uint32_t* gsel,
                             float scale, void* Op, float* lse, float* o_f32, cudaStream_t s);
prism_status_t attn_bwd_simt(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* Op,
                             const float* o_f32, const void* dOp, const float* lse, const uint32_t* gsel,
                             const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp, float* delta,
                             cudaStream_t s);

static std::atomic<unsigned long long> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// bf16: enough for either entry point (the raster one adds the per-granule positions)
size_t attn_fwd_ws_bytes(const Dims& d) { return d.dtype == PRISM_BF16 ? attn_fwd_raster_ws_bytes(d) : 0; }
size_t attn_bwd_ws_bytes(const Dims& d) {
    return d.dtype == PRISM_BF16 ? attn_bwd_sm100_ws_bytes(d) : (size_t)d.heads * d.N * sizeof(float);
}
}  // namespace prism

using namespace prism;

extern "C" prism_status_t prism_query_sizes(const prism_problem_t* prob, prism_sizes_t* sizes) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!sizes) return PRISM_ERR_INVALID_ARG;
    sizes->n_tokens = d.N;
    sizes->n_zones = d.Z;
    sizes->max_blocks = d.MB;
    sizes->sel_words = d.SW;
    sizes->ws_indicator = zone_indicator_ws_bytes(d);
    sizes->ws_attn_fwd = attn_fwd_ws_bytes(d);
    sizes->ws_attn_bwd = attn_bwd_ws_bytes(d);
    sizes->bytes_P_max = (size_t)d.heads * d.MB * d.MB * sizeof(float);
    return PRISM_OK;
}

extern "C" prism_status_t prism_sparse_attn_fwd(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                                const void* Vp, const uint32_t* gsel, float scale, void* Op,
                                                float* lse, float* o_f32, uint32_t* dev_status, void* ws,
                                                size_t ws_bytes, cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(Qp) || !ok_ptr(Kp) || !ok_ptr(Vp) || !ok_ptr(gsel) || !ok_ptr(Op) || !ok_opt(lse) ||
        !ok_opt(o_f32) || !ok_ptr(dev_status) || !ok_opt(ws))
        return PRISM_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return PRISM_ERR_INVALID_ARG;
    if (ws_bytes < attn_fwd_ws_bytes(d)) return PRISM_ERR_WORKSPACE;
    if (d.dtype == PRISM_BF16)
        return attn_fwd_sm100(d, Qp, Kp, Vp, gsel, scale, Op, lse, o_f32, dev_status, ws, stream);
    return attn_fwd_simt(d, Qp, Kp, Vp, gsel, scale, Op, lse, o_f32, stream);
}

extern "C" prism_status_t prism_sparse_attn_fwd_raster(const prism_problem_t* prob, const void* Q, const void* K,
                                                       const void* V, const int32_t* perm, const uint8_t* shape_id,
                                                       const uint32_t* gsel, float scale, void* O, float* lse,
                                                       float* o_f32, uint32_t* dev_status, void* ws, size_t ws_bytes,
                                                       cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (d.dtype != PRISM_BF16) return PRISM_ERR_UNSUPPORTED;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(perm) || !ok_ptr(shape_id) || !ok_ptr(gsel) || !ok_ptr(O) ||
        !ok_opt(lse) || !ok_opt(o_f32) || !ok_ptr(dev_status) || !ok_ptr(ws))
        return PRISM_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return PRISM_ERR_INVALID_ARG;
    if (ws_bytes < attn_fwd_raster_ws_bytes(d)) return PRISM_ERR_WORKSPACE;
    return attn_fwd_raster(d, Q, K, V, perm, shape_id, gsel, scale, O, lse, o_f32, dev_status, ws, stream);
}

namespace {
// argument checks shared by the backward entry points; ds == nullptr: no handoff
prism_status_t bwd_blocked(const prism_problem_t* prob, const void* Qp, const void* Kp, const void* Vp,
                           const void* Op, const float* o_f32, const void* dOp, const float* lse,
                           const uint32_t* gsel, const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp,
                           uint32_t* dev_status, void* ws, size_t ws_bytes, void* ds, size_t ds_bytes,
                           cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(Qp) || !ok_ptr(Kp) || !ok_ptr(Vp) || !ok_ptr(Op) || !ok_opt(o_f32) || !ok_ptr(dOp) ||
        !ok_ptr(lse) || !ok_ptr(gsel) || !ok_ptr(gselT) || !ok_ptr(dQp) || !ok_ptr(dKp) || !ok_ptr(dVp) ||
        !ok_ptr(dev_status) || !ok_ptr(ws) || !ok_opt(ds))
        return PRISM_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return PRISM_ERR_INVALID_ARG;
    if (ws_bytes < attn_bwd_ws_bytes(d)) return PRISM_ERR_WORKSPACE;
    if (d.dtype == PRISM_BF16)
        return attn_bwd_sm100(d, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, ws,
                              stream, ds, ds_bytes);
    if (ds) return PRISM_ERR_UNSUPPORTED;
    return attn_bwd_simt(d, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, (float*)ws, stream);
}

prism_status_t bwd_raster(const prism_problem_t* prob, const void* Q, const void* K, const void* V,
                          const float* o_f32, const void* dO, const float* lse, const int32_t* perm,
                          const uint8_t* shape_id, const uint32_t* gsel, const uint32_t* gselT, float scale, void* dQ,
                          void* dK, void* dV, uint32_t* dev_status, void* ws, size_t ws_bytes, void* ds,
                          size_t ds_bytes, cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (d.dtype != PRISM_BF16) return PRISM_ERR_UNSUPPORTED;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(o_f32) || !ok_ptr(dO) || !ok_ptr(lse) || !ok_ptr(perm) ||
        !ok_ptr(shape_id) || !ok_ptr(gsel) || !ok_ptr(gselT) || !ok_ptr(dQ) || !ok_ptr(dK) || !ok_ptr(dV) ||
        !ok_ptr(dev_status) || !ok_ptr(ws) || !ok_opt(ds))
        return PRISM_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return PRISM_ERR_INVALID_ARG;
    if (ws_bytes < attn_bwd_ws_bytes(d)) return PRISM_ERR_WORKSPACE;
    return attn_bwd_raster(d, Q, K, V, o_f32, dO, lse, perm, shape_id, gsel, gselT, scale, dQ, dK, dV, dev_status, ws,
                           stream, ds, ds_bytes);
}
}  // namespace

extern "C" prism_status_t prism_sparse_attn_bwd(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                                const void* Vp, const void* Op, const float* o_f32,
                                                const void* dOp, const float* lse, const uint32_t* gsel,
                                                const uint32_t* gselT, float scale, void* dQp, void* dKp,
                                                void* dVp, uint32_t* dev_status, void* ws, size_t ws_bytes,
                                                cudaStream_t stream) {
    return bwd_blocked(prob, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, ws,
                       ws_bytes, nullptr, 0, stream);
}

extern "C" prism_status_t prism_sparse_attn_bwd_raster(const prism_problem_t* prob, const void* Q, const void* K,
                                                       const void* V, const float* o_f32, const void* dO,
                                                       const float* lse, const int32_t* perm, const uint8_t* shape_id,
                                                       const uint32_t* gsel, const uint32_t* gselT, float scale,
                                                       void* dQ, void* dK, void* dV, uint32_t* dev_status, void* ws,
                                                       size_t ws_bytes, cudaStream_t stream) {
    return bwd_raster(prob, Q, K, V, o_f32, dO, lse, perm, shape_id, gsel, gselT, scale, dQ, dK, dV, dev_status, ws,
                      ws_bytes, nullptr, 0, stream);
}

extern "C" prism_status_t prism_attn_bwd_ds_bytes(const prism_problem_t* prob, int64_t pieces, size_t* bytes) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!bytes || pieces < 1 || pieces > ds::kMaxPieces) return PRISM_ERR_INVALID_ARG;
    *bytes = attn_bwd_ds_bytes(d, pieces);
    return PRISM_OK;
}

extern "C" prism_status_t prism_sparse_attn_bwd_ds(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                                   const void* Vp, const void* Op, const float* o_f32,
                                                   const void* dOp, const float* lse, const uint32_t* gsel,
                                                   const uint32_t* gselT, float scale, void* dQp, void* dKp,
                                                   void* dVp, uint32_t* dev_status, void* ws, size_t ws_bytes,
                                                   void* ds, size_t ds_bytes, cudaStream_t stream) {
    if (!ok_ptr(ds)) return PRISM_ERR_INVALID_ARG;
    return bwd_blocked(prob, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, ws,
                       ws_bytes, ds, ds_bytes, stream);
}

extern "C" prism_status_t prism_sparse_attn_bwd_raster_ds(const prism_problem_t* prob, const void* Q, const void* K,
                                                          const void* V, const float* o_f32, const void* dO,
                                                          const float* lse, const int32_t* perm,
                                                          const uint8_t* shape_id, const uint32_t* gsel,
                                                          const uint32_t* gselT, float scale, void* dQ, void* dK,
                                                          void* dV, uint32_t* dev_status, void* ws, size_t ws_bytes,
                                                          void* ds, size_t ds_bytes, cudaStream_t stream) {
    if (!ok_ptr(ds)) return PRISM_ERR_INVALID_ARG;
    return bwd_raster(prob, Q, K, V, o_f32, dO, lse, perm, shape_id, gsel, gselT, scale, dQ, dK, dV, dev_status, ws,
                      ws_bytes, ds, ds_bytes, stream);
}

extern "C" prism_status_t prism_read_status(const uint32_t* dev_status, uint32_t* host_out, cudaStream_t stream) {
    if (!dev_status || !host_out) return PRISM_ERR_INVALID_ARG;
    if (cudaMemcpyAsync(host_out, dev_status, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return PRISM_ERR_CUDA;
    return cudaStreamSynchronize(stream) == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

extern "C" const char* prism_status_string(prism_status_t s) {
    switch (s) {
        case PRISM_OK: return "ok";
        case PRISM_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad scalar)";
        case PRISM_ERR_SHAPE: return "grid axes must be positive multiples of 8";
        case PRISM_ERR_UNSUPPORTED: return "unsupported dtype, head_dim, heads, audio_dim or size";
        case PRISM_ERR_WORKSPACE: return "workspace too small";
        case PRISM_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

extern "C" const char* prism_version(void) { return "prism-b200 0.1.0 sm_100a"; }

extern "C" unsigned long long prism_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }
