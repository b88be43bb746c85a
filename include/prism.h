/*
 * prism.h — C ABI of the B200 (sm_100a) implementation of Prism's dynamic,
 * content-adaptive block-sparse video self-attention.
 *
 * Source of the operations: "Prism: Dynamic Sparse Attention for Native 2K
 * Joint Video-Audio Generation Model Training" (arXiv 2610.05416).  Section
 * names below refer to its Portuguese reading guide ("Método" 1-3, "Ideias
 * centrais"), its Chinese reading guide (FAQ) and the sd114.wiki news page
 * ("工作原理", how it works).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument except `prob`, `sizes` and `host_out` is a DEVICE
 *    pointer, 16-byte aligned.  The caller allocates and owns every buffer
 *    (sizes from prism_query_sizes); the library allocates nothing and keeps
 *    no state between calls.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream).
 *    Data-dependent counts (the number of blocks n_blk, selection counts)
 *    stay in device memory; no call synchronises except prism_read_status.
 *  - Argument and shape errors are returned before any launch, and then no
 *    output is touched.  A failed launch returns PRISM_ERR_CUDA.  Conditions
 *    only the device can see set bits in `dev_status` (PRISM_DEV_*); kernels
 *    then return early instead of trapping.  No C++ exception crosses the ABI.
 *  - Supported: dtype PRISM_F32 or PRISM_BF16, head_dim 64 or 128,
 *    1 <= heads <= 64, even audio_dim <= 1024, T, H, W positive multiples of
 *    8 with N = T*H*W <= 2^24.  Anything else -> PRISM_ERR_UNSUPPORTED or
 *    PRISM_ERR_SHAPE.
 *
 * Notation: N = T*H*W tokens, raster token index r = (t*H + h)*W + w;
 * Z = N/512 macro-zones of 8x8x8 tokens in raster zone order; D = heads*head_dim.
 * Layouts (batch 1):
 *    raster  [N][heads][head_dim]   (Q, K, V, O, dO, dQ, dK, dV as a DiT holds them)
 *    blocked [heads][N][head_dim]   (tokens in permutation order; block j is the
 *                                    row range [blk_start[j], blk_start[j+1]))
 *    hhat    [N][audio_dim]
 * Storage dtype of every tensor above is prob->dtype; per-zone, per-block and
 * probability arrays are float32.
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PRISM_OK = 0,
    PRISM_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad scalar        */
    PRISM_ERR_SHAPE = 2,         /* grid axes not positive multiples of 8        */
    PRISM_ERR_UNSUPPORTED = 3,   /* dtype, head_dim, heads, audio_dim, N too big */
    PRISM_ERR_WORKSPACE = 4,     /* workspace smaller than prism_query_sizes says */
    PRISM_ERR_CUDA = 5           /* a CUDA launch or runtime call failed          */
} prism_status_t;

typedef enum { PRISM_F32 = 0, PRISM_BF16 = 1 } prism_dtype_t;

/* Device status bits (written with atomicOr into a caller-owned uint32). */
#define PRISM_DEV_TIMEOUT   0x1u   /* a bounded wait in a kernel gave up          */
#define PRISM_DEV_BAD_INDEX 0x2u   /* an index read from device memory was out of range */

typedef struct {
    int32_t T, H, W;       /* latent video grid                                  */
    int32_t heads;         /* attention heads                                    */
    int32_t head_dim;      /* d                                                  */
    int32_t audio_dim;     /* channels of hhat                                   */
    int32_t dtype;         /* prism_dtype_t: storage dtype of the token tensors  */
} prism_problem_t;

typedef struct {
    int64_t n_tokens;       /* N                                                 */
    int64_t n_zones;        /* Z = N / 512                                       */
    int64_t max_blocks;     /* N / 64: upper bound of n_blk                      */
    int64_t sel_words;      /* uint32 words per selection row = ceil(max_blocks/32) */
    size_t  ws_indicator;   /* workspace bytes of prism_zone_indicator           */
    size_t  ws_attn_fwd;    /* workspace bytes of prism_sparse_attn_fwd          */
    size_t  ws_attn_bwd;    /* workspace bytes of prism_sparse_attn_bwd          */
    size_t  bytes_P_max;    /* bytes of P at n_blk = max_blocks (worst case)     */
} prism_sizes_t;

/* Sizes of every buffer of the path (host only, no CUDA call). */
prism_status_t prism_query_sizes(const prism_problem_t* prob, prism_sizes_t* sizes);

/*
 * Stage 1 — macro-zones and the dual-guidance variation indicator
 * ("Ideias centrais": 8x8x8 macro-zones; "Método" 1: sigma^2_{v,d}, r_{v,d},
 * a = ||hhat||_2, abar, vhat_{a,d}, g_d = r_{v,d} + abar*vhat_{a,d} + eps).
 *   V          raster [N][heads*head_dim] (all heads' channels form D)
 *   hhat       [N][audio_dim], cached audio-to-video cross-attention output
 *   eps        the indicator's epsilon (> 0)
 * Outputs (float32, zone-major, raster zone order):
 *   g [Z][3] (T, H, W);  rho [Z] = max(rho_v, abar) where rho_v is the zone's
 *   channel-averaged token variance of V over its grid maximum;  abar [Z] =
 *   A(m)/max A, A = zone mean of a;  zone_stats [Z][8] (nullable) =
 *   (sigma2_vT, sigma2_vH, sigma2_vW, rho_raw, A, sigma2_aT, sigma2_aH, sigma2_aW).
 * ws: >= sizes.ws_indicator bytes of scratch.
 * V is read through a TMA tensor map, one 8x8x8-zone box of 128 bytes of
 * channels per copy (V 16-byte aligned, like every pointer argument);
 * PRISM_ERR_CUDA if the map cannot be encoded.  A copy that never lands (a
 * failing device; the wait gives up after 2 s) leaves NaN statistics for the
 * zones that CTA had left, rather than stale ones.
 */
prism_status_t prism_zone_indicator(const prism_problem_t* prob, const void* V, const void* hhat,
                                    float eps, float* g, float* rho, float* abar,
                                    float* zone_stats, void* ws, size_t ws_bytes,
                                    cudaStream_t stream);

/*
 * Stage 1 with one guidance term removed (the pages' ablations of the dual
 * guidance; Portuguese reading guide, "Método" 1 and the ablations of its
 * experiments).  guidance = PRISM_GUIDE_JOINT gives prism_zone_indicator;
 * PRISM_GUIDE_VIDEO drops the audio term from both outputs that combine the
 * two (g_d = r_{v,d} + eps, rho = rho_v); PRISM_GUIDE_AUDIO drops the video
 * term (g_d = abar*vhat_{a,d} + eps, rho = abar).  abar and zone_stats are as
 * in prism_zone_indicator.  Any other guidance value: PRISM_ERR_INVALID_ARG.
 */
typedef enum { PRISM_GUIDE_JOINT = 0, PRISM_GUIDE_VIDEO = 1, PRISM_GUIDE_AUDIO = 2 } prism_guidance_t;
prism_status_t prism_zone_indicator_ex(const prism_problem_t* prob, const void* V, const void* hhat,
                                       float eps, int32_t guidance, float* g, float* rho, float* abar,
                                       float* zone_stats, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Stage 1 split for heads spread over several GPUs.  The indicator's video
 * statistics are sums over all D = heads*head_dim channels of V (the pages
 * form D from every channel; one shape per zone serves every head), so a rank
 * holding some of the heads computes the sums over its own channels, the
 * ranks add them with one all-reduce, and each rank finishes alone:
 *   prism_zone_partials(prob_local, V_local, hhat, partials, ws, ...)
 *       prob_local: the problem with heads = this rank's heads;
 *       V_local raster [N][local heads * head_dim];  hhat whole, [N][audio_dim];
 *       partials [2][Z][4] float32: [0] per zone the sums over the local
 *       channels of (8 sigma2_vT, 8 sigma2_vH, 8 sigma2_vW, 512 rho_raw) times
 *       the channel count (un-normalised sums of squared deviations);
 *       [1] the audio statistics (A, sigma2_aT, sigma2_aH, sigma2_aW), the
 *       same on every rank.  ws >= sizes.ws_indicator of prob_local.
 *   all-reduce (sum) of partials[0] ([Z][4] floats, contiguous) over the ranks
 *   prism_zone_finalize(prob, partials, eps, guidance, g, rho, abar, zone_stats, ws, ...)
 *       prob: the whole problem (all heads); outputs as prism_zone_indicator_ex;
 *       ws >= Z*16 bytes of scratch.
 * The result equals prism_zone_indicator_ex up to the order of the fp32 sums.
 */
prism_status_t prism_zone_partials(const prism_problem_t* prob_local, const void* V_local, const void* hhat,
                                   float* partials, void* ws, size_t ws_bytes, cudaStream_t stream);
prism_status_t prism_zone_finalize(const prism_problem_t* prob, const float* partials, float eps,
                                   int32_t guidance, float* g, float* rho, float* abar, float* zone_stats,
                                   void* ws, size_t ws_bytes, cudaStream_t stream);

/* Size of the library-owned scratch array behind prism_zone_indicator_noalloc. */
#define PRISM_NOALLOC_SCRATCH_BYTES (2u << 20)

/*
 * prism_zone_indicator without a workspace argument: same inputs, outputs
 * and results, for callers that cannot allocate device memory themselves (a
 * C host with no device allocator of its own, or a service whose device
 * footprint is fixed at start-up).  The paper has no counterpart; this is a
 * library convenience.
 *  - Scratch is a fixed PRISM_NOALLOC_SCRATCH_BYTES (2 MiB) array inside the
 *    library, held by every GPU that loads it until the process exits.  A
 *    problem needing more (zones * (4*D/CH + 8) floats, CH = 64 channels for
 *    bf16, 32 for f32; the 1,032,192-token bf16 grid needs 1.6 MB) returns
 *    PRISM_ERR_WORKSPACE before any launch.
 *  - Nothing is allocated: no cudaMalloc/cudaFree or allocating library call.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The address is kept for the life of the
 *    process: it does not survive cudaDeviceReset or any other teardown of
 *    the device's primary context, after which this entry point must not be
 *    called again on that device in the same process.
 *  - All calls share the array: calls whose kernels overlap on the GPU (two
 *    streams, two host threads) race on it and must be serialised by the caller.
 */
prism_status_t prism_zone_indicator_noalloc(const prism_problem_t* prob, const void* V,
                                            const void* hhat, float eps, float* g, float* rho,
                                            float* abar, float* zone_stats, cudaStream_t stream);

/*
 * Stage 2 — block volume and shape quantisation ("Método" 2): B(m) = 64 if
 * rho >= tau128, 128 if tau256 <= rho < tau128, else 256; l*_d =
 * -1/2 log2 g_d + (log2 B + 1/2 sum log2 g)/3; the shape is the candidate of
 * volume B nearest to l* in log2 space (edges in {2,4,8}: 16 candidates
 * numbered by (volume, b_T, b_H, b_W) ascending; exact ties go to the smaller
 * id).  Also builds the token permutation (zones in raster order, blocks in
 * raster order inside a zone, tokens in raster order inside a block).
 *   shape_id  [Z] uint8           perm [N] int32: perm[p] = raster index of row p
 *   inv_perm  [N] int32 (nullable): inv_perm[perm[p]] = p
 *   blk_start [max_blocks+1] int32: entries past n_blk hold N
 *   gran_blk  [N/64] int32: block index of each 64-row granule
 *   n_blk     [1] int32 (device)  margin [Z][2] float32 (nullable): (second-best
 *             minus best squared distance, min |rho - tau|)
 */
prism_status_t prism_assign_shapes(const prism_problem_t* prob, const float* g, const float* rho,
                                   float tau128, float tau256, uint8_t* shape_id, int32_t* perm,
                                   int32_t* inv_perm, int32_t* blk_start, int32_t* gran_blk,
                                   int32_t* n_blk, float* margin, cudaStream_t stream);

/*
 * Stage 2 with the fixed-shape block-sparse baseline the pages compare
 * against: fixed_shape = -1 is prism_assign_shapes; fixed_shape in [0, 15]
 * gives every zone that candidate (ids as above: 0-6 volume 64, 7-12 volume
 * 128, 13-15 volume 256), ignoring g, rho and the thresholds; margin (if
 * given) is then +inf (no decision is taken).  Outside [-1, 15]:
 * PRISM_ERR_INVALID_ARG.
 */
prism_status_t prism_assign_shapes_ex(const prism_problem_t* prob, const float* g, const float* rho,
                                      float tau128, float tau256, int32_t fixed_shape, uint8_t* shape_id,
                                      int32_t* perm, int32_t* inv_perm, int32_t* blk_start,
                                      int32_t* gran_blk, int32_t* n_blk, float* margin,
                                      cudaStream_t stream);

/*
 * Stage 3 — gather raster tokens into block order and head-major layout
 * (news page, "工作原理" step 4, and its inverse that restores the layout).
 *   prism_permute:   dst_blocked[h][p][:] = src_raster[perm[p]][h][:]
 *   prism_unpermute: dst_raster[perm[p]][h][:] = src_blocked[h][p][:]
 * Bit copies in prob->dtype.
 */
prism_status_t prism_permute(const prism_problem_t* prob, const void* src_raster,
                             const int32_t* perm, void* dst_blocked, cudaStream_t stream);
prism_status_t prism_unpermute(const prism_problem_t* prob, const void* src_blocked,
                               const int32_t* perm, void* dst_raster, cudaStream_t stream);

/*
 * Stage 4 — pooled block representatives and block probabilities ("Método" 3):
 * Qbar_i, Kbar_j = means over the block's rows (float32 [heads][max_blocks][d]);
 * s_ij = scale * Qbar_i . Kbar_j;  P_i = softmax_j over all n_blk key blocks.
 * P is packed with the device n_blk: P[(h*n_blk + i)*n_blk + j]; it needs
 * heads*n_blk^2 floats (at most sizes.bytes_P_max bytes).
 */
prism_status_t prism_block_pool_score(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                      const int32_t* blk_start, const int32_t* n_blk, float scale,
                                      float* Qbar, float* Kbar, float* P, cudaStream_t stream);

/*
 * Stage 5 — hybrid selection S_i = Top-k(P_i, k) U Top-p(P_i, p) ("Método" 3).
 * Both are prefixes of the order (P desc, j asc): Top-p is the shortest prefix
 * whose sum reaches p (all blocks if p >= 1 or it never does), so S_i is the
 * first max(min(k, n_blk), n_p) blocks.  k >= 0 and 0 < p: k = 0 is the
 * Top-p-only ablation and a tiny p (n_p = 1) the Top-k-only one; k < 0 or
 * p <= 0 (or not finite): PRISM_ERR_INVALID_ARG.
 *   sel       [heads][max_blocks][sel_words] uint32 bitmask, bit j of row i
 *   sel_count [heads][max_blocks] int32 (|S_i|; rows past n_blk are 0)
 *   gsel      [heads][N/64][sel_words] uint32: the same selection at granule
 *             level, the view the attention kernels read: row qg (64-row query
 *             granule) has bit kg set when the block of key granule kg is in S
 *             of the block of qg (blk_start, gran_blk from prism_assign_shapes)
 *   gselT     [heads][N/64][sel_words] uint32 (nullable): transpose of gsel, the
 *             key-major view of the backward (inference passes NULL)
 *   margin    [heads][max_blocks] float32 (nullable): the smallest change of the
 *             row (L1 size) that could change S_i: the gap between the last
 *             selected and the first unselected value; the sum of S_i above p
 *             (while n < n_blk); when Top-p sets n (n_p > n_k), p above the sum
 *             of the n-1 largest.  inf when nothing can change S_i.
 *   dev_status  PRISM_DEV_BAD_INDEX if n_blk exceeds 16384, the longest row the
 *             selection holds on chip (rows of up to 4096 blocks sit in registers,
 *             longer ones in shared memory); every row is then left empty.
 * Rows i >= n_blk are written as empty rows with count 0.
 */
prism_status_t prism_block_select(const prism_problem_t* prob, const float* P, const int32_t* blk_start,
                                  const int32_t* gran_blk, const int32_t* n_blk, int32_t top_k,
                                  float top_p, uint32_t* sel, int32_t* sel_count, uint32_t* gsel,
                                  uint32_t* gselT, float* margin, uint32_t* dev_status,
                                  cudaStream_t stream);

/*
 * Stage 6 — exact online-softmax attention of every query block over the tokens
 * of its selected key blocks ("Método" 3; non-causal, scale usually 1/sqrt(d)).
 *   Qp, Kp, Vp blocked [heads][N][d];  gsel granule-level selection from
 *   prism_block_select;  Op blocked;  lse [heads][N] float32 (nullable: the
 *   backward's input only, so inference passes NULL) = natural log of the
 *   softmax denominator; -inf for an empty S_i, whose O is 0.
 *   o_f32 (nullable) blocked [heads][N][d] float32: the unrounded O, for the
 *   backward's Delta (with a bf16 O, rowsum(dO*O) carries O's rounding error,
 *   which dominates dQ/dK when the attention is diffuse).
 * ws: >= sizes.ws_attn_fwd bytes (may be NULL when that is 0).
 * bf16 runs on tcgen05 tensor cores (fp32 accumulation); f32 on CUDA cores.
 */
prism_status_t prism_sparse_attn_fwd(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                     const void* Vp, const uint32_t* gsel, float scale, void* Op,
                                     float* lse, float* o_f32, uint32_t* dev_status, void* ws,
                                     size_t ws_bytes, cudaStream_t stream);

/*
 * Stage 7 — gradients of stage 6 under the fixed selection (Chinese guide,
 * FAQ on error propagation: rho, g and P_i are constants; gradients flow only
 * through the attention over the selected blocks).  Delta = rowsum(dO*O),
 * P = exp(s - lse), dV = P^T dO, dS = P*(dO V^T - Delta), dQ = scale*dS K,
 * dK = scale*dS^T Q.  Keys no query selected get dK = dV = 0.
 * Delta uses o_f32 when it is given (the forward's unrounded O), else Op.
 * gsel, gselT from prism_block_select.  All tensors blocked;
 * ws >= sizes.ws_attn_bwd bytes.
 */
prism_status_t prism_sparse_attn_bwd(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                     const void* Vp, const void* Op, const float* o_f32,
                                     const void* dOp, const float* lse, const uint32_t* gsel,
                                     const uint32_t* gselT, float scale, void* dQp, void* dKp,
                                     void* dVp, uint32_t* dev_status, void* ws, size_t ws_bytes,
                                     cudaStream_t stream);

/*
 * Stages 4, 6 and 7 straight from the raster layout (news page, "工作原理" step 4:
 * the kernel runs over the permuted blocks and the original layout comes back;
 * here the permutation is applied inside the loads and stores instead of by
 * copies).  Q, K, V, O raster [N][heads][head_dim]; perm and shape_id from
 * prism_assign_shapes.  The results equal, bit for bit, those of the blocked
 * calls on prism_permute'd inputs followed by prism_unpermute of O.
 *   prism_block_pool_score_raster: as prism_block_pool_score, rows read
 *     through perm.
 *   prism_sparse_attn_fwd_raster: as prism_sparse_attn_fwd; every 64-row
 *     granule of the blocked order is one tensor-map box of the raster tensor
 *     (its tokens are an (n_T, b_H, b_W) sub-box of the block), so Q, K and V are
 *     loaded and O is stored in place.  lse and o_f32 (nullable) stay in
 *     permutation order ([heads][N]).  bf16 only (PRISM_ERR_UNSUPPORTED else);
 *     ws >= sizes.ws_attn_fwd.
 */
prism_status_t prism_block_pool_score_raster(const prism_problem_t* prob, const void* Q, const void* K,
                                             const int32_t* perm, const int32_t* blk_start, const int32_t* n_blk,
                                             float scale, float* Qbar, float* Kbar, float* P, cudaStream_t stream);
prism_status_t prism_sparse_attn_fwd_raster(const prism_problem_t* prob, const void* Q, const void* K,
                                            const void* V, const int32_t* perm, const uint8_t* shape_id,
                                            const uint32_t* gsel, float scale, void* O, float* lse, float* o_f32,
                                            uint32_t* dev_status, void* ws, size_t ws_bytes, cudaStream_t stream);
/*
 * Stage 7 on raster operands: as prism_sparse_attn_bwd with Q, K, V, dO, dQ,
 * dK, dV raster [N][heads][head_dim]; o_f32 (required: the forward's unrounded
 * O) and lse in permutation order, as prism_sparse_attn_fwd_raster leaves
 * them.  Bit for bit the blocked call's results, unpermuted.  bf16 only;
 * ws >= sizes.ws_attn_bwd.
 */
prism_status_t prism_sparse_attn_bwd_raster(const prism_problem_t* prob, const void* Q, const void* K,
                                            const void* V, const float* o_f32, const void* dO, const float* lse,
                                            const int32_t* perm, const uint8_t* shape_id, const uint32_t* gsel,
                                            const uint32_t* gselT, float scale, void* dQ, void* dK, void* dV,
                                            uint32_t* dev_status, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Stage 7 with a dS handoff (same gradients as the FAQ formulas above; a
 * different split of the work).  The key-stationary kernel forms dS^T for
 * every selected (128-key tile, 64-query granule) pair anyway.  Given a
 * caller-owned buffer `ds` of ds_bytes, it also stores those blocks there as
 * bf16, and dQ = scale*dS K is then one GEMM per selected key granule, in
 * place of recomputing S = Q K^T and dP = dO V^T for dQ.
 *   Pieces: one 16 KB block (128 keys x 64 queries) per unit of the
 *   key-stationary walk, i.e. per (key tile, query granule that selected one of
 *   its two key granules).
 *   Whether the selection's pieces fit is decided on the device, with no host
 *   synchronisation.  When they do not fit, the call recomputes S and dP, as
 *   prism_sparse_attn_bwd does.
 *   dQ may differ from the recomputing call's in the last bf16 bit: S^T and S
 *   are accumulated in different orders.  dK and dV are the same.
 *   ds: 16-byte aligned, not aliased with any other argument.  ds_bytes: at
 *   least prism_attn_bwd_ds_bytes(prob, 1), else PRISM_ERR_WORKSPACE.
 *   prism_attn_bwd_ds_bytes: the bytes for a buffer that holds `pieces`
 *   pieces, 1 <= pieces < 2^24 (PRISM_ERR_INVALID_ARG else).  A selection
 *   needs at most the number of its selected (query granule, key granule)
 *   pairs.
 *   bf16 only: PRISM_ERR_UNSUPPORTED for f32.
 */
prism_status_t prism_attn_bwd_ds_bytes(const prism_problem_t* prob, int64_t pieces, size_t* bytes);
prism_status_t prism_sparse_attn_bwd_ds(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                        const void* Vp, const void* Op, const float* o_f32,
                                        const void* dOp, const float* lse, const uint32_t* gsel,
                                        const uint32_t* gselT, float scale, void* dQp, void* dKp,
                                        void* dVp, uint32_t* dev_status, void* ws, size_t ws_bytes,
                                        void* ds, size_t ds_bytes, cudaStream_t stream);
prism_status_t prism_sparse_attn_bwd_raster_ds(const prism_problem_t* prob, const void* Q, const void* K,
                                               const void* V, const float* o_f32, const void* dO,
                                               const float* lse, const int32_t* perm, const uint8_t* shape_id,
                                               const uint32_t* gsel, const uint32_t* gselT, float scale,
                                               void* dQ, void* dK, void* dV, uint32_t* dev_status, void* ws,
                                               size_t ws_bytes, void* ds, size_t ds_bytes, cudaStream_t stream);

/* Copy a device status word to the host (synchronises `stream`). */
prism_status_t prism_read_status(const uint32_t* dev_status, uint32_t* host_out, cudaStream_t stream);

/* Static description of a status code. */
const char* prism_status_string(prism_status_t status);

/* Library version, e.g. "prism-b200 0.1.0 sm_100a". */
const char* prism_version(void);

/* Number of kernels this library has launched since it was loaded (all
 * threads, all devices); a diagnostics counter for profiling harnesses. */
unsigned long long prism_launch_count(void);

/* ==========================================================================
 * The whole layer as one object.  The pages describe the stages; this is their
 * call sequence, in the order above, over buffers carved from one caller-owned
 * device arena, for hosts that want one call per direction (a C program, a
 * binding).  The struct is transparent: after prism_layer_bind every buffer
 * pointer is set and may be read (or, with the same sizes, set by a caller that
 * allocates the buffers one by one instead of binding an arena).
 * ========================================================================== */
typedef struct {
    /* parameters (prism_layer_init sets the defaults shown) */
    prism_problem_t prob;
    int32_t top_k;          /* 8                                                    */
    float top_p;            /* 0.9                                                  */
    float eps;              /* 1e-6: the indicator's epsilon                        */
    float tau128, tau256;   /* 0.5, 0.25: the block-volume thresholds on rho        */
    float scale;            /* 1/sqrt(head_dim)                                     */
    int32_t guidance;       /* PRISM_GUIDE_JOINT                                    */
    int32_t fixed_shape;    /* -1: adaptive shapes                                  */
    int32_t with_backward;  /* 1; 0 = inference: no LSE, fp32 O, gselT, backward buffers */
    int32_t with_io;        /* 0; 1 = also the raster inputs/outputs, for prism_layer_step_host */
    int32_t raster;         /* 0; 1 = the attention reads Q, K, V, dO and writes O, dQ, dK, dV
                               in the raster layout: no blocked copies (bf16 only)          */
    int64_t p_blocks;       /* 0: P sized for max_blocks; else a caller-known bound on n_blk */
    /* device buffers; shapes and layouts as the stage calls above describe them */
    float *g, *rho, *abar, *zone_stats;
    void* ws_ind;
    size_t ws_ind_bytes;
    uint8_t* shape_id;
    int32_t *perm, *blk_start, *gran_blk, *n_blk;
    float* margin_shape;
    void *Qp, *Kp, *Vp;
    float *Qbar, *Kbar, *P;
    uint32_t *sel, *gsel, *gselT;
    int32_t* sel_count;
    float* margin_sel;
    uint32_t* dev_status;   /* cleared by the caller before the first step          */
    void* Op;
    float *Of32, *lse;
    void* ws_fwd;
    size_t ws_fwd_bytes;
    void *dOp, *dQp, *dKp, *dVp;
    void* ws_bwd;
    size_t ws_bwd_bytes;
    /* raster Q, K, V, hhat, O, dO, dQ, dK, dV on the device (with_io only) */
    void *Q, *K, *V, *hhat, *O, *dO, *dQ, *dK, *dV;
    /* library-owned state of prism_layer_step_host (two CUDA events that carry
       "this step has read its raster inputs" to the next call): NULL after
       prism_layer_init, created by the first host-buffer step, destroyed by
       prism_layer_release.  Callers do not touch it. */
    void* io_events;
} prism_layer_t;

/* Fill L with the defaults above for `prob` and no buffers (host only). */
prism_status_t prism_layer_init(prism_layer_t* L, const prism_problem_t* prob);
/* Bytes of the arena prism_layer_bind needs for L's parameters (host only). */
prism_status_t prism_layer_arena_bytes(const prism_layer_t* L, size_t* bytes);
/* Carve every buffer of L from `arena` (device memory, 256-byte aligned, at
 * least prism_layer_arena_bytes; caller-owned).  Host only: no CUDA call. */
prism_status_t prism_layer_bind(prism_layer_t* L, void* arena, size_t bytes);
/* Stages 1-6 and the unpermute of O on `stream`: raster device Q, K, V, hhat in,
 * raster O out.  Asynchronous; read L->dev_status (prism_read_status) after. */
prism_status_t prism_layer_forward(const prism_layer_t* L, const void* Q, const void* K, const void* V,
                                   const void* hhat, void* O, cudaStream_t stream);
/* Stage 7 for the last forward on `stream`: raster device dO in, raster dQ, dK,
 * dV out.  Q, K, V: the last forward's raster inputs, unchanged since (read
 * only when L->raster; may be NULL otherwise).  PRISM_ERR_UNSUPPORTED when L
 * has no backward buffers. */
prism_status_t prism_layer_backward(const prism_layer_t* L, const void* Q, const void* K, const void* V,
                                    const void* dO, void* dQ, void* dK, void* dV, cudaStream_t stream);
/* One whole step from HOST buffers (L bound with with_io = 1): uploads Q, K,
 * V, hhat (and dO with a backward), runs the layer, downloads O (and dQ, dK,
 * dV), with one cudaMemcpyAsync per tensor on the two copy streams: V and
 * hhat first, dO during the forward, O during the backward.  Three distinct
 * streams.  Host buffers should be page-locked, or the copies do not overlap.
 * Asynchronous: every device step of the call precedes its last download on
 * `d2h`, so the host outputs are final once `d2h` has passed this call (e.g.
 * cudaStreamSynchronize(d2h)).  Consecutive calls with the same streams are
 * ordered.  The next call's uploads wait only until this call has read the
 * raster inputs.  In the blocked layout that is the permutes at the start of
 * the forward (Q, K, V, hhat) and of the backward (dO), so the next uploads
 * overlap this call's attention and downloads; with L->raster it is the end of
 * the backward.  The next call's writes of O and the gradients wait for this
 * call's downloads.  Host input buffers must stay unchanged and output buffers
 * unread until then.  The first call creates L->io_events (two CUDA events);
 * prism_layer_release destroys them. */
prism_status_t prism_layer_step_host(prism_layer_t* L, const void* hQ, const void* hK, const void* hV,
                                     const void* hhhat, const void* hdO, void* hO, void* hdQ, void* hdK,
                                     void* hdV, cudaStream_t compute, cudaStream_t h2d, cudaStream_t d2h);
/* Destroy the CUDA events a host-buffer step created in L (L->io_events),
 * after every call that used them has completed; a no-op when there are none.
 * The device buffers stay the caller's. */
prism_status_t prism_layer_release(prism_layer_t* L);
/* sizeof(prism_layer_t) as compiled into the library (a check for bindings). */
size_t prism_layer_sizeof(void);

#ifdef __cplusplus
}
#endif
#endif /* PRISM_H */
