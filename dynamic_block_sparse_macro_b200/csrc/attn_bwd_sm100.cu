// Stage 7 on sm_100a tensor cores: block-sparse attention backward for bf16.
//
// Chinese reading guide of the Prism paper, FAQ on error propagation: rho, g
// and the block probabilities P_i are constants in the backward; gradients
// flow only through the attention over the selected key-value blocks.  With
// P = exp(s - lse) over the selected keys and Delta = rowsum(dO * O):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),  dQ = scale dS K,
//   dK = scale dS^T Q.
//
// Two persistent kernels (one CTA per SM looping over the work plan's items),
// no atomics (deterministic):
//   k_bwd_dq_persist    query-stationary: per (128-row query tile, head) walk the
//                       key granules of the union of its two granule-level rows;
//                       Q and dO sit in TMEM as bf16; per 64-key granule S = Q K^T
//                       and dP = dO V^T (M=128, N=64, A from TMEM) into TMEM, dS
//                       as bf16 back into TMEM, dQ += dS K (K MN-major in smem).
//   k_bwd_dkdv_persist  key-stationary: per (128-key tile, head) walk the query
//                       granules whose blocks selected the tile's key blocks (the
//                       transposed granule-level selection); per 64-query granule
//                       S^T = K Q^T and dP^T = V dO^T, then P^T and dS^T as bf16
//                       in TMEM, dV += P^T dO and dK += dS^T Q.
// With a dS handoff buffer (ds_handoff.cuh) the key-stationary kernel also
// stores its dS^T blocks, and k_bwd_dq_ds replaces the query-stationary kernel
// with one GEMM per key granule, dQ += dS K, so that S and dP are formed once.
// Both double-buffer the granule products in TMEM so that the tensor core
// works on granule g+1 while the elementwise warps work on granule g, and
// stream granules through a TMA ring as deep as shared memory allows; ring
// stages, buffers and barrier phases carry across item edges, so the next
// item's loads and first products overlap the current item's epilogue.
// Roles: warp 0 TMA (one lane per ring stage and stream, one whole-row copy
// per granule), warp 1 TMEM allocation; MMA issue (the whole warp, one elected
// lane issues) by warps 1, 10, 11 in dQ (S, dP, dQ) and warps 1, 2 in dK/dV
// (S^T and dP^T; dV and dK), one accumulation chain each, so that one warp's
// barrier waits leave the others' MMAs in the tensor pipe; the elementwise
// warps one tile row per thread.
// Every wait is bounded; a timeout sets PRISM_DEV_TIMEOUT.
#include "attn_plan.cuh"
#include "common.cuh"
#include "ds_handoff.cuh"
#include "sm100.cuh"

namespace prism {

using namespace sm100;

prism_status_t bwd_delta(const Dims& d, const void* Op, const float* o_f32, const void* dOp, float* delta,
                         const float* lse, float* nld, cudaStream_t s, const int32_t* perm);

namespace {

constexpr int kTile = 128 * 128;           // bytes: 128 rows x 64 bf16 columns
constexpr int kGran = 64 * 128;            // bytes: 64 rows x 64 bf16 columns
constexpr int kStages = 8;                 // barrier slots; the ring uses nst <= kStages of them
constexpr int kCtrl = 512;                 // bytes of barriers and flags
constexpr int kXs = 512;                   // per stage (dK/dV only): -lse*log2(e) and -Delta of 64 query rows
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSmemMax = 227 * 1024;
// dK/dV kernel register split: 384 threads launch with 168 each; warpgroup 0
// (TMA, MMA) drops to 152 and the two elementwise warpgroups rise to 176
// (128 * (152 + 2 * 176) = 384 * 168); the persistent item loop needs more
// than 136 registers on the TMA/MMA side and fits 176 on the elementwise side
constexpr uint32_t kRegsLow = 152, kRegsHigh = 176;

// descriptor offsets: K-major operand, k-th 16-element step of the contraction over d
__device__ __forceinline__ uint32_t kmaj_off(int k, int region) { return (k >> 2) * region + (k & 3) * 32; }

// ============================================================================ dQ (persistent)
// One CTA per SM takes items blockIdx.x, blockIdx.x + gridDim.x, ...  Granules
// are numbered G = 0, 1, ... over all of the CTA's items, so the ring stages,
// the double-buffered S/dP columns and every phase carry across item edges:
// the producer runs ahead into the next item while the current one finishes,
// the next item's Q and dO go into TMEM as soon as the current item's last
// products are consumed, and its first S/dP MMAs overlap the current epilogue.
// Per local item j:
//   rows[j & 1]  the tile's two selection rows: the producer's 32 lanes write
//                them (rows_full, 32 arrivals), the four elementwise warps
//                release them after their walk (rows_empty, 4 arrivals)
// Per non-empty item k (items with no granule, ng = 0, never reach the MMA
// warp: their dQ is zero and written without TMEM, so that no barrier can
// complete two phases before its waiter has seen the first):
//   qdo_full     Q, dO of item k in TMEM (128 arrivals), phase k & 1
//   fin          every MMA of item k complete, phase k & 1
// The dQ columns are free for item j+1's first dQ MMA once the elementwise
// warps have arrived on that granule's elem barrier: they do so only after the
// epilogue of item j has read dQ.
// Raster operands (no blocked copies): the kernels read Q, K, V, dO and write
// dQ, dK, dV in the raster layout [N][heads][d] through the permutation, every
// 64-row granule being one 5-D box per 64-column region (make_map_raster); the
// fp32 partials of split tiles stay in their blocked slots.
enum { kRK = 0, kRV = 1, kRdQ = 2, kRQ = 2, kRdO = 3, kRdK = 4, kRdV = 5 };
template <bool RASTER, int T> using BwdRasterMaps = RasterMaps<RASTER ? T : 1>;
struct BwdRaster {
    const int4* gpos;          // [N/64] granule positions (gran_positions)
    const int32_t* perm;       // [N]
    int heads;
};

// Device side of the dS handoff (ds_handoff.cuh): `on` is written by k_ds_bases
// before any kernel that reads it, 1 when every piece and entry fits
struct DsDev {
    int* on;
    int64_t* base_q;           // [tiles] exclusive prefix of the query tiles' units
    int64_t* base_kv;          // [tiles] exclusive prefix of the key tiles' units
    int32_t* pre;              // [tiles][SW] word prefixes of the key tiles' unions
    int4* entries;             // [cap_q] look-up entries of the query-stationary walk
    __nv_bfloat16* pieces;     // [1 + cap_units][128][64] dS^T; piece 0 stays zero
};

constexpr int kStagingP = 2 * kTile;       // 32 KB: two 128-byte regions of 128 rows

template <int D>
struct DqpLayout {
    static constexpr int NR = D / 64;
    static constexpr int STAGE = 2 * NR * kGran;       // K and V of one granule
    __host__ __device__ static int staging(int nst) { return nst * STAGE; }
    __host__ __device__ static int ctrl(int nst) { return staging(nst) + kStagingP; }
    __host__ __device__ static int rows(int nst) { return ctrl(nst) + kCtrl; }
    static int alloc(int nst, int SW) { return rows(nst) + 16 * SW + 1024; }   // 2 slots x 2 rows
    static int stages(int SW) {
        int n = kStages;
        while (n > 2 && alloc(n, SW) > kSmemMax) --n;
        return n;
    }
};

struct BarsP {
    uint64_t* full0;           // [kStages] K and V of a granule landed (two arrivals)
    uint64_t* empty;           // [kStages]
    uint64_t* prod;            // [2]
    uint64_t* elem;            // [2]
    uint64_t* qdo_full;
    uint64_t* fin;
    uint64_t* drain;           // [3] teardown after an abort: every MMA an issuer issued complete
    uint64_t* rows_full;       // [2]
    uint64_t* rows_empty;      // [2]
    uint64_t* dq_done;         // [2] dQ MMAs of the buffer's granule complete (its dS read)
    uint32_t* tmem_slot;
    volatile int* abort_flag;
};

__device__ __forceinline__ BarsP carve_p(uint8_t* ctrl) {
    uint64_t* b = reinterpret_cast<uint64_t*>(ctrl);
    BarsP r;
    r.full0 = b;
    r.empty = b + 2 * kStages;
    r.prod = b + 3 * kStages;
    r.elem = b + 3 * kStages + 2;
    r.qdo_full = b + 3 * kStages + 4;
    r.fin = b + 3 * kStages + 5;
    r.drain = b + 3 * kStages + 6;
    r.rows_full = b + 3 * kStages + 9;
    r.rows_empty = b + 3 * kStages + 11;
    r.dq_done = b + 3 * kStages + 13;
    r.tmem_slot = reinterpret_cast<uint32_t*>(b + 3 * kStages + 15);
    r.abort_flag = reinterpret_cast<volatile int*>(r.tmem_slot + 1);
    return r;
}
static_assert((3 * kStages + 15) * 8 + 8 <= kCtrl, "barriers overflow the control block");

// Epilogue with a 32 KB staging area of its own (the ring is busy with the
// next item), shared by the two elementwise warpgroups, warpgroup wg owning
// accumulator columns 64 wg .. 64 wg + 63: the bf16 tile (D/64 regions) in one
// store, each warpgroup writing its own region; the fp32 partial (D/32
// regions) in passes of two regions, pass p written by warpgroup p.  The
// barrier at the top of every pass makes the staging free: the leader passes
// it only after its previous store has finished reading shared memory.  Every
// thread of both warpgroups runs the same barriers whatever `ok` is (passes
// depend on `part` only).
// With `rmaps` (raster output), the bf16 tile goes out as one box per (query
// granule, region): granule hg's position gp[hg], head-region base hreg.
template <int D>
__device__ void store_tile_p(uint32_t tacc, int row, int wg, bool ok, bool zero, bool part, float mul,
                             uint8_t* stage, const CUtensorMap* map_bf16, const CUtensorMap* map_f32h, int y_bf16,
                             int y_f32, int bar_id, int nthreads, bool leader, const CUtensorMap* rmaps = nullptr,
                             int4 gp0 = int4{}, int4 gp1 = int4{}, int hreg = 0, int store_lane = 0) {
    static_assert(D == 128 || D == 64, "head_dim");
    const int regions = part ? D / 32 : D / 64;            // 128-byte regions of a row
    const int per_pass = regions < 2 ? regions : 2;
    const int passes = regions / per_pass;
    const uint32_t sw = (uint32_t)(row & 7);
    constexpr int kColsWg = D / 2;                          // accumulator columns of one warpgroup
#pragma unroll 1
    for (int p = 0; p < passes; ++p) {
        named_sync(bar_id, nthreads);
        // fp32 pass p covers columns 32 p * per_pass ..; bf16 covers every column in one pass
        const int c0 = part ? 32 * per_pass * p : 0, c1 = part ? c0 + 32 * per_pass : D;
        const int w0 = kColsWg * wg, w1 = w0 + kColsWg;     // this warpgroup's columns
        const int q0 = (c0 > w0 ? c0 : w0) / 32, q1 = (c1 < w1 ? c1 : w1) / 32;
        if (ok && q0 < q1) {
#pragma unroll 1
            for (int q = q0; q < q1; ++q) {                   // 32 fp32 TMEM columns per load
                uint32_t r[32];
                if (zero) {                                   // an empty item: TMEM is not read
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                } else {
                    tmem_ld32(tacc + 32 * q, r);
                    tmem_wait_ld();
                }
                if (!part) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int g = 4 * q + k;              // 16-byte chunk of the bf16 row
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(r[8 * k + 0]) * mul, __uint_as_float(r[8 * k + 1]) * mul);
                        v.y = pack_bf16x2(__uint_as_float(r[8 * k + 2]) * mul, __uint_as_float(r[8 * k + 3]) * mul);
                        v.z = pack_bf16x2(__uint_as_float(r[8 * k + 4]) * mul, __uint_as_float(r[8 * k + 5]) * mul);
                        v.w = pack_bf16x2(__uint_as_float(r[8 * k + 6]) * mul, __uint_as_float(r[8 * k + 7]) * mul);
                        *reinterpret_cast<uint4*>(stage + (g >> 3) * kTile + row * 128 + (((g & 7) ^ sw) << 4)) = v;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int g = 8 * (q - c0 / 32) + k;  // 16-byte chunk within this pass
                        const float4 v = make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                                                     __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]));
                        *reinterpret_cast<float4*>(stage + (g >> 3) * kTile + row * 128 + (((g & 7) ^ sw) << 4)) = v;
                    }
                }
            }
            fence_proxy_async_smem();
        }
        named_sync(bar_id, nthreads);
        // leader: lane 0 of the storing warp, or (raster bf16 tile) the lanes
        // store_lane = 0 .. 2 D/64 - 1, each with its own (granule, region) box
        if (ok && leader && (store_lane == 0 || (rmaps && !part))) {
            if (part) {
                tma_store_3d(map_f32h, stage, 0, y_f32, p * per_pass);
            } else if (rmaps) {
                const int hg = store_lane / (D / 64), r = store_lane % (D / 64);
                const int4 gp = hg ? gp1 : gp0;
                tma_store_5d(rmaps + gp.w, stage + r * kTile + hg * kGran, 0, hreg + r, gp.z, gp.y, gp.x);
            } else {
                tma_store_3d(map_bf16, stage, 0, y_bf16, 0);
            }
            bulk_commit();
            bulk_wait_read();
        }
    }
}

// One row of Q or dO into TMEM as bf16 (two per 32-bit column)
template <int D>
__device__ __forceinline__ void load_row_tmem(uint32_t taddr, const __nv_bfloat16* src_rows, int64_t grow) {
    const uint4* src = reinterpret_cast<const uint4*>(src_rows + grow * D);
#pragma unroll
    for (int q = 0; q < D / 64; ++q) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 v = __ldg(src + 8 * q + i);
            r[4 * i] = v.x;
            r[4 * i + 1] = v.y;
            r[4 * i + 2] = v.z;
            r[4 * i + 3] = v.w;
        }
        tmem_st32(taddr + 32 * q, r);
    }
    tmem_wait_st();
}

// DS: launched beside k_bwd_dq_ds, which does the work when *ds_on is set
template <int D, bool RASTER, bool DS = false>
__global__ void __launch_bounds__(384, 1)
k_bwd_dq_persist(const __nv_bfloat16* __restrict__ Qg, const __nv_bfloat16* __restrict__ dOg,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmPqh,
                 const __grid_constant__ BwdRasterMaps<RASTER, 3> rmaps, BwdRaster ras,
                 const uint32_t* __restrict__ gsel, const PlanHeader* __restrict__ hdr,
                 const int4* __restrict__ items, const float* __restrict__ lse,
                 const float* __restrict__ delta, int64_t N, int64_t MB, int SW, int nst, float scale,
                 uint32_t* __restrict__ dev_status, const int* __restrict__ ds_on) {
    if constexpr (DS) {
        if (*ds_on) return;                           // uniform: dQ comes from the stored dS
    }
    using L = DqpLayout<D>;
    constexpr int kRL = RASTER ? L::NR : 1;            // copy lanes per (stream, stage)
    constexpr uint32_t cdQ = 0, cS = 128, cP = 192;   // + 128 * buffer for S / dP
    constexpr uint32_t cQ = 384, cdO = 384 + D / 2;
    const int n_items = hdr->n_items;
    if ((int)blockIdx.x >= n_items) return;           // uniform: more CTAs than items
    const int tiles_per_head = (int)(N / 128);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BarsP B = carve_p(sm + L::ctrl(nst));
    uint32_t* rows_base = reinterpret_cast<uint32_t*>(sm + L::rows(nst));   // [2 slots][2 rows][SW]
    uint8_t* staging = sm + L::staging(nst);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wn = SW;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(B.full0 + s, 2 * kRL);           // each K and V copy lane arrives
            mbar_init(B.empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(B.prod + b, 2);                  // the S and the dP issuer each commit
            mbar_init(B.elem + b, 256);
            mbar_init(B.rows_full + b, 32);
            mbar_init(B.rows_empty + b, 8);
            mbar_init(B.dq_done + b, 1);
        }
        mbar_init(B.qdo_full, 256);
        mbar_init(B.fin, 1);
        for (int i = 0; i < 3; ++i) mbar_init(B.drain + i, 1);
        *B.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *B.tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // lane kind * nst + stage (kind 0: K, 1: V) issues its stream's copies for
        // the granules of that stage; all 32 lanes copy the selection rows
        // lane (kind * nst + stage) * kRL + region: a raster granule is one box per
        // 64-column region, each from a lane of its own (copies of one thread
        // complete one after another)
        const int kind = lane / (nst * kRL), stage = (lane / kRL) % nst, region = lane % kRL;
        const bool copier = lane < 2 * nst * kRL;
        uint64_t* full = B.full0;                          // one barrier for both copies of a stage
        const CUtensorMap* mg = kind == 0 ? &tmK : &tmV;
        if (copier && !RASTER) tma_prefetch_desc(mg);
        bool ok = true;
        int last_cyc = -1;                                 // ring cycle of this lane's last copy
        int st0 = 0, cyc0 = 0;                             // stage and ring cycle of the item's first granule
        for (int it = blockIdx.x, j = 0; it < n_items; it += gridDim.x, ++j) {
            const int4 item = items[it];
            const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
            const int g_begin = item.y, ng = item.z - item.y;
            const int64_t row0 = (int64_t)hh * N;
            uint32_t* u0 = rows_base + (j & 1) * 2 * SW;
            uint32_t* u1 = u0 + SW;
            if (ok && j >= 2) ok = mbar_wait(B.rows_empty + (j & 1), ((j >> 1) - 1) & 1, B.abort_flag, dev_status);
            if (ok) {
                const uint32_t* s0 = gsel + ((int64_t)hh * MB + 2 * tile) * SW;
                for (int w = lane; w < wn; w += 32) {
                    u0[w] = s0[w];
                    u1[w] = s0[SW + w];
                }
            }
            mbar_arrive(B.rows_full + (j & 1));
            __syncwarp();                                  // every lane's rows visible to the walkers
            int s_ = st0, c_ = cyc0;
            if (copier && ok) {
                GranuleWalk walk;
                walk.init(u0, u1, wn);
                walk.skip(g_begin);
                for (int g = 0; g < ng; ++g) {
                    int row;
                    uint32_t m;
                    walk.next(row, m);
                    if (s_ == stage) {
                        if (c_ >= 1 && !mbar_wait(B.empty + stage, (uint32_t)(c_ - 1) & 1, B.abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        uint8_t* dst = sm + stage * L::STAGE + kind * L::NR * kGran;
                        if constexpr (RASTER) {
                            const int4 gp = ras.gpos[row >> 6];
                            mbar_expect_tx(full + stage, kGran);
                            tma_load_5d(dst + region * kGran, rmaps.m + (kind ? kRV : kRK) * kRasterKinds + gp.w,
                                        full + stage, 0, hh * L::NR + region, gp.z, gp.y, gp.x);
                        } else {
                            mbar_expect_tx(full + stage, L::NR * kGran);
                            tma_load_3d(dst, mg, full + stage, 0, (int)(row0 + row), 0);
                        }
                        last_cyc = c_;
                    }
                    if (++s_ == nst) { s_ = 0; ++c_; }
                }
            }
            __syncwarp();                                  // no lane walks rows a later item overwrites
            if (*B.abort_flag) ok = false;
            // every lane advances the ring position by the item's granules
            const int tot = st0 + ng;
            cyc0 += tot / nst;
            st0 = tot % nst;
        }
        if (!ok && copier && last_cyc >= 0) {
            volatile int no_abort = 0;                     // let this lane's last copy land
            mbar_wait(full + stage, (uint32_t)last_cyc & 1, &no_abort, dev_status);
        }
    } else if (warp == 1 || warp >= 10) {
        // ---------------------------------------------------------------- MMA issue, three warps
        // Three accumulation chains, each issued in order by one warp on its own
        // SM sub-partition: warp 1 S = Q K^T, warp 10 dP = dO V^T, warp 11
        // dQ += dS K.  Per TMEM buffer b and its u-th use (granule GG, b = GG & 1,
        // u = GG >> 1): S(GG) waits elem(b) and dq_done(b) of use u - 1 (its
        // columns consumed and dS read), dP(GG) waits elem(b) of use u - 1,
        // dQ(GG) waits elem(b) of use u; prod(b) completes when both S and dP
        // have.  No barrier can run two phases ahead of its waiter: every phase
        // needs the waiter's own earlier issue.
        const int role = warp == 1 ? 0 : warp - 9;          // 0: S, 1: dP, 2: dQ
        const uint32_t idPS = idesc_bf16_f32(128, 64, false, false);
        const uint32_t idQ = idesc_bf16_f32(128, D, false, true);
        const uint32_t aR = smem_u32(sm);
        bool ok = true;
        int G = 0;                                         // granules of this CTA so far
        int s_ = 0, c_ = 0;                                // stage and ring cycle of granule G
        int kq = 0;                                        // non-empty items so far
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            const int4 item = items[it];
            const int ng = item.z - item.y;
            if (ng == 0) continue;
            if (role < 2) {
                ok = mbar_wait_w(B.qdo_full, kq & 1, B.abort_flag, dev_status);
                if (!ok) break;
                tc_fence_after();
            }
            for (int g = 0; g < ng; ++g) {
                const int GG = G + g;
                const int s = s_, b = GG & 1, u = GG >> 1;
                const uint32_t ph = (uint32_t)c_ & 1;
                if (++s_ == nst) { s_ = 0; ++c_; }
                if (role < 2) {
                    if (!mbar_wait_w(B.full0 + s, ph, B.abort_flag, dev_status)) { ok = false; break; }
                    if (GG >= 2) {
                        if (!mbar_wait_w(B.elem + b, (uint32_t)(u - 1) & 1, B.abort_flag, dev_status) ||
                            (role == 0 && !mbar_wait_w(B.dq_done + b, (uint32_t)(u - 1) & 1, B.abort_flag, dev_status))) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint64_t dK = sdesc_sw128(aR + s * L::STAGE, 16, 1024);
                    if (role == 0) {
#pragma unroll
                        for (int k = 0; k < D / 16; ++k)
                            mma_ts_w(tb + cS + 128 * b, tb + cQ + 8 * k, sdesc_add(dK, kmaj_off(k, kGran)), idPS, k > 0);
                    } else {
                        const uint64_t dV = sdesc_add(dK, L::NR * kGran);
#pragma unroll
                        for (int k = 0; k < D / 16; ++k)
                            mma_ts_w(tb + cP + 128 * b, tb + cdO + 8 * k, sdesc_add(dV, kmaj_off(k, kGran)), idPS,
                                     k > 0);
                    }
                    tc_commit_w(B.prod + b);
                } else {
                    if (!mbar_wait_w(B.elem + b, (uint32_t)u & 1, B.abort_flag, dev_status)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t dKq = sdesc_sw128(aR + s * L::STAGE, kGran, 1024);
#pragma unroll
                    for (int k = 0; k < 4; ++k)              // dS keys 16 k ..: warpgroup k / 2's columns
                        mma_ts_w(tb + cdQ, tb + cS + 128 * b + 32 * (k >> 1) + 8 * (k & 1), sdesc_add(dKq, k * 2048),
                                 idQ, (g > 0 || k > 0) ? 1u : 0u);
                    tc_commit_w(B.empty + s);
                    tc_commit_w(B.dq_done + b);
                }
            }
            if (!ok) break;
            if (role == 2) tc_commit_w(B.fin);
            G += ng;
            ++kq;
        }
        if (!ok) {
            tc_commit_w(B.drain + role);                   // every MMA this warp issued complete
            volatile int no_abort = 0;
            mbar_wait(B.drain + role, 0, &no_abort, dev_status);
        }
    } else {
        // ---------------------------------------------------------------- elementwise + epilogue
        // Two warpgroups (warps 2-5, 6-9) on every granule: warpgroup wg turns key
        // columns 32 wg .. 32 wg + 31 of S and dP into dS and writes it, as bf16,
        // over the first 16 of those columns, so neither touches the other's
        // columns and no barrier joins them per granule.
        const int wg = (warp - 2) >> 2;
        const int sub = warp & 3, row = sub * 32 + lane, half = row >> 6;
        const uint32_t tl = tb + ((uint32_t)(sub * 32) << 16);
        const float sl2 = scale * kLog2e;
        const uint64_t sl2x2 = f2pack(sl2, sl2);
        bool ok = true;
        int G = 0;
        int kf = 0;                                        // non-empty items so far
        // Q (warpgroup 0) and dO (warpgroup 1) of a non-empty item go into TMEM
        // once both warpgroups have consumed every S/dP product of the previous
        // non-empty item; the first one before the loop
        auto qdo_ahead = [&](int itn) {
            if (itn >= n_items) return;
            const int4 nx = items[itn];
            if (nx.z == nx.y) return;                      // empty: never reaches the MMA warp
            if (ok) {
                const int nh = nx.x / tiles_per_head;
                const int64_t nrow = 128 * (int64_t)(nx.x % tiles_per_head) + row;     // within the head
                const int64_t src = RASTER ? (int64_t)ras.perm[nrow] * ras.heads + nh : (int64_t)nh * N + nrow;
                load_row_tmem<D>(tl + (wg ? cdO : cQ), wg ? dOg : Qg, src);
                tc_fence_before();
            }
            mbar_arrive(B.qdo_full);
        };
        qdo_ahead(blockIdx.x);
        for (int it = blockIdx.x, j = 0; it < n_items; it += gridDim.x, ++j) {
            const int4 item = items[it];
            const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
            const int g_begin = item.y, ng = item.z - item.y, slot = item.w;
            const int64_t row0 = (int64_t)hh * N;
            const int64_t grow = row0 + 128 * tile + row;
            const float lse2 = lse[grow] * kLog2e, dl = delta[grow];
            const uint64_t nlse2 = f2pack(-lse2, -lse2), ndl2 = f2pack(-dl, -dl);
            const uint32_t* u0 = rows_base + (j & 1) * 2 * SW;
            GranuleWalk walk;
            if (lane == 0) {
                const bool got = ok && mbar_wait(B.rows_full + (j & 1), (j >> 1) & 1, B.abort_flag, dev_status);
                if (got) {
                    walk.init(u0, u0 + SW, wn);
                    walk.skip(g_begin);
                } else {
                    walk.init(u0, u0 + SW, 0);             // empty walk; ok drops below
                }
                ok = got;
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int g = 0; ok && g < ng; ++g) {
                const int GG = G + g;
                const int b = GG & 1;
                uint32_t mk = 0;
                if (lane == 0) {
                    int rr;
                    walk.next(rr, mk);
                }
                mk = __shfl_sync(0xffffffffu, mk, 0);
                const bool valid = (mk >> half) & 1u;          // warp-uniform
                const bool got = mbar_wait(B.prod + b, (uint32_t)(GG >> 1) & 1, B.abort_flag, dev_status);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                const uint32_t cs = cS + 128 * b + 32 * wg, cp = cP + 128 * b + 32 * wg;
                uint32_t sv[32], pv[32];
                if (valid) {                                   // both loads in flight before one wait
                    tmem_ld32(tl + cs, sv);
                    tmem_ld32(tl + cp, pv);
                    tmem_wait_ld();
                }
                uint32_t o[16];
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float x0, x1;
                        f2unpack(ffma2(f2pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2x2,
                                       nlse2),
                                 x0, x1);
                        const uint64_t pp = f2pack(ex2(x0), ex2(x1));
                        const uint64_t dp =
                            fadd2(f2pack(__uint_as_float(pv[2 * i]), __uint_as_float(pv[2 * i + 1])), ndl2);
                        float d0, d1;
                        f2unpack(fmul2(pp, dp), d0, d1);
                        o[i] = pack_bf16x2(d0, d1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = 0u;
                }
                tmem_st16(tl + cs, o);                         // dS (bf16) over this warpgroup's S columns
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(B.elem + b);
            }
            if (lane == 0) mbar_arrive(B.rows_empty + (j & 1));
            // the next non-empty item's Q and dO: this warpgroup has seen every S/dP
            // product of this item complete, and so has the other before its own load
            qdo_ahead(it + (int)gridDim.x);
            bool fin = ok;
            if (ng > 0) {
                fin = __all_sync(0xffffffffu, ok && mbar_wait(B.fin, kf & 1, B.abort_flag, dev_status));
                if (fin) tc_fence_after();
                ++kf;
            }
            ok = fin;
            // the item's dQ (or zeros when nothing was selected: ng == 0)
            if constexpr (RASTER)
                store_tile_p<D>(tl + cdQ, row, wg, fin, ng == 0, slot >= 0, scale, staging, &tmdQ, &tmPqh,
                                (int)(row0 + 128 * tile), slot * 128, 1, 256, warp == 2 && lane < 2 * (D / 64),
                                rmaps.m + kRdQ * kRasterKinds, ras.gpos[2 * tile], ras.gpos[2 * tile + 1],
                                hh * (D / 64), lane);
            else
                store_tile_p<D>(tl + cdQ, row, wg, fin, ng == 0, slot >= 0, scale, staging, &tmdQ, &tmPqh,
                                (int)(row0 + 128 * tile), slot * 128, 1, 256, warp == 2 && lane == 0);
            G += ng;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, kTmemCols);
}

// ============================================================================ dK, dV (persistent)
// One CTA per SM takes items blockIdx.x, blockIdx.x + gridDim.x, ...; granules
// are numbered over all of the CTA's items, so the ring and the double-buffered
// S^T/dP^T columns carry across item edges.  The next non-empty item's K and V
// tiles are loaded as soon as the current item's last S^T/dP^T MMAs complete
// (kv_free), which hides the load behind the current item's tail and epilogue.
// Items with no granule (no query selected these keys) never reach the MMA
// warp; their dK and dV are zero, written without TMEM.  The epilogue shares one
// 16 KB staging region: one 128-row region of dK or dV per pass.
template <int D>
struct DkvpLayout {
    static constexpr int NR = D / 64;
    static constexpr int A0 = 0;                       // K tile
    static constexpr int A1 = NR * kTile;              // V tile
    static constexpr int STG = 2 * NR * kTile;         // one region of 128 rows x 128 bytes
    static constexpr int RING = STG + kTile;
    static constexpr int STAGE = 2 * NR * kGran;       // Q and dO of one granule
    __host__ __device__ static int xs(int nst) { return RING + nst * STAGE; }
    __host__ __device__ static int ctrl(int nst) { return xs(nst) + nst * kXs; }
    __host__ __device__ static int rows(int nst) { return ctrl(nst) + kCtrl; }
    static int alloc(int nst, int SW) { return rows(nst) + 16 * SW + 1024; }   // 2 slots x 2 rows
    static int stages(int SW) {
        int n = kStages;
        while (n > 2 && alloc(n, SW) > kSmemMax) --n;
        return n;
    }
};

struct BarsKV {
    uint64_t* full0;           // [kStages] Q and dO of a granule landed (two arrivals)
    uint64_t* fullx;           // [kStages] row data landed
    uint64_t* empty;           // [kStages]
    uint64_t* prod;            // [2]
    uint64_t* elem;            // [2] (256 arrivals)
    uint64_t* stat;            // K, V tiles of a non-empty item landed (2 copies)
    uint64_t* kv_free;         // the item's last S^T/dP^T MMAs complete
    uint64_t* fin;
    uint64_t* drain;           // [2] teardown after an abort, per MMA-issuing warp
    uint64_t* kv_done;         // [2] dV/dK MMAs of the buffer's granule complete (its P^T, dS^T read)
    uint64_t* rows_full;       // [2] (32 arrivals)
    uint64_t* rows_empty;      // [2] (8 arrivals: one per elementwise warp)
    uint32_t* tmem_slot;
    volatile int* abort_flag;
};

__device__ __forceinline__ BarsKV carve_kv(uint8_t* ctrl) {
    uint64_t* b = reinterpret_cast<uint64_t*>(ctrl);
    BarsKV r;
    r.full0 = b;
    r.fullx = b + 2 * kStages;
    r.empty = b + 3 * kStages;
    r.prod = b + 4 * kStages;
    r.elem = b + 4 * kStages + 2;
    r.stat = b + 4 * kStages + 4;
    r.kv_free = b + 4 * kStages + 5;
    r.fin = b + 4 * kStages + 6;
    r.drain = b + 4 * kStages + 7;
    r.rows_full = b + 4 * kStages + 9;
    r.rows_empty = b + 4 * kStages + 11;
    r.kv_done = b + 4 * kStages + 13;
    r.tmem_slot = reinterpret_cast<uint32_t*>(b + 4 * kStages + 15);
    r.abort_flag = reinterpret_cast<volatile int*>(r.tmem_slot + 1);
    return r;
}
static_assert((4 * kStages + 15) * 8 + 8 <= kCtrl, "barriers overflow the control block");

// DS: the elementwise warps also store the dS^T blocks (pieces, ds_handoff.cuh)
// when *ds.on is set
template <int D, bool RASTER, bool DS = false>
__global__ void __launch_bounds__(384, 1)
k_bwd_dkdv_persist(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                   const __grid_constant__ CUtensorMap tmdK1, const __grid_constant__ CUtensorMap tmdV1,
                   const __grid_constant__ CUtensorMap tmPkv1,
                   const __grid_constant__ BwdRasterMaps<RASTER, 6> rmaps, BwdRaster ras,
                   const uint32_t* __restrict__ gselT, const PlanHeader* __restrict__ hdr,
                   const int4* __restrict__ items, const float* __restrict__ nld,
                   int64_t N, int64_t MB, int SW, int nst, float scale, uint32_t* __restrict__ dev_status,
                   DsDev ds) {
    using L = DkvpLayout<D>;
    constexpr int kRL = RASTER ? L::NR : 1;            // copy lanes per (stream, stage)
    constexpr int kStatLanes = RASTER ? 2 * 2 * L::NR : 2;   // stationary copies: (tensor, granule, region)
    constexpr uint32_t cdK = 0, cdV = 128, cS = 256, cP = 320;   // + 128 * buffer for S^T / dP^T
    const int n_items = hdr->n_items;
    if ((int)blockIdx.x >= n_items) return;
    const int tiles_per_head = (int)(N / 128);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BarsKV B = carve_kv(sm + L::ctrl(nst));
    uint8_t* xs = sm + L::xs(nst);
    uint32_t* rows_base = reinterpret_cast<uint32_t*>(sm + L::rows(nst));
    uint8_t* staging = sm + L::STG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wn = SW;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(B.full0 + s, 2 * kRL);           // each Q and dO copy lane arrives
            mbar_init(B.fullx + s, 1);
            mbar_init(B.empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(B.prod + b, 1);
            mbar_init(B.elem + b, 256);
            mbar_init(B.rows_full + b, 32);
            mbar_init(B.rows_empty + b, 8);
            mbar_init(B.kv_done + b, 1);
            mbar_init(B.drain + b, 1);
        }
        mbar_init(B.stat, kStatLanes);
        mbar_init(B.kv_free, 1);
        mbar_init(B.fin, 1);
        *B.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *B.tmem_slot;

    if (warp < 4) {
      regs_dec<kRegsLow>();
      if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // lanes (kind * nst + stage) * kRL + region stream Q (kind 0) and dO
        // (kind 1) of the ring, one 64-column region each in the raster layout;
        // the next nst lanes the granules' row data (kind 2); the top kStatLanes
        // lanes load the stationary K and V tiles of each non-empty item once the
        // previous one's S^T/dP^T MMAs are done (copies of one thread complete
        // one after another, so each copy has a lane)
        const int nqd = 2 * nst * kRL;                     // Q and dO copy lanes
        const int kind = lane < nqd ? lane / (nst * kRL) : 2;
        const int stage = lane < nqd ? (lane / kRL) % nst : lane - nqd;
        const int region = lane < nqd ? lane % kRL : 0;
        const bool copier = lane < nqd + nst;
        const int si = lane - (32 - kStatLanes);           // stationary copy index
        const bool stat_lane = si >= 0;
        uint64_t* full = kind < 2 ? B.full0 : B.fullx;     // Q and dO share one barrier per stage
        const CUtensorMap* mg = kind == 0 ? &tmQ : &tmdO;
        if (copier && kind < 2 && !RASTER) tma_prefetch_desc(mg);
        bool ok = true;
        int last_cyc = -1;
        int last_stat = -1;                                // index of the last stationary copy issued
        int st0 = 0, cyc0 = 0;
        int kq = 0;                                        // non-empty items so far
        for (int it = blockIdx.x, j = 0; it < n_items; it += gridDim.x, ++j) {
            const int4 item = items[it];
            const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
            const int g_begin = item.y, ng = item.z - item.y;
            const int64_t row0 = (int64_t)hh * N;
            uint32_t* u0 = rows_base + (j & 1) * 2 * SW;
            uint32_t* u1 = u0 + SW;
            if (ok && j >= 2) ok = mbar_wait(B.rows_empty + (j & 1), ((j >> 1) - 1) & 1, B.abort_flag, dev_status);
            if (ok) {
                const uint32_t* s0 = gselT + ((int64_t)hh * MB + 2 * tile) * SW;
                for (int w = lane; w < wn; w += 32) {
                    u0[w] = s0[w];
                    u1[w] = s0[SW + w];
                }
            }
            mbar_arrive(B.rows_full + (j & 1));
            __syncwarp();
            if (ng > 0) {
                if (stat_lane && ok) {
                    if (kq >= 1) ok = mbar_wait(B.kv_free, (uint32_t)(kq - 1) & 1, B.abort_flag, dev_status);
                    if (ok) {
                        if constexpr (RASTER) {
                            // copy si: tensor si / (2 NR), key granule (si / NR) % 2, region si % NR
                            const int tens = si / (2 * L::NR), hg = (si / L::NR) % 2, r = si % L::NR;
                            const int4 gp = ras.gpos[2 * tile + hg];
                            mbar_expect_tx(B.stat, kGran);
                            tma_load_5d(sm + (tens ? L::A1 : L::A0) + r * kTile + hg * kGran,
                                        rmaps.m + (tens ? kRV : kRK) * kRasterKinds + gp.w, B.stat, 0, hh * L::NR + r,
                                        gp.z, gp.y, gp.x);
                        } else {
                            mbar_expect_tx(B.stat, L::NR * kTile);
                            tma_load_3d(sm + (si ? L::A1 : L::A0), si ? &tmV : &tmK, B.stat, 0,
                                        (int)(row0 + 128 * tile), 0);
                        }
                        last_stat = kq;
                    }
                }
                ++kq;
            }
            int s_ = st0, c_ = cyc0;
            if (copier && ok) {
                GranuleWalk walk;
                walk.init(u0, u1, wn);
                walk.skip(g_begin);
                for (int g = 0; g < ng; ++g) {
                    int row;
                    uint32_t m;
                    walk.next(row, m);
                    if (s_ == stage) {
                        if (c_ >= 1 && !mbar_wait(B.empty + stage, (uint32_t)(c_ - 1) & 1, B.abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        if (kind == 2) {
                            mbar_expect_tx(full + stage, kXs);
                            bulk_load(xs + stage * kXs, nld + ((row0 + row) >> 6) * 128, kXs, full + stage);
                        } else {
                            uint8_t* dst = sm + L::RING + stage * L::STAGE + kind * L::NR * kGran;
                            if constexpr (RASTER) {
                                const int4 gp = ras.gpos[row >> 6];
                                mbar_expect_tx(full + stage, kGran);
                                tma_load_5d(dst + region * kGran,
                                            rmaps.m + (kind ? kRdO : kRQ) * kRasterKinds + gp.w, full + stage, 0,
                                            hh * L::NR + region, gp.z, gp.y, gp.x);
                            } else {
                                mbar_expect_tx(full + stage, L::NR * kGran);
                                tma_load_3d(dst, mg, full + stage, 0, (int)(row0 + row), 0);
                            }
                            }
                        last_cyc = c_;
                    }
                    if (++s_ == nst) { s_ = 0; ++c_; }
                }
            }
            __syncwarp();
            if (*B.abort_flag) ok = false;
            const int tot = st0 + ng;
            cyc0 += tot / nst;
            st0 = tot % nst;
        }
        if (!ok && copier && last_cyc >= 0) {
            volatile int no_abort = 0;
            mbar_wait(full + stage, (uint32_t)last_cyc & 1, &no_abort, dev_status);
        }
        // a stationary copy in flight lands before the CTA goes away
        if (!ok && stat_lane && last_stat >= 0) {
            volatile int no_abort = 0;                     // bounded: the other lane's copy may be missing
            mbar_wait(B.stat, (uint32_t)last_stat & 1, &no_abort, dev_status);
        }
      } else if (warp == 1 || warp == 2) {
        // ---------------------------------------------------------------- MMA, two warps
        // Two accumulation chains, each issued in order by one warp (whole warp,
        // elected issue): warp 1 S^T = K Q^T and dP^T = V dO^T, warp 2 dV += P^T dO
        // and dK += dS^T Q, so that one warp's waits leave the other's MMAs in the
        // tensor pipe.  Per TMEM buffer b and its u-th use (granule GG, b = GG & 1,
        // u = GG >> 1): S^T/dP^T(GG) wait kv_done(b) of use u - 1 (the previous
        // granule's P^T and dS^T in those columns read), dV/dK(GG) wait elem(b) of
        // use u.  No barrier can run two phases ahead of its waiter: every phase
        // needs the waiter's own earlier issue.
        const int role = warp - 1;                         // 0: S^T, dP^T; 1: dV, dK
        const uint32_t idPS = idesc_bf16_f32(128, 64, false, false);
        const uint32_t idKV = idesc_bf16_f32(128, D, false, true);
        const uint32_t aR = smem_u32(sm + L::RING);
        const uint64_t dKs = sdesc_sw128(smem_u32(sm + L::A0), 16, 1024);   // stationary K, V tiles
        const uint64_t dVs = sdesc_sw128(smem_u32(sm + L::A1), 16, 1024);
        bool ok = true;
        int G = 0, s_ = 0, c_ = 0, kq = 0;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            const int4 item = items[it];
            const int ng = item.z - item.y;
            if (ng == 0) continue;
            if (role == 0) {
                ok = mbar_wait_w(B.stat, kq & 1, B.abort_flag, dev_status);
                if (!ok) break;
                tc_fence_after();
            }
            for (int g = 0; g < ng; ++g) {
                const int GG = G + g;
                const int s = s_, b = GG & 1, u = GG >> 1;
                const uint32_t ph = (uint32_t)c_ & 1;
                if (++s_ == nst) { s_ = 0; ++c_; }
                if (role == 0) {
                    if (!mbar_wait_w(B.full0 + s, ph, B.abort_flag, dev_status) ||
                        (GG >= 2 && !mbar_wait_w(B.kv_done + b, (uint32_t)(u - 1) & 1, B.abort_flag, dev_status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dQ = sdesc_sw128(aR + s * L::STAGE, 16, 1024);
                    const uint64_t ddO = sdesc_add(dQ, L::NR * kGran);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ss_w(tb + cS + 128 * b, sdesc_add(dKs, kmaj_off(k, kTile)), sdesc_add(dQ, kmaj_off(k, kGran)),
                                 idPS, k > 0);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ss_w(tb + cP + 128 * b, sdesc_add(dVs, kmaj_off(k, kTile)),
                                 sdesc_add(ddO, kmaj_off(k, kGran)), idPS, k > 0);
                    tc_commit_w(B.prod + b);
                    if (g == ng - 1) tc_commit_w(B.kv_free);   // K and V no longer read by this item
                } else {
                    if (!mbar_wait_w(B.elem + b, (uint32_t)u & 1, B.abort_flag, dev_status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dQn = sdesc_sw128(aR + s * L::STAGE, kGran, 1024);
                    const uint64_t ddOn = sdesc_add(dQn, L::NR * kGran);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {            // queries 16 k ..: warpgroup k / 2's columns
                        const uint32_t acc = (g > 0 || k > 0) ? 1u : 0u;
                        const uint32_t ck = 128 * b + 32 * (k >> 1) + 8 * (k & 1);
                        mma_ts_w(tb + cdV, tb + cS + ck, sdesc_add(ddOn, k * 2048), idKV, acc);
                        mma_ts_w(tb + cdK, tb + cP + ck, sdesc_add(dQn, k * 2048), idKV, acc);
                    }
                    tc_commit_w(B.empty + s);
                    tc_commit_w(B.kv_done + b);
                }
            }
            if (!ok) break;
            if (role == 1) tc_commit_w(B.fin);
            G += ng;
            ++kq;
        }
        if (!ok) {
            tc_commit_w(B.drain + role);                   // every MMA this warp issued complete
            volatile int no_abort = 0;
            mbar_wait(B.drain + role, 0, &no_abort, dev_status);
        }
      }
    } else {
        regs_inc<kRegsHigh>();
        // Both warpgroups on every granule, warpgroup wg on query columns 32 wg ..
        // 32 wg + 31 of S^T and dP^T; it writes P^T and dS^T as bf16 over the first
        // 16 of its own columns, so no barrier joins the two per granule.  Every
        // thread runs every named barrier of the epilogue.
        const int wg = (warp - 4) >> 2;
        const int sub = warp & 3, row = sub * 32 + lane, half = row >> 6;
        const uint32_t tl = tb + ((uint32_t)(sub * 32) << 16);
        const float sl2 = scale * kLog2e;
        const uint64_t sl2x2 = f2pack(sl2, sl2);
        bool ok = true;
        int G = 0, kf = 0;
        int st_ = 0, cy_ = 0;                              // ring stage and cycle of granule G
        bool ds_live = false;
        if constexpr (DS) ds_live = *ds.on != 0;
        for (int it = blockIdx.x, j = 0; it < n_items; it += gridDim.x, ++j) {
            const int4 item = items[it];
            const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
            const int g_begin = item.y, ng = item.z - item.y, slot = item.w;
            const int64_t row0 = (int64_t)hh * N;
            // this thread's 64 bytes (key `row`, queries 32 wg ..) of the item's first piece
            uint8_t* ds_row = nullptr;
            if constexpr (DS) {
                if (ds_live && ng > 0)
                    ds_row = reinterpret_cast<uint8_t*>(ds.pieces) +
                             ds::piece_row_offset(ds.base_kv[item.x], g_begin, row) + 64 * wg;
            }
            const uint32_t* u0 = rows_base + (j & 1) * 2 * SW;
            GranuleWalk walk;
            if (lane == 0) {
                const bool got = ok && mbar_wait(B.rows_full + (j & 1), (j >> 1) & 1, B.abort_flag, dev_status);
                walk.init(u0, u0 + SW, got ? wn : 0);
                if (got) walk.skip(g_begin);
                ok = got;
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int g = 0; g < ng; ++g) {
                const int GG = G + g;
                const int b = GG & 1;
                const int st = st_;
                const uint32_t cph = (uint32_t)cy_ & 1;
                if (++st_ == nst) { st_ = 0; ++cy_; }
                uint32_t mk = 0;
                int qrow = 0;
                if (lane == 0) walk.next(qrow, mk);
                mk = __shfl_sync(0xffffffffu, mk, 0);
                const bool valid = (mk >> half) & 1u;
                const float4* nl4 = reinterpret_cast<const float4*>(xs + st * kXs) + 8 * wg;
                const float4* nd4 = nl4 + 16;
                if (ok)
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(B.prod + b, (uint32_t)(GG >> 1) & 1, B.abort_flag, dev_status) &&
                                        mbar_wait(B.fullx + st, cph, B.abort_flag, dev_status));
                uint32_t sv[32], pv[32];
                if (ok) {
                    tc_fence_after();
                    if (valid) {
                        tmem_ld32(tl + cS + 128 * b + 32 * wg, sv);
                        tmem_ld32(tl + cP + 128 * b + 32 * wg, pv);
                    }
                    tmem_wait_ld();
                }
                if (!ok) continue;
                uint32_t op[16], od[16];
                if (valid) {
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 l4 = nl4[i4];
                        const float4 d4 = nd4[i4];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int i = 4 * i4 + 2 * u;
                            const uint64_t nl = u ? f2pack(l4.z, l4.w) : f2pack(l4.x, l4.y);
                            const uint64_t nd = u ? f2pack(d4.z, d4.w) : f2pack(d4.x, d4.y);
                            float x0, x1;
                            f2unpack(ffma2(f2pack(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), sl2x2, nl), x0,
                                     x1);
                            const float p0 = ex2(x0), p1 = ex2(x1);
                            float d0, d1;
                            f2unpack(fmul2(f2pack(p0, p1),
                                           fadd2(f2pack(__uint_as_float(pv[i]), __uint_as_float(pv[i + 1])), nd)),
                                     d0, d1);
                            op[2 * i4 + u] = pack_bf16x2(p0, p1);
                            od[2 * i4 + u] = pack_bf16x2(d0, d1);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) { op[i] = 0u; od[i] = 0u; }
                }
                if constexpr (DS) {
                    // the piece's unread halves (a key granule this query granule did
                    // not select) are never stored: the look-up sends those to piece 0
                    if (ds_row && valid) {
                        uint4* dst = reinterpret_cast<uint4*>(ds_row + (int64_t)g * ds::kPieceBytes);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            __stcs(dst + k, make_uint4(od[4 * k], od[4 * k + 1], od[4 * k + 2], od[4 * k + 3]));
                    }
                }
                tmem_st16(tl + cS + 128 * b + 32 * wg, op);       // over this warpgroup's own S^T columns
                tmem_st16(tl + cP + 128 * b + 32 * wg, od);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(B.elem + b);
            }
            if (lane == 0) mbar_arrive(B.rows_empty + (j & 1));
            bool fin = ok;
            if (ng > 0) {
                fin = __all_sync(0xffffffffu, ok && mbar_wait(B.fin, kf & 1, B.abort_flag, dev_status));
                if (fin) tc_fence_after();
                ++kf;
            }
            ok = fin;
            // epilogue: dK (warpgroup 0) then dV (warpgroup 1), one 128-row region a pass
            const bool part = slot >= 0, zero = ng == 0;
            const int regions = part ? D / 32 : D / 64;
            const uint32_t sw = (uint32_t)(row & 7);
#pragma unroll 1
            for (int out = 0; out < 2; ++out) {
#pragma unroll 1
                for (int r = 0; r < regions; ++r) {
                    named_sync(2, 256);                    // the previous store has read the staging
                    if (ok && wg == out) {
                        const float mul = out ? 1.f : scale;
                        const uint32_t tacc = tl + (out ? cdV : cdK);
                        // bf16: region r = TMEM columns 64 r .. 64 r + 63; fp32: 32 r .. 32 r + 31
                        const int nq = part ? 1 : 2;
#pragma unroll 1
                        for (int qq = 0; qq < nq; ++qq) {
                            const int q = part ? r : 2 * r + qq;
                            uint32_t v[32];
                            if (zero) {
#pragma unroll
                                for (int i = 0; i < 32; ++i) v[i] = 0u;
                            } else {
                                tmem_ld32(tacc + 32 * q, v);
                                tmem_wait_ld();
                            }
                            if (!part) {
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const int c = 4 * qq + k;              // 16-byte chunk within the region
                                    uint4 w4;
                                    w4.x = pack_bf16x2(__uint_as_float(v[8 * k + 0]) * mul, __uint_as_float(v[8 * k + 1]) * mul);
                                    w4.y = pack_bf16x2(__uint_as_float(v[8 * k + 2]) * mul, __uint_as_float(v[8 * k + 3]) * mul);
                                    w4.z = pack_bf16x2(__uint_as_float(v[8 * k + 4]) * mul, __uint_as_float(v[8 * k + 5]) * mul);
                                    w4.w = pack_bf16x2(__uint_as_float(v[8 * k + 6]) * mul, __uint_as_float(v[8 * k + 7]) * mul);
                                    *reinterpret_cast<uint4*>(staging + row * 128 + ((c ^ sw) << 4)) = w4;
                                }
                            } else {
#pragma unroll
                                for (int k = 0; k < 8; ++k) {
                                    const float4 w4 = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                                                  __uint_as_float(v[4 * k + 2]),
                                                                  __uint_as_float(v[4 * k + 3]));
                                    *reinterpret_cast<float4*>(staging + row * 128 + ((k ^ sw) << 4)) = w4;
                                }
                            }
                        }
                        fence_proxy_async_smem();
                    }
                    named_sync(2, 256);
                    // lane 0 of the warpgroup's first warp stores; in the raster layout
                    // lanes 0 and 1 store the region's two key granules
                    if (ok && wg == out && (warp & 3) == 0 && (lane == 0 || (RASTER && !part && lane == 1))) {
                        if (part) {
                            tma_store_3d(&tmPkv1, staging, 0, (slot * 2 + out) * 128, r);
                        } else if constexpr (RASTER) {
                            const int4 gp = ras.gpos[2 * tile + lane];
                            tma_store_5d(rmaps.m + (out ? kRdV : kRdK) * kRasterKinds + gp.w, staging + lane * kGran, 0,
                                         hh * L::NR + r, gp.z, gp.y, gp.x);
                        } else {
                            tma_store_3d(out ? &tmdV1 : &tmdK1, staging, 0, (int)(row0 + 128 * tile), r);
                        }
                        bulk_commit();
                        bulk_wait_read();
                    }
                }
            }
            G += ng;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, kTmemCols);
}

// ============================================================================ dS handoff
// Set-up kernels of the handoff (index arithmetic in ds_handoff.cuh), run after
// the two work plans and before the backward kernels:
//   k_ds_bases    one CTA: base_q, base_kv (exclusive prefix sums of the plans'
//                 per-tile units) and the gate `on`
//   k_ds_prefix   one warp per key tile: word prefixes of its gselT union
//   k_ds_entries  one warp per query tile: an entry per key granule of its walk
__global__ void __launch_bounds__(1024) k_ds_bases(const int32_t* __restrict__ units_q,
                                                   const int32_t* __restrict__ units_kv, int64_t tiles,
                                                   const PlanHeader* __restrict__ hq,
                                                   const PlanHeader* __restrict__ hkv, int64_t cap_units,
                                                   int64_t cap_q, DsDev ds) {
    __shared__ long long wsum[2][32];
    __shared__ long long carry[2];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    if (tid == 0) {
        carry[0] = carry[1] = 0;
        *ds.on = ((long long)hkv->total_units <= cap_units && (long long)hq->total_units <= cap_q) ? 1 : 0;
    }
    __syncthreads();
    for (int64_t base = 0; base < tiles; base += blockDim.x) {
        const int64_t t = base + tid;
        const long long v0 = t < tiles ? units_q[t] : 0, v1 = t < tiles ? units_kv[t] : 0;
        long long a = v0, b = v1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
            if (lane >= o) { a += x; b += y; }
        }
        if (lane == 31) { wsum[0][wid] = a; wsum[1][wid] = b; }
        __syncthreads();
        if (wid == 0) {
            long long x = lane < nw ? wsum[0][lane] : 0, y = lane < nw ? wsum[1][lane] : 0;
            const long long x0 = x, y0 = y;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long p = __shfl_up_sync(0xffffffffu, x, o), q = __shfl_up_sync(0xffffffffu, y, o);
                if (lane >= o) { x += p; y += q; }
            }
            if (lane < nw) { wsum[0][lane] = x - x0; wsum[1][lane] = y - y0; }
        }
        __syncthreads();
        if (t < tiles) {
            ds.base_q[t] = carry[0] + wsum[0][wid] + a - v0;
            ds.base_kv[t] = carry[1] + wsum[1][wid] + b - v1;
        }
        __syncthreads();
        if (tid == blockDim.x - 1) {
            carry[0] += wsum[0][wid] + a;
            carry[1] += wsum[1][wid] + b;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(256) k_ds_prefix(const uint32_t* __restrict__ gselT, int64_t MB, int64_t SW,
                                                   int64_t tph, int heads, DsDev ds) {
    if (!*ds.on) return;
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= tph * heads) return;                          // whole warps
    const int64_t r = (t / tph) * MB + 2 * (t % tph);       // the key tile's first gselT row
    int carry = 0;
    for (int64_t w0 = 0; w0 < SW; w0 += 32) {
        const int64_t w = w0 + lane;
        const int x = w < SW ? ds::popc32(ds::union_word(gselT, r, SW, w)) : 0;
        int inc = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (w < SW) ds.pre[t * SW + w] = carry + inc - x;
        carry += __shfl_sync(0xffffffffu, inc, 31);
    }
}

__global__ void __launch_bounds__(256) k_ds_entries(const uint32_t* __restrict__ gsel,
                                                    const uint32_t* __restrict__ gselT, int64_t MB, int64_t SW,
                                                    int64_t tph, int heads, DsDev ds) {
    if (!*ds.on) return;
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= tph * heads) return;
    const int hh = (int)(t / tph);
    const int64_t tq = t % tph, r = (int64_t)hh * MB + 2 * tq;
    int64_t j = ds.base_q[t];                               // entry of the walk's next granule
    for (int64_t w0 = 0; w0 < SW; w0 += 32) {
        const int64_t w = w0 + lane;
        uint32_t bits = w < SW ? ds::union_word(gsel, r, SW, w) : 0u;
        const int x = ds::popc32(bits);
        int inc = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        int64_t e = j + inc - x;
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            int32_t o4[4];
            ds::make_entry(gsel, gselT, ds.pre, ds.base_kv, hh, MB, SW, tph, tq, (int)(32 * w + b), o4);
            ds.entries[e++] = make_int4(o4[0], o4[1], o4[2], o4[3]);
        }
        j += __shfl_sync(0xffffffffu, inc, 31);
    }
}

// ============================================================================ dQ from stored dS (persistent)
// With the handoff the query-stationary pass is one GEMM per key granule,
// dQ += dS K: dS as two 64 x 64 blocks of stored dS^T (the MN-major A operand,
// queries contiguous), K a whole-row granule (the MN-major B operand).  One CTA
// per SM over the same plan items as k_bwd_dq_persist; the accumulator is
// double-buffered in TMEM so that the next item's MMAs run during this item's
// epilogue.
//   warp 0      copies: a lane per (stage, K region) and per (stage, query
//               granule half); each lane reads the entries of its own stage's
//               granules, so no selection rows are needed
//   warp 1      TMEM allocation and MMA issue (4 MMAs of K = 16 a granule)
//   warps 2-9   epilogue (store_tile_p), warpgroup wg on accumulator columns
//               D/2 wg .. D/2 wg + D/2 - 1
// Per non-empty item k (buffer b = k & 1): fin(b) completes when the item's
// MMAs have; acc_free(b) when the epilogue has read the buffer (256
// arrivals).  The MMA warp waits acc_free(b) of item k - 2 before the first
// MMA of item k, and the epilogue waits fin(b) of item k only after its own
// arrival for item k - 2, so neither barrier runs two phases ahead of its waiter.
template <int D>
struct DqdLayout {
    static constexpr int NR = D / 64;
    static constexpr int STAGE = NR * kGran + 2 * kGran;   // K granule, then dS^T of the two query granules
    __host__ __device__ static int staging(int nst) { return nst * STAGE; }
    __host__ __device__ static int ctrl(int nst) { return staging(nst) + kStagingP; }
    static int alloc(int nst) { return ctrl(nst) + kCtrl + 1024; }
    static int stages(int lanes_per_stage) {
        int n = kStages;
        while (n > 2 && (alloc(n) > kSmemMax || n * lanes_per_stage > 32)) --n;
        return n;
    }
};

struct BarsD {
    uint64_t* full;            // [kStages] K and both dS^T blocks of a granule landed
    uint64_t* empty;           // [kStages]
    uint64_t* fin;             // [2]
    uint64_t* acc_free;        // [2]
    uint64_t* drain;
    uint32_t* tmem_slot;
    volatile int* abort_flag;
};

__device__ __forceinline__ BarsD carve_d(uint8_t* ctrl) {
    uint64_t* b = reinterpret_cast<uint64_t*>(ctrl);
    BarsD r;
    r.full = b;
    r.empty = b + kStages;
    r.fin = b + 2 * kStages;
    r.acc_free = b + 2 * kStages + 2;
    r.drain = b + 2 * kStages + 4;
    r.tmem_slot = reinterpret_cast<uint32_t*>(b + 2 * kStages + 5);
    r.abort_flag = reinterpret_cast<volatile int*>(r.tmem_slot + 1);
    return r;
}
static_assert((2 * kStages + 5) * 8 + 8 <= kCtrl, "barriers overflow the control block");

template <int D, bool RASTER>
__global__ void __launch_bounds__(320, 1)
k_bwd_dq_ds(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmS,
            const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmPqh,
            const __grid_constant__ BwdRasterMaps<RASTER, 3> rmaps, BwdRaster ras, DsDev ds,
            const PlanHeader* __restrict__ hdr, const int4* __restrict__ items, int64_t N, int nst, float scale,
            uint32_t* __restrict__ dev_status) {
    using L = DqdLayout<D>;
    constexpr int kRL = RASTER ? L::NR : 1;                // K copy lanes per stage
    constexpr uint32_t kCols = 2 * D;                      // two accumulators
    if (!*ds.on) return;                                   // uniform: k_bwd_dq_persist does the work
    const int n_items = hdr->n_items;
    if ((int)blockIdx.x >= n_items) return;
    const int tiles_per_head = (int)(N / 128);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BarsD B = carve_d(sm + L::ctrl(nst));
    uint8_t* staging = sm + L::staging(nst);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(B.full + s, kRL + 2);                // every K and dS^T copy lane arrives
            mbar_init(B.empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(B.fin + b, 1);
            mbar_init(B.acc_free + b, 256);
        }
        mbar_init(B.drain, 1);
        *B.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(B.tmem_slot, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *B.tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // lanes stage * kRL + region copy K; lanes nst * kRL + 2 * stage + h copy
        // the dS^T block of query granule h
        const int nk = nst * kRL;
        const bool is_k = lane < nk;
        const int stage = is_k ? lane / kRL : (lane - nk) >> 1;
        const int part = is_k ? lane % kRL : (lane - nk) & 1;  // K region or query granule
        const bool copier = lane < nk + 2 * nst;
        if (copier) {
            if (!is_k) tma_prefetch_desc(&tmS);
            else if (!RASTER) tma_prefetch_desc(&tmK);
        }
        bool ok = true;
        int last_cyc = -1;
        int st0 = 0, cyc0 = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int4 item = items[it];
            const int hh = item.x / tiles_per_head;
            const int ng = item.z - item.y;
            const int64_t row0 = (int64_t)hh * N;
            int s_ = st0, c_ = cyc0;
            if (copier && ok && ng > 0) {
                const int4* ent = ds.entries + ds.base_q[item.x] + item.y;
                for (int g = 0; g < ng; ++g) {
                    if (s_ == stage) {
                        const int4 e = ent[g];             // read before the wait
                        if (c_ >= 1 && !mbar_wait(B.empty + stage, (uint32_t)(c_ - 1) & 1, B.abort_flag, dev_status)) {
                            ok = false;
                            break;
                        }
                        uint8_t* dst = sm + stage * L::STAGE;
                        if (is_k) {
                            if constexpr (RASTER) {
                                const int4 gp = ras.gpos[e.x >> 6];
                                mbar_expect_tx(B.full + stage, kGran);
                                tma_load_5d(dst + part * kGran, rmaps.m + kRK * kRasterKinds + gp.w, B.full + stage, 0,
                                            hh * L::NR + part, gp.z, gp.y, gp.x);
                            } else {
                                mbar_expect_tx(B.full + stage, L::NR * kGran);
                                tma_load_3d(dst, &tmK, B.full + stage, 0, (int)(row0 + e.x), 0);
                            }
                        } else {
                            mbar_expect_tx(B.full + stage, kGran);
                            tma_load_2d(dst + (L::NR + part) * kGran, &tmS, B.full + stage, 0, part ? e.z : e.y);
                        }
                        last_cyc = c_;
                    }
                    if (++s_ == nst) { s_ = 0; ++c_; }
                }
            }
            __syncwarp();
            if (*B.abort_flag) ok = false;
            const int tot = st0 + ng;                      // every lane advances the ring position
            cyc0 += tot / nst;
            st0 = tot % nst;
        }
        if (!ok && copier && last_cyc >= 0) {
            volatile int no_abort = 0;                     // let this lane's last copy land
            mbar_wait(B.full + stage, (uint32_t)last_cyc & 1, &no_abort, dev_status);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        const uint32_t idQ = idesc_bf16_f32(128, D, true, true);
        const uint32_t aR = smem_u32(sm);
        bool ok = true;
        int s_ = 0, c_ = 0, kq = 0;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            const int4 item = items[it];
            const int ng = item.z - item.y;
            if (ng == 0) continue;
            const int b = kq & 1;
            if (kq >= 2) {
                if (!mbar_wait_w(B.acc_free + b, (uint32_t)((kq >> 1) - 1) & 1, B.abort_flag, dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            for (int g = 0; g < ng; ++g) {
                const int s = s_;
                const uint32_t ph = (uint32_t)c_ & 1;
                if (++s_ == nst) { s_ = 0; ++c_; }
                if (!mbar_wait_w(B.full + s, ph, B.abort_flag, dev_status)) { ok = false; break; }
                tc_fence_after();
                const uint64_t dK = sdesc_sw128(aR + s * L::STAGE, kGran, 1024);
                const uint64_t dS = sdesc_sw128(aR + s * L::STAGE + L::NR * kGran, kGran, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k)                // keys 16 k .. 16 k + 15
                    mma_ss_w(tb + D * b, sdesc_add(dS, k * 2048), sdesc_add(dK, k * 2048), idQ,
                             (g > 0 || k > 0) ? 1u : 0u);
                tc_commit_w(B.empty + s);
            }
            if (!ok) break;
            tc_commit_w(B.fin + b);
            ++kq;
        }
        if (!ok) {
            tc_commit_w(B.drain);                          // every MMA this warp issued complete
            volatile int no_abort = 0;
            mbar_wait(B.drain, 0, &no_abort, dev_status);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int wg = (warp - 2) >> 2;
        const int sub = warp & 3, row = sub * 32 + lane;
        const uint32_t tl = tb + ((uint32_t)(sub * 32) << 16);
        bool ok = true;
        int kq = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int4 item = items[it];
            const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
            const int ng = item.z - item.y, slot = item.w;
            const int64_t row0 = (int64_t)hh * N;
            const int b = kq & 1;
            if (ng > 0) {
                ok = __all_sync(0xffffffffu, ok && mbar_wait(B.fin + b, (uint32_t)(kq >> 1) & 1, B.abort_flag, dev_status));
                if (ok) tc_fence_after();
            }
            // the item's dQ (or zeros when nothing was selected: ng == 0)
            if constexpr (RASTER)
                store_tile_p<D>(tl + D * b, row, wg, ok, ng == 0, slot >= 0, scale, staging, &tmdQ, &tmPqh,
                                (int)(row0 + 128 * tile), slot * 128, 1, 256, warp == 2 && lane < 2 * (D / 64),
                                rmaps.m + kRdQ * kRasterKinds, ras.gpos[2 * tile], ras.gpos[2 * tile + 1],
                                hh * (D / 64), lane);
            else
                store_tile_p<D>(tl + D * b, row, wg, ok, ng == 0, slot >= 0, scale, staging, &tmdQ, &tmPqh,
                                (int)(row0 + 128 * tile), slot * 128, 1, 256, warp == 2 && lane == 0);
            if (ng > 0) {
                tc_fence_before();
                mbar_arrive(B.acc_free + b);
                ++kq;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, kCols);
}

// ------------------------------------------------------------------ host side
// whole-row view of a [rows][d] fp32 tensor (d/32 regions of 32 columns) whose
// box covers `box_regions` regions: the persistent dQ epilogue stores an fp32
// partial tile in passes of two regions
bool make_map_bf16_rows_box(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows, int box_regions) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(d / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, 128};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_regions};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_f32_rows_box(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows, int box_regions) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(d / 32)};
    cuuint64_t strides[2] = {(cuuint64_t)d * 4, 128};
    cuuint32_t box[3] = {32, (cuuint32_t)box_rows, (cuuint32_t)box_regions};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct BwdWs {
    float* delta;
    float* nld;         // [heads*N/64][128]: per 64-row granule -lse*log2(e), then -Delta
    Plan pq, pkv;
    float* part_q;      // [slots][128][D]
    float* part_kv;     // [slots][2][128][D]
    int4* gpos;         // [N/64] granule positions (raster operands only)
};

BwdWs carve_bwd(void* ws, const Dims& d, size_t* total) {
    const int64_t tiles = (int64_t)d.heads * (d.N / 128);
    const int target = plan_target(device_sms());
    const int64_t slots = 2 * (int64_t)target;
    uint8_t* p = static_cast<uint8_t*>(ws);
    BwdWs w;
    w.delta = reinterpret_cast<float*>(p);
    p += align16((int64_t)d.heads * d.N * 4);
    w.nld = reinterpret_cast<float*>(p);
    p += align16((int64_t)d.heads * d.N * 8);
    w.pq = carve_plan(p, tiles, target);
    p += plan_bytes(tiles, target);
    w.pkv = carve_plan(p, tiles, target);
    p += plan_bytes(tiles, target);
    w.part_q = reinterpret_cast<float*>(p);
    p += align16(slots * 128 * d.d * 4);
    w.part_kv = reinterpret_cast<float*>(p);
    p += align16(slots * 2 * 128 * d.d * 4);
    w.gpos = reinterpret_cast<int4*>(p);
    p += align16(d.MB * (int64_t)sizeof(int4));
    if (total) *total = (size_t)(p - static_cast<uint8_t*>(ws));
    return w;
}

// Host view of a dS handoff buffer: [gate 256 B][base_q][base_kv][pre][entries]
// [pieces], the pieces 256-byte aligned: cap_units pieces after the zero piece,
// and cap_q = 2 cap_units entries.  Every selected (query granule, key granule)
// pair lies in exactly one unit of each walk, and a unit holds one or two
// pairs, so the query walk never has more than twice the key walk's units:
// whenever the pieces fit, so do the entries.
struct DsHost {
    DsDev dev;
    int64_t cap_units = 0, cap_q = 0;
};

size_t ds_fixed_bytes(const Dims& d) {
    const int64_t tiles = (int64_t)d.heads * (d.N / 128);
    return 256 + 2 * align16(tiles * 8) + align16(tiles * d.SW * 4) + 256;
}

constexpr int64_t kDsUnitBytes = ds::kPieceBytes + 2 * ds::kEntryBytes;

bool carve_ds(void* buf, size_t bytes, const Dims& d, DsHost* h) {
    const size_t fixed = ds_fixed_bytes(d);
    if (!buf || bytes < fixed + (size_t)(ds::kPieceBytes + kDsUnitBytes)) return false;
    int64_t cap = (int64_t)((bytes - fixed - (size_t)ds::kPieceBytes) / (size_t)kDsUnitBytes);
    if (cap > ds::kMaxPieces) cap = ds::kMaxPieces;
    const int64_t tiles = (int64_t)d.heads * (d.N / 128);
    uint8_t* p = static_cast<uint8_t*>(buf);
    h->dev.on = reinterpret_cast<int*>(p);
    p += 256;
    h->dev.base_q = reinterpret_cast<int64_t*>(p);
    p += align16(tiles * 8);
    h->dev.base_kv = reinterpret_cast<int64_t*>(p);
    p += align16(tiles * 8);
    h->dev.pre = reinterpret_cast<int32_t*>(p);
    p += align16(tiles * d.SW * 4);
    h->dev.entries = reinterpret_cast<int4*>(p);
    p += 2 * cap * ds::kEntryBytes;
    p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 255) & ~uintptr_t(255));
    h->dev.pieces = reinterpret_cast<__nv_bfloat16*>(p);
    h->cap_units = cap;
    h->cap_q = 2 * cap;
    return true;
}

// RASTER: Qp, Kp, Vp, dOp, dQp, dKp, dVp are the raster tensors; perm and
// shape_id give every granule's box (gran_positions, into the workspace)
template <int D, bool RASTER>
prism_status_t launch_bwd(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* dOp,
                          const float* lse, const uint32_t* gsel, const uint32_t* gselT, float scale, void* dQp,
                          void* dKp, void* dVp, uint32_t* dev_status, const BwdWs& w, const int32_t* perm,
                          const uint8_t* shape_id, cudaStream_t s, const DsHost* ds = nullptr) {
    const int64_t rows = (int64_t)d.heads * d.N;
    const int target = plan_target(device_sms());
    const int64_t slots = 2 * (int64_t)target;
    CUtensorMap tK, tV, gQ, gdO, gK, gV, tdQ, tdK1, tdV1, tPqh, tPkv1;
    // fp32 partials of split tiles stay blocked (their slots) in both layouts
    if (!make_map_f32_rows_box(&tPqh, w.part_q, slots * 128, D, 128, D / 32 < 2 ? D / 32 : 2) ||
        !make_map_f32_rows_box(&tPkv1, w.part_kv, slots * 2 * 128, D, 128, 1))
        return PRISM_ERR_CUDA;
    BwdRasterMaps<RASTER, 3> rq;
    BwdRasterMaps<RASTER, 6> rkv;
    BwdRaster ras{nullptr, perm, d.heads};
    if constexpr (RASTER) {
        const void* bq[3] = {Kp, Vp, dQp};
        const void* bkv[6] = {Kp, Vp, Qp, dOp, dKp, dVp};
        for (int k = 0; k < kRasterKinds; ++k) {
            for (int t = 0; t < 3; ++t)
                if (!make_map_raster(&rq.m[t * kRasterKinds + k], bq[t], d.heads, D, d.T, d.H, d.W, k))
                    return PRISM_ERR_CUDA;
            for (int t = 0; t < 6; ++t)
                if (!make_map_raster(&rkv.m[t * kRasterKinds + k], bkv[t], d.heads, D, d.T, d.H, d.W, k))
                    return PRISM_ERR_CUDA;
        }
        if (gran_positions(perm, shape_id, d, w.gpos, s) != PRISM_OK) return PRISM_ERR_CUDA;
        ras.gpos = w.gpos;
        tK = tV = gQ = gdO = gK = gV = tdQ = tdK1 = tdV1 = tPqh;      // the blocked maps: never used
    } else {
        if (!make_map_bf16_rows(&tK, Kp, rows, D, 128) || !make_map_bf16_rows(&tV, Vp, rows, D, 128) ||
            !make_map_bf16_rows(&gQ, Qp, rows, D, 64) || !make_map_bf16_rows(&gdO, dOp, rows, D, 64) ||
            !make_map_bf16_rows(&gK, Kp, rows, D, 64) || !make_map_bf16_rows(&gV, Vp, rows, D, 64))
            return PRISM_ERR_CUDA;
        // output maps: dQ whole rows; dK, dV one 128-byte region a box
        if (!make_map_bf16_rows(&tdQ, dQp, rows, D, 128) || !make_map_bf16_rows_box(&tdK1, dKp, rows, D, 128, 1) ||
            !make_map_bf16_rows_box(&tdV1, dVp, rows, D, 128, 1))
            return PRISM_ERR_CUDA;
        rq.m[0] = rkv.m[0] = tPqh;                                      // never used
    }
    prism_status_t st = plan_work(w.pq, gsel, d, 2, 1, target, kSegMinGranules, s);
    if (st == PRISM_OK) st = plan_work(w.pkv, gselT, d, 2, 1, target, kSegMinGranules, s);
    if (st != PRISM_OK) return st;
    const int nq = DqpLayout<D>::stages((int)d.SW), nk = DkvpLayout<D>::stages((int)d.SW);
    const int smq = DqpLayout<D>::alloc(nq, (int)d.SW);
    const int smk = DkvpLayout<D>::alloc(nk, (int)d.SW);
    if (smq > kSmemMax || smk > kSmemMax) return PRISM_ERR_UNSUPPORTED;   // selection rows too long
    const int64_t gq = w.pq.items_max < device_sms() ? w.pq.items_max : device_sms();
    const int64_t gk = w.pkv.items_max < device_sms() ? w.pkv.items_max : device_sms();
    if (!ds) {
        auto kq = k_bwd_dq_persist<D, RASTER, false>;
        auto kk = k_bwd_dkdv_persist<D, RASTER, false>;
        if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smq) != cudaSuccess ||
            cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smk) != cudaSuccess)
            return PRISM_ERR_CUDA;
        // persistent: one CTA per SM (all 512 TMEM columns each), items strided over the CTAs
        kq<<<(unsigned)gq, 384, smq, s>>>((const __nv_bfloat16*)Qp, (const __nv_bfloat16*)dOp, gK, gV, tdQ, tPqh,
                                          rq, ras, gsel, w.pq.hdr, w.pq.items, lse, w.delta, d.N, d.MB, (int)d.SW, nq,
                                          scale, dev_status, nullptr);
        kk<<<(unsigned)gk, 384, smk, s>>>(tK, tV, gQ, gdO, tdK1, tdV1, tPkv1, rkv, ras, gselT, w.pkv.hdr,
                                          w.pkv.items, w.nld, d.N, d.MB, (int)d.SW, nk, scale, dev_status, DsDev{});
        st = launch_status(2);
    } else {
        // dS handoff: the gate and the look-up tables, then dK/dV (storing dS^T),
        // then dQ from the stored dS, or, when the selection does not fit, the
        // recomputing dQ kernel (each of the two exits at once when it is not chosen)
        const int64_t tiles = (int64_t)d.heads * (d.N / 128), tph = d.N / 128;
        const unsigned gw = (unsigned)((tiles * 32 + 255) / 256);
        CUtensorMap tS;
        if (!make_map_bf16(&tS, ds->dev.pieces, (1 + ds->cap_units) * ds::kPieceRows, 64, 64)) return PRISM_ERR_CUDA;
        constexpr int kRLd = RASTER ? D / 64 : 1;
        const int nd = DqdLayout<D>::stages(kRLd + 2);
        const int smd = DqdLayout<D>::alloc(nd);
        auto kq = k_bwd_dq_persist<D, RASTER, true>;
        auto kk = k_bwd_dkdv_persist<D, RASTER, true>;
        auto kd = k_bwd_dq_ds<D, RASTER>;
        if (smd > kSmemMax || cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smq) != cudaSuccess ||
            cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smk) != cudaSuccess ||
            cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, smd) != cudaSuccess)
            return PRISM_ERR_CUDA;
        if (cudaMemsetAsync(ds->dev.pieces, 0, (size_t)ds::kPieceBytes, s) != cudaSuccess) return PRISM_ERR_CUDA;
        k_ds_bases<<<1, 1024, 0, s>>>(w.pq.tile_units, w.pkv.tile_units, tiles, w.pq.hdr, w.pkv.hdr, ds->cap_units,
                                      ds->cap_q, ds->dev);
        k_ds_prefix<<<gw, 256, 0, s>>>(gselT, d.MB, d.SW, tph, d.heads, ds->dev);
        k_ds_entries<<<gw, 256, 0, s>>>(gsel, gselT, d.MB, d.SW, tph, d.heads, ds->dev);
        kk<<<(unsigned)gk, 384, smk, s>>>(tK, tV, gQ, gdO, tdK1, tdV1, tPkv1, rkv, ras, gselT, w.pkv.hdr,
                                          w.pkv.items, w.nld, d.N, d.MB, (int)d.SW, nk, scale, dev_status, ds->dev);
        kq<<<(unsigned)gq, 384, smq, s>>>((const __nv_bfloat16*)Qp, (const __nv_bfloat16*)dOp, gK, gV, tdQ, tPqh,
                                          rq, ras, gsel, w.pq.hdr, w.pq.items, lse, w.delta, d.N, d.MB, (int)d.SW, nq,
                                          scale, dev_status, ds->dev.on);
        kd<<<(unsigned)gq, 320, smd, s>>>(gK, tS, tdQ, tPqh, rq, ras, ds->dev, w.pq.hdr, w.pq.items, d.N, nd, scale,
                                          dev_status);
        st = launch_status(6);
    }
    const int32_t* cperm = RASTER ? perm : nullptr;
    if (st == PRISM_OK) st = bwd_combine(w.pq, d, 1, w.part_q, dQp, scale, nullptr, 0.f, s, cperm);
    if (st == PRISM_OK) st = bwd_combine(w.pkv, d, 2, w.part_kv, dKp, scale, dVp, 1.f, s, cperm);
    return st;
}

}  // namespace

size_t attn_bwd_sm100_ws_bytes(const Dims& d) {
    size_t total = 0;
    carve_bwd(reinterpret_cast<void*>(uintptr_t(256)), d, &total);
    return total;
}

size_t attn_bwd_ds_bytes(const Dims& d, int64_t pieces) {
    return ds_fixed_bytes(d) + (size_t)ds::kPieceBytes + (size_t)pieces * (size_t)kDsUnitBytes;
}

// ds/ds_bytes: a dS handoff buffer (ds_handoff.cuh), or nullptr: S and dP are
// recomputed by the query-stationary kernel
prism_status_t attn_bwd_sm100(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* Op,
                              const float* o_f32, const void* dOp, const float* lse, const uint32_t* gsel,
                              const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp,
                              uint32_t* dev_status, void* ws, cudaStream_t s, void* ds, size_t ds_bytes) {
    BwdWs w = carve_bwd(ws, d, nullptr);
    DsHost dh;
    const DsHost* dsp = carve_ds(ds, ds_bytes, d, &dh) ? &dh : nullptr;
    if (ds && !dsp) return PRISM_ERR_WORKSPACE;
    prism_status_t st = bwd_delta(d, Op, o_f32, dOp, w.delta, lse, w.nld, s, nullptr);
    if (st != PRISM_OK) return st;
    if (d.d == 128)
        return launch_bwd<128, false>(d, Qp, Kp, Vp, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, w,
                                      nullptr, nullptr, s, dsp);
    return launch_bwd<64, false>(d, Qp, Kp, Vp, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, w, nullptr,
                                 nullptr, s, dsp);
}

// raster Q, K, V, dO, dQ, dK, dV ([N][heads][d]); o_f32 and lse in permutation order
prism_status_t attn_bwd_raster(const Dims& d, const void* Q, const void* K, const void* V, const float* o_f32,
                               const void* dO, const float* lse, const int32_t* perm, const uint8_t* shape_id,
                               const uint32_t* gsel, const uint32_t* gselT, float scale, void* dQ, void* dK, void* dV,
                               uint32_t* dev_status, void* ws, cudaStream_t s, void* ds, size_t ds_bytes) {
    BwdWs w = carve_bwd(ws, d, nullptr);
    DsHost dh;
    const DsHost* dsp = carve_ds(ds, ds_bytes, d, &dh) ? &dh : nullptr;
    if (ds && !dsp) return PRISM_ERR_WORKSPACE;
    prism_status_t st = bwd_delta(d, nullptr, o_f32, dO, w.delta, lse, w.nld, s, perm);
    if (st != PRISM_OK) return st;
    if (d.d == 128)
        return launch_bwd<128, true>(d, Q, K, V, dO, lse, gsel, gselT, scale, dQ, dK, dV, dev_status, w, perm, shape_id,
                                     s, dsp);
    return launch_bwd<64, true>(d, Q, K, V, dO, lse, gsel, gselT, scale, dQ, dK, dV, dev_status, w, perm, shape_id, s,
                                dsp);
}

}  // namespace prism
