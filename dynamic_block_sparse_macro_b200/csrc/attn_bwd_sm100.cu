// Stage 7 on sm_100a tensor cores: block-sparse attention backward for bf16.
//
// Chinese reading guide of the Prism paper, FAQ on error propagation: rho, g
// and the block probabilities P_i are constants in the backward; gradients
// flow only through the attention over the selected key-value blocks.  With
// P = exp(s - lse) over the selected keys and Delta = rowsum(dO * O):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),  dQ = scale dS K,
//   dK = scale dS^T Q.
//
// Two kernels, no atomics (deterministic):
//   k_bwd_dq_sm100    query-stationary: per (128-row query tile, head) walk the
//                     key granules of the union of its two granule-level rows;
//                     Q and dO sit in TMEM as bf16; per 64-key granule S = Q K^T
//                     and dP = dO V^T (M=128, N=64, A from TMEM) into TMEM, dS
//                     as bf16 back into TMEM, dQ += dS K (K MN-major in smem).
//   k_bwd_dkdv_sm100  key-stationary: per (128-key tile, head) walk the query
//                     granules whose blocks selected the tile's key blocks (the
//                     transposed granule-level selection); per 64-query granule
//                     S^T = K Q^T and dP^T = V dO^T, then P^T and dS^T as bf16
//                     in TMEM, dV += P^T dO and dK += dS^T Q.
// Both double-buffer the granule products in TMEM so that the tensor core
// works on granule g+1 while four warps do the elementwise step of granule g,
// and stream granules through a TMA ring as deep as shared memory allows.
// Roles: warp 0 TMA (one lane per ring stage and stream, one whole-row copy
// per granule), warp 1 TMEM allocation + MMA issue (the whole warp, one
// elected lane issues), warps 2-5 one tile row per thread.
// Every wait is bounded; a timeout sets PRISM_DEV_TIMEOUT.
#include "attn_plan.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace prism {

using namespace sm100;

prism_status_t bwd_delta(const Dims& d, const void* Op, const float* o_f32, const void* dOp, float* delta,
                         const float* lse, float* nld, cudaStream_t s);

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
// (TMA, MMA) drops to 120 and the two elementwise warpgroups rise to 192
// (128 * (120 + 2 * 192) = 384 * 168)
constexpr uint32_t kRegsLow = 120, kRegsHigh = 192;

// Shared memory: stationary tiles (dK/dV only; the dQ kernel keeps Q and dO
// in TMEM), then a ring of nst granule stages (as many as fit: the TMA latency
// under load is about 4000 cycles, a granule's MMAs take about 800), then
// barriers and the two selection rows.
template <int D, bool STAT>
struct BwdLayout {
    static constexpr int NR = D / 64;
    static constexpr int A0 = 0;                       // stationary operand 1 (K)
    static constexpr int A1 = NR * kTile;              // stationary operand 2 (V)
    static constexpr int RING = STAT ? 2 * NR * kTile : 0;   // streamed granules
    static constexpr int STAGE = 2 * NR * kGran;       // two operands per stage
    // xs: bytes of per-granule row data staged beside each stage (0 or kXs)
    __host__ __device__ static int xs(int nst) { return RING + nst * STAGE; }
    __host__ __device__ static int ctrl(int nst, int xsb) { return xs(nst) + nst * xsb; }
    __host__ __device__ static int rows(int nst, int xsb) { return ctrl(nst, xsb) + kCtrl; }
    static int alloc(int nst, int xsb, int SW) { return rows(nst, xsb) + 8 * SW + 1024; }
    static int stages(int xsb, int SW) {               // deepest ring that fits, at least 2
        int n = kStages;
        while (n > 2 && alloc(n, xsb, SW) > kSmemMax) --n;
        return n;
    }
};

struct Bars {
    uint64_t* stat;            // stationary tiles landed (one arrival per producer)
    uint64_t* full0;           // [kStages] streamed operand 0 of a granule landed
    uint64_t* full1;           // [kStages] streamed operand 1 of a granule landed
    uint64_t* fullx;           // [kStages] row data of a granule landed (dK/dV only)
    uint64_t* empty;           // [kStages] granule stage free
    uint64_t* prod;            // [2] products of a granule in TMEM
    uint64_t* elem;            // [2] elementwise results of a granule in TMEM (128 arrivals)
    uint64_t* fin;             // all MMAs done
    uint32_t* tmem_slot;
    volatile int* abort_flag;
    int* ng_slot;
};

__device__ __forceinline__ Bars carve(uint8_t* ctrl) {
    uint64_t* b = reinterpret_cast<uint64_t*>(ctrl);
    Bars r;
    r.stat = b;
    r.full0 = b + 1;
    r.full1 = b + 1 + kStages;
    r.fullx = b + 1 + 2 * kStages;
    r.empty = b + 1 + 3 * kStages;
    r.prod = b + 1 + 4 * kStages;
    r.elem = b + 3 + 4 * kStages;
    r.fin = b + 5 + 4 * kStages;
    r.tmem_slot = reinterpret_cast<uint32_t*>(b + 6 + 4 * kStages);
    r.abort_flag = reinterpret_cast<volatile int*>(r.tmem_slot + 1);
    r.ng_slot = reinterpret_cast<int*>(r.tmem_slot + 2);
    return r;
}
static_assert((6 + 4 * kStages) * 8 + 12 <= kCtrl, "barriers overflow the control block");

__device__ __forceinline__ void init_bars(const Bars& B, int nst, int stat_arrivals, int elem_arrivals) {
    mbar_init(B.stat, stat_arrivals);
    for (int s = 0; s < nst; ++s) {
        mbar_init(B.full0 + s, 1);
        mbar_init(B.full1 + s, 1);
        mbar_init(B.fullx + s, 1);
        mbar_init(B.empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
        mbar_init(B.prod + b, 1);
        mbar_init(B.elem + b, elem_arrivals);
    }
    mbar_init(B.fin, 1);
    *B.abort_flag = 0;
    fence_mbar_init();
}

// descriptor offsets: K-major operand, k-th 16-element step of the contraction over d
__device__ __forceinline__ uint32_t kmaj_off(int k, int region) { return (k >> 2) * region + (k & 3) * 32; }

// The TMA producer warp.  A copy engine completes the copies issued by one
// thread one after another, so every (ring stage, stream) pair gets a lane of
// its own: lane kind * nst + stage issues stream `kind` (0: operand 0, 1:
// operand 1, 2: the 512 bytes of row data, dK/dV only) of the granules that
// use that stage, one copy per granule, and never has more than one copy in
// flight.  With stationary tiles in shared memory (dK/dV), lanes 0 and nst
// also copy those.
template <int D, bool STAT>
__device__ void produce(const CUtensorMap* m0, const CUtensorMap* m1, const CUtensorMap* g0, const CUtensorMap* g1,
                        const float* nld, uint8_t* xs, uint8_t* sm, const Bars& B, int64_t row0, int tile_row,
                        const uint32_t* u0, const uint32_t* u1, int wn, int g_begin, int ng, int nst,
                        uint32_t* dev_status) {
    using L = BwdLayout<D, STAT>;
    const int lane = threadIdx.x & 31;
    if (lane >= (nld ? 3 : 2) * nst) return;
    const int kind = lane / nst, stage = lane % nst;
    uint64_t* full = kind == 0 ? B.full0 : kind == 1 ? B.full1 : B.fullx;
    const CUtensorMap* mg = kind == 0 ? g0 : g1;
    if (kind < 2) tma_prefetch_desc(mg);
    if (STAT && stage == 0 && kind < 2) {
        const CUtensorMap* ms = kind == 0 ? m0 : m1;
        mbar_expect_tx(B.stat, L::NR * kTile);
        tma_load_3d(sm + (kind ? L::A1 : L::A0), ms, B.stat, 0, (int)(row0 + tile_row), 0);
    }
    GranuleWalk walk;
    walk.init(u0, u1, wn);
    walk.skip(g_begin);
    int last = -1;
    for (int g = 0; g < ng && !*B.abort_flag; ++g) {
        int row;
        uint32_t m;
        walk.next(row, m);
        if (g % nst != stage) continue;
        if (g >= nst && !mbar_wait(B.empty + stage, ((g / nst) - 1) & 1, B.abort_flag, dev_status)) break;
        if (kind == 2) {
            mbar_expect_tx(full + stage, kXs);
            bulk_load(xs + stage * kXs, nld + ((row0 + row) >> 6) * 128, kXs, full + stage);
        } else {
            mbar_expect_tx(full + stage, L::NR * kGran);
            tma_load_3d(sm + L::RING + stage * L::STAGE + kind * L::NR * kGran, mg, full + stage, 0,
                        (int)(row0 + row), 0);
        }
        last = g;
    }
    if (*B.abort_flag && last >= 0) {
        // let this lane's copy land before the CTA goes away
        volatile int no_abort = 0;
        mbar_wait(full + stage, (last / nst) & 1, &no_abort, dev_status);
    }
}

// Epilogue of a 128-row accumulator tile (D fp32 columns in TMEM; this thread
// holds row `row`, TMEM address `tacc` = its lane quarter + first column):
// scaled bf16 (a finished tile) or raw fp32 (the partial of a split tile),
// written as 16-byte chunks in the 128-byte-swizzled image of the whole-row
// TMA maps into `stage` (free shared memory, 1024-byte aligned), then stored by
// the group's leader with one TMA copy.  Per-row 16-byte stores straight to
// global memory would touch 32 lines per warp instruction.  Every thread of
// the group (nthreads, named barrier bar_id) runs the barrier, also when `ok`
// is false after a timeout.
template <int D>
__device__ void store_tile(uint32_t tacc, int row, bool ok, bool zero, bool part, float mul, uint8_t* stage,
                           const CUtensorMap* map_bf16, const CUtensorMap* map_f32, int y_bf16, int y_f32,
                           int bar_id, int nthreads, bool leader) {
    if (ok) {
        const uint32_t sw = (uint32_t)(row & 7);
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
            uint32_t r[32];
            tmem_ld32(tacc + 32 * q, r);
            tmem_wait_ld();
            if (zero) {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = 0u;
            }
            if (!part) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {                          // 4 chunks of 8 bf16
                    const int g = 4 * q + k;
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[8 * k + 0]) * mul, __uint_as_float(r[8 * k + 1]) * mul);
                    v.y = pack_bf16x2(__uint_as_float(r[8 * k + 2]) * mul, __uint_as_float(r[8 * k + 3]) * mul);
                    v.z = pack_bf16x2(__uint_as_float(r[8 * k + 4]) * mul, __uint_as_float(r[8 * k + 5]) * mul);
                    v.w = pack_bf16x2(__uint_as_float(r[8 * k + 6]) * mul, __uint_as_float(r[8 * k + 7]) * mul);
                    *reinterpret_cast<uint4*>(stage + (g >> 3) * kTile + row * 128 + (((g & 7) ^ sw) << 4)) = v;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {                          // 8 chunks of 4 fp32
                    const int g = 8 * q + k;
                    const float4 v = make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                                                 __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3]));
                    *reinterpret_cast<float4*>(stage + (g >> 3) * kTile + row * 128 + (((g & 7) ^ sw) << 4)) = v;
                }
            }
        }
        fence_proxy_async_smem();
    }
    named_sync(bar_id, nthreads);
    if (ok && leader) {
        tma_store_3d(part ? map_f32 : map_bf16, stage, 0, part ? y_f32 : y_bf16, 0);
        bulk_commit();
        bulk_wait_read();                                              // shared memory stays valid until read
    }
}

// ============================================================================ dQ
template <int D>
__global__ void __launch_bounds__(192, 1)
k_bwd_dq_sm100(const __nv_bfloat16* __restrict__ Qg, const __nv_bfloat16* __restrict__ dOg,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmPq,
               const uint32_t* __restrict__ gsel, const PlanHeader* __restrict__ hdr,
               const int4* __restrict__ items, const float* __restrict__ lse,
               const float* __restrict__ delta, int64_t N, int64_t MB, int SW, int nst, float scale,
               uint32_t* __restrict__ dev_status) {
    using L = BwdLayout<D, false>;
    // TMEM: dQ, S / dP of two granules, and the tile's Q and dO as bf16 (the A
    // operands of S = Q K^T and dP = dO V^T, read by the tensor core from TMEM)
    constexpr uint32_t cdQ = 0, cS = 128, cP = 192;   // + 128 * buffer for S / dP
    constexpr uint32_t cQ = 384, cdO = 384 + D / 2;
    if ((int)blockIdx.x >= hdr->n_items) return;      // uniform: beyond the item list
    const int4 item = items[blockIdx.x];
    const int tiles_per_head = (int)(N / 128);
    const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
    const int g_begin = item.y, ng = item.z - item.y, slot = item.w;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars B = carve(sm + L::ctrl(nst, 0));
    uint32_t* u0 = reinterpret_cast<uint32_t*>(sm + L::rows(nst, 0));
    uint32_t* u1 = u0 + SW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wn = SW;
    const int64_t row0 = (int64_t)hh * N;

    load_rows(u0, u1, gsel + ((int64_t)hh * MB + 2 * tile) * SW, gsel + ((int64_t)hh * MB + 2 * tile + 1) * SW, wn);
    if (threadIdx.x == 0) init_bars(B, nst, 128, 128);   // Q, dO: one arrival per tile row
    if (warp == 1) {
        tmem_alloc(B.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *B.tmem_slot;

    if (warp == 0) {
        produce<D, false>(nullptr, nullptr, &tmK, &tmV, nullptr, nullptr, sm, B, row0, 128 * tile, u0, u1, wn,
                          g_begin, ng, nst, dev_status);
    } else if (warp == 1) {
        {   // the whole warp, converged; one elected lane issues
            const uint32_t idPS = idesc_bf16_f32(128, 64, false, false);
            const uint32_t idQ = idesc_bf16_f32(128, D, false, true);
            const uint32_t aR = smem_u32(sm + L::RING);
            bool ok = mbar_wait_w(B.stat, 0, B.abort_flag, dev_status);
            tc_fence_after();
            for (int g = 0; ok && g <= ng; ++g) {
                if (g < ng) {
                    const int s = g % nst, b = g & 1;
                    if (!mbar_wait_w(B.full0 + s, (g / nst) & 1, B.abort_flag, dev_status) ||
                        !mbar_wait_w(B.full1 + s, (g / nst) & 1, B.abort_flag, dev_status))
                        break;
                    tc_fence_after();
                    const uint32_t aK = aR + s * L::STAGE, aV = aK + L::NR * kGran;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ts_w(tb + cS + 128 * b, tb + cQ + 8 * k, sdesc_sw128(aK + kmaj_off(k, kGran), 16, 1024),
                                 idPS, k > 0);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ts_w(tb + cP + 128 * b, tb + cdO + 8 * k, sdesc_sw128(aV + kmaj_off(k, kGran), 16, 1024),
                                 idPS, k > 0);
                    tc_commit_w(B.prod + b);
                }
                if (g > 0) {
                    const int gp = g - 1, s = gp % nst, b = gp & 1;
                    if (!mbar_wait_w(B.elem + b, (gp >> 1) & 1, B.abort_flag, dev_status)) break;
                    tc_fence_after();
                    const uint32_t aK = aR + s * L::STAGE;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_ts_w(tb + cdQ, tb + cS + 128 * b + 8 * k, sdesc_sw128(aK + k * 2048, kGran, 1024), idQ,
                                 (gp > 0 || k > 0) ? 1u : 0u);
                    tc_commit_w(B.empty + s);
                }
            }
            tc_commit_w(B.fin);
            if (*B.abort_flag) {
                volatile int no_abort = 0;
                mbar_wait(B.fin, 0, &no_abort, dev_status);
            }
        }
    } else {
        const int sub = warp & 3, row = sub * 32 + lane, half = row >> 6;
        const uint32_t tl = tb + ((uint32_t)(sub * 32) << 16);
        const int64_t grow = row0 + 128 * tile + row;
        {
            // this row of Q and of dO into TMEM (two bf16 per column)
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint4* src = reinterpret_cast<const uint4*>((which ? dOg : Qg) + grow * D);
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
                    tmem_st32(tl + (which ? cdO : cQ) + 32 * q, r);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(B.stat);
        }
        const float lse2 = lse[grow] * kLog2e, dl = delta[grow];
        const float sl2 = scale * kLog2e;
        const uint64_t sl2x2 = f2pack(sl2, sl2), nlse2 = f2pack(-lse2, -lse2), ndl2 = f2pack(-dl, -dl);
        GranuleWalk walk;
        if (lane == 0) {
            walk.init(u0, u1, wn);
            walk.skip(g_begin);
        }
        bool ok = true;
        for (int g = 0; g < ng; ++g) {
            const int b = g & 1;
            uint32_t mk = 0;
            if (lane == 0) {
                int rr;
                walk.next(rr, mk);
            }
            mk = __shfl_sync(0xffffffffu, mk, 0);
            const bool valid = (mk >> half) & 1u;              // warp-uniform
            const bool got = mbar_wait(B.prod + b, (g >> 1) & 1, B.abort_flag, dev_status);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            // S and dP of the granule: all TMEM loads in flight before one wait
            uint32_t sv[2][32], pv[2][32];
            if (valid) {
                tmem_ld32(tl + cS + 128 * b, sv[0]);
                tmem_ld32(tl + cP + 128 * b, pv[0]);
                tmem_ld32(tl + cS + 128 * b + 32, sv[1]);
                tmem_ld32(tl + cP + 128 * b + 32, pv[1]);
                tmem_wait_ld();
            }
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
                uint32_t o[16];
                if (valid) {
                    const uint32_t (&s)[32] = sv[hq];
                    const uint32_t (&p)[32] = pv[hq];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float x0, x1;
                        f2unpack(ffma2(f2pack(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), sl2x2, nlse2),
                                 x0, x1);
                        const uint64_t pp = f2pack(ex2(x0), ex2(x1));
                        const uint64_t dp = fadd2(f2pack(__uint_as_float(p[2 * i]), __uint_as_float(p[2 * i + 1])), ndl2);
                        float d0, d1;
                        f2unpack(fmul2(pp, dp), d0, d1);
                        o[i] = pack_bf16x2(d0, d1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = 0u;
                }
                tmem_st16(tl + cS + 128 * b + 16 * hq, o);     // dS (bf16) over the consumed S columns
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(B.elem + b);
        }
        const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(B.fin, 0, B.abort_flag, dev_status));
        if (fin) tc_fence_after();
        // nothing selected (ng == 0): TMEM never written, the tile is zero.  The ring is free.
        store_tile<D>(tl + cdQ, row, fin, ng == 0, slot >= 0, scale, sm + L::RING, &tmdQ, &tmPq,
                      (int)(row0 + 128 * tile), slot * 128, 1, 128, warp == 2 && lane == 0);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, kTmemCols);
}

// ============================================================================ dK, dV
template <int D>
__global__ void __launch_bounds__(384, 1)
k_bwd_dkdv_sm100(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                 const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                 const __grid_constant__ CUtensorMap tmPkv,
                 const uint32_t* __restrict__ gselT, const PlanHeader* __restrict__ hdr,
                 const int4* __restrict__ items, const float* __restrict__ nld,
                 int64_t N, int64_t MB, int SW, int nst, float scale, uint32_t* __restrict__ dev_status) {
    using L = BwdLayout<D, true>;
    constexpr uint32_t cdK = 0, cdV = 128, cS = 256, cP = 320;   // + 128 * buffer for S^T / dP^T
    if ((int)blockIdx.x >= hdr->n_items) return;      // uniform: beyond the item list
    const int4 item = items[blockIdx.x];
    const int tiles_per_head = (int)(N / 128);
    const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
    const int g_begin = item.y, ng = item.z - item.y, slot = item.w;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars B = carve(sm + L::ctrl(nst, kXs));
    uint8_t* xs = sm + L::xs(nst);
    uint32_t* u0 = reinterpret_cast<uint32_t*>(sm + L::rows(nst, kXs));
    uint32_t* u1 = u0 + SW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wn = SW;
    const int64_t row0 = (int64_t)hh * N;

    load_rows(u0, u1, gselT + ((int64_t)hh * MB + 2 * tile) * SW, gselT + ((int64_t)hh * MB + 2 * tile + 1) * SW, wn);
    if (threadIdx.x == 0) init_bars(B, nst, 2, 256);     // K, V: one arrival per stationary copy
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
        produce<D, true>(&tmK, &tmV, &tmQ, &tmdO, nld, xs, sm, B, row0, 128 * tile, u0, u1, wn, g_begin, ng, nst,
                         dev_status);
      } else if (warp == 1) {
        {   // the whole warp, converged; one elected lane issues
            const uint32_t idPS = idesc_bf16_f32(128, 64, false, false);
            const uint32_t idKV = idesc_bf16_f32(128, D, false, true);
            const uint32_t aK = smem_u32(sm + L::A0), aV = smem_u32(sm + L::A1), aR = smem_u32(sm + L::RING);
            bool ok = mbar_wait_w(B.stat, 0, B.abort_flag, dev_status);
            tc_fence_after();
            for (int g = 0; ok && g <= ng; ++g) {
                if (g < ng) {
                    const int s = g % nst, b = g & 1;
                    if (!mbar_wait_w(B.full0 + s, (g / nst) & 1, B.abort_flag, dev_status) ||
                        !mbar_wait_w(B.full1 + s, (g / nst) & 1, B.abort_flag, dev_status))
                        break;
                    tc_fence_after();
                    const uint32_t aQ = aR + s * L::STAGE, adO = aQ + L::NR * kGran;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ss_w(tb + cS + 128 * b, sdesc_sw128(aK + kmaj_off(k, kTile), 16, 1024),
                                 sdesc_sw128(aQ + kmaj_off(k, kGran), 16, 1024), idPS, k > 0);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ss_w(tb + cP + 128 * b, sdesc_sw128(aV + kmaj_off(k, kTile), 16, 1024),
                                 sdesc_sw128(adO + kmaj_off(k, kGran), 16, 1024), idPS, k > 0);
                    tc_commit_w(B.prod + b);
                }
                if (g > 0) {
                    const int gp = g - 1, s = gp % nst, b = gp & 1;
                    if (!mbar_wait_w(B.elem + b, (gp >> 1) & 1, B.abort_flag, dev_status)) break;
                    tc_fence_after();
                    const uint32_t aQ = aR + s * L::STAGE, adO = aQ + L::NR * kGran;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t acc = (gp > 0 || k > 0) ? 1u : 0u;
                        mma_ts_w(tb + cdV, tb + cS + 128 * b + 8 * k, sdesc_sw128(adO + k * 2048, kGran, 1024), idKV,
                                 acc);
                        mma_ts_w(tb + cdK, tb + cP + 128 * b + 8 * k, sdesc_sw128(aQ + k * 2048, kGran, 1024), idKV,
                                 acc);
                    }
                    tc_commit_w(B.empty + s);
                }
            }
            tc_commit_w(B.fin);
            if (*B.abort_flag) {
                volatile int no_abort = 0;
                mbar_wait(B.fin, 0, &no_abort, dev_status);
            }
        }
      }
    } else {
        regs_inc<kRegsHigh>();
        // Both elementwise warpgroups work on every granule, warpgroup wg on
        // its 32 query columns (16 wg .. 16 wg + 15 of P^T / dS^T), which halves
        // the latency from the granule's products to its dK/dV MMAs.  bf16 P^T
        // and dS^T of warpgroup 1 overwrite fp32 columns that warpgroup 0
        // reads, so the stores wait at a named barrier for both warpgroups'
        // loads; every thread runs every barrier, also after a timeout.
        const int wg = (warp - 4) >> 2;
        const int sub = warp & 3, row = sub * 32 + lane, half = row >> 6;
        const uint32_t tl = tb + ((uint32_t)(sub * 32) << 16);
        const float sl2 = scale * kLog2e;
        const uint64_t sl2x2 = f2pack(sl2, sl2);
        GranuleWalk walk;
        if (lane == 0) {
            walk.init(u0, u1, wn);
            walk.skip(g_begin);
        }
        bool ok = true;
        for (int g = 0; g < ng; ++g) {
            const int b = g & 1, st = g % nst;
            uint32_t mk = 0;
            int qrow = 0;
            if (lane == 0) walk.next(qrow, mk);
            mk = __shfl_sync(0xffffffffu, mk, 0);
            const bool valid = (mk >> half) & 1u;              // warp-uniform
            const float4* nl4 = reinterpret_cast<const float4*>(xs + st * kXs) + 8 * wg;   // -lse*log2(e)
            const float4* nd4 = nl4 + 16;                                                   // -Delta
            if (ok)
                ok = __all_sync(0xffffffffu, mbar_wait(B.prod + b, (g >> 1) & 1, B.abort_flag, dev_status) &&
                                                 mbar_wait(B.fullx + st, (g / nst) & 1, B.abort_flag, dev_status));
            // 32 columns of S^T and of dP^T: both TMEM loads in flight before one wait
            uint32_t sv[32], pv[32];
            if (ok) {
                tc_fence_after();
                if (valid) {
                    tmem_ld32(tl + cS + 128 * b + 32 * wg, sv);
                    tmem_ld32(tl + cP + 128 * b + 32 * wg, pv);
                }
                tmem_wait_ld();
            }
            named_sync(1, 256);                                // both warpgroups hold their columns
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
                        f2unpack(ffma2(f2pack(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), sl2x2, nl), x0, x1);
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
            tmem_st16(tl + cS + 128 * b + 16 * wg, op);        // P^T
            tmem_st16(tl + cP + 128 * b + 16 * wg, od);        // dS^T
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(B.elem + b);
        }
        const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(B.fin, 0, B.abort_flag, dev_status));
        if (fin) tc_fence_after();
        // warpgroup 0 writes dK, warpgroup 1 dV, each staged in its half of the (now free) ring;
        // no query selected these keys (ng == 0): TMEM never written, zeros
        store_tile<D>(tl + (wg ? cdV : cdK), row, fin, ng == 0, slot >= 0, wg ? 1.f : scale,
                      sm + L::RING + wg * 2 * L::NR * kTile, wg ? &tmdV : &tmdK, &tmPkv, (int)(row0 + 128 * tile),
                      (slot * 2 + wg) * 128, 2 + wg, 128, (warp & 3) == 0 && lane == 0);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tb, kTmemCols);
}

// ------------------------------------------------------------------ host side
struct BwdWs {
    float* delta;
    float* nld;         // [heads*N/64][128]: per 64-row granule -lse*log2(e), then -Delta
    Plan pq, pkv;
    float* part_q;      // [slots][128][D]
    float* part_kv;     // [slots][2][128][D]
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
    if (total) *total = (size_t)(p - static_cast<uint8_t*>(ws));
    return w;
}

template <int D>
prism_status_t launch_bwd(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* dOp,
                          const float* lse, const uint32_t* gsel, const uint32_t* gselT, float scale, void* dQp,
                          void* dKp, void* dVp, uint32_t* dev_status, const BwdWs& w, cudaStream_t s) {
    const int64_t rows = (int64_t)d.heads * d.N;
    CUtensorMap tK, tV, gQ, gdO, gK, gV;
    if (!make_map_bf16_rows(&tK, Kp, rows, D, 128) || !make_map_bf16_rows(&tV, Vp, rows, D, 128) ||
        !make_map_bf16_rows(&gQ, Qp, rows, D, 64) || !make_map_bf16_rows(&gdO, dOp, rows, D, 64) ||
        !make_map_bf16_rows(&gK, Kp, rows, D, 64) || !make_map_bf16_rows(&gV, Vp, rows, D, 64))
        return PRISM_ERR_CUDA;
    const int target = plan_target(device_sms());
    const int64_t slots = 2 * (int64_t)target;
    CUtensorMap tdQ, tdK, tdV, tPq, tPkv;
    if (!make_map_bf16_rows(&tdQ, dQp, rows, D, 128) || !make_map_bf16_rows(&tdK, dKp, rows, D, 128) ||
        !make_map_bf16_rows(&tdV, dVp, rows, D, 128) || !make_map_f32_rows(&tPq, w.part_q, slots * 128, D, 128) ||
        !make_map_f32_rows(&tPkv, w.part_kv, slots * 2 * 128, D, 128))
        return PRISM_ERR_CUDA;
    prism_status_t st = plan_work(w.pq, gsel, d, 2, 1, target, kSegMinGranules, s);
    if (st == PRISM_OK) st = plan_work(w.pkv, gselT, d, 2, 1, target, kSegMinGranules, s);
    if (st != PRISM_OK) return st;
    const int nq = BwdLayout<D, false>::stages(0, (int)d.SW), nk = BwdLayout<D, true>::stages(kXs, (int)d.SW);
    const int smq = BwdLayout<D, false>::alloc(nq, 0, (int)d.SW);
    const int smk = BwdLayout<D, true>::alloc(nk, kXs, (int)d.SW);
    if (smq > kSmemMax || smk > kSmemMax) return PRISM_ERR_UNSUPPORTED;   // selection rows too long
    auto kq = k_bwd_dq_sm100<D>;
    auto kk = k_bwd_dkdv_sm100<D>;
    if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smq) != cudaSuccess ||
        cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, smk) != cudaSuccess)
        return PRISM_ERR_CUDA;
    kq<<<(unsigned)w.pq.items_max, 192, smq, s>>>((const __nv_bfloat16*)Qp, (const __nv_bfloat16*)dOp, gK, gV, tdQ, tPq,
                                                  gsel, w.pq.hdr, w.pq.items, lse,
                                                  w.delta, d.N, d.MB, (int)d.SW, nq, scale, dev_status);
    kk<<<(unsigned)w.pkv.items_max, 384, smk, s>>>(tK, tV, gQ, gdO, tdK, tdV, tPkv, gselT, w.pkv.hdr, w.pkv.items,
                                                   w.nld, d.N, d.MB, (int)d.SW, nk, scale, dev_status);
    st = launch_status(2);
    if (st == PRISM_OK) st = bwd_combine(w.pq, d, 1, w.part_q, dQp, scale, nullptr, 0.f, s);
    if (st == PRISM_OK) st = bwd_combine(w.pkv, d, 2, w.part_kv, dKp, scale, dVp, 1.f, s);
    return st;
}

}  // namespace

size_t attn_bwd_sm100_ws_bytes(const Dims& d) {
    size_t total = 0;
    carve_bwd(reinterpret_cast<void*>(uintptr_t(256)), d, &total);
    return total;
}

prism_status_t attn_bwd_sm100(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* Op,
                              const float* o_f32, const void* dOp, const float* lse, const uint32_t* gsel,
                              const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp,
                              uint32_t* dev_status, void* ws, cudaStream_t s) {
    BwdWs w = carve_bwd(ws, d, nullptr);
    prism_status_t st = bwd_delta(d, Op, o_f32, dOp, w.delta, lse, w.nld, s);
    if (st != PRISM_OK) return st;
    if (d.d == 128)
        return launch_bwd<128>(d, Qp, Kp, Vp, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, w, s);
    return launch_bwd<64>(d, Qp, Kp, Vp, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, dev_status, w, s);
}

}  // namespace prism
