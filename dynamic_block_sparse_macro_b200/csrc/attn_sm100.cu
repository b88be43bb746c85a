// Stage 6 on sm_100a tensor cores: block-sparse attention forward for bf16.
//
// Prism, Portuguese reading guide, "Método" 3: an online-softmax kernel runs
// the attention only over the selected set S_i of each query block.
//
// Work unit: one CTA per (128-row query tile, head).  Blocks are whole 64-row
// granules, so a tile holds either half of a 256-block, one 128-block, or two
// 64-blocks b0, b1 (rows 0-63 and 64-127).  The key stream is the union of
// S_b0 and S_b1 walked as 64-row granules in block order; two granules form
// one 128-key chunk, and a per-granule 2-bit mask says which half of the tile
// selected it (an odd tail repeats its last granule with mask 0).
//
// Roles (6 warps):
//   warp 0      TMA producer: Q once, then per chunk K and V (64x64 bf16 boxes,
//               128-byte swizzle) into one K and one V buffer.
//   warp 1      allocates 256 TMEM columns; lane 0 issues tcgen05.mma:
//               S = Q K^T (M=128, N=128, fp32 in TMEM), then O += P V with
//               P read from TMEM (aliasing S) and V MN-major from shared memory.
//   warps 2-5   one query row per thread: S row from TMEM, masked online
//               softmax in the exp2 domain with lazy rescaling (the running
//               max only moves when it grows by more than 2^8), P as bf16 back
//               into TMEM, then the epilogue (O / l, LSE).
// Two CTAs share an SM (96 KB shared memory and 256 TMEM columns each), so
// one CTA's softmax overlaps the other's MMAs.  Every wait is bounded; a
// timeout sets PRISM_DEV_TIMEOUT and the CTA winds down without trapping.
#include "common.cuh"
#include "sm100.cuh"

namespace prism {

using namespace sm100;

namespace {

constexpr int kRegion = 128 * 128;         // bytes of a 128-row x 64-col bf16 tile region
constexpr int kGranBytes = 64 * 128;       // 64 rows x 64 cols bf16
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0;              // O accumulator: D columns
constexpr uint32_t kColS = 128;            // S (fp32, 128 columns); P (bf16) aliases its first 64
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct FwdLayout {
    static constexpr int NR = D / 64;
    static constexpr int Q = 0;
    static constexpr int K = NR * kRegion;
    static constexpr int V = 2 * NR * kRegion;
    static constexpr int CTRL = 3 * NR * kRegion;
    static constexpr int BYTES = CTRL + 256;
    // + slack for 1024-byte alignment; at least 80 KB so that no more than two
    // CTAs (2 x 256 of the SM's 512 TMEM columns) are ever resident on an SM
    static constexpr int ALLOC = (BYTES + 1024) > 80 * 1024 ? (BYTES + 1024) : 80 * 1024;
};

template <int D>
__global__ void __launch_bounds__(192, 2)
k_attn_fwd_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ blk_start,
                 const int32_t* __restrict__ gran_blk, const int32_t* __restrict__ n_blk,
                 const uint32_t* __restrict__ sel, int64_t N, int64_t MB, int SW, float scale,
                 __nv_bfloat16* __restrict__ O, float* __restrict__ lse, float* __restrict__ o_f32,
                 uint32_t* __restrict__ dev_status) {
    using L = FwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = sm + L::Q;
    uint8_t* sK = sm + L::K;
    uint8_t* sV = sm + L::V;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::CTRL);
    uint64_t* bar_q = bars + 0;
    uint64_t* bar_kf = bars + 1;
    uint64_t* bar_ke = bars + 2;
    uint64_t* bar_vf = bars + 3;
    uint64_t* bar_ve = bars + 4;
    uint64_t* bar_s = bars + 5;
    uint64_t* bar_p = bars + 6;
    uint64_t* bar_o = bars + 7;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* nch_slot = reinterpret_cast<int*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x, hh = blockIdx.y;
    const int nb = *n_blk;
    const int b0 = gran_blk[2 * tile], b1 = gran_blk[2 * tile + 1];
    if (b0 < 0 || b0 >= nb || b1 < 0 || b1 >= nb) {      // uniform across the CTA
        if (threadIdx.x == 0) atomicOr(dev_status, PRISM_DEV_BAD_INDEX);
        return;
    }
    const uint32_t* r0 = sel + ((int64_t)hh * MB + b0) * SW;
    const uint32_t* r1 = sel + ((int64_t)hh * MB + b1) * SW;
    const int wn = (nb + 31) >> 5;
    const int64_t row0 = (int64_t)hh * N;                  // first row of this head in [heads*N, D]

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_kf, 1);
        mbar_init(bar_ke, 1);
        mbar_init(bar_vf, 1);
        mbar_init(bar_ve, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_p, 128);
        mbar_init(bar_o, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {                                       // count granules of the union
        const int cnt = count_granules(r0, r1, blk_start, wn, lane);
        if (lane == 0) *nch_slot = (cnt + 1) >> 1;
    } else if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const int nch = *nch_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_expect_tx(bar_q, L::NR * kRegion);
            for (int r = 0; r < L::NR; ++r)
                tma_load_2d(sQ + r * kRegion, &tmQ, bar_q, 64 * r, (int)(row0 + 128 * tile));
            GranuleWalk walk;
            walk.init(r0, r1, blk_start, wn);
            int issued_k = 0, issued_v = 0;
            for (int c = 0; c < nch && !*abort_flag; ++c) {
                int ra = 0, rb = 0;
                uint32_t ma, mb;
                walk.next(ra, ma);
                if (!walk.next(rb, mb)) rb = ra;
                if (c > 0 && !mbar_wait(bar_ke, (c - 1) & 1, abort_flag, dev_status)) break;
                mbar_expect_tx(bar_kf, 2 * L::NR * kGranBytes);
                for (int r = 0; r < L::NR; ++r) {
                    tma_load_2d(sK + r * kRegion, &tmK, bar_kf, 64 * r, (int)(row0 + ra));
                    tma_load_2d(sK + r * kRegion + kGranBytes, &tmK, bar_kf, 64 * r, (int)(row0 + rb));
                }
                ++issued_k;
                if (c > 0 && !mbar_wait(bar_ve, (c - 1) & 1, abort_flag, dev_status)) break;
                mbar_expect_tx(bar_vf, 2 * L::NR * kGranBytes);
                for (int r = 0; r < L::NR; ++r) {
                    tma_load_2d(sV + r * kRegion, &tmV, bar_vf, 64 * r, (int)(row0 + ra));
                    tma_load_2d(sV + r * kRegion + kGranBytes, &tmV, bar_vf, 64 * r, (int)(row0 + rb));
                }
                ++issued_v;
            }
            if (*abort_flag) {
                // let the copies already in flight land before the CTA goes away
                volatile int no_abort = 0;
                if (issued_k) mbar_wait(bar_kf, (issued_k - 1) & 1, &no_abort, dev_status);
                if (issued_v) mbar_wait(bar_vf, (issued_v - 1) & 1, &no_abort, dev_status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t idS = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idO = idesc_bf16_f32(128, D, false, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait(bar_q, 0, abort_flag, dev_status);
            tc_fence_after();
            for (int c = 0; ok && c < nch; ++c) {
                if (!mbar_wait(bar_kf, c & 1, abort_flag, dev_status)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
                    mma_ss(tbase + kColS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024), idS,
                           k > 0 ? 1u : 0u);
                }
                tc_commit(bar_ke);
                tc_commit(bar_s);
                if (!mbar_wait(bar_p, c & 1, abort_flag, dev_status)) break;
                tc_fence_after();
                if (!mbar_wait(bar_vf, c & 1, abort_flag, dev_status)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts(tbase + kColO, tbase + kColS + 8 * k, sdesc_sw128(aV + k * 2048, kRegion, 1024), idO,
                           (c > 0 || k > 0) ? 1u : 0u);
                tc_commit(bar_ve);
            }
            tc_commit(bar_o);
            if (*abort_flag) {
                volatile int no_abort = 0;
                mbar_wait(bar_o, 0, &no_abort, dev_status);
            }
        }
    } else {
        // ---------------------------------------------------- softmax + epilogue
        const int sub = warp & 3;                          // TMEM lane quarter of this warp
        const int row = sub * 32 + lane;                   // query row within the tile
        const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
        const int half = row >> 6;
        const float sl2 = scale * kLog2e;
        float m_run = -INFINITY, l = 0.f;
        GranuleWalk walk;
        if (lane == 0) walk.init(r0, r1, blk_start, wn);
        bool ok = true;
        for (int c = 0; c < nch; ++c) {
            uint32_t mk = 0;
            if (lane == 0) {
                int ra, rb;
                uint32_t ma = 0, mb = 0;
                walk.next(ra, ma);
                if (!walk.next(rb, mb)) mb = 0;
                mk = ma | (mb << 2);
            }
            mk = __shfl_sync(0xffffffffu, mk, 0);
            const bool v0 = (mk >> half) & 1u, v1 = (mk >> (2 + half)) & 1u;
            const bool got = mbar_wait(bar_s, c & 1, abort_flag, dev_status);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }   // warp-uniform exit
            tc_fence_after();
            // pass 1: row max over the valid columns
            float mx = -INFINITY;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (!(q < 2 ? v0 : v1)) continue;
                uint32_t r[32];
                tmem_ld32(tl + kColS + 32 * q, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(r[i]));
            }
            const float mx2 = mx * sl2;
            const bool need = mx2 > m_run + kRescaleThreshold || (m_run == -INFINITY && mx2 > -INFINITY);
            const float alpha = need ? exp2f(m_run - mx2) : 1.f;   // 0 when m_run = -inf
            // O holds chunks < c, all complete (S of chunk c was issued after them).
            // TMEM access is warp-collective: the whole warp rescales if any row must.
            if (c > 0 && __any_sync(0xffffffffu, need && m_run > -INFINITY)) {
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t r[32];
                    tmem_ld32(tl + kColO + 32 * q, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(tl + kColO + 32 * q, r);
                }
            }
            if (need) {
                l *= alpha;
                m_run = mx2;
            }
            // pass 2: P = exp2(s * scale * log2e - m) as bf16 into the first 64 columns of S
            float rs = 0.f;
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
                const bool v = hq == 0 ? v0 : v1;
                uint32_t pk[32];
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t r[32];
                    tmem_ld32(tl + kColS + 64 * hq + 32 * q2, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float p0 = 0.f, p1 = 0.f;
                        if (v && m_run > -INFINITY) {
                            p0 = exp2f(fmaf(__uint_as_float(r[2 * i]), sl2, -m_run));
                            p1 = exp2f(fmaf(__uint_as_float(r[2 * i + 1]), sl2, -m_run));
                        }
                        rs += p0 + p1;
                        pk[16 * q2 + i] = pack_bf16x2(p0, p1);
                    }
                }
                tmem_st32(tl + kColS + 32 * hq, pk);
            }
            l += rs;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p);
        }
        const bool fin = ok && mbar_wait(bar_o, 0, abort_flag, dev_status);
        if (__all_sync(0xffffffffu, fin)) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int64_t grow = row0 + 128 * tile + row;
            __nv_bfloat16* orow = O + grow * D;
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                uint32_t r[32];
                tmem_ld32(tl + kColO + 32 * q, r);
                tmem_wait_ld();
                if (!(l > 0.f)) {                          // empty selection: O = 0 (TMEM never written)
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
                uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                if (o_f32) {
                    float4* df = reinterpret_cast<float4*>(o_f32 + grow * D + 32 * q);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        df[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                            __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
                }
            }
            lse[grow] = l > 0.f ? (m_run + log2f(l)) * kLn2 : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ host side
template <int D>
prism_status_t launch_fwd(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const int32_t* blk_start,
                          const int32_t* gran_blk, const int32_t* n_blk, const uint32_t* sel, float scale, void* Op,
                          float* lse, float* o_f32, uint32_t* dev_status, cudaStream_t s) {
    CUtensorMap mQ, mK, mV;
    const int64_t rows = (int64_t)d.heads * d.N;
    if (!make_map_bf16(&mQ, Qp, rows, D, 128) || !make_map_bf16(&mK, Kp, rows, D, 64) ||
        !make_map_bf16(&mV, Vp, rows, D, 64))
        return PRISM_ERR_CUDA;
    auto k = k_attn_fwd_sm100<D>;
    const int smem = FwdLayout<D>::ALLOC;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PRISM_ERR_CUDA;
    dim3 grid((unsigned)(d.N / 128), (unsigned)d.heads);
    k<<<grid, 192, smem, s>>>(mQ, mK, mV, blk_start, gran_blk, n_blk, sel, d.N, d.MB, (int)d.SW, scale,
                              (__nv_bfloat16*)Op, lse, o_f32, dev_status);
    return launch_status(1);
}

}  // namespace

prism_status_t attn_fwd_sm100(const Dims& d, const void* Qp, const void* Kp, const void* Vp,
                              const int32_t* blk_start, const int32_t* gran_blk, const int32_t* n_blk,
                              const uint32_t* sel, float scale, void* Op, float* lse, float* o_f32,
                              uint32_t* dev_status, cudaStream_t s) {
    if (d.d == 128)
        return launch_fwd<128>(d, Qp, Kp, Vp, blk_start, gran_blk, n_blk, sel, scale, Op, lse, o_f32, dev_status, s);
    return launch_fwd<64>(d, Qp, Kp, Vp, blk_start, gran_blk, n_blk, sel, scale, Op, lse, o_f32, dev_status, s);
}

}  // namespace prism
