// Stage 5: hybrid Top-k / Top-p block selection.
//
// Prism, Portuguese reading guide, "Método" 3: S_i = Top-k(P_i, k) U
// Top-p(P_i, p); the Chinese guide's glossary describes Top-k as the
// guaranteed minimum context and Top-p as the adaptive cumulative threshold
// for queries with dispersed attention.  Read here as two prefixes of the
// same order (P desc, j asc): Top-p is the shortest prefix whose sum reaches
// p (everything if p >= 1 or it never does), so S_i is the longer prefix,
// max(min(k, n_blk), n_p) blocks.
//
// For P >= 0 the float bit pattern orders like the value, so thresholds are
// found by binary search over bit patterns, each step a pass over the row
// and a fixed-order reduction (deterministic):
//   v_k = largest t with #{P_j >= t} >= k       (k-th value of the order),
//   v*  = largest t with sum{P_j : P_j >= t} >= p (Top-p crossing value).
// One search per row suffices.  With S_k the sum of the first k entries, Top-k
// sets the size when S_k >= p (then n_p <= k, and n_p = k exactly when
// S_k - v_k < p); otherwise n_p > k and the Top-p search gives both n_p and the
// threshold.  S_i = {P > v_n} plus the lowest-index ties at v_n.
//
// k_select_reg<C>  one warp per (row, head), the row in registers (C values a
//                  lane, rows of 32*CLO < n_blk <= 32*C blocks); one kernel
//                  per size class, each exits for the others' rows.
// k_select_cta     one 256-thread CTA per row above 4096 blocks, the row in
//                  shared memory.
// k_sel_expand     granule-level view of the selection for the attention
//                  kernels; k_bit_transpose its key-major transpose.
#include "common.cuh"

namespace prism {

constexpr int kSelectThreads = 256;
constexpr int kSelectMaxRow = 16384;    // P values of a row held in shared memory (CTA form)
constexpr int kWarpRowMax = 4096;       // rows up to this many blocks: one warp each, in registers
constexpr int kWarpRowsPerCta = 4;
static_assert(kWarpRowMax == 32 * 128, "the largest register class holds 128 values a lane");

struct SelRed {
    float f[kSelectThreads / 32];
    int i[kSelectThreads / 32];
};

// fixed-order block reductions (every thread gets the result)
__device__ __forceinline__ float sel_sum(float v, SelRed& r) {
    v = warp_sum(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) r.f[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kSelectThreads / 32; ++w) s += r.f[w];
    return s;
}
__device__ __forceinline__ int sel_count_i(int v, SelRed& r) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) r.i[threadIdx.x >> 5] = v;
    __syncthreads();
    int s = 0;
#pragma unroll
    for (int w = 0; w < kSelectThreads / 32; ++w) s += r.i[w];
    return s;
}
__device__ __forceinline__ float sel_max(float v, SelRed& r) {
    v = warp_max(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) r.f[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = r.f[0];
#pragma unroll
    for (int w = 1; w < kSelectThreads / 32; ++w) s = fmaxf(s, r.f[w]);
    return s;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// size of S_i and its threshold: the first n entries of (P desc, j asc) are
// {P > vb} plus the first need_eq ties at vb (all of the row when n >= nb)
struct SelCut {
    int n;
    uint32_t vb;
    int need_eq;
    float gap_p;     // cumulative-sum margin: the sum of the n selected above p (when n can
                     // still grow) and, when Top-p sets n (n_p > n_k), p above the sum of n-1
};

// count_ge(t) = #{P >= t}, sum_ge(t) = sum{P >= t} for bit patterns t (row-wide)
template <class CountGe, class SumGe>
__device__ __forceinline__ SelCut select_cut(int nb, int top_k, float top_p, CountGe count_ge, SumGe sum_ge) {
    SelCut c{nb, 0u, nb, INFINITY};
    const int n_k = min(top_k, nb);
    const float total = sum_ge(0u);
    if (!(top_p < 1.f) || total < top_p) {       // Top-p takes the whole row
        if (top_p < 1.f && nb > n_k && nb >= 2) {
            // n_p = nb falls to nb - 1 once the nb - 1 largest reach p
            uint32_t lo = 0u, hi = 0x3F800001u;      // smallest value: count{P >= lo} == nb
            while (hi - lo > 1u) {
                const uint32_t mid = lo + ((hi - lo) >> 1);
                if (count_ge(mid) >= nb) lo = mid;
                else hi = mid;
            }
            c.gap_p = top_p - (total - __uint_as_float(lo));
        }
        return c;
    }
    constexpr uint32_t kHi = 0x3F800001u;        // (1.0f bits) + 1: no P reaches it
    // Top-k threshold and S_k
    uint32_t lo_k = 0u;
    int gt_k = 0;
    bool k_sets = false;
    if (n_k > 0) {
        uint32_t lo = 0u, hi = kHi;              // count{P >= lo} >= n_k > count{P >= hi}
        while (hi - lo > 1u) {
            const uint32_t mid = lo + ((hi - lo) >> 1);
            if (count_ge(mid) >= n_k) lo = mid;
            else hi = mid;
        }
        lo_k = lo;
        gt_k = count_ge(lo + 1u);
        const float vk = __uint_as_float(lo);
        const float S_k = sum_ge(lo + 1u) + (float)(n_k - gt_k) * vk;
        if (S_k >= top_p) {                      // n_p <= n_k: Top-k sets n; a shorter Top-p
            k_sets = true;                       // prefix changes nothing, a longer one does
            if (n_k < nb) c.gap_p = S_k - top_p;
        }
    }
    if (!k_sets) {
        // largest bit pattern t with sum{P >= t} >= p: lo keeps the property, hi does not
        uint32_t lo = 0u, hi = kHi;
        while (hi - lo > 1u) {
            const uint32_t mid = lo + ((hi - lo) >> 1);
            if (sum_ge(mid) >= top_p) lo = mid;
            else hi = mid;
        }
        const float vstar = __uint_as_float(lo);
        const float s_gt = sum_ge(lo + 1u);
        const int c_gt = count_ge(lo + 1u), c_eq = count_ge(lo) - c_gt;
        int m = c_eq;                                           // fewest ties at v* reaching p
        if (vstar > 0.f) {
            const float need = ceilf((top_p - s_gt) / vstar);
            m = need < 1.f ? 1 : (need > (float)c_eq ? c_eq : (int)need);
        }
        const int n_p = c_gt + m;
        if (n_p >= n_k) {
            const float c_at = s_gt + (float)m * vstar;
            const float up = n_p < nb ? c_at - top_p : INFINITY;
            const float down = (n_p > n_k && n_p >= 2) ? top_p - (c_at - vstar) : INFINITY;
            c.gap_p = fminf(up, down);
            c.n = n_p;
            c.vb = lo;
            c.need_eq = m;
            return c;
        }
        // rounding put n_p below n_k after S_k fell short of p: Top-k sets n
    }
    c.n = n_k;
    c.vb = lo_k;
    c.need_eq = n_k - gt_k;
    return c;
}

__device__ __forceinline__ void clear_row(uint32_t* srow, int SW, int lane, int nthreads, int32_t* cnt, float* mg) {
    for (int w = lane; w < SW; w += nthreads) srow[w] = 0u;
    if (lane == 0) {
        *cnt = 0;
        if (mg) *mg = INFINITY;
    }
}

// One warp per row, C values a lane in registers (value j = 32 c + lane; the
// padding lanes hold -1, below every threshold since thresholds are >= 0).
template <int C, int CLO>
__global__ void __launch_bounds__(32 * kWarpRowsPerCta) k_select_reg(const float* __restrict__ P,
                                                                     const int32_t* __restrict__ n_blk, int64_t MB,
                                                                     int SW, int top_k, float top_p,
                                                                     uint32_t* __restrict__ sel,
                                                                     int32_t* __restrict__ sel_count,
                                                                     float* __restrict__ margin) {
    const int nb = *n_blk;
    if ((CLO > 0 && nb <= 32 * CLO) || nb > 32 * C) return;          // another size class
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * kWarpRowsPerCta + (threadIdx.x >> 5), hh = blockIdx.y;
    if (i >= MB) return;                                             // warp-uniform
    const int64_t ri = (int64_t)hh * MB + i;
    uint32_t* srow = sel + ri * SW;
    if (i >= nb) {
        clear_row(srow, SW, lane, 32, sel_count + ri, margin ? margin + ri : nullptr);
        return;
    }
    const float* prow = P + ((int64_t)hh * nb + i) * nb;
    float x[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const int j = 32 * c + lane;
        x[c] = j < nb ? __ldg(prow + j) : -1.f;
    }
    // four accumulators in a fixed pattern, then a butterfly: a fixed order
    auto count_ge = [&](uint32_t t) {
        const float tf = __uint_as_float(t);
        int a[4] = {0, 0, 0, 0};
#pragma unroll
        for (int c = 0; c < C; ++c) a[c & 3] += x[c] >= tf ? 1 : 0;
        return warp_sum_i((a[0] + a[1]) + (a[2] + a[3]));
    };
    auto sum_ge = [&](uint32_t t) {
        const float tf = __uint_as_float(t);
        float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < C; ++c) a[c & 3] += x[c] >= tf ? x[c] : 0.f;
        return warp_sum((a[0] + a[1]) + (a[2] + a[3]));
    };
    const SelCut cut = select_cut(nb, top_k, top_p, count_ge, sum_ge);
    const bool all = cut.n >= nb;
    const float vbf = __uint_as_float(cut.vb);
    // bitmask in index order: word c is chunk c; a running count ranks ties by index
    const uint32_t below_me = (1u << lane) - 1u;
    int eq_seen = 0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        if (32 * c < nb) {                                           // warp-uniform
            const bool in = 32 * c + lane < nb;
            const bool gt = in && (all || x[c] > vbf);
            const bool eq = in && !all && x[c] == vbf;
            const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
            const int rank = eq_seen + __popc(eqmask & below_me);
            const uint32_t word = __ballot_sync(0xffffffffu, gt || (eq && rank < cut.need_eq));
            eq_seen += __popc(eqmask);
            if (lane == 0) srow[c] = word;
        }
    }
    for (int w = (nb + 31) / 32 + lane; w < SW; w += 32) srow[w] = 0u;
    // margins: order gap at the boundary, and the cumulative-sum gap
    float gap_o = INFINITY;
    if (!all) {
        const int c_ge = count_ge(cut.vb);
        float below = -INFINITY;
#pragma unroll
        for (int c = 0; c < C; ++c)
            if (x[c] >= 0.f && x[c] < vbf) below = fmaxf(below, x[c]);
        below = warp_max(below);
        gap_o = c_ge > cut.n ? 0.f : vbf - below;
    }
    if (lane == 0) {
        sel_count[ri] = cut.n;
        if (margin) margin[ri] = fminf(gap_o, cut.gap_p);
    }
}

// One CTA per row, the row in shared memory (rows above kWarpRowMax blocks).
__global__ void __launch_bounds__(kSelectThreads) k_select_cta(const float* __restrict__ P,
                                                              const int32_t* __restrict__ n_blk, int64_t MB,
                                                              int SW, int top_k, float top_p,
                                                              uint32_t* __restrict__ sel,
                                                              int32_t* __restrict__ sel_count,
                                                              float* __restrict__ margin,
                                                              uint32_t* __restrict__ dev_status) {
    extern __shared__ float row[];
    __shared__ SelRed red;
    const int nb = *n_blk;
    if (nb <= kWarpRowMax) return;                                  // the warp form's rows
    const int tid = threadIdx.x;
    const int i = blockIdx.x, hh = blockIdx.y;
    const int64_t ri = (int64_t)hh * MB + i;
    uint32_t* srow = sel + ri * SW;
    if (i >= nb || nb > kSelectMaxRow) {
        clear_row(srow, SW, tid, kSelectThreads, sel_count + ri, margin ? margin + ri : nullptr);
        if (tid == 0 && nb > kSelectMaxRow && i == 0 && hh == 0) atomicOr(dev_status, PRISM_DEV_BAD_INDEX);
        return;
    }
    const float* prow = P + ((int64_t)hh * nb + i) * nb;
    for (int j = tid; j < nb; j += kSelectThreads) row[j] = prow[j];
    __syncthreads();
    auto sum_ge = [&](uint32_t tb) {
        float s = 0.f;
        for (int j = tid; j < nb; j += kSelectThreads) {
            const float x = row[j];
            if (__float_as_uint(x) >= tb) s += x;
        }
        return sel_sum(s, red);
    };
    auto count_ge = [&](uint32_t tb) {
        int c = 0;
        for (int j = tid; j < nb; j += kSelectThreads) c += __float_as_uint(row[j]) >= tb;
        return sel_count_i(c, red);
    };
    const SelCut cut = select_cut(nb, top_k, top_p, count_ge, sum_ge);
    const bool all = cut.n >= nb;
    // bitmask in index order (warp 0; a running count ranks ties by index)
    if (tid < 32) {
        int eq_seen = 0;
        const int wn = (nb + 31) >> 5;
        for (int w = 0; w < SW; ++w) {
            uint32_t word = 0u;
            if (w < wn) {
                const int j = w * 32 + tid;
                const bool in = j < nb;
                const uint32_t xb = in ? __float_as_uint(row[j]) : 0u;
                const bool gt = in && (all || xb > cut.vb);
                const bool eq = in && !all && xb == cut.vb;
                const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
                const int rank = eq_seen + __popc(eqmask & ((1u << tid) - 1u));
                word = __ballot_sync(0xffffffffu, gt || (eq && rank < cut.need_eq));
                eq_seen += __popc(eqmask);
            }
            if (tid == 0) srow[w] = word;
        }
    }
    float gap_o = INFINITY;
    if (!all) {
        const int c_ge = count_ge(cut.vb);
        float below = -INFINITY;
        for (int j = tid; j < nb; j += kSelectThreads)
            if (__float_as_uint(row[j]) < cut.vb) below = fmaxf(below, row[j]);
        below = sel_max(below, red);
        gap_o = c_ge > cut.n ? 0.f : __uint_as_float(cut.vb) - below;
    }
    if (tid == 0) {
        sel_count[ri] = cut.n;
        if (margin) margin[ri] = fminf(gap_o, cut.gap_p);
    }
}

// Granule-level view of the selection for the attention kernels: row qg (a
// 64-row query granule) has bit kg set when the block of key granule kg is
// in S of the block of qg.  Same size as the block-level mask (N/64 rows of
// N/64 bits), but a kernel reads key rows straight from the bit position.
__global__ void __launch_bounds__(128) k_sel_expand(const uint32_t* __restrict__ sel,
                                                    const int32_t* __restrict__ blk_start,
                                                    const int32_t* __restrict__ gran_blk,
                                                    const int32_t* __restrict__ n_blk, int64_t MB, int SW,
                                                    uint32_t* __restrict__ gsel) {
    extern __shared__ uint32_t gwords[];
    const int qg = blockIdx.x, hh = blockIdx.y;
    const int nb = *n_blk;
    for (int w = threadIdx.x; w < SW; w += blockDim.x) gwords[w] = 0u;
    __syncthreads();
    const int i = gran_blk[qg];
    if (i >= 0 && i < nb) {
        const uint32_t* srow = sel + ((int64_t)hh * MB + i) * SW;
        const int wn = (nb + 31) >> 5;
        for (int w = threadIdx.x; w < wn; w += blockDim.x) {
            uint32_t b = srow[w];
            while (b) {
                const int j = w * 32 + __ffs(b) - 1;
                b &= b - 1;
                const int g0 = blk_start[j] >> 6, g1 = blk_start[j + 1] >> 6;   // granules [g0, g1)
                for (int g = g0; g < g1; ++g) atomicOr(&gwords[g >> 5], 1u << (g & 31));
            }
        }
    }
    __syncthreads();
    uint32_t* out = gsel + ((int64_t)hh * MB + qg) * SW;
    for (int w = threadIdx.x; w < SW; w += blockDim.x) out[w] = gwords[w];
}

// Bit-matrix transpose, one warp per 32x32 tile: lane l holds row (32 rt + l)
// word wc; ballot over bit b gives row (32 wc + b) of the transpose.
__global__ void __launch_bounds__(256) k_bit_transpose(const uint32_t* __restrict__ in, int64_t MB, int SW,
                                                       uint32_t* __restrict__ out) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int wc = blockIdx.x;                         // source word column
    const int rt = blockIdx.y * 8 + wid;               // source row tile
    const int hh = blockIdx.z;
    if (rt >= SW) return;                              // warp-uniform
    const int64_t r = (int64_t)rt * 32 + lane;
    const uint32_t x = r < MB ? in[((int64_t)hh * MB + r) * SW + wc] : 0u;
    uint32_t mine = 0u;
#pragma unroll
    for (int b = 0; b < 32; ++b) {
        const uint32_t t = __ballot_sync(0xffffffffu, (x >> b) & 1u);
        if (lane == b) mine = t;
    }
    const int64_t orow = (int64_t)wc * 32 + lane;
    if (orow < MB) out[((int64_t)hh * MB + orow) * SW + rt] = mine;
}

}  // namespace prism

using namespace prism;

extern "C" prism_status_t prism_block_select(const prism_problem_t* prob, const float* P,
                                             const int32_t* blk_start, const int32_t* gran_blk,
                                             const int32_t* n_blk, int32_t top_k, float top_p,
                                             uint32_t* sel, int32_t* sel_count, uint32_t* gsel,
                                             uint32_t* gselT, float* margin, uint32_t* dev_status,
                                             cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(P) || !ok_ptr(blk_start) || !ok_ptr(gran_blk) || !ok_ptr(n_blk) || !ok_ptr(sel) ||
        !ok_ptr(sel_count) || !ok_ptr(gsel) || !ok_opt(gselT) || !ok_opt(margin) || !ok_ptr(dev_status))
        return PRISM_ERR_INVALID_ARG;
    if (top_k < 0 || !(top_p > 0.f) || !isfinite(top_p)) return PRISM_ERR_INVALID_ARG;
    // n_blk is known on the device only: every size class that n_blk <= MB can
    // reach is launched, and each kernel handles only the rows of its own class
    const dim3 wgrid((unsigned)((d.MB + kWarpRowsPerCta - 1) / kWarpRowsPerCta), (unsigned)d.heads);
    const int wthreads = 32 * kWarpRowsPerCta;
    int launches = 0;
#define PRISM_SELECT_CLASS(C, CLO)                                                                        \
    if (d.MB > 32 * (CLO)) {                                                                             \
        k_select_reg<C, CLO><<<wgrid, wthreads, 0, stream>>>(P, n_blk, d.MB, (int)d.SW, top_k, top_p, sel, \
                                                              sel_count, margin);                        \
        ++launches;                                                                                      \
    }
    PRISM_SELECT_CLASS(16, 0)
    PRISM_SELECT_CLASS(32, 16)
    PRISM_SELECT_CLASS(64, 32)
    PRISM_SELECT_CLASS(128, 64)
#undef PRISM_SELECT_CLASS
    if (d.MB > kWarpRowMax) {
        const int rowcap = (int)(d.MB < kSelectMaxRow ? d.MB : kSelectMaxRow);
        const size_t smem = (size_t)rowcap * sizeof(float);
        if (cudaFuncSetAttribute(k_select_cta, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return PRISM_ERR_CUDA;
        k_select_cta<<<dim3((unsigned)d.MB, (unsigned)d.heads), kSelectThreads, smem, stream>>>(
            P, n_blk, d.MB, (int)d.SW, top_k, top_p, sel, sel_count, margin, dev_status);
        ++launches;
    }
    k_sel_expand<<<dim3((unsigned)d.MB, (unsigned)d.heads), 128, (size_t)d.SW * 4, stream>>>(
        sel, blk_start, gran_blk, n_blk, d.MB, (int)d.SW, gsel);
    if (gselT)
        k_bit_transpose<<<dim3((unsigned)d.SW, (unsigned)((d.SW + 7) / 8), (unsigned)d.heads), 256, 0, stream>>>(
            gsel, d.MB, (int)d.SW, gselT);
    return launch_status(launches + (gselT ? 2 : 1));
}
