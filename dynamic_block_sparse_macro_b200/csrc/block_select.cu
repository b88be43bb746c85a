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
// k_block_select   one warp per (row, head) for rows of up to 4096 blocks, one
//                  256-thread CTA per row above that; no sort.  For P >= 0 the float bit
//                  pattern orders like the value, so thresholds are found by
//                  binary search over bit patterns with block reductions over
//                  the row held in shared memory:
//                    v* = largest t with sum{P_j : P_j >= t} >= p   (Top-p
//                         crossing value; n_p = #{P > v*} + the fewest ties
//                         at v* that reach p),
//                    v_n = largest t with #{P_j >= t} >= n  (n-th value),
//                  then S_i = {P > v_n} plus the lowest-index ties at v_n.
//                  All reductions run in a fixed order (deterministic).  Every
//                  search step is a pass over the row and a reduction, so the
//                  warp form (shuffles, no block barrier) does the same work
//                  in a fraction of the time.
// k_sel_expand     granule-level view of the selection for the attention
//                  kernels; k_bit_transpose its key-major transpose.
#include "common.cuh"

namespace prism {

constexpr int kSelectThreads = 256;
constexpr int kSelectMaxRow = 16384;    // P values of a row held in shared memory
constexpr int kWarpRowMax = 4096;       // rows up to this many blocks: one warp each
constexpr int kWarpRowsPerCta = 4;

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
// the same reductions over one warp (butterfly: every lane gets the result)
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
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

// TPR threads per row: 32 (one warp per row, kWarpRowsPerCta rows per CTA)
// or kSelectThreads (one CTA per row); each form leaves the other's rows alone.
template <int TPR>
__global__ void __launch_bounds__(kSelectThreads) k_block_select(const float* __restrict__ P,
                                                                 const int32_t* __restrict__ n_blk, int64_t MB,
                                                                 int SW, int rowcap, int top_k, float top_p,
                                                                 uint32_t* __restrict__ sel,
                                                                 int32_t* __restrict__ sel_count,
                                                                 float* __restrict__ margin,
                                                                 uint32_t* __restrict__ dev_status) {
    constexpr bool kWarp = TPR == 32;
    extern __shared__ float smem_rows[];
    __shared__ SelRed red;
    const int nb = *n_blk;
    if (kWarp ? nb > kWarpRowMax : nb <= kWarpRowMax) return;      // the other form's rows
    const int tid = kWarp ? (threadIdx.x & 31) : threadIdx.x;
    const int i = kWarp ? blockIdx.x * kWarpRowsPerCta + (threadIdx.x >> 5) : blockIdx.x, hh = blockIdx.y;
    if (kWarp && i >= MB) return;                                   // warp-uniform
    float* row = smem_rows + (kWarp ? (threadIdx.x >> 5) * rowcap : 0);
    uint32_t* srow = sel + ((int64_t)hh * MB + i) * SW;
    if (i >= nb || nb > kSelectMaxRow) {
        for (int w = tid; w < SW; w += TPR) srow[w] = 0u;
        if (tid == 0) {
            sel_count[(int64_t)hh * MB + i] = 0;
            if (margin) margin[(int64_t)hh * MB + i] = INFINITY;
            if (nb > kSelectMaxRow && i == 0 && hh == 0) atomicOr(dev_status, PRISM_DEV_BAD_INDEX);
        }
        return;
    }
    const float* prow = P + ((int64_t)hh * nb + i) * nb;
    for (int j = tid; j < nb; j += TPR) row[j] = prow[j];
    if (kWarp) __syncwarp();
    else __syncthreads();

    // sum and count of {P >= t}, {P > t}, {P == t} over the row
    auto sum_ge = [&](uint32_t tb) {
        float s = 0.f;
        for (int j = tid; j < nb; j += TPR) {
            const float x = row[j];
            if (__float_as_uint(x) >= tb) s += x;
        }
        return kWarp ? warp_sum(s) : sel_sum(s, red);
    };
    auto count_ge = [&](uint32_t tb) {
        int c = 0;
        for (int j = tid; j < nb; j += TPR) c += __float_as_uint(row[j]) >= tb;
        return kWarp ? warp_sum_i(c) : sel_count_i(c, red);
    };

    const int n_k = min(top_k, nb);
    int n_p = nb;
    float gap_p = INFINITY;
    const float total = sum_ge(0u);
    if (top_p < 1.f) {
        float c_at, c_before;
        if (total >= top_p) {
            // largest bit pattern t with sum{P >= t} >= p: lo keeps the property, hi does not
            uint32_t lo = 0u, hi = 0x3F800001u;                 // (1.0f bits) + 1
            while (hi - lo > 1u) {
                const uint32_t mid = lo + ((hi - lo) >> 1);
                if (sum_ge(mid) >= top_p) lo = mid;
                else hi = mid;
            }
            const float vstar = __uint_as_float(lo);
            const float s_gt = sum_ge(lo + 1u);
            const int c_gt = count_ge(lo + 1u), c_eq = count_ge(lo) - c_gt;
            int m = c_eq;                                       // fewest ties at v* reaching p
            if (vstar > 0.f) {
                const float need = ceilf((top_p - s_gt) / vstar);
                m = need < 1.f ? 1 : (need > (float)c_eq ? c_eq : (int)need);
            }
            n_p = c_gt + m;
            c_at = s_gt + (float)m * vstar;
            c_before = n_p >= 2 ? c_at - vstar : -INFINITY;
        } else {                                                // the sum never reaches p: everything
            n_p = nb;
            c_at = total;
            c_before = -INFINITY;                               // refined below if it matters
        }
        if (n_p >= n_k) gap_p = fminf(fabsf(c_at - top_p), fabsf(top_p - c_before));
    }
    const int n = max(n_k, n_p);

    // threshold of the first n entries of the order (P desc, j asc)
    uint32_t vb = 0u;
    int c_gt = 0, need_eq = n;
    if (n < nb) {
        uint32_t lo = 0u, hi = 0x3F800001u;                     // count{P >= lo} >= n > count{P >= hi}
        while (hi - lo > 1u) {
            const uint32_t mid = lo + ((hi - lo) >> 1);
            if (count_ge(mid) >= n) lo = mid;
            else hi = mid;
        }
        vb = lo;
        c_gt = count_ge(lo + 1u);
        need_eq = n - c_gt;
    }
    // bitmask in index order (warp 0; a running count ranks ties by index)
    if (tid < 32) {
        int eq_seen = 0;
        const int wn = (nb + 31) >> 5;
        for (int w = 0; w < SW; ++w) {
            uint32_t word = 0u;
            if (w < wn) {
                const int j = w * 32 + tid;
                const uint32_t xb = j < nb ? __float_as_uint(row[j]) : 0u;
                const bool in = j < nb;
                const bool gt = in && (n >= nb || xb > vb);
                const bool eq = in && n < nb && xb == vb;
                const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
                const int rank = eq_seen + __popc(eqmask & ((1u << tid) - 1u));
                word = __ballot_sync(0xffffffffu, gt || (eq && rank < need_eq));
                eq_seen += __popc(eqmask);
            }
            if (tid == 0) srow[w] = word;
        }
    }
    // margins: order gap at the boundary, and the cumulative-sum gap
    float gap_o = INFINITY;
    if (n < nb) {
        const int c_ge = count_ge(vb);
        float below = -INFINITY;
        for (int j = tid; j < nb; j += TPR)
            if (__float_as_uint(row[j]) < vb) below = fmaxf(below, row[j]);
        below = kWarp ? warp_max(below) : sel_max(below, red);
        gap_o = c_ge > n ? 0.f : __uint_as_float(vb) - below;
    }
    if (tid == 0) {
        sel_count[(int64_t)hh * MB + i] = n;
        if (margin) margin[(int64_t)hh * MB + i] = fminf(gap_o, gap_p);
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
    // n_blk is known on the device only: both forms are launched and each
    // handles the rows of its own size class (the other exits at once)
    const int rowcap = (int)(d.MB < kSelectMaxRow ? d.MB : kSelectMaxRow);
    const int wrowcap = (int)(d.MB < kWarpRowMax ? d.MB : kWarpRowMax);
    const size_t smem = (size_t)rowcap * sizeof(float), wsmem = (size_t)kWarpRowsPerCta * wrowcap * sizeof(float);
    if (cudaFuncSetAttribute(k_block_select<kSelectThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess ||
        cudaFuncSetAttribute(k_block_select<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wsmem) !=
            cudaSuccess)
        return PRISM_ERR_CUDA;
    k_block_select<32><<<dim3((unsigned)((d.MB + kWarpRowsPerCta - 1) / kWarpRowsPerCta), (unsigned)d.heads),
                         32 * kWarpRowsPerCta, wsmem, stream>>>(P, n_blk, d.MB, (int)d.SW, wrowcap, top_k, top_p,
                                                                sel, sel_count, margin, dev_status);
    k_block_select<kSelectThreads><<<dim3((unsigned)d.MB, (unsigned)d.heads), kSelectThreads, smem, stream>>>(
        P, n_blk, d.MB, (int)d.SW, rowcap, top_k, top_p, sel, sel_count, margin, dev_status);
    k_sel_expand<<<dim3((unsigned)d.MB, (unsigned)d.heads), 128, (size_t)d.SW * 4, stream>>>(
        sel, blk_start, gran_blk, n_blk, d.MB, (int)d.SW, gsel);
    if (gselT)
        k_bit_transpose<<<dim3((unsigned)d.SW, (unsigned)((d.SW + 7) / 8), (unsigned)d.heads), 256, 0, stream>>>(
            gsel, d.MB, (int)d.SW, gselT);
    return launch_status(gselT ? 4 : 3);
}
