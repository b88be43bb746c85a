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
// k_block_select     one CTA per (row, head): the row's (P, j) pairs packed
//                    into 64-bit keys (P's bits are order-preserving since
//                    P >= 0; ~j breaks ties towards smaller j), bitonic sort
//                    in shared memory, block scan of the sorted probabilities,
//                    bitmask of the first n entries.
// k_select_transpose key-major copy of the bitmask for the backward pass.
#include "common.cuh"

namespace prism {

constexpr int kSelectMaxRow = 16384;    // keys per row held in shared memory

__device__ __forceinline__ float key_p(unsigned long long k) { return __uint_as_float((unsigned)(k >> 32)); }
__device__ __forceinline__ int key_j(unsigned long long k) { return (int)(0xffffffffu - (unsigned)(k & 0xffffffffu)); }

__global__ void __launch_bounds__(512) k_block_select(const float* __restrict__ P,
                                                      const int32_t* __restrict__ n_blk, int64_t MB,
                                                      int SW, int keycap, int top_k, float top_p,
                                                      uint32_t* __restrict__ sel,
                                                      int32_t* __restrict__ sel_count,
                                                      float* __restrict__ margin,
                                                      uint32_t* __restrict__ dev_status) {
    extern __shared__ unsigned long long keys[];
    __shared__ int s_first;
    __shared__ float s_cat, s_cbef, s_tot;
    __shared__ float wsum[16];
    uint32_t* bits = reinterpret_cast<uint32_t*>(keys + keycap);   // SW words

    const int i = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x, nt = blockDim.x;
    const int nb = *n_blk;
    uint32_t* srow = sel + ((int64_t)hh * MB + i) * SW;
    if (i >= nb || nb > keycap) {
        for (int w = tid; w < SW; w += nt) srow[w] = 0u;
        if (tid == 0) {
            sel_count[(int64_t)hh * MB + i] = 0;
            if (margin) margin[(int64_t)hh * MB + i] = INFINITY;
            if (nb > keycap && i == 0 && hh == 0) atomicOr(dev_status, PRISM_DEV_BAD_INDEX);
        }
        return;
    }
    int n2 = 1;
    while (n2 < nb) n2 <<= 1;
    const float* prow = P + ((int64_t)hh * nb + i) * nb;
    for (int j = tid; j < n2; j += nt)
        keys[j] = j < nb ? (((unsigned long long)__float_as_uint(prow[j]) << 32) | (0xffffffffu - (unsigned)j))
                         : 0ull;
    for (int w = tid; w < SW; w += nt) bits[w] = 0u;
    if (tid == 0) s_first = nb;
    __syncthreads();

    // bitonic sort, descending
    for (int k = 2; k <= n2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int q = tid; q < (n2 >> 1); q += nt) {
                const int a = 2 * j * (q / j) + (q % j), b = a + j;
                const unsigned long long ka = keys[a], kb = keys[b];
                const bool desc = (a & k) == 0;
                if (desc ? (ka < kb) : (ka > kb)) { keys[a] = kb; keys[b] = ka; }
            }
            __syncthreads();
        }
    }

    // cumulative sum in sorted order: contiguous segment per thread
    const int L = (nb + nt - 1) / nt;
    const int s0 = tid * L, s1 = min(nb, s0 + L);
    float local = 0.f;
    for (int q = s0; q < s1; ++q) local += key_p(keys[q]);
    // exclusive scan of `local` over threads
    const int lane = tid & 31, wid = tid >> 5;
    float incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    float woff = 0.f;
    for (int w = 0; w < wid; ++w) woff += wsum[w];
    float c = woff + incl - local;
    if (tid == nt - 1) s_tot = c + local;
    bool found = false;
    float cat = 0.f, cbef = 0.f;
    int first = nb;
    for (int q = s0; q < s1 && !found; ++q) {
        const float prev = c;
        c += key_p(keys[q]);
        if (c >= top_p) { found = true; first = q; cat = c; cbef = prev; }
    }
    if (found) atomicMin(&s_first, first);
    __syncthreads();
    if (found && first == s_first) { s_cat = cat; s_cbef = cbef; }
    __syncthreads();

    const int n_k = min(top_k, nb);
    int n_p;
    float gap_p = INFINITY;
    if (top_p >= 1.f) {
        n_p = nb;
    } else {
        float c_at, c_before;
        if (s_first < nb) {
            n_p = s_first + 1;
            c_at = s_cat;
            c_before = n_p >= 2 ? s_cbef : -INFINITY;
        } else {
            n_p = nb;
            c_at = s_tot;
            c_before = nb >= 2 ? s_tot - key_p(keys[nb - 1]) : -INFINITY;
        }
        if (n_p >= n_k) gap_p = fminf(fabsf(c_at - top_p), fabsf(top_p - c_before));
    }
    const int n = max(n_k, n_p);
    for (int q = tid; q < n; q += nt) {
        const int j = key_j(keys[q]);
        atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    for (int w = tid; w < SW; w += nt) srow[w] = bits[w];
    if (tid == 0) {
        sel_count[(int64_t)hh * MB + i] = n;
        if (margin) {
            const float gap_o = n < nb ? key_p(keys[n - 1]) - key_p(keys[n]) : INFINITY;
            margin[(int64_t)hh * MB + i] = fminf(gap_o, gap_p);
        }
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
    extern __shared__ uint32_t row[];
    const int qg = blockIdx.x, hh = blockIdx.y;
    const int nb = *n_blk;
    for (int w = threadIdx.x; w < SW; w += blockDim.x) row[w] = 0u;
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
                for (int g = g0; g < g1; ++g) atomicOr(&row[g >> 5], 1u << (g & 31));
            }
        }
    }
    __syncthreads();
    uint32_t* out = gsel + ((int64_t)hh * MB + qg) * SW;
    for (int w = threadIdx.x; w < SW; w += blockDim.x) out[w] = row[w];
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

int select_keycap(const Dims& d) {
    int cap = 1;
    while (cap < d.MB && cap < kSelectMaxRow) cap <<= 1;
    return cap;
}

size_t select_smem_bytes(const Dims& d) {
    return (size_t)select_keycap(d) * 8 + (size_t)d.SW * 4;
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
    if (top_k < 1 || !(top_p > 0.f) || !isfinite(top_p)) return PRISM_ERR_INVALID_ARG;
    size_t smem = select_smem_bytes(d);
    if (smem > 227 * 1024) return PRISM_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(k_block_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return PRISM_ERR_CUDA;
    k_block_select<<<dim3((unsigned)d.MB, (unsigned)d.heads), 512, smem, stream>>>(
        P, n_blk, d.MB, (int)d.SW, select_keycap(d), top_k, top_p, sel, sel_count, margin, dev_status);
    k_sel_expand<<<dim3((unsigned)d.MB, (unsigned)d.heads), 128, (size_t)d.SW * 4, stream>>>(
        sel, blk_start, gran_blk, n_blk, d.MB, (int)d.SW, gsel);
    if (gselT)
        k_bit_transpose<<<dim3((unsigned)d.SW, (unsigned)((d.SW + 7) / 8), (unsigned)d.heads), 256, 0, stream>>>(
            gsel, d.MB, (int)d.SW, gselT);
    return launch_status(gselT ? 3 : 2);
}
