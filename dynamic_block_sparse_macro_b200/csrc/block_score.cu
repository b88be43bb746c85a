// Stage 4: pooled block representatives and block probabilities.
//
// Prism, Portuguese reading guide, "Método" 3 (Atenção Híbrida Top-k /
// Top-p): key blocks are mean-pooled into representatives Kbar_j and scored
// against the query blocks to give block probabilities P_i.  Read here as:
// Qbar_i and Kbar_j are the means over the block's rows, s_ij =
// scale * Qbar_i . Kbar_j (scale 1/sqrt(d)), P_i = softmax_j s_ij over all
// key blocks, per head.
//
// k_block_pool    grid (max_blocks, heads, {Q,K}): one CTA per block, 16-byte
//                 row loads, fixed-order fp32 reduction (HBM bound).
// k_block_score   64x64 fp32 SIMT tiles of Qbar Kbar^T (kept in fp32: the
//                 scores feed discrete decisions compared against an fp64
//                 definition, so no reduced-precision tensor path here).
// k_row_softmax   one CTA per row, in place, fixed-order reductions.
#include "common.cuh"

namespace prism {

// perm == nullptr: Qp, Kp blocked [heads][N][d]; otherwise raster [N][heads][d],
// row r of the block order read at token perm[r]
template <typename T>
__global__ void __launch_bounds__(256) k_block_pool(const T* __restrict__ Qp, const T* __restrict__ Kp,
                                                    const int32_t* __restrict__ blk_start,
                                                    const int32_t* __restrict__ n_blk, int64_t N,
                                                    int64_t MB, int d, float* __restrict__ Qbar,
                                                    float* __restrict__ Kbar, const int32_t* __restrict__ perm,
                                                    int heads) {
    constexpr int VE = 16 / sizeof(T);
    __shared__ float red[256 * VE];
    const int j = blockIdx.x, hh = blockIdx.y, which = blockIdx.z;
    float* out = (which ? Kbar : Qbar) + ((int64_t)hh * MB + j) * d;
    const int nb = *n_blk;
    if (j >= nb) {
        for (int c = threadIdx.x; c < d; c += blockDim.x) out[c] = 0.f;
        return;
    }
    const T* base = which ? Kp : Qp;
    const T* src = perm ? base : base + (int64_t)hh * N * d;
    const int s = blk_start[j], e = blk_start[j + 1];
    const int lpr = d / VE, rg = threadIdx.x / lpr, v = threadIdx.x % lpr, RG = blockDim.x / lpr;
    float acc[VE];
#pragma unroll
    for (int k = 0; k < VE; ++k) acc[k] = 0.f;
    for (int r = s + rg; r < e; r += RG) {
        const int64_t row = perm ? (int64_t)__ldg(perm + r) * heads + hh : (int64_t)r;
        const int4 raw = __ldg(reinterpret_cast<const int4*>(src + row * d) + v);
        const T* x = reinterpret_cast<const T*>(&raw);
#pragma unroll
        for (int k = 0; k < VE; ++k) acc[k] += to_f32(x[k]);
    }
#pragma unroll
    for (int k = 0; k < VE; ++k) red[rg * d + v * VE + k] = acc[k];
    __syncthreads();
    const float inv = 1.f / (float)(e - s);
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float sum = 0.f;
        for (int q = 0; q < RG; ++q) sum += red[q * d + c];
        out[c] = sum * inv;
    }
}

// S[h][i][j] = scale * sum_c Qbar[h][i][c] * Kbar[h][j][c], written packed at (h*nb + i)*nb + j
__global__ void __launch_bounds__(256) k_block_score(const float* __restrict__ Qbar,
                                                     const float* __restrict__ Kbar,
                                                     const int32_t* __restrict__ n_blk, int64_t MB,
                                                     int d, float scale, float* __restrict__ P) {
    __shared__ float As[16][68];
    __shared__ float Bs[16][68];
    const int nb = *n_blk;
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64, hh = blockIdx.z;
    if (i0 >= nb || j0 >= nb) return;
    const float* A = Qbar + (int64_t)hh * MB * d;
    const float* B = Kbar + (int64_t)hh * MB * d;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += 16) {
        // 64 rows x 16 columns of each operand, 4 elements per thread
        for (int q = threadIdx.x; q < 64 * 16; q += 256) {
            const int r = q >> 4, c = q & 15;
            As[c][r] = (i0 + r < nb) ? A[(int64_t)(i0 + r) * d + k0 + c] : 0.f;
            Bs[c][r] = (j0 + r < nb) ? B[(int64_t)(j0 + r) * d + k0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            float a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { a[u] = As[c][ty * 4 + u]; b[u] = Bs[c][tx * 4 + u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty * 4 + u;
        if (i >= nb) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int j = j0 + tx * 4 + v;
            if (j < nb) P[((int64_t)hh * nb + i) * nb + j] = acc[u][v] * scale;
        }
    }
}

__device__ __forceinline__ float block_reduce(float v, float* sm, bool is_max) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = is_max ? warp_max(v) : warp_sum(v);
    __syncthreads();
    if (lane == 0) sm[wid] = v;
    __syncthreads();
    float r = sm[0];
    for (int k = 1; k < nw; ++k) r = is_max ? fmaxf(r, sm[k]) : r + sm[k];
    return r;
}

__global__ void __launch_bounds__(256) k_row_softmax(float* __restrict__ P,
                                                     const int32_t* __restrict__ n_blk) {
    __shared__ float sm[32];
    const int nb = *n_blk;
    const int i = blockIdx.x, hh = blockIdx.y;
    if (i >= nb) return;
    float* row = P + ((int64_t)hh * nb + i) * nb;
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) mx = fmaxf(mx, row[j]);
    mx = block_reduce(mx, sm, true);
    float s = 0.f;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s += expf(row[j] - mx);
    s = block_reduce(s, sm, false);
    const float inv = 1.f / s;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) row[j] = expf(row[j] - mx) * inv;
}

}  // namespace prism

using namespace prism;

static prism_status_t pool_score(const prism_problem_t* prob, const void* Qp, const void* Kp,
                                 const int32_t* perm, const int32_t* blk_start, const int32_t* n_blk, float scale,
                                 float* Qbar, float* Kbar, float* P, cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(Qp) || !ok_ptr(Kp) || !ok_ptr(blk_start) || !ok_ptr(n_blk) || !ok_ptr(Qbar) ||
        !ok_ptr(Kbar) || !ok_ptr(P))
        return PRISM_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return PRISM_ERR_INVALID_ARG;
    dim3 gp((unsigned)d.MB, (unsigned)d.heads, 2);
    if (d.dtype == PRISM_BF16)
        k_block_pool<__nv_bfloat16><<<gp, 256, 0, stream>>>((const __nv_bfloat16*)Qp,
                                                            (const __nv_bfloat16*)Kp, blk_start,
                                                            n_blk, d.N, d.MB, d.d, Qbar, Kbar, perm, d.heads);
    else
        k_block_pool<float><<<gp, 256, 0, stream>>>((const float*)Qp, (const float*)Kp, blk_start,
                                                    n_blk, d.N, d.MB, d.d, Qbar, Kbar, perm, d.heads);
    const unsigned tiles = (unsigned)((d.MB + 63) / 64);
    k_block_score<<<dim3(tiles, tiles, (unsigned)d.heads), 256, 0, stream>>>(Qbar, Kbar, n_blk, d.MB,
                                                                             d.d, scale, P);
    k_row_softmax<<<dim3((unsigned)d.MB, (unsigned)d.heads), 256, 0, stream>>>(P, n_blk);
    return launch_status(3);
}

extern "C" prism_status_t prism_block_pool_score(const prism_problem_t* prob, const void* Qp,
                                                 const void* Kp, const int32_t* blk_start,
                                                 const int32_t* n_blk, float scale, float* Qbar,
                                                 float* Kbar, float* P, cudaStream_t stream) {
    return pool_score(prob, Qp, Kp, nullptr, blk_start, n_blk, scale, Qbar, Kbar, P, stream);
}

// Stage 4 from raster Q, K ([N][heads][d]) through the permutation
extern "C" prism_status_t prism_block_pool_score_raster(const prism_problem_t* prob, const void* Q, const void* K,
                                                        const int32_t* perm, const int32_t* blk_start,
                                                        const int32_t* n_blk, float scale, float* Qbar, float* Kbar,
                                                        float* P, cudaStream_t stream) {
    if (!ok_ptr(perm)) return PRISM_ERR_INVALID_ARG;
    return pool_score(prob, Q, K, perm, blk_start, n_blk, scale, Qbar, Kbar, P, stream);
}
