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
// k_block_score   128x128 fp32 SIMT tiles of Qbar Kbar^T, 8x8 outputs a
//                 thread (kept in fp32: the scores feed discrete decisions
//                 compared against an fp64 definition, so no reduced-precision
//                 tensor path here).
// k_row_softmax   one warp per row, in place, fixed-order reductions.
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

// S[h][i][j] = scale * sum_c Qbar[h][i][c] * Kbar[h][j][c], written packed at (h*nb + i)*nb + j.
// A 128x128 tile per CTA; 256 threads as 16x16, each owning an 8x8 sub-grid (rows ty*4+u and
// 64+ty*4+u, columns tx*4+v and 64+tx*4+v) so that every step over c reads four 16-byte words
// of shared memory for 64 FMAs.  The operands move in panels of 16 columns, stored transposed
// ([c][row]) and double-buffered, the next panel held in registers while the current one is
// multiplied.  Each output is one fp32 FMA chain over c = 0..d-1 in order.
constexpr int kScT = 128, kScK = 16, kScLd = kScT + 4;

__global__ void __launch_bounds__(256, 2) k_block_score(const float* __restrict__ Qbar,
                                                        const float* __restrict__ Kbar,
                                                        const int32_t* __restrict__ n_blk, int64_t MB,
                                                        int d, float scale, float* __restrict__ P) {
    __shared__ __align__(16) float As[2][kScK][kScLd];
    __shared__ __align__(16) float Bs[2][kScK][kScLd];
    const int nb = *n_blk;
    const int i0 = blockIdx.y * kScT, j0 = blockIdx.x * kScT, hh = blockIdx.z;
    if (i0 >= nb || j0 >= nb) return;
    const float* A = Qbar + (int64_t)hh * MB * d;
    const float* B = Kbar + (int64_t)hh * MB * d;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    // panel fetch: 128 rows x 4 column quads per operand, two quads a thread, row-fastest so
    // that the transposed shared-memory stores of a warp fall on 32 distinct banks
    float4 pa[2], pb[2];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int q = threadIdx.x + u * 256, r = q & (kScT - 1), c = k0 + (q >> 7) * 4;
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            pa[u] = i0 + r < nb ? __ldg(reinterpret_cast<const float4*>(A + (int64_t)(i0 + r) * d + c)) : z;
            pb[u] = j0 + r < nb ? __ldg(reinterpret_cast<const float4*>(B + (int64_t)(j0 + r) * d + c)) : z;
        }
    };
    auto stash = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int q = threadIdx.x + u * 256, r = q & (kScT - 1), c = (q >> 7) * 4;
            As[buf][c + 0][r] = pa[u].x; As[buf][c + 1][r] = pa[u].y;
            As[buf][c + 2][r] = pa[u].z; As[buf][c + 3][r] = pa[u].w;
            Bs[buf][c + 0][r] = pb[u].x; Bs[buf][c + 1][r] = pb[u].y;
            Bs[buf][c + 2][r] = pb[u].z; Bs[buf][c + 3][r] = pb[u].w;
        }
    };
    float acc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
    const int nk = d / kScK;
    fetch(0);
    stash(0);
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < nk) fetch((kt + 1) * kScK);
#pragma unroll
        for (int c = 0; c < kScK; ++c) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][c][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][c][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][c][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][c][64 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
        }
        // the buffer written next was last read before the previous barrier
        if (kt + 1 < nk) stash(buf ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int i = i0 + (u < 4 ? ty * 4 + u : 64 + ty * 4 + u - 4);
        if (i >= nb) continue;
        float* row = P + ((int64_t)hh * nb + i) * nb;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int j = j0 + (v < 4 ? tx * 4 + v : 64 + tx * 4 + v - 4);
            if (j < nb) row[j] = acc[u][v] * scale;
        }
    }
}

// one warp per row of P (rows h*nb + i, all heads): max, sum of exponentials, normalise, in
// place.  The row is read three times; the second and third reads find it in L1.
__global__ void __launch_bounds__(256) k_row_softmax(float* __restrict__ P, const int32_t* __restrict__ n_blk,
                                                     int heads) {
    const int nb = *n_blk;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= (int64_t)heads * nb) return;
    const int lane = threadIdx.x & 31;
    float* r = P + row * nb;
    float mx = -INFINITY;
    for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, r[j]);
    mx = warp_max(mx);
    float s = 0.f;
    for (int j = lane; j < nb; j += 32) s += expf(r[j] - mx);
    s = warp_sum(s);
    const float inv = 1.f / s;
    for (int j = lane; j < nb; j += 32) r[j] = expf(r[j] - mx) * inv;
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
    const unsigned tiles = (unsigned)((d.MB + kScT - 1) / kScT);
    k_block_score<<<dim3(tiles, tiles, (unsigned)d.heads), 256, 0, stream>>>(Qbar, Kbar, n_blk, d.MB,
                                                                             d.d, scale, P);
    const unsigned rows8 = (unsigned)(((int64_t)d.heads * d.MB + 7) / 8);
    k_row_softmax<<<rows8, 256, 0, stream>>>(P, n_blk, d.heads);
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
