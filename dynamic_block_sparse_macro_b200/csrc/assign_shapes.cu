// Stage 2: block volume, shape quantisation and the token permutation.
//
// Prism, Portuguese reading guide, "Método" 2 (Volume do Bloco e Quantização
// do Formato): B(m) in {64,128,256} from rho(m) against tau_128 = 0.5 and
// tau_256 = 0.25; minimising sum_d g_d (b_d^2 - 1) under prod_d b_d = B gives
// b*_d proportional to g_d^{-1/2}, i.e. in log2 space
//   l*_d = -1/2 log2 g_d + (S + 1/2 sum_d' log2 g_d') / 3,  S = log2 B,
// and the shape is the candidate of C_B nearest to l* (Euclidean distance).
// The 16 candidates (never listed on the pages) are read as the power-of-two
// edge triples in {2,4,8} with product B: 7 of volume 64, 6 of 128, 3 of 256.
// Higher rho unlocks the smaller volume; exact distance ties go to the
// smaller shape id (ids ordered by volume, then b_T, b_H, b_W).
//
// The news page ("工作原理" step 4) runs the sparse kernel over blocks and
// then restores the original layout; the permutation here places zones in
// raster order, blocks in raster order inside a zone and tokens in raster
// order inside a block, so zone m owns rows [512 m, 512 m + 512).
//
// k_assign_shapes   one CTA: per-zone decision, block-count scan, blk_start,
//                   gran_blk, n_blk.
// k_build_perm      one thread per permuted row.
#include "common.cuh"

namespace prism {

constexpr int kMaxZonesPerThread = 32;   // N <= 2^24 -> Z <= 32768 = 32 * 1024

__global__ void __launch_bounds__(1024) k_assign_shapes(const float* __restrict__ g,
                                                        const float* __restrict__ rho, int Z,
                                                        float tau128, float tau256, int64_t MB,
                                                        int N, uint8_t* __restrict__ shape_id,
                                                        int32_t* __restrict__ blk_start,
                                                        int32_t* __restrict__ gran_blk,
                                                        int32_t* __restrict__ n_blk,
                                                        float* __restrict__ margin, int fixed) {
    __shared__ int sE[16][3];
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int tid = threadIdx.x, nt = blockDim.x;
    if (tid < 16) shape_exponents(tid, &sE[tid][0], &sE[tid][1], &sE[tid][2]);
    if (tid == 0) carry = 0;
    __syncthreads();

    int myB[kMaxZonesPerThread];
    int nz = 0;
    for (int m = tid; m < Z; m += nt, ++nz) {
        const float r = rho[m];
        const int S = fixed >= 0 ? sE[fixed][0] + sE[fixed][1] + sE[fixed][2]   // fixed-shape baseline
                                 : (r >= tau128 ? 6 : (r >= tau256 ? 7 : 8));
        const float l0 = log2f(g[m * 3 + 0]), l1 = log2f(g[m * 3 + 1]), l2 = log2f(g[m * 3 + 2]);
        const float common_term = ((float)S + 0.5f * (l0 + l1 + l2)) / 3.f;
        const float e0 = -0.5f * l0 + common_term, e1 = -0.5f * l1 + common_term,
                    e2 = -0.5f * l2 + common_term;
        float best = INFINITY, second = INFINITY;
        int bid = -1;
        for (int id = 0; id < 16; ++id) {
            if (sE[id][0] + sE[id][1] + sE[id][2] != S) continue;
            const float a = (float)sE[id][0] - e0, b = (float)sE[id][1] - e1,
                        c = (float)sE[id][2] - e2;
            const float dd = a * a + b * b + c * c;
            if (dd < best) { second = best; best = dd; bid = id; }
            else if (dd < second) second = dd;
        }
        shape_id[m] = (uint8_t)(fixed >= 0 ? fixed : bid);
        myB[nz] = 1 << S;
        if (margin) {                                   // no decision is taken for a fixed shape
            margin[m * 2 + 0] = fixed >= 0 ? INFINITY : second - best;
            margin[m * 2 + 1] = fixed >= 0 ? INFINITY : fminf(fabsf(r - tau128), fabsf(r - tau256));
        }
    }

    // exclusive scan of blocks-per-zone (512 / B) in zone order, 1024 zones per round
    nz = 0;
    const int lane = tid & 31, wid = tid >> 5;
    for (int base = 0; base < Z; base += nt, ++nz) {
        const int m = base + tid;
        const int cnt = m < Z ? 512 / myB[nz] : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int v = lane < (nt >> 5) ? warp_tot[lane] : 0;
            int vi = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int u = __shfl_up_sync(0xffffffffu, vi, o);
                if (lane >= o) vi += u;
            }
            warp_tot[lane] = vi - v;               // exclusive prefix of warp totals
        }
        __syncthreads();
        const int boff = carry + warp_tot[wid] + incl - cnt;
        if (m < Z) {
            const int B = myB[nz];
            for (int k = 0; k < 512 / B; ++k) blk_start[boff + k] = m * 512 + k * B;
            for (int q = 0; q < 8; ++q) gran_blk[m * 8 + q] = boff + (q * 64) / B;
        }
        __syncthreads();
        if (tid == nt - 1) carry = boff + cnt;
        __syncthreads();
    }
    const int total = carry;
    for (int64_t j = total + tid; j <= MB; j += nt) blk_start[j] = N;
    if (tid == 0) *n_blk = total;
}

__global__ void k_build_perm(const uint8_t* __restrict__ shape_id, int H, int W, int N,
                             int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
    __shared__ int sE[16][3];
    if (threadIdx.x < 16)
        shape_exponents(threadIdx.x, &sE[threadIdx.x][0], &sE[threadIdx.x][1], &sE[threadIdx.x][2]);
    __syncthreads();
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= N) return;
    const int m = p >> 9, l = p & 511;
    const int ZH = H / 8, ZW = W / 8;
    const int zt = m / (ZH * ZW), zh = (m / ZW) % ZH, zw = m % ZW;
    const int sid = shape_id[m];
    const int bT = 1 << sE[sid][0], bH = 1 << sE[sid][1], bW = 1 << sE[sid][2];
    const int B = bT * bH * bW;
    const int nbH = 8 / bH, nbW = 8 / bW;
    const int blk = l / B, o = l % B;
    const int bt = blk / (nbH * nbW), bh = (blk / nbW) % nbH, bw = blk % nbW;
    const int ot = o / (bH * bW), oh = (o / bW) % bH, ow = o % bW;
    const int t = zt * 8 + bt * bT + ot, h = zh * 8 + bh * bH + oh, w = zw * 8 + bw * bW + ow;
    const int r = (t * H + h) * W + w;
    perm[p] = r;
    if (inv_perm) inv_perm[r] = p;
}

}  // namespace prism

using namespace prism;

extern "C" prism_status_t prism_assign_shapes_ex(const prism_problem_t* prob, const float* g,
                                                 const float* rho, float tau128, float tau256,
                                                 int32_t fixed_shape, uint8_t* shape_id, int32_t* perm,
                                                 int32_t* inv_perm, int32_t* blk_start, int32_t* gran_blk,
                                                 int32_t* n_blk, float* margin, cudaStream_t stream) {
    if (fixed_shape < -1 || fixed_shape > 15) return PRISM_ERR_INVALID_ARG;
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(g) || !ok_ptr(rho) || !ok_ptr(shape_id) || !ok_ptr(perm) || !ok_opt(inv_perm) ||
        !ok_ptr(blk_start) || !ok_ptr(gran_blk) || !ok_ptr(n_blk) || !ok_opt(margin))
        return PRISM_ERR_INVALID_ARG;
    if (!isfinite(tau128) || !isfinite(tau256) || !(tau256 <= tau128)) return PRISM_ERR_INVALID_ARG;
    k_assign_shapes<<<1, 1024, 0, stream>>>(g, rho, (int)d.Z, tau128, tau256, d.MB, (int)d.N,
                                            shape_id, blk_start, gran_blk, n_blk, margin, fixed_shape);
    const int thr = 256;
    k_build_perm<<<(unsigned)((d.N + thr - 1) / thr), thr, 0, stream>>>(shape_id, d.H, d.W,
                                                                         (int)d.N, perm, inv_perm);
    return launch_status(2);
}

extern "C" prism_status_t prism_assign_shapes(const prism_problem_t* prob, const float* g,
                                              const float* rho, float tau128, float tau256,
                                              uint8_t* shape_id, int32_t* perm, int32_t* inv_perm,
                                              int32_t* blk_start, int32_t* gran_blk,
                                              int32_t* n_blk, float* margin, cudaStream_t stream) {
    return prism_assign_shapes_ex(prob, g, rho, tau128, tau256, -1, shape_id, perm, inv_perm, blk_start,
                                  gran_blk, n_blk, margin, stream);
}
