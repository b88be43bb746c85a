// Stage 3: gather raster tokens into block order (head-major) and the inverse
// scatter that restores the original spatio-temporal layout (Prism news page,
// "工作原理" step 4).  Pure bit copies, bound by HBM bandwidth.
//
// One warp moves one token: the token's raster row of heads*d elements is
// contiguous, and its heads land in `heads` contiguous rows of d elements in
// the blocked tensor, so both sides are read/written as 16-byte vectors and
// every 32-byte sector is used in full.  Grid-stride over tokens with a grid of
// a few CTAs per SM.
#include "common.cuh"

namespace prism {

// row_vec = 16-byte vectors per (token, head) row; heads rows per token
template <bool kGather>
__global__ void __launch_bounds__(256) k_permute(const int4* __restrict__ src, int4* __restrict__ dst,
                                                 const int32_t* __restrict__ perm, int64_t N,
                                                 int heads, int row_vec) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int tok_vec = heads * row_vec;
    for (int64_t p = warp; p < N; p += nwarps) {
        const int64_t r = perm[p];
        if ((uint64_t)r >= (uint64_t)N) continue;   // corrupt permutation: skip, never fault
        for (int v = lane; v < tok_vec; v += 32) {
            const int hh = v / row_vec, c = v - hh * row_vec;
            const int64_t blocked = ((int64_t)hh * N + p) * row_vec + c;
            const int64_t raster = r * tok_vec + v;
            if (kGather) dst[blocked] = __ldg(src + raster);
            else dst[raster] = __ldg(src + blocked);
        }
    }
}

static int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

static prism_status_t run(const prism_problem_t* prob, const void* src, const int32_t* perm,
                          void* dst, cudaStream_t stream, bool gather) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(src) || !ok_ptr(perm) || !ok_ptr(dst) || src == dst) return PRISM_ERR_INVALID_ARG;
    const int row_vec = (int)(d.d * d.esz / 16);
    const int64_t want = (d.N + 7) / 8;                    // 8 warps (tokens) per CTA
    const int64_t cap = (int64_t)num_sms() * 8;            // 8 resident CTAs per SM
    const unsigned grid = (unsigned)(want < cap ? want : cap);
    if (gather)
        k_permute<true><<<grid, 256, 0, stream>>>((const int4*)src, (int4*)dst, perm, d.N, d.heads, row_vec);
    else
        k_permute<false><<<grid, 256, 0, stream>>>((const int4*)src, (int4*)dst, perm, d.N, d.heads, row_vec);
    return launch_status(1);
}

}  // namespace prism

extern "C" prism_status_t prism_permute(const prism_problem_t* prob, const void* src_raster,
                                        const int32_t* perm, void* dst_blocked, cudaStream_t stream) {
    return prism::run(prob, src_raster, perm, dst_blocked, stream, true);
}

extern "C" prism_status_t prism_unpermute(const prism_problem_t* prob, const void* src_blocked,
                                          const int32_t* perm, void* dst_raster, cudaStream_t stream) {
    return prism::run(prob, src_blocked, perm, dst_raster, stream, false);
}
