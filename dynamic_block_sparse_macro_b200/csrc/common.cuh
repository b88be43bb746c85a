// Shared host/device helpers of the Prism CUDA library (argument checks,
// problem dimensions, dtype loads).  Nothing here computes the method itself.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <math.h>

#include "prism.h"

namespace prism {

constexpr int kZone = 8;          // 8x8x8 macro-zones
constexpr int kZoneTokens = 512;
constexpr int kGranule = 64;      // every block is a whole number of 64-row granules

struct Dims {
    int T, H, W, heads, d, Da, dtype;
    int64_t N, Z, D, MB, SW;      // tokens, zones, heads*d, max blocks, sel words per row
    size_t esz;                   // bytes per stored element
};

inline prism_status_t make_dims(const prism_problem_t* p, Dims* o) {
    if (!p || !o) return PRISM_ERR_INVALID_ARG;
    if (p->T <= 0 || p->H <= 0 || p->W <= 0 || p->T % kZone || p->H % kZone || p->W % kZone)
        return PRISM_ERR_SHAPE;
    if (p->dtype != PRISM_F32 && p->dtype != PRISM_BF16) return PRISM_ERR_UNSUPPORTED;
    if (p->head_dim != 64 && p->head_dim != 128) return PRISM_ERR_UNSUPPORTED;
    if (p->heads < 1 || p->heads > 64) return PRISM_ERR_UNSUPPORTED;
    if (p->audio_dim < 1 || p->audio_dim > 1024) return PRISM_ERR_UNSUPPORTED;
    int64_t N = (int64_t)p->T * p->H * p->W;
    if (N > (int64_t(1) << 24)) return PRISM_ERR_UNSUPPORTED;
    o->T = p->T; o->H = p->H; o->W = p->W;
    o->heads = p->heads; o->d = p->head_dim; o->Da = p->audio_dim; o->dtype = p->dtype;
    o->N = N;
    o->Z = N / kZoneTokens;
    o->D = (int64_t)p->heads * p->head_dim;
    o->MB = N / kGranule;
    o->SW = (o->MB + 31) / 32;
    o->esz = p->dtype == PRISM_BF16 ? 2 : 4;
    return PRISM_OK;
}

inline bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }
inline bool ok_ptr(const void* ptr) { return ptr != nullptr && aligned16(ptr); }
inline bool ok_opt(const void* ptr) { return ptr == nullptr || aligned16(ptr); }

// kernels launched by the library since it was loaded (diagnostics)
void note_launches(int n);

inline prism_status_t launch_status(int launches) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return PRISM_ERR_CUDA;
    note_launches(launches);
    return PRISM_OK;
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// two consecutive elements as float2
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Candidate block shapes: edges in {2,4,8} (log2 exponents in {1,2,3}) whose
// product is 64, 128 or 256; numbered by (volume, b_T, b_H, b_W) ascending.
// Exponent triples are enumerated in lexicographic order inside each volume.
__host__ __device__ inline void shape_exponents(int id, int* eT, int* eH, int* eW) {
    int k = 0;
    for (int S = 6; S <= 8; ++S)
        for (int a = 1; a <= 3; ++a)
            for (int b = 1; b <= 3; ++b) {
                int c = S - a - b;
                if (c < 1 || c > 3) continue;
                if (k == id) { *eT = a; *eH = b; *eW = c; return; }
                ++k;
            }
    *eT = *eH = *eW = 0;
}

}  // namespace prism
