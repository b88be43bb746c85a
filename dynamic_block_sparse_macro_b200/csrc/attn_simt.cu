// Stages 6-7 on CUDA cores: exact block-sparse attention forward and backward
// with fp32 arithmetic (the path for float32 problems, whose 1e-5 accuracy a
// reduced-precision tensor-core product cannot give).
//
// Prism, Portuguese reading guide, "Método" 3: an online-softmax kernel runs
// the attention only over S_i.  Chinese guide, FAQ on error propagation: the
// gradients flow only through the attention over the selected blocks.
//
// Work unit: a 64-row tile of one head.  Blocks are whole 64-row granules,
// so a query tile lies in one query block and every selected 64-key
// granule (a bit of the granule-level selection row) is unmasked.
//   k_fwd_simt     query tile x selected key chunks, online softmax (exp2 form)
//   k_bwd_delta    Delta = rowsum(dO * O)
//   k_bwd_dkdv     key tile x query granules of the blocks that selected it (gselT)
//   k_bwd_dq       query tile x selected key chunks
// Shared tiles are row-major with one float of padding (row stride = 1 mod 32
// banks); thread (ty, tx) owns rows ty + 16u and columns tx + 16v.
#include "common.cuh"

namespace prism {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D> struct Tile { static constexpr int LD = D + 1; };

template <typename T, int D>
__device__ __forceinline__ void load_tile(float* dst, const T* src, int tid) {
    constexpr int LD = D + 1;
    for (int q = tid; q < 64 * D; q += 256) {
        const int r = q / D, c = q % D;
        dst[r * LD + c] = to_f32(src[(int64_t)r * D + c]);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_fwd_simt(const T* __restrict__ Q, const T* __restrict__ K,
                                                  const T* __restrict__ V,
                                                  const uint32_t* __restrict__ gsel, int64_t N,
                                                  int64_t MB, int SW, float scale, T* __restrict__ O,
                                                  float* __restrict__ lse, float* __restrict__ o_f32) {
    constexpr int LD = D + 1, CW = D / 16;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* Ks = Qs + 64 * LD;
    float* Vs = Ks + 64 * LD;
    float* Ps = Vs + 64 * LD;            // [64][65]
    const int g = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int64_t q0 = (int64_t)g * 64;
    const int64_t hoff = (int64_t)hh * N * D;
    load_tile<T, D>(Qs, Q + hoff + q0 * D, tid);

    const float sl2 = scale * kLog2e;
    float m2[4], l[4], acc[4][CW];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        m2[u] = -INFINITY;
        l[u] = 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) acc[u][w] = 0.f;
    }
    const uint32_t* srow = gsel + ((int64_t)hh * MB + g) * SW;
    for (int wi = 0; wi < SW; ++wi) {
        uint32_t bits = srow[wi];
        while (bits) {
            const int j = wi * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            const int ks = 64 * j, ke = ks + 64;        // key granule j
            for (int k0 = ks; k0 < ke; k0 += 64) {
                __syncthreads();
                load_tile<T, D>(Ks, K + hoff + (int64_t)k0 * D, tid);
                load_tile<T, D>(Vs, V + hoff + (int64_t)k0 * D, tid);
                __syncthreads();
                float s[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) s[u][v] = 0.f;
                for (int c = 0; c < D; ++c) {
                    float a[4], b[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) a[u] = Qs[(ty + 16 * u) * LD + c];
#pragma unroll
                    for (int v = 0; v < 4; ++v) b[v] = Ks[(tx + 16 * v) * LD + c];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int v = 0; v < 4; ++v) s[u][v] = fmaf(a[u], b[v], s[u][v]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int v = 0; v < 4; ++v) { s[u][v] *= sl2; mx = fmaxf(mx, s[u][v]); }
#pragma unroll
                    for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    const float mnew = fmaxf(m2[u], mx);
                    const float alpha = exp2f(m2[u] - mnew);
                    float rs = 0.f;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float p = exp2f(s[u][v] - mnew);
                        rs += p;
                        Ps[(ty + 16 * u) * 65 + tx + 16 * v] = p;
                    }
#pragma unroll
                    for (int o = 1; o < 16; o <<= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
                    l[u] = l[u] * alpha + rs;
                    m2[u] = mnew;
#pragma unroll
                    for (int w = 0; w < CW; ++w) acc[u][w] *= alpha;
                }
                __syncthreads();
                for (int k = 0; k < 64; ++k) {
                    float p[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) p[u] = Ps[(ty + 16 * u) * 65 + k];
#pragma unroll
                    for (int w = 0; w < CW; ++w) {
                        const float v = Vs[k * LD + tx + 16 * w];
#pragma unroll
                        for (int u = 0; u < 4; ++u) acc[u][w] = fmaf(p[u], v, acc[u][w]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t r = q0 + ty + 16 * u;
        const float inv = l[u] > 0.f ? 1.f / l[u] : 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) {
            const float o = acc[u][w] * inv;
            O[hoff + r * D + tx + 16 * w] = from_f32<T>(o);
            if (o_f32) o_f32[hoff + r * D + tx + 16 * w] = o;
        }
        if (tx == 0 && lse) lse[(int64_t)hh * N + r] = l[u] > 0.f ? (m2[u] + log2f(l[u])) * kLn2 : -INFINITY;
    }
}

// Delta = rowsum(dO * O), from the unrounded fp32 O when the forward kept it.
// Each lane reads 4 consecutive elements (16-byte fp32 / 8-byte bf16 vectors);
// D/4 lanes cover a row, so a warp covers 128/D rows.
template <typename T> __device__ __forceinline__ float4 load4(const T* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <typename T, int D>
__global__ void k_bwd_delta(const T* __restrict__ O, const float* __restrict__ o_f32,
                            const T* __restrict__ dO, int64_t rows, float* __restrict__ delta,
                            const float* __restrict__ lse, float* __restrict__ nld,
                            const int32_t* __restrict__ perm = nullptr, int64_t N = 0, int heads = 0) {
    constexpr int LPR = D / 4;                                // lanes per row
    const int64_t gl = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t r = gl / LPR;
    const int c = (int)(gl % LPR) * 4;
    float s = 0.f;
    if (r < rows) {
        // with perm, dO is raster [N][heads][D]: blocked row r of head r / N is token perm[r % N]
        const int64_t dr = perm ? (int64_t)perm[r % N] * heads + r / N : r;
        const float4 g = load4<T>(dO + dr * D + c);
        const float4 o = o_f32 ? __ldg(reinterpret_cast<const float4*>(o_f32 + r * D + c)) : load4<T>(O + r * D + c);
        s = o.x * g.x + o.y * g.y + o.z * g.z + o.w * g.w;
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (r < rows && (gl % LPR) == 0) {
        delta[r] = s;
        if (nld) {                       // per 64-row granule: -lse*log2(e) [64], then -Delta [64]
            float* blk = nld + (r >> 6) * 128;
            blk[r & 63] = -lse[r] * kLog2e;
            blk[64 + (r & 63)] = -s;
        }
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_bwd_dkdv_simt(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
    const T* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
    const uint32_t* __restrict__ gselT, int64_t N, int64_t MB,
    int SW, float scale, T* __restrict__ dK, T* __restrict__ dV) {
    constexpr int LD = D + 1, CW = D / 16;
    extern __shared__ float sm[];
    float* Ks = sm;
    float* Vs = Ks + 64 * LD;
    float* Qs = Vs + 64 * LD;
    float* dOs = Qs + 64 * LD;
    float* Pt = dOs + 64 * LD;           // [64 keys][65]
    float* dSt = Pt + 64 * 65;
    float* lse2 = dSt + 64 * 65;         // [64]
    float* dl = lse2 + 64;               // [64]
    const int g = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int64_t k0 = (int64_t)g * 64;
    const int64_t hoff = (int64_t)hh * N * D;
    load_tile<T, D>(Ks, K + hoff + k0 * D, tid);
    load_tile<T, D>(Vs, V + hoff + k0 * D, tid);
    const float sl2 = scale * kLog2e;
    float aK[4][CW], aV[4][CW];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < CW; ++w) aK[u][w] = aV[u][w] = 0.f;

    const uint32_t* trow = gselT + ((int64_t)hh * MB + g) * SW;
    for (int wi = 0; wi < SW; ++wi) {
        uint32_t bits = trow[wi];
        while (bits) {
            const int i = wi * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            const int qs = 64 * i, qe = qs + 64;        // query granule i
            for (int qc = qs; qc < qe; qc += 64) {
                __syncthreads();
                load_tile<T, D>(Qs, Q + hoff + (int64_t)qc * D, tid);
                load_tile<T, D>(dOs, dO + hoff + (int64_t)qc * D, tid);
                if (tid < 64) {
                    lse2[tid] = lse[(int64_t)hh * N + qc + tid] * kLog2e;
                    dl[tid] = delta[(int64_t)hh * N + qc + tid];
                }
                __syncthreads();
                // rows = keys (ty + 16u), cols = queries (tx + 16v)
                float s[4][4], dp[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) s[u][v] = dp[u][v] = 0.f;
                for (int c = 0; c < D; ++c) {
                    float kk[4], vv[4], qq[4], oo[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) { kk[u] = Ks[(ty + 16 * u) * LD + c]; vv[u] = Vs[(ty + 16 * u) * LD + c]; }
#pragma unroll
                    for (int v = 0; v < 4; ++v) { qq[v] = Qs[(tx + 16 * v) * LD + c]; oo[v] = dOs[(tx + 16 * v) * LD + c]; }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            s[u][v] = fmaf(kk[u], qq[v], s[u][v]);
                            dp[u][v] = fmaf(vv[u], oo[v], dp[u][v]);
                        }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int qcol = tx + 16 * v;
                        const float p = exp2f(s[u][v] * sl2 - lse2[qcol]);
                        Pt[(ty + 16 * u) * 65 + qcol] = p;
                        dSt[(ty + 16 * u) * 65 + qcol] = p * (dp[u][v] - dl[qcol]);
                    }
                __syncthreads();
                for (int q = 0; q < 64; ++q) {
                    float p[4], ds[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) { p[u] = Pt[(ty + 16 * u) * 65 + q]; ds[u] = dSt[(ty + 16 * u) * 65 + q]; }
#pragma unroll
                    for (int w = 0; w < CW; ++w) {
                        const float o = dOs[q * LD + tx + 16 * w], x = Qs[q * LD + tx + 16 * w];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            aV[u][w] = fmaf(p[u], o, aV[u][w]);
                            aK[u][w] = fmaf(ds[u], x, aK[u][w]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t r = k0 + ty + 16 * u;
#pragma unroll
        for (int w = 0; w < CW; ++w) {
            dK[hoff + r * D + tx + 16 * w] = from_f32<T>(aK[u][w] * scale);
            dV[hoff + r * D + tx + 16 * w] = from_f32<T>(aV[u][w]);
        }
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_bwd_dq_simt(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
    const T* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
    const uint32_t* __restrict__ gsel, int64_t N, int64_t MB,
    int SW, float scale, T* __restrict__ dQ) {
    constexpr int LD = D + 1, CW = D / 16;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* dOs = Qs + 64 * LD;
    float* Ks = dOs + 64 * LD;
    float* Vs = Ks + 64 * LD;
    float* dSs = Vs + 64 * LD;           // [64 queries][65]
    const int g = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int64_t q0 = (int64_t)g * 64;
    const int64_t hoff = (int64_t)hh * N * D;
    load_tile<T, D>(Qs, Q + hoff + q0 * D, tid);
    load_tile<T, D>(dOs, dO + hoff + q0 * D, tid);
    const float sl2 = scale * kLog2e;
    float lse2[4], dl[4], acc[4][CW];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        lse2[u] = lse[(int64_t)hh * N + q0 + ty + 16 * u] * kLog2e;
        dl[u] = delta[(int64_t)hh * N + q0 + ty + 16 * u];
#pragma unroll
        for (int w = 0; w < CW; ++w) acc[u][w] = 0.f;
    }
    const uint32_t* srow = gsel + ((int64_t)hh * MB + g) * SW;
    for (int wi = 0; wi < SW; ++wi) {
        uint32_t bits = srow[wi];
        while (bits) {
            const int j = wi * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            const int ks = 64 * j, ke = ks + 64;        // key granule j
            for (int kc = ks; kc < ke; kc += 64) {
                __syncthreads();
                load_tile<T, D>(Ks, K + hoff + (int64_t)kc * D, tid);
                load_tile<T, D>(Vs, V + hoff + (int64_t)kc * D, tid);
                __syncthreads();
                float s[4][4], dp[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) s[u][v] = dp[u][v] = 0.f;
                for (int c = 0; c < D; ++c) {
                    float qq[4], oo[4], kk[4], vv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) { qq[u] = Qs[(ty + 16 * u) * LD + c]; oo[u] = dOs[(ty + 16 * u) * LD + c]; }
#pragma unroll
                    for (int v = 0; v < 4; ++v) { kk[v] = Ks[(tx + 16 * v) * LD + c]; vv[v] = Vs[(tx + 16 * v) * LD + c]; }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            s[u][v] = fmaf(qq[u], kk[v], s[u][v]);
                            dp[u][v] = fmaf(oo[u], vv[v], dp[u][v]);
                        }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float p = exp2f(s[u][v] * sl2 - lse2[u]);
                        dSs[(ty + 16 * u) * 65 + tx + 16 * v] = p * (dp[u][v] - dl[u]);
                    }
                __syncthreads();
                for (int k = 0; k < 64; ++k) {
                    float ds[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) ds[u] = dSs[(ty + 16 * u) * 65 + k];
#pragma unroll
                    for (int w = 0; w < CW; ++w) {
                        const float kv = Ks[k * LD + tx + 16 * w];
#pragma unroll
                        for (int u = 0; u < 4; ++u) acc[u][w] = fmaf(ds[u], kv, acc[u][w]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t r = q0 + ty + 16 * u;
#pragma unroll
        for (int w = 0; w < CW; ++w) dQ[hoff + r * D + tx + 16 * w] = from_f32<T>(acc[u][w] * scale);
    }
}

template <int D> constexpr size_t fwd_smem() { return (3 * 64 * (D + 1) + 64 * 65) * sizeof(float); }
template <int D> constexpr size_t dkdv_smem() { return (4 * 64 * (D + 1) + 2 * 64 * 65 + 128) * sizeof(float); }
template <int D> constexpr size_t dq_smem() { return (4 * 64 * (D + 1) + 64 * 65) * sizeof(float); }

template <typename T, int D>
prism_status_t simt_fwd(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const uint32_t* gsel,
                        float scale, void* Op, float* lse, float* o_f32, cudaStream_t s) {
    auto k = k_fwd_simt<T, D>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fwd_smem<D>()) != cudaSuccess)
        return PRISM_ERR_CUDA;
    k<<<dim3((unsigned)d.MB, (unsigned)d.heads), 256, fwd_smem<D>(), s>>>(
        (const T*)Qp, (const T*)Kp, (const T*)Vp, gsel, d.N, d.MB, (int)d.SW, scale, (T*)Op, lse, o_f32);
    return launch_status(1);
}

template <typename T, int D>
prism_status_t simt_bwd(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* Op,
                        const float* o_f32, const void* dOp, const float* lse, const uint32_t* gsel,
                        const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp, float* delta,
                        cudaStream_t s) {
    const int64_t rows = (int64_t)d.heads * d.N;
    k_bwd_delta<T, D><<<(unsigned)((rows * (D / 4) + 255) / 256), 256, 0, s>>>((const T*)Op, o_f32,
                                                                                (const T*)dOp, rows, delta, lse, nullptr);
    auto kk = k_bwd_dkdv_simt<T, D>;
    auto kq = k_bwd_dq_simt<T, D>;
    if (cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dkdv_smem<D>()) != cudaSuccess ||
        cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem<D>()) != cudaSuccess)
        return PRISM_ERR_CUDA;
    dim3 grid((unsigned)d.MB, (unsigned)d.heads);
    kk<<<grid, 256, dkdv_smem<D>(), s>>>((const T*)Qp, (const T*)Kp, (const T*)Vp, (const T*)dOp, lse, delta,
                                         gselT, d.N, d.MB, (int)d.SW, scale, (T*)dKp, (T*)dVp);
    kq<<<grid, 256, dq_smem<D>(), s>>>((const T*)Qp, (const T*)Kp, (const T*)Vp, (const T*)dOp, lse, delta,
                                       gsel, d.N, d.MB, (int)d.SW, scale, (T*)dQp);
    return launch_status(3);
}

prism_status_t attn_fwd_simt(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const uint32_t* gsel,
                             float scale, void* Op, float* lse, float* o_f32, cudaStream_t s) {
#define PRISM_FWD_ARGS d, Qp, Kp, Vp, gsel, scale, Op, lse, o_f32, s
    if (d.dtype == PRISM_F32)
        return d.d == 64 ? simt_fwd<float, 64>(PRISM_FWD_ARGS) : simt_fwd<float, 128>(PRISM_FWD_ARGS);
    return d.d == 64 ? simt_fwd<__nv_bfloat16, 64>(PRISM_FWD_ARGS) : simt_fwd<__nv_bfloat16, 128>(PRISM_FWD_ARGS);
#undef PRISM_FWD_ARGS
}

// Delta = rowsum(dO * O) for every blocked row (shared by both backward families)
// (perm != nullptr: dO raster, read through the permutation; O then comes from o_f32)
prism_status_t bwd_delta(const Dims& d, const void* Op, const float* o_f32, const void* dOp, float* delta,
                         const float* lse, float* nld, cudaStream_t s, const int32_t* perm) {
    const int64_t rows = (int64_t)d.heads * d.N;
    const unsigned grid = (unsigned)((rows * (d.d / 4) + 255) / 256);
    const int64_t N = d.N;
    const int h = d.heads;
    if (d.dtype == PRISM_F32) {
        if (d.d == 64) k_bwd_delta<float, 64><<<grid, 256, 0, s>>>((const float*)Op, o_f32, (const float*)dOp, rows, delta, lse, nld, perm, N, h);
        else k_bwd_delta<float, 128><<<grid, 256, 0, s>>>((const float*)Op, o_f32, (const float*)dOp, rows, delta, lse, nld, perm, N, h);
    } else {
        using B = __nv_bfloat16;
        if (d.d == 64) k_bwd_delta<B, 64><<<grid, 256, 0, s>>>((const B*)Op, o_f32, (const B*)dOp, rows, delta, lse, nld, perm, N, h);
        else k_bwd_delta<B, 128><<<grid, 256, 0, s>>>((const B*)Op, o_f32, (const B*)dOp, rows, delta, lse, nld, perm, N, h);
    }
    return launch_status(1);
}

prism_status_t attn_bwd_simt(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const void* Op,
                             const float* o_f32, const void* dOp, const float* lse, const uint32_t* gsel,
                             const uint32_t* gselT, float scale, void* dQp, void* dKp, void* dVp, float* delta,
                             cudaStream_t s) {
#define PRISM_BWD_ARGS d, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp, delta, s
    if (d.dtype == PRISM_F32)
        return d.d == 64 ? simt_bwd<float, 64>(PRISM_BWD_ARGS) : simt_bwd<float, 128>(PRISM_BWD_ARGS);
    return d.d == 64 ? simt_bwd<__nv_bfloat16, 64>(PRISM_BWD_ARGS) : simt_bwd<__nv_bfloat16, 128>(PRISM_BWD_ARGS);
#undef PRISM_BWD_ARGS
}

}  // namespace prism
