// Stage 1: macro-zone statistics and the dual-guidance variation indicator.
//
// Prism, Portuguese reading guide, "Método" 1 (Formulação do Indicador de
// Variação): for each 8x8x8 macro-zone m and axis d in {T,H,W},
//   sigma^2_{v,d}(m) = (1/D) sum_c (1/8) sum_i (Vbar^{(d)}_{m,i,c} - mu_{m,c})^2,
//   r_{v,d} = sigma^2_{v,d} / sum_d' sigma^2_{v,d'},
//   a = ||hhat||_2 per token, abar(m) in [0,1], vhat_{a,d}(m),
//   g_d = r_{v,d} + abar * vhat_{a,d} + eps.
// Readings of the unstated parts: D spans every head's channels; abar =
// A / max A with A the zone mean of a; vhat_{a,d} is the r construction on
// the scalar field a; rho = max(rho_v, abar) with rho_v the zone's mean
// token variance of V over its grid maximum; zero total variance gives 1/3.
//
// Kernels (all reductions in a fixed order, no float atomics, so the result
// is deterministic):
//   k_zone_video    persistent, one CTA per SM over the (zone, 128-byte channel
//                   chunk) items, chunks fastest; each item's 8x8x8 x 128-byte
//                   slice lands in shared memory as one 64 KB TMA copy, two
//                   stages deep; warp w holds temporal slice t = w of the
//                   zone, each lane CPL channels, 64 tokens kept in registers
//                   for the two-pass (mean first, then squared deviations)
//                   variance.
//   k_zone_audio    grid Z: one thread per token of the zone.
//   k_zone_finalize one CTA: per-zone sums over chunks, grid maxima, outputs.
#include <mutex>

#include "attn_plan.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace prism {

using namespace sm100;

template <typename T> struct VidTraits;
template <> struct VidTraits<__nv_bfloat16> { static constexpr int CPL = 2; };  // 4 B per lane
template <> struct VidTraits<float> { static constexpr int CPL = 1; };          // 4 B per lane

constexpr int kZoneStage = 512 * 128;                       // one zone x 128 bytes of channels
constexpr int kZoneScratch = 2 * 8 * 8 * 64 * 4 + 8 * 64 * 4 + 8 * 4 * 4;   // sH, sW, sT, red (bf16 sizes)
constexpr int kZoneSmem = 2 * kZoneStage + kZoneScratch + 64 + 1024;       // + barriers, + alignment

// bounded wait on a copy this thread issued, for the wind-down after a timeout
__device__ __forceinline__ void zone_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kWaitLimitNs) {
    }
}

// ws layout: video partial sums [Z][nchunk][4] then audio stats [Z][4].
// Persistent: CTA b takes items b, b + gridDim.x, ... (item = zone * nchunk +
// chunk, chunks fastest, so the CTAs in flight together read whole token rows
// of a few zones); each item's zone slice comes in as one 64 KB TMA copy, two
// stages deep, the next-but-one copy issued as soon as a stage has been read.
// If a copy never lands (2 s), the CTA marks its remaining items' sums NaN,
// lets its copies in flight land (bounded) and exits.
template <typename T>
__global__ void __launch_bounds__(256, 1) k_zone_video(const __grid_constant__ CUtensorMap tmV, int H, int W,
                                                       int nchunk, int n_items, float* __restrict__ part) {
    constexpr int CPL = VidTraits<T>::CPL;
    constexpr int CH = 32 * CPL;                    // channels per item (128 bytes)
    extern __shared__ uint8_t zraw[];
    uint8_t* zs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(zraw) + 1023) & ~uintptr_t(1023));
    float(*sH)[8][CH] = reinterpret_cast<float(*)[8][CH]>(zs + 2 * kZoneStage);              // [t][h][c]
    float(*sW)[8][CH] = reinterpret_cast<float(*)[8][CH]>(zs + 2 * kZoneStage + 256 * CH);    // [t][w][c]
    float(*sT)[CH] = reinterpret_cast<float(*)[CH]>(zs + 2 * kZoneStage + 512 * CH);          // [t][c]
    float(*red)[4] = reinterpret_cast<float(*)[4]>(zs + 2 * kZoneStage + 544 * CH);
    uint64_t* full = reinterpret_cast<uint64_t*>(zs + 2 * kZoneStage + kZoneScratch);
    int* abort_flag = reinterpret_cast<int*>(full + 2);
    uint32_t* wstat = reinterpret_cast<uint32_t*>(abort_flag + 1);

    const int lane = threadIdx.x & 31, t = threadIdx.x >> 5;
    const int ZH = H / 8, ZW = W / 8;
    auto issue = [&](int it, int buf) {
        const int chunk = it % nchunk, m = it / nchunk;
        const int zt = m / (ZH * ZW), zh = (m / ZW) % ZH, zw = m % ZW;
        mbar_expect_tx(full + buf, kZoneStage);
        tma_load_4d(zs + buf * kZoneStage, &tmV, full + buf, chunk * CH, zw * 8, zh * 8, zt * 8);
    };
    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init(full + 1, 1);
        *abort_flag = 0;
        *wstat = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        for (int b = 0; b < 2; ++b)
            if (blockIdx.x + b * gridDim.x < n_items) issue(blockIdx.x + b * gridDim.x, b);

    for (int it = blockIdx.x, k = 0; it < n_items; it += gridDim.x, ++k) {
        const int buf = k & 1;
        const bool got = mbar_wait(full + buf, (uint32_t)(k >> 1) & 1u, abort_flag, wstat);
        // one 32-bit word per token (a bf16 pair or one float) of this warp's slice t
        // keeps the slice at 64 registers for the second (deviation) pass
        const uint32_t* src = reinterpret_cast<const uint32_t*>(zs + buf * kZoneStage) + t * 2048 + lane;
        uint32_t raw[8][8];
#pragma unroll
        for (int h = 0; h < 8; ++h)
#pragma unroll
            for (int w = 0; w < 8; ++w) raw[h][w] = src[(h * 8 + w) * 32];
        // the stage has been read by every thread, and sH, sW, sT, red are free
        if (__syncthreads_or(!got)) {
            if (threadIdx.x == 0) {
                zone_drain(full + buf, (uint32_t)(k >> 1) & 1u);
                if (it + gridDim.x < n_items) zone_drain(full + (buf ^ 1), (uint32_t)((k + 1) >> 1) & 1u);
            }
            for (int r = it; r < n_items; r += gridDim.x)
                if (threadIdx.x < 4) part[(int64_t)r * 4 + threadIdx.x] = __int_as_float(0x7fc00000);
            return;
        }
        if (threadIdx.x == 0 && it + 2 * gridDim.x < n_items) issue(it + 2 * gridDim.x, buf);
        auto val = [&](int h, int w, int c) -> float {
            if constexpr (CPL == 2) return __uint_as_float(c == 0 ? (raw[h][w] << 16) : (raw[h][w] & 0xffff0000u));
            else return __uint_as_float(raw[h][w]);
        };
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            float tot = 0.f;
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                float rs = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) rs += val(h, w, c);
                sH[t][h][lane * CPL + c] = rs;
                tot += rs;
            }
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                float cs = 0.f;
#pragma unroll
                for (int h = 0; h < 8; ++h) cs += val(h, w, c);
                sW[t][w][lane * CPL + c] = cs;
            }
            sT[t][lane * CPL + c] = tot;
        }
        __syncthreads();

        // this thread handles profile index i = t along every axis
        float aT = 0.f, aH = 0.f, aW = 0.f, aTok = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int ch = lane * CPL + c;
            float zsum = 0.f, hsum = 0.f, wsum = 0.f;
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) {
                zsum += sT[tt][ch];
                hsum += sH[tt][t][ch];
                wsum += sW[tt][t][ch];
            }
            const float mu = zsum * (1.f / 512.f);
            const float pT = sT[t][ch] * (1.f / 64.f) - mu;
            const float pH = hsum * (1.f / 64.f) - mu;
            const float pW = wsum * (1.f / 64.f) - mu;
            aT += pT * pT;
            aH += pH * pH;
            aW += pW * pW;
            float tv = 0.f;
#pragma unroll
            for (int h = 0; h < 8; ++h)
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    const float dv = val(h, w, c) - mu;
                    tv += dv * dv;
                }
            aTok += tv;
        }
        aT = warp_sum(aT); aH = warp_sum(aH); aW = warp_sum(aW); aTok = warp_sum(aTok);
        if (lane == 0) { red[t][0] = aT; red[t][1] = aH; red[t][2] = aW; red[t][3] = aTok; }
        __syncthreads();
        if (threadIdx.x < 4) {
            float sum = 0.f;
            for (int q = 0; q < 8; ++q) sum += red[q][threadIdx.x];
            part[(int64_t)it * 4 + threadIdx.x] = sum;
        }
    }
}

// Launch of k_zone_video over V ([T][H][W][D] raster, bf16 or fp32)
static prism_status_t launch_zone_video(const Dims& d, const void* V, int nchunk, float* part, cudaStream_t s) {
    CUtensorMap tm;
    if (!make_map_zone(&tm, V, d.dtype == PRISM_BF16, d.T, d.H, d.W, d.D)) return PRISM_ERR_CUDA;
    const int n_items = (int)(d.Z * nchunk);
    const int grid = n_items < device_sms() ? n_items : device_sms();
    if (d.dtype == PRISM_BF16) {
        if (cudaFuncSetAttribute(k_zone_video<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kZoneSmem) != cudaSuccess)
            return PRISM_ERR_CUDA;
        k_zone_video<__nv_bfloat16><<<grid, 256, kZoneSmem, s>>>(tm, d.H, d.W, nchunk, n_items, part);
    } else {
        if (cudaFuncSetAttribute(k_zone_video<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, kZoneSmem) !=
            cudaSuccess)
            return PRISM_ERR_CUDA;
        k_zone_video<float><<<grid, 256, kZoneSmem, s>>>(tm, d.H, d.W, nchunk, n_items, part);
    }
    return PRISM_OK;
}

template <typename T>
__global__ void __launch_bounds__(512) k_zone_audio(const T* __restrict__ hh, int H, int W, int Da,
                                                    float* __restrict__ astat) {
    __shared__ float a[512];
    __shared__ float prof[3][8];
    const int m = blockIdx.x, tid = threadIdx.x;
    const int ZH = H / 8, ZW = W / 8;
    const int zt = m / (ZH * ZW), zh = (m / ZW) % ZH, zw = m % ZW;
    const int t = tid >> 6, h = (tid >> 3) & 7, w = tid & 7;
    const int64_t r = ((int64_t)(zt * 8 + t) * H + zh * 8 + h) * W + zw * 8 + w;
    const T* p = hh + r * Da;
    float s = 0.f;
    for (int c = 0; c < Da; c += 2) {
        float2 v = load2(p + c);
        s += v.x * v.x + v.y * v.y;
    }
    a[tid] = sqrtf(s);
    __syncthreads();
    if (tid < 24) {
        const int ax = tid >> 3, i = tid & 7;
        float acc = 0.f;
        for (int u = 0; u < 8; ++u)
            for (int v = 0; v < 8; ++v) {
                int tt, hy, wx;
                if (ax == 0) { tt = i; hy = u; wx = v; }
                else if (ax == 1) { tt = u; hy = i; wx = v; }
                else { tt = u; hy = v; wx = i; }
                acc += a[tt * 64 + hy * 8 + wx];
            }
        prof[ax][i] = acc;
    }
    __syncthreads();
    if (tid == 0) {
        float tot = 0.f;
        for (int i = 0; i < 8; ++i) tot += prof[0][i];
        const float A = tot * (1.f / 512.f);
        astat[m * 4 + 0] = A;
        for (int ax = 0; ax < 3; ++ax) {
            float v = 0.f;
            for (int i = 0; i < 8; ++i) {
                float dv = prof[ax][i] * (1.f / 64.f) - A;
                v += dv * dv;
            }
            astat[m * 4 + 1 + ax] = v * (1.f / 8.f);
        }
    }
}

__global__ void __launch_bounds__(1024) k_zone_finalize(const float* __restrict__ part,
                                                        const float* __restrict__ astat, int Z,
                                                        int nchunk, float invD, float eps,
                                                        float* __restrict__ g, float* __restrict__ rho,
                                                        float* __restrict__ abar,
                                                        float* __restrict__ zstat,
                                                        float* __restrict__ vsum, int guide) {
    // guidance ablation: the video term, the audio term or both (g and rho)
    const float wv = guide == PRISM_GUIDE_AUDIO ? 0.f : 1.f, wa = guide == PRISM_GUIDE_VIDEO ? 0.f : 1.f;
    __shared__ float rmx[32], amx[32];
    const int tid = threadIdx.x;
    float rmax = 0.f, Amax = 0.f;
    for (int m = tid; m < Z; m += blockDim.x) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        const float* pp = part + (int64_t)m * nchunk * 4;
        for (int k = 0; k < nchunk; ++k)
#pragma unroll
            for (int q = 0; q < 4; ++q) s[q] += pp[k * 4 + q];
        // sigma^2_{v,d} = S_d / (8 D), rho_raw = S_tok / (512 D)
        vsum[m * 4 + 0] = s[0] * (1.f / 8.f) * invD;
        vsum[m * 4 + 1] = s[1] * (1.f / 8.f) * invD;
        vsum[m * 4 + 2] = s[2] * (1.f / 8.f) * invD;
        const float rr = s[3] * (1.f / 512.f) * invD;
        vsum[m * 4 + 3] = rr;
        rmax = fmaxf(rmax, rr);
        Amax = fmaxf(Amax, astat[m * 4]);
    }
    rmax = warp_max(rmax);
    Amax = warp_max(Amax);
    if ((tid & 31) == 0) { rmx[tid >> 5] = rmax; amx[tid >> 5] = Amax; }
    __syncthreads();
    if (tid < 32) {
        float a = tid < (int)(blockDim.x >> 5) ? rmx[tid] : 0.f;
        float b = tid < (int)(blockDim.x >> 5) ? amx[tid] : 0.f;
        a = warp_max(a);
        b = warp_max(b);
        if (tid == 0) { rmx[0] = a; amx[0] = b; }
    }
    __syncthreads();
    rmax = rmx[0];
    Amax = amx[0];
    for (int m = tid; m < Z; m += blockDim.x) {
        const float sv0 = vsum[m * 4 + 0], sv1 = vsum[m * 4 + 1], sv2 = vsum[m * 4 + 2];
        const float rr = vsum[m * 4 + 3];
        const float A = astat[m * 4], sa0 = astat[m * 4 + 1], sa1 = astat[m * 4 + 2],
                    sa2 = astat[m * 4 + 3];
        const float tv = sv0 + sv1 + sv2, ta = sa0 + sa1 + sa2;
        const float third = 1.f / 3.f;
        const float r0 = tv > 0.f ? sv0 / tv : third, r1 = tv > 0.f ? sv1 / tv : third,
                    r2 = tv > 0.f ? sv2 / tv : third;
        const float v0 = ta > 0.f ? sa0 / ta : third, v1 = ta > 0.f ? sa1 / ta : third,
                    v2 = ta > 0.f ? sa2 / ta : third;
        const float ab = Amax > 0.f ? A / Amax : 0.f;
        g[m * 3 + 0] = wv * r0 + wa * ab * v0 + eps;
        g[m * 3 + 1] = wv * r1 + wa * ab * v1 + eps;
        g[m * 3 + 2] = wv * r2 + wa * ab * v2 + eps;
        const float rv = rmax > 0.f ? rr / rmax : 0.f;
        rho[m] = fmaxf(wv * rv, wa * ab);
        abar[m] = ab;
        if (zstat) {
            float* o = zstat + (int64_t)m * 8;
            o[0] = sv0; o[1] = sv1; o[2] = sv2; o[3] = rr;
            o[4] = A; o[5] = sa0; o[6] = sa1; o[7] = sa2;
        }
    }
}

size_t zone_indicator_ws_bytes(const Dims& d) {
    const int CH = d.dtype == PRISM_BF16 ? 64 : 32;
    const int64_t nchunk = d.D / CH;
    return (size_t)d.Z * (nchunk * 4 + 4 + 4) * sizeof(float);
}

}  // namespace prism

using namespace prism;

extern "C" prism_status_t prism_zone_indicator_ex(const prism_problem_t* prob, const void* V,
                                                  const void* hhat, float eps, int32_t guidance, float* g,
                                                  float* rho, float* abar, float* zone_stats, void* ws,
                                                  size_t ws_bytes, cudaStream_t stream) {
    if (guidance != PRISM_GUIDE_JOINT && guidance != PRISM_GUIDE_VIDEO && guidance != PRISM_GUIDE_AUDIO)
        return PRISM_ERR_INVALID_ARG;
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(V) || !ok_ptr(hhat) || !ok_ptr(g) || !ok_ptr(rho) || !ok_ptr(abar) ||
        !ok_opt(zone_stats) || !ok_ptr(ws))
        return PRISM_ERR_INVALID_ARG;
    if (!(eps > 0.f) || !isfinite(eps)) return PRISM_ERR_INVALID_ARG;
    if (d.Da & 1) return PRISM_ERR_UNSUPPORTED;
    if (ws_bytes < zone_indicator_ws_bytes(d)) return PRISM_ERR_WORKSPACE;
    const int CH = d.dtype == PRISM_BF16 ? 64 : 32;
    const int nchunk = (int)(d.D / CH);
    float* part = (float*)ws;
    float* astat = part + d.Z * nchunk * 4;
    float* vsum = astat + d.Z * 4;
    st = launch_zone_video(d, V, nchunk, part, stream);
    if (st != PRISM_OK) return st;
    if (d.dtype == PRISM_BF16)
        k_zone_audio<__nv_bfloat16><<<(unsigned)d.Z, 512, 0, stream>>>((const __nv_bfloat16*)hhat,
                                                                       d.H, d.W, d.Da, astat);
    else
        k_zone_audio<float><<<(unsigned)d.Z, 512, 0, stream>>>((const float*)hhat, d.H, d.W, d.Da,
                                                               astat);
    k_zone_finalize<<<1, 1024, 0, stream>>>(part, astat, (int)d.Z, nchunk, 1.f / (float)d.D, eps, g,
                                            rho, abar, zone_stats, vsum, guidance);
    return launch_status(3);
}

extern "C" prism_status_t prism_zone_indicator(const prism_problem_t* prob, const void* V,
                                               const void* hhat, float eps, float* g, float* rho,
                                               float* abar, float* zone_stats, void* ws,
                                               size_t ws_bytes, cudaStream_t stream) {
    return prism_zone_indicator_ex(prob, V, hhat, eps, PRISM_GUIDE_JOINT, g, rho, abar, zone_stats, ws,
                                   ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// Head-sharded indicator: a rank holding some of the heads computes the
// per-zone sums over its own channels (prism_zone_partials); one all-reduce
// (sum) of the [Z][4] video sums over the ranks makes them the sums over all
// D channels; prism_zone_finalize then forms g, rho and abar exactly as
// prism_zone_indicator does.  The audio statistics come from hhat, which every
// rank holds whole, so they need no reduction.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_zone_chunk_sum(const float* __restrict__ part, int Z, int nchunk,
                                                        float* __restrict__ out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;      // (zone, statistic)
    if (i >= Z * 4) return;
    const int m = i >> 2, q = i & 3;
    float s = 0.f;
    for (int k = 0; k < nchunk; ++k) s += part[((int64_t)m * nchunk + k) * 4 + q];
    out[i] = s;
}

extern "C" prism_status_t prism_zone_partials(const prism_problem_t* prob_local, const void* V_local,
                                              const void* hhat, float* partials, void* ws, size_t ws_bytes,
                                              cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob_local, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(V_local) || !ok_ptr(hhat) || !ok_ptr(partials) || !ok_ptr(ws)) return PRISM_ERR_INVALID_ARG;
    if (d.Da & 1) return PRISM_ERR_UNSUPPORTED;
    if (ws_bytes < zone_indicator_ws_bytes(d)) return PRISM_ERR_WORKSPACE;
    const int CH = d.dtype == PRISM_BF16 ? 64 : 32;
    const int nchunk = (int)(d.D / CH);
    float* part = (float*)ws;
    st = launch_zone_video(d, V_local, nchunk, part, stream);
    if (st != PRISM_OK) return st;
    if (d.dtype == PRISM_BF16)
        k_zone_audio<__nv_bfloat16><<<(unsigned)d.Z, 512, 0, stream>>>((const __nv_bfloat16*)hhat, d.H, d.W,
                                                                       d.Da, partials + d.Z * 4);
    else
        k_zone_audio<float><<<(unsigned)d.Z, 512, 0, stream>>>((const float*)hhat, d.H, d.W, d.Da,
                                                               partials + d.Z * 4);
    k_zone_chunk_sum<<<(unsigned)((d.Z * 4 + 255) / 256), 256, 0, stream>>>(part, (int)d.Z, nchunk, partials);
    return launch_status(3);
}

extern "C" prism_status_t prism_zone_finalize(const prism_problem_t* prob, const float* partials, float eps,
                                              int32_t guidance, float* g, float* rho, float* abar,
                                              float* zone_stats, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (guidance != PRISM_GUIDE_JOINT && guidance != PRISM_GUIDE_VIDEO && guidance != PRISM_GUIDE_AUDIO)
        return PRISM_ERR_INVALID_ARG;
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (!ok_ptr(partials) || !ok_ptr(g) || !ok_ptr(rho) || !ok_ptr(abar) || !ok_opt(zone_stats) || !ok_ptr(ws))
        return PRISM_ERR_INVALID_ARG;
    if (!(eps > 0.f) || !isfinite(eps)) return PRISM_ERR_INVALID_ARG;
    if (ws_bytes < (size_t)d.Z * 4 * sizeof(float)) return PRISM_ERR_WORKSPACE;
    k_zone_finalize<<<1, 1024, 0, stream>>>(partials, partials + d.Z * 4, (int)d.Z, 1, 1.f / (float)d.D, eps, g,
                                            rho, abar, zone_stats, (float*)ws, guidance);
    return launch_status(1);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of prism_zone_indicator.
//
// Some callers cannot hand us a workspace: a host that has no device
// allocator wired in (a plain C program driving the library through this
// ABI), or a service whose memory footprint is fixed at start-up and which
// forbids device allocations afterwards.  For them the indicator's scratch
// (per zone x channel-chunk partial sums, per-zone audio statistics and
// per-zone totals) lives in a fixed array inside this library instead.
//
// The array is a file-scope __device__ symbol, so every GPU that loads the
// library holds PRISM_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Host code cannot use the symbol's name as a device address; the address is
// looked up with cudaGetSymbolAddress once per device, the first time the
// entry point runs with that device current (so that first call should come
// before any stream capture), and kept for the life of the process: a
// cudaDeviceReset (or any teardown of the primary context) invalidates it.  Every call shares the one array: two calls
// whose kernels overlap on the GPU race on it.  Each call writes every
// scratch word it later reads, so nothing has to be cleared between calls.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[PRISM_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

prism_status_t noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PRISM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return PRISM_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PRISM_OK;
}
}  // namespace

extern "C" prism_status_t prism_zone_indicator_noalloc(const prism_problem_t* prob, const void* V,
                                                       const void* hhat, float eps, float* g, float* rho,
                                                       float* abar, float* zone_stats,
                                                       cudaStream_t stream) {
    Dims d;
    prism_status_t st = make_dims(prob, &d);
    if (st != PRISM_OK) return st;
    if (zone_indicator_ws_bytes(d) > (size_t)PRISM_NOALLOC_SCRATCH_BYTES) return PRISM_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != PRISM_OK) return st;
    return prism_zone_indicator(prob, V, hhat, eps, g, rho, abar, zone_stats, scratch,
                                (size_t)PRISM_NOALLOC_SCRATCH_BYTES, stream);
}
