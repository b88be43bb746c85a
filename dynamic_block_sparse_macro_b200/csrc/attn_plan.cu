// Work planning for the tensor-core attention kernels.
//
// A tile's work is the union of the granule-level selection rows of its
// 64-row granules (two: forward and backward both use 128-row tiles).  That
// union is data dependent and very uneven (a query block with flat block
// probabilities makes Top-p select most keys), so one CTA per tile would
// leave a few CTAs running long after the rest.  The
// plan cuts every tile into segments of at most `seg` work units, choosing
// seg from the total so that the item count stays near a fixed target, and
// gives each segment of a split tile a slot for its partial result; a
// combine kernel merges the slots afterwards.  Units are 128-key chunks
// (forward) or 64-row granules (backward).
//
//   k_plan_count   one warp per tile: popcount of the union -> units
//   k_plan_items   one CTA: seg, exclusive scans, item list, slot table
//   k_fwd_combine  merges (O, m, l) partials of split forward tiles
//   k_bwd_combine  sums dQ (or dK, dV) partials of split backward tiles
#include "common.cuh"
#include "attn_plan.cuh"

namespace prism {

__global__ void __launch_bounds__(256) k_plan_count(const uint32_t* __restrict__ rows, int64_t MB, int SW,
                                                    int tiles_per_head, int heads, int tile_gran, int unit_granules,
                                                    int32_t* __restrict__ tile_units, PlanHeader* hdr) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= (int64_t)tiles_per_head * heads) return;
    const int hh = (int)(t / tiles_per_head), tile = (int)(t % tiles_per_head);
    const uint32_t* r0 = rows + ((int64_t)hh * MB + (int64_t)tile_gran * tile) * SW;
    int cnt = 0;
    for (int w = lane; w < SW; w += 32) {
        uint32_t u = 0u;
        for (int i = 0; i < tile_gran; ++i) u |= r0[(int64_t)i * SW + w];
        cnt += __popc(u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) {
        const int units = (cnt + unit_granules - 1) / unit_granules;
        tile_units[t] = units;
        atomicAdd(&hdr->total_units, (unsigned long long)units);
    }
}

__global__ void __launch_bounds__(1024) k_plan_items(const int32_t* __restrict__ tile_units, int tiles,
                                                     int target, int seg_min, int2* __restrict__ tile_split,
                                                     int4* __restrict__ items, PlanHeader* hdr) {
    __shared__ int wsum_i[32], wsum_s[32];
    __shared__ int carry_i, carry_s;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    const unsigned long long total = hdr->total_units;
    int seg = (int)((total + (unsigned long long)target - 1) / (unsigned long long)target);
    if (seg < seg_min) seg = seg_min;
    if (tid == 0) { carry_i = 0; carry_s = 0; }
    __syncthreads();
    for (int base = 0; base < tiles; base += blockDim.x) {
        const int t = base + tid;
        const int u = t < tiles ? tile_units[t] : 0;
        const int nseg = t < tiles ? (u > seg ? (u + seg - 1) / seg : 1) : 0;
        const int nslot = nseg > 1 ? nseg : 0;
        int ii = nseg, is = nslot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, ii, o), b = __shfl_up_sync(0xffffffffu, is, o);
            if (lane >= o) { ii += a; is += b; }
        }
        if (lane == 31) { wsum_i[wid] = ii; wsum_s[wid] = is; }
        __syncthreads();
        if (wid == 0) {
            int a = lane < nw ? wsum_i[lane] : 0, b = lane < nw ? wsum_s[lane] : 0;
            const int a0 = a, b0 = b;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
                if (lane >= o) { a += x; b += y; }
            }
            wsum_i[lane] = a - a0;
            wsum_s[lane] = b - b0;
        }
        __syncthreads();
        const int ioff = carry_i + wsum_i[wid] + ii - nseg;
        const int soff = carry_s + wsum_s[wid] + is - nslot;
        if (t < tiles) {
            tile_split[t] = make_int2(nslot ? soff : -1, nseg);
            for (int k = 0; k < nseg; ++k) {
                const int u0 = k * seg, u1 = (k + 1) * seg < u ? (k + 1) * seg : u;
                items[ioff + k] = make_int4(t, u0, nseg == 1 ? u : u1, nslot ? soff + k : -1);
            }
        }
        __syncthreads();
        if (tid == blockDim.x - 1) { carry_i = ioff + nseg; carry_s = soff + nslot; }
        __syncthreads();
    }
    if (tid == 0) {
        hdr->seg = seg;
        hdr->n_items = carry_i;
        hdr->n_slots = carry_s;
    }
}

// ------------------------------------------------------------------ combine
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, lse = (M + log2 L) ln 2
__global__ void __launch_bounds__(128) k_fwd_combine(const int2* __restrict__ tile_split, int tiles_per_head,
                                                     int tile_rows, int64_t N, int D, const float* __restrict__ opart,
                                                     const float* __restrict__ mpart,
                                                     const float* __restrict__ lpart,
                                                     __nv_bfloat16* __restrict__ O, float* __restrict__ o_f32,
                                                     float* __restrict__ lse, const int32_t* __restrict__ perm,
                                                     int heads) {
    const int t = blockIdx.x;
    const int2 sp = tile_split[t];
    if (sp.y <= 1) return;
    const int hh = t / tiles_per_head, tile = t % tiles_per_head;
    const int64_t grow0 = (int64_t)hh * N + (int64_t)tile_rows * tile;
    for (int r = 0; r < tile_rows; ++r) {
        float M = -INFINITY;
        for (int s = 0; s < sp.y; ++s) M = fmaxf(M, mpart[(int64_t)(sp.x + s) * tile_rows + r]);
        float L = 0.f, acc = 0.f;
        for (int s = 0; s < sp.y; ++s) {
            const int64_t slot = sp.x + s;
            const float m = mpart[slot * tile_rows + r];
            const float w = m > -INFINITY ? exp2f(m - M) : 0.f;
            L += w * lpart[slot * tile_rows + r];
            if (threadIdx.x < D) acc += w * opart[(slot * tile_rows + r) * D + threadIdx.x];
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        if (threadIdx.x < D) {
            const float o = acc * inv;
            // with perm, O is raster [N][heads][D] and the row goes to its token's place
            const int64_t orow = perm ? (int64_t)perm[(int64_t)tile_rows * tile + r] * heads + hh : grow0 + r;
            O[orow * D + threadIdx.x] = __float2bfloat16_rn(o);
            if (o_f32) o_f32[(grow0 + r) * D + threadIdx.x] = o;
        }
        if (threadIdx.x == 0 && lse) lse[grow0 + r] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
}

// out_k = mul_k * sum_s part_k[s] for k < nout (dQ; or dK, dV)
__global__ void __launch_bounds__(256) k_bwd_combine(const int2* __restrict__ tile_split, int tiles_per_head,
                                                     int64_t N, int D, int nout, const float* __restrict__ part,
                                                     __nv_bfloat16* __restrict__ out0, float mul0,
                                                     __nv_bfloat16* __restrict__ out1, float mul1,
                                                     const int32_t* __restrict__ perm, int heads) {
    const int t = blockIdx.x;
    const int2 sp = tile_split[t];
    if (sp.y <= 1) return;
    const int hh = t / tiles_per_head, tile = t % tiles_per_head;
    const int64_t grow0 = (int64_t)hh * N + 128 * (int64_t)tile;
    const int per = 128 * D;                                  // elements of one output tile
    for (int k = 0; k < nout; ++k) {
        __nv_bfloat16* out = k ? out1 : out0;
        const float mul = k ? mul1 : mul0;
        for (int e = threadIdx.x; e < per; e += blockDim.x) {
            float acc = 0.f;
            for (int s = 0; s < sp.y; ++s) acc += part[((int64_t)(sp.x + s) * nout + k) * per + e];
            // with perm, the outputs are raster [N][heads][D]: row r goes to its token's place
            const int64_t orow = perm ? (int64_t)perm[128 * (int64_t)tile + e / D] * heads + hh : grow0 + e / D;
            out[orow * D + e % D] = __float2bfloat16_rn(acc * mul);
        }
    }
}

size_t plan_bytes(int64_t tiles, int target) {
    return sizeof(PlanHeader) + align16(tiles * 4) + align16(tiles * 8) + align16((tiles + target) * 16);
}

Plan carve_plan(void* base, int64_t tiles, int target) {
    uint8_t* p = static_cast<uint8_t*>(base);
    Plan pl;
    pl.hdr = reinterpret_cast<PlanHeader*>(p);
    p += sizeof(PlanHeader);
    pl.tile_units = reinterpret_cast<int32_t*>(p);
    p += align16(tiles * 4);
    pl.tile_split = reinterpret_cast<int2*>(p);
    p += align16(tiles * 8);
    pl.items = reinterpret_cast<int4*>(p);
    pl.tiles = tiles;
    pl.items_max = tiles + target;
    return pl;
}

prism_status_t plan_work(const Plan& pl, const uint32_t* rows, const Dims& d, int tile_gran, int unit_granules,
                         int target, int seg_min, cudaStream_t s) {
    if (cudaMemsetAsync(pl.hdr, 0, sizeof(PlanHeader), s) != cudaSuccess) return PRISM_ERR_CUDA;
    const int tph = (int)(d.N / (64 * tile_gran));
    const unsigned grid = (unsigned)((pl.tiles * 32 + 255) / 256);
    k_plan_count<<<grid, 256, 0, s>>>(rows, d.MB, (int)d.SW, tph, d.heads, tile_gran, unit_granules, pl.tile_units,
                                      pl.hdr);
    k_plan_items<<<1, 1024, 0, s>>>(pl.tile_units, (int)pl.tiles, target, seg_min, pl.tile_split, pl.items,
                                    pl.hdr);
    return launch_status(2);
}

__global__ void __launch_bounds__(256) k_gran_pos(const int32_t* __restrict__ perm,
                                                  const uint8_t* __restrict__ shape_id, int64_t MB, int H, int W,
                                                  int4* __restrict__ gpos) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= MB) return;
    const int r0 = perm[64 * g];
    const int t0 = r0 / (H * W), h0 = (r0 / W) % H, w0 = r0 % W;
    const int zone = ((t0 >> 3) * (H >> 3) + (h0 >> 3)) * (W >> 3) + (w0 >> 3);
    int eT, eH, eW;
    shape_exponents(shape_id[zone], &eT, &eH, &eW);
    gpos[g] = make_int4(t0, h0, w0, 3 * (eH - 1) + (eW - 1));
}

prism_status_t gran_positions(const int32_t* perm, const uint8_t* shape_id, const Dims& d, int4* gpos,
                              cudaStream_t s) {
    k_gran_pos<<<(unsigned)((d.MB + 255) / 256), 256, 0, s>>>(perm, shape_id, d.MB, d.H, d.W, gpos);
    return launch_status(1);
}

prism_status_t fwd_combine(const Plan& pl, const Dims& d, int tile_rows, const float* opart, const float* mpart,
                           const float* lpart, void* Op, float* o_f32, float* lse, const int32_t* perm, cudaStream_t s) {
    k_fwd_combine<<<(unsigned)pl.tiles, 128, 0, s>>>(pl.tile_split, (int)(d.N / tile_rows), tile_rows, d.N, d.d,
                                                     opart, mpart, lpart, (__nv_bfloat16*)Op, o_f32, lse, perm,
                                                     d.heads);
    return launch_status(1);
}

prism_status_t bwd_combine(const Plan& pl, const Dims& d, int nout, const float* part, void* out0, float mul0,
                           void* out1, float mul1, cudaStream_t s, const int32_t* perm) {
    k_bwd_combine<<<(unsigned)pl.tiles, 256, 0, s>>>(pl.tile_split, (int)(d.N / 128), d.N, d.d, nout, part,
                                                     (__nv_bfloat16*)out0, mul0, (__nv_bfloat16*)out1, mul1, perm,
                                                     d.heads);
    return launch_status(1);
}

}  // namespace prism
