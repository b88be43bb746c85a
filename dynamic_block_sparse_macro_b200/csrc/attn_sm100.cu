// Stage 6 on sm_100a tensor cores: block-sparse attention forward for bf16.
//
// Prism, Portuguese reading guide, "Método" 3: an online-softmax kernel runs
// the attention only over the selected set S_i of each query block.
//
// Tiles: 128 query rows (two 64-row granules, which lie in one block or in two
// 64-blocks).  A tile's keys are the union of the granule-level selection rows
// of its two granules, walked in ascending order; two key granules form one
// 128-key chunk, and a per-granule 2-bit mask says which half of the tile
// selected it (an odd tail repeats its last granule with mask 0).  The work
// plan (attn_plan.cu) cuts heavy tiles into segments of chunks; one CTA runs
// one segment, and split tiles leave (O, m, l) partials for k_fwd_combine.
//
// Roles (6 warps):
//   warp 0      TMA producer: Q once, then per chunk K and V (64x64 bf16 boxes,
//               128-byte swizzle) into one K and one V buffer.
//   warp 1      allocates 256 TMEM columns and issues tcgen05.mma (the whole
//               warp, one elected lane):
//               S = Q K^T (M=128, N=128, fp32 in TMEM), then O += P V with
//               P read from TMEM (aliasing S) and V MN-major from shared memory.
//   warps 2-9   two softmax warpgroups, one query row per thread, warpgroup g
//               owning key granule g of every chunk (S columns 64 g ..) and O
//               columns (D/2) g ..; the row maxima are exchanged through shared
//               memory once a chunk.  Per row: S from TMEM, masked online
//               softmax in the exp2 domain with lazy rescaling (the running
//               max only moves when it grows by more than 2^8), packed fp32
//               arithmetic, P as bf16 back into TMEM, then the epilogue.
// Two CTAs share an SM (about 100 KB shared memory and 256 TMEM columns
// each), so one CTA's softmax overlaps the other's MMAs.  Every wait is
// bounded; a timeout sets PRISM_DEV_TIMEOUT and the CTA winds down.
#include "attn_plan.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace prism {

using namespace sm100;

namespace {

constexpr int kRegion = 128 * 128;         // bytes of a 128-row x 64-col bf16 tile region
constexpr int kGranBytes = 64 * 128;       // 64 rows x 64 cols bf16
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0;              // O accumulator: D columns
constexpr uint32_t kColS = 128;            // S (fp32, 128 columns); P (bf16) over the first 32 of each granule's 64
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct FwdLayout {
    static constexpr int NR = D / 64;
    static constexpr int Q = 0;
    static constexpr int K = NR * kRegion;
    static constexpr int V = 2 * NR * kRegion;
    static constexpr int CTRL = 3 * NR * kRegion;
    static constexpr int XCH = CTRL + 256;         // [3][2][128] floats: row maxima (two parities), denominators
    static constexpr int ROWS = XCH + 3 * 2 * 128 * 4;   // two selection rows of SW words follow
    // bytes to request: + slack for 1024-byte alignment; at least 80 KB so that
    // no more than two CTAs (2 x 256 of the SM's 512 TMEM columns) share an SM
    static int alloc(int SW) {
        const int b = ROWS + 8 * SW + 1024;
        return b > 80 * 1024 ? b : 80 * 1024;
    }
};

struct FwdParts {
    float* o;       // [slots][128][D] unnormalised O
    float* m;       // [slots][128] running max, log2 domain
    float* l;       // [slots][128] denominator
};

// ------------------------------------------------------------------ raster (unpermuted) operands
enum { kMapQ = 0, kMapK = 1, kMapV = 2, kMapO = 3, kRasterMaps = 4 };

// one map, unused, in the blocked-layout kernel
template <bool RASTER>
using FwdRasterMaps = RasterMaps<RASTER ? kRasterMaps : 1>;
struct RasterOps {
    const int4* gpos;           // [N/64] per-granule raster positions (gran_positions)
};

template <int D, bool RASTER>
__global__ void __launch_bounds__(320, 2)
k_attn_fwd_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                 const __grid_constant__ CUtensorMap tmOf, const __grid_constant__ CUtensorMap tmPo,
                 const __grid_constant__ FwdRasterMaps<RASTER> rmaps, RasterOps ras,
                 const uint32_t* __restrict__ gsel,
                 const PlanHeader* __restrict__ hdr, const int4* __restrict__ items, FwdParts parts,
                 int64_t N, int64_t MB, int SW, float scale, __nv_bfloat16* __restrict__ O,
                 float* __restrict__ lse, float* __restrict__ o_f32, uint32_t* __restrict__ dev_status) {
    using L = FwdLayout<D>;
    if ((int)blockIdx.x >= hdr->n_items) return;              // uniform: beyond the item list
    const int4 item = items[blockIdx.x];
    const int tiles_per_head = (int)(N / 128);
    const int hh = item.x / tiles_per_head, tile = item.x % tiles_per_head;
    const int c_begin = item.y, nch = item.z - item.y, slot = item.w;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = sm + L::Q;
    uint8_t* sK = sm + L::K;
    uint8_t* sV = sm + L::V;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::CTRL);
    uint64_t* bar_q = bars + 0;
    uint64_t* bar_kf = bars + 1;
    uint64_t* bar_ke = bars + 2;
    uint64_t* bar_vf = bars + 3;
    uint64_t* bar_ve = bars + 4;
    uint64_t* bar_s = bars + 5;
    uint64_t* bar_p = bars + 6;
    uint64_t* bar_o = bars + 7;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    uint32_t* u0 = reinterpret_cast<uint32_t*>(sm + L::ROWS);
    uint32_t* u1 = u0 + SW;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wn = SW;
    const int64_t row0 = (int64_t)hh * N;                  // first row of this head in [heads*N, D]

    // the selection rows of the tile's two query granules
    load_rows(u0, u1, gsel + ((int64_t)hh * MB + 2 * tile) * SW, gsel + ((int64_t)hh * MB + 2 * tile + 1) * SW, wn);
    if (threadIdx.x == 0) {
        mbar_init(bar_q, L::NR);                           // one copy lane per region
        mbar_init(bar_kf, L::NR);
        mbar_init(bar_ke, 1);
        mbar_init(bar_vf, L::NR);
        mbar_init(bar_ve, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_o, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        // A copy engine completes the copies of one issuing thread one after
        // another, so each (tensor, 64-column region) has a lane of its own:
        // lane tensor * NR + r loads region r of Q (tensor 0 only, once), then of
        // K (tensor 0) or V (tensor 1) for both key granules of every chunk.
        if (lane < 2 * L::NR) {
            const int tensor = lane / L::NR, r = lane % L::NR;
            const CUtensorMap* mt = tensor ? &tmV : &tmK;
            uint64_t* bfull = tensor ? bar_vf : bar_kf;
            uint64_t* bempty = tensor ? bar_ve : bar_ke;
            uint8_t* buf = tensor ? sV : sK;
            if constexpr (!RASTER) tma_prefetch_desc(mt);
            if (tensor == 0) {
                mbar_expect_tx(bar_q, kRegion);
                if constexpr (RASTER) {
                    for (int hg = 0; hg < 2; ++hg) {             // the tile's two query granules
                        const int4 gp = ras.gpos[2 * tile + hg];
                        tma_load_5d(sQ + r * kRegion + hg * kGranBytes, rmaps.m + kMapQ * kRasterKinds + gp.w, bar_q,
                                    0, hh * L::NR + r, gp.z, gp.y, gp.x);
                    }
                } else {
                    tma_prefetch_desc(&tmQ);
                    tma_load_2d(sQ + r * kRegion, &tmQ, bar_q, 64 * r, (int)(row0 + 128 * tile));
                }
            }
            GranuleWalk walk;
            walk.init(u0, u1, wn);
            walk.skip(2 * c_begin);
            int issued = 0;
            for (int c = 0; c < nch && !*abort_flag; ++c) {
                int ra = 0, rb = 0;
                uint32_t ma, mb;
                walk.next(ra, ma);
                if (!walk.next(rb, mb)) rb = ra;
                if (c > 0 && !mbar_wait(bempty, (c - 1) & 1, abort_flag, dev_status)) break;
                mbar_expect_tx(bfull, 2 * kGranBytes);
                if constexpr (RASTER) {
                    const CUtensorMap* mk = rmaps.m + (tensor ? kMapV : kMapK) * kRasterKinds;
                    const int4 pa = ras.gpos[ra >> 6], pb = ras.gpos[rb >> 6];
                    tma_load_5d(buf + r * kRegion, mk + pa.w, bfull, 0, hh * L::NR + r, pa.z, pa.y, pa.x);
                    tma_load_5d(buf + r * kRegion + kGranBytes, mk + pb.w, bfull, 0, hh * L::NR + r, pb.z, pb.y, pb.x);
                } else {
                    tma_load_2d(buf + r * kRegion, mt, bfull, 64 * r, (int)(row0 + ra));
                    tma_load_2d(buf + r * kRegion + kGranBytes, mt, bfull, 64 * r, (int)(row0 + rb));
                }
                ++issued;
            }
            if (*abort_flag && issued) {
                // let this lane's copies land before the CTA goes away
                volatile int no_abort = 0;
                mbar_wait(bfull, (issued - 1) & 1, &no_abort, dev_status);
            }
        }
    } else if (warp == 1) {
        {   // the whole warp, converged; one elected lane issues
            // ------------------------------------------------ MMA issuer
            const uint32_t idS = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idO = idesc_bf16_f32(128, D, false, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait_w(bar_q, 0, abort_flag, dev_status);
            tc_fence_after();
            for (int c = 0; ok && c < nch; ++c) {
                if (!mbar_wait_w(bar_kf, c & 1, abort_flag, dev_status)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
                    mma_ss_w(tbase + kColS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024), idS,
                             k > 0 ? 1u : 0u);
                }
                tc_commit_w(bar_ke);
                tc_commit_w(bar_s);
                if (!mbar_wait_w(bar_p, c & 1, abort_flag, dev_status)) break;
                tc_fence_after();
                if (!mbar_wait_w(bar_vf, c & 1, abort_flag, dev_status)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts_w(tbase + kColO, tbase + kColS + 64 * (k >> 2) + 8 * (k & 3),
                             sdesc_sw128(aV + k * 2048, kRegion, 1024), idO,
                             (c > 0 || k > 0) ? 1u : 0u);
                tc_commit_w(bar_ve);
            }
            tc_commit_w(bar_o);
            if (*abort_flag) {
                volatile int no_abort = 0;
                mbar_wait(bar_o, 0, &no_abort, dev_status);
            }
        }
    } else {
        // ---------------------------------------------------- softmax + epilogue
        // Warpgroup g (warps 2-5: 0, 6-9: 1) owns key granule g of every chunk; both keep
        // the same running max (the row maxima are exchanged through shared memory, two
        // buffers by chunk parity so that one barrier a chunk suffices) and each sums its
        // own part of the denominator, added in a fixed order at the end.
        const int g = (warp - 2) >> 2;
        const int sub = warp & 3;                          // TMEM lane quarter of this warp
        const int row = sub * 32 + lane;                   // query row within the tile
        const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
        const int half = row >> 6;
        float* xmax = reinterpret_cast<float*>(sm + L::XCH);   // [parity][g][128]
        float* xden = xmax + 2 * 2 * 128;                      // [g][128]
        const float sl2 = scale * kLog2e;
        const uint64_t sl2x2 = f2pack(sl2, sl2);
        float m_run = -INFINITY, l = 0.f;
        GranuleWalk walk;
        if (lane == 0) {
            walk.init(u0, u1, wn);
            walk.skip(2 * c_begin);
        }
        bool ok = true;
        for (int c = 0; c < nch; ++c) {
            uint32_t mk = 0;
            if (lane == 0) {
                int ra, rb;
                uint32_t ma = 0, mb = 0;
                walk.next(ra, ma);
                if (!walk.next(rb, mb)) mb = 0;
                mk = ma | (mb << 2);
            }
            mk = __shfl_sync(0xffffffffu, mk, 0);
            const bool vg = (mk >> (2 * g + half)) & 1u;                     // warp-uniform
            const uint32_t tS = tl + kColS + 64 * g;                          // this granule's S
            bool got = ok && mbar_wait(bar_s, c & 1, abort_flag, dev_status);
            got = __all_sync(0xffffffffu, got);
            if (got) tc_fence_after();
            // pass 1: this granule's row max, then the other warpgroup's
            float mx = -INFINITY;
            if (got && vg) {
                uint32_t r[32];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_ld32(tS + 32 * q, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 2) mx = fmax3(mx, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
                }
            }
            xmax[((c & 1) * 2 + g) * 128 + row] = mx;
            named_sync(2, 256);                                // every thread, also after a timeout
            mx = fmaxf(mx, xmax[((c & 1) * 2 + (g ^ 1)) * 128 + row]);
            ok = ok && got;
            if (!ok) continue;                                 // winds down: barriers only
            const float mx2 = mx * sl2;
            const bool need = mx2 > m_run + kRescaleThreshold || (m_run == -INFINITY && mx2 > -INFINITY);
            const float alpha = need ? ex2(m_run - mx2) : 1.f;      // 0 when m_run = -inf
            // O holds chunks < c, all complete (S of chunk c was issued after them).
            // TMEM access is warp-collective: the whole warp rescales if any row must (both
            // warpgroups see the same rows and maxima, so they agree), each its O columns.
            if (c > 0 && __any_sync(0xffffffffu, need && m_run > -INFINITY)) {
                const uint64_t a2 = f2pack(alpha, alpha);
#pragma unroll
                for (int q = (D / 64) * g; q < (D / 64) * (g + 1); ++q) {
                    uint32_t r[32];
                    tmem_ld32(tl + kColO + 32 * q, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float x, y;
                        f2unpack(fmul2(f2pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), a2), x, y);
                        r[i] = __float_as_uint(x);
                        r[i + 1] = __float_as_uint(y);
                    }
                    tmem_st32(tl + kColO + 32 * q, r);
                }
            }
            if (need) {
                l *= alpha;
                m_run = mx2;
            }
            // pass 2: P = 2^(s * scale * log2e - m) as bf16 over the first 32 of the granule's
            // own 64 S columns (already read), 32 S columns per load
            const bool v = vg && m_run > -INFINITY;
            const uint64_t negm = f2pack(-m_run, -m_run);
            uint64_t rs2 = f2pack(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t pk[16];
                if (v) {
                    uint32_t r[32];
                    tmem_ld32(tS + 32 * q, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float x0, x1;
                        f2unpack(ffma2(f2pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), sl2x2, negm),
                                 x0, x1);
                        const float p0 = ex2(x0), p1 = ex2(x1);
                        rs2 = fadd2(rs2, f2pack(p0, p1));
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                }
                tmem_st16(tl + kColS + 64 * g + 16 * q, pk);
            }
            float rsa, rsb;
            f2unpack(rs2, rsa, rsb);
            l += rsa + rsb;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p);
        }
        const bool fin = __all_sync(0xffffffffu, ok && mbar_wait(bar_o, 0, abort_flag, dev_status));
        if (fin) tc_fence_after();
        // the denominator: the two warpgroups' parts, added in a fixed order
        xden[g * 128 + row] = l;
        named_sync(2, 256);
        const float lt = xden[row] + xden[128 + row];
        // Epilogue.  Every MMA is complete, so Q, K and V are free: O (bf16) is
        // staged in the Q buffer and the fp32 O or a split tile's partial in the
        // K and V buffers, as 16-byte chunks in the 128-byte-swizzled image of the
        // whole-row maps, each warpgroup its own columns, and each goes out in one
        // TMA store.  Every thread runs the barrier, also after a timeout.
        const int64_t grow = row0 + 128 * tile + row;
        const bool part = slot >= 0;
        const bool zero = part ? nch == 0 : (!(lt > 0.f) || nch == 0);   // nothing selected: O = 0
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const uint32_t sw = (uint32_t)(row & 7);
        if (fin) {
#pragma unroll 1
            for (int q = (D / 64) * g; q < (D / 64) * (g + 1); ++q) {
                uint32_t r[32];
                if (zero) {                                 // TMEM never written
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                } else {
                    tmem_ld32(tl + kColO + 32 * q, r);
                    tmem_wait_ld();
                }
                if (!part) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {           // 4 chunks of 8 bf16
                        const int gc = 4 * q + k;
                        uint4 v4;
                        v4.x = pack_bf16x2(__uint_as_float(r[8 * k + 0]) * inv, __uint_as_float(r[8 * k + 1]) * inv);
                        v4.y = pack_bf16x2(__uint_as_float(r[8 * k + 2]) * inv, __uint_as_float(r[8 * k + 3]) * inv);
                        v4.z = pack_bf16x2(__uint_as_float(r[8 * k + 4]) * inv, __uint_as_float(r[8 * k + 5]) * inv);
                        v4.w = pack_bf16x2(__uint_as_float(r[8 * k + 6]) * inv, __uint_as_float(r[8 * k + 7]) * inv);
                        *reinterpret_cast<uint4*>(sQ + (gc >> 3) * kRegion + row * 128 + (((gc & 7) ^ sw) << 4)) = v4;
                    }
                }
                if (part || o_f32) {
                    const float mul = part ? 1.f : inv;     // the partial stays unnormalised
#pragma unroll
                    for (int k = 0; k < 8; ++k) {           // 8 chunks of 4 fp32
                        const int gc = 8 * q + k;
                        const float4 v4 = make_float4(__uint_as_float(r[4 * k]) * mul, __uint_as_float(r[4 * k + 1]) * mul,
                                                      __uint_as_float(r[4 * k + 2]) * mul,
                                                      __uint_as_float(r[4 * k + 3]) * mul);
                        *reinterpret_cast<float4*>(sK + (gc >> 3) * kRegion + row * 128 + (((gc & 7) ^ sw) << 4)) = v4;
                    }
                }
            }
            fence_proxy_async_smem();
            if (g == 0) {
                if (!part) {
                    if (lse) lse[grow] = lt > 0.f ? (m_run + log2f(lt)) * kLn2 : -INFINITY;
                } else {
                    parts.m[(int64_t)slot * 128 + row] = m_run;
                    parts.l[(int64_t)slot * 128 + row] = lt;
                }
            }
        }
        named_sync(1, 256);
        if constexpr (RASTER) {
            // O back to the raster layout: one box per (query granule, region), a lane each;
            // the fp32 O (kept in permutation order) and the partials as whole-row tiles
            if (fin && warp == 2) {
                bool issued = false;
                if (!part && lane < 2 * L::NR) {
                    const int hg = lane / L::NR, r = lane % L::NR;
                    const int4 gp = ras.gpos[2 * tile + hg];
                    tma_store_5d(rmaps.m + kMapO * kRasterKinds + gp.w, sQ + r * kRegion + hg * kGranBytes, 0,
                                 hh * L::NR + r, gp.z, gp.y, gp.x);
                    issued = true;
                } else if (lane == 31) {
                    if (!part && o_f32) { tma_store_3d(&tmOf, sK, 0, (int)(row0 + 128 * tile), 0); issued = true; }
                    if (part) { tma_store_3d(&tmPo, sK, 0, slot * 128, 0); issued = true; }
                }
                if (issued) {
                    bulk_commit();
                    bulk_wait_read();
                }
            }
        } else {
            if (fin && warp == 2 && lane == 0) {
                if (!part) {
                    tma_store_3d(&tmO, sQ, 0, (int)(row0 + 128 * tile), 0);
                    if (o_f32) tma_store_3d(&tmOf, sK, 0, (int)(row0 + 128 * tile), 0);
                } else {
                    tma_store_3d(&tmPo, sK, 0, slot * 128, 0);
                }
                bulk_commit();
                bulk_wait_read();                           // shared memory stays valid until read
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------ host side
struct FwdWs {
    Plan plan;
    FwdParts parts;
};

size_t fwd_ws_bytes_d(const Dims& d) {
    const int64_t tiles = (int64_t)d.heads * (d.N / 128);
    const int target = plan_target(device_sms());
    const int64_t slots = 2 * (int64_t)target;
    return plan_bytes(tiles, target) + align16(slots * 128 * d.d * 4) + 2 * align16(slots * 128 * 4);
}

FwdWs carve_fwd(void* ws, const Dims& d) {
    const int64_t tiles = (int64_t)d.heads * (d.N / 128);
    const int target = plan_target(device_sms());
    const int64_t slots = 2 * (int64_t)target;
    FwdWs w;
    w.plan = carve_plan(ws, tiles, target);
    uint8_t* p = static_cast<uint8_t*>(ws) + plan_bytes(tiles, target);
    w.parts.o = reinterpret_cast<float*>(p);
    p += align16(slots * 128 * d.d * 4);
    w.parts.m = reinterpret_cast<float*>(p);
    p += align16(slots * 128 * 4);
    w.parts.l = reinterpret_cast<float*>(p);
    return w;
}

// Raster operands: the workspace also holds the per-granule positions after the
// blocked-layout workspace.
size_t fwd_raster_extra_bytes(const Dims& d) { return align16(d.MB * (int64_t)sizeof(int4)); }

template <int D, bool RASTER>
prism_status_t launch_fwd(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const int32_t* perm,
                          const uint8_t* shape_id, const uint32_t* gsel, float scale, void* Op, float* lse,
                          float* o_f32, uint32_t* dev_status, void* ws, cudaStream_t s) {
    CUtensorMap mQ, mK, mV, mO, mOf, mPo;
    const int64_t rows = (int64_t)d.heads * d.N;
    FwdWs w = carve_fwd(ws, d);
    const int64_t slots = 2 * (int64_t)plan_target(device_sms());
    // fp32 outputs stay in permutation order: whole 128-row tiles (the fp32 O map only when o_f32 is given)
    if (!make_map_f32_rows(&mPo, w.parts.o, slots * 128, D, 128) ||
        (o_f32 && !make_map_f32_rows(&mOf, o_f32, rows, D, 128)))
        return PRISM_ERR_CUDA;
    if (!o_f32) mOf = mPo;                              // never used
    FwdRasterMaps<RASTER> rm;
    RasterOps ras{nullptr};
    if constexpr (RASTER) {
        const void* bases[kRasterMaps] = {Qp, Kp, Vp, Op};
        for (int t = 0; t < kRasterMaps; ++t)
            for (int k = 0; k < kRasterKinds; ++k)
                if (!make_map_raster(&rm.m[t * kRasterKinds + k], bases[t], d.heads, D, d.T, d.H, d.W, k))
                    return PRISM_ERR_CUDA;
        int4* gpos = reinterpret_cast<int4*>(static_cast<uint8_t*>(ws) + fwd_ws_bytes_d(d));
        if (gran_positions(perm, shape_id, d, gpos, s) != PRISM_OK) return PRISM_ERR_CUDA;
        ras.gpos = gpos;
        mQ = mK = mV = mO = mPo;                        // never used
    } else {
        if (!make_map_bf16(&mQ, Qp, rows, D, 128) || !make_map_bf16(&mK, Kp, rows, D, 64) ||
            !make_map_bf16(&mV, Vp, rows, D, 64) || !make_map_bf16_rows(&mO, Op, rows, D, 128))
            return PRISM_ERR_CUDA;
        rm.m[0] = mPo;                                  // never used
    }
    const int target = plan_target(device_sms());
    prism_status_t st = plan_work(w.plan, gsel, d, 2, 2, target, kSegMinChunks, s);
    if (st != PRISM_OK) return st;
    auto k = k_attn_fwd_sm100<D, RASTER>;
    const int smem = FwdLayout<D>::alloc((int)d.SW);
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PRISM_ERR_CUDA;
    k<<<(unsigned)w.plan.items_max, 320, smem, s>>>(mQ, mK, mV, mO, mOf, mPo, rm, ras, gsel, w.plan.hdr, w.plan.items,
                                                    w.parts, d.N, d.MB, (int)d.SW, scale, (__nv_bfloat16*)Op, lse,
                                                    o_f32, dev_status);
    st = launch_status(1);
    if (st != PRISM_OK) return st;
    return fwd_combine(w.plan, d, 128, w.parts.o, w.parts.m, w.parts.l, Op, o_f32, lse, RASTER ? perm : nullptr, s);
}

}  // namespace

size_t attn_fwd_sm100_ws_bytes(const Dims& d) { return fwd_ws_bytes_d(d); }
size_t attn_fwd_raster_ws_bytes(const Dims& d) { return fwd_ws_bytes_d(d) + fwd_raster_extra_bytes(d); }

prism_status_t attn_fwd_sm100(const Dims& d, const void* Qp, const void* Kp, const void* Vp, const uint32_t* gsel,
                              float scale, void* Op, float* lse, float* o_f32, uint32_t* dev_status, void* ws,
                              cudaStream_t s) {
    if (d.d == 128)
        return launch_fwd<128, false>(d, Qp, Kp, Vp, nullptr, nullptr, gsel, scale, Op, lse, o_f32, dev_status, ws, s);
    return launch_fwd<64, false>(d, Qp, Kp, Vp, nullptr, nullptr, gsel, scale, Op, lse, o_f32, dev_status, ws, s);
}

// raster Q, K, V, O ([N][heads][d]); perm and shape_id from prism_assign_shapes; lse and
// o_f32 (nullable) stay in permutation order
prism_status_t attn_fwd_raster(const Dims& d, const void* Q, const void* K, const void* V, const int32_t* perm,
                               const uint8_t* shape_id, const uint32_t* gsel, float scale, void* O, float* lse,
                               float* o_f32, uint32_t* dev_status, void* ws, cudaStream_t s) {
    if (d.d == 128)
        return launch_fwd<128, true>(d, Q, K, V, perm, shape_id, gsel, scale, O, lse, o_f32, dev_status, ws, s);
    return launch_fwd<64, true>(d, Q, K, V, perm, shape_id, gsel, scale, O, lse, o_f32, dev_status, ws, s);
}

}  // namespace prism
