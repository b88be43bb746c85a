// Work plan shared by the tensor-core attention kernels (see attn_plan.cu).
#pragma once

#include <atomic>

#include "common.cuh"

namespace prism {

struct PlanHeader {
    unsigned long long total_units;   // work units over all tiles
    int seg;                          // units per segment
    int n_items;                      // items in the list
    int n_slots;                      // partial-result slots used by split tiles
    int pad[11];                      // 64 bytes
};

struct Plan {
    PlanHeader* hdr;
    int32_t* tile_units;              // [tiles] units per tile
    int2* tile_split;                 // [tiles] (first slot or -1, segments)
    int4* items;                      // [tiles + target] (tile, unit begin, unit end, slot or -1)
    int64_t tiles;                    // heads * N / tile rows
    int64_t items_max;
};

inline int64_t align16(int64_t b) { return (b + 15) & ~int64_t(15); }

// items stay near this many per launch; at most 2*target partial slots
inline int plan_target(int num_sms) { return 4 * 2 * num_sms; }
constexpr int kSegMinChunks = 8;      // forward: 128-key chunks
constexpr int kSegMinGranules = 16;   // backward: 64-row granules

size_t plan_bytes(int64_t tiles, int target);
Plan carve_plan(void* base, int64_t tiles, int target);
// tile_gran: 64-row granules per tile (2: the 128-row tiles of the forward and
// the backward); unit_granules: granules per work unit
prism_status_t plan_work(const Plan& pl, const uint32_t* rows, const Dims& d, int tile_gran, int unit_granules,
                         int target, int seg_min, cudaStream_t s);
prism_status_t fwd_combine(const Plan& pl, const Dims& d, int tile_rows, const float* opart, const float* mpart,
                           const float* lpart, void* Op, float* o_f32, float* lse, const int32_t* perm,
                           cudaStream_t s);
// perm != nullptr: the outputs are raster [N][heads][d] (rows scattered through it)
prism_status_t bwd_combine(const Plan& pl, const Dims& d, int nout, const float* part, void* out0, float mul0,
                           void* out1, float mul1, cudaStream_t s, const int32_t* perm = nullptr);

// per 64-row granule g of the blocked order: (t0, h0, w0, box kind) of its first
// token perm[64 g] (the raster maps' coordinates; see make_map_raster)
prism_status_t gran_positions(const int32_t* perm, const uint8_t* shape_id, const Dims& d, int4* gpos,
                              cudaStream_t s);

// number of SMs of the current device (cached per device ordinal; the plan
// target and the workspace sizes depend on it)
inline int device_sms() {
    constexpr int kMaxDev = 64;
    static std::atomic<int> cache[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
    int sms = dev < kMaxDev ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
        if (dev < kMaxDev) cache[dev].store(sms, std::memory_order_relaxed);
    }
    return sms;
}

}  // namespace prism
