// Host check of the dS handoff's index arithmetic (csrc/ds_handoff.cuh), built
// with g++ by tests/test_ds_handoff_index.py.
//
// Input (binary file argv[1]): int32 heads, MB, SW, then gsel as
// uint32 [heads][MB][SW].  The program forms the transpose, the plan units
// and prefix sums and the key tiles' word prefixes in plain loops, then uses
// the header's functions for both sides of the handoff:
//   - the key-stationary side writes, for every unit (key tile tk, u-th query
//     granule gq of its union) and every key row r selected by gq, the values
//     tag(head, key granule, key, gq, query) at piece_row_offset(base_kv[tk], u, r);
//   - the query-stationary side reads, for every unit (query tile tq, u-th key
//     granule of its union), the two 64 x 64 blocks at rows y0, y1 of its entry
//     and compares every value with the tag (or zero where gq did not select gk).
// Output (stdout): one line "E t u x y0 y1" per entry in walk order, then
// "checked <values> mismatches <count>".
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "ds_handoff.cuh"

using namespace prism;

static int64_t tag(int64_t hh, int64_t gk, int64_t key, int64_t gq, int64_t q, int64_t MB) {
    return ((((hh * MB + gk) * 64 + key) * MB + gq) * 64 + q) + 1;   // never zero
}

int main(int argc, char** argv) {
    if (argc < 2) return 2;
    FILE* f = std::fopen(argv[1], "rb");
    if (!f) return 2;
    int32_t dims[3];
    if (std::fread(dims, 4, 3, f) != 3) return 2;
    const int heads = dims[0];
    const int64_t MB = dims[1], SW = dims[2], tph = MB / 2;
    std::vector<uint32_t> gsel((size_t)(heads * MB * SW)), gselT(gsel.size(), 0u);
    if (std::fread(gsel.data(), 4, gsel.size(), f) != gsel.size()) return 2;
    std::fclose(f);
    auto bit = [&](const std::vector<uint32_t>& s, int64_t hh, int64_t row, int64_t g) {
        return (s[(size_t)((hh * MB + row) * SW + (g >> 5))] >> (g & 31)) & 1u;
    };
    for (int64_t hh = 0; hh < heads; ++hh)
        for (int64_t gq = 0; gq < MB; ++gq)
            for (int64_t gk = 0; gk < MB; ++gk)
                if (bit(gsel, hh, gq, gk)) gselT[(size_t)((hh * MB + gk) * SW + (gq >> 5))] |= 1u << (gq & 31);
    // union of rows 2t, 2t + 1, ascending
    auto walk = [&](const std::vector<uint32_t>& s, int64_t hh, int64_t t) {
        std::vector<int> out;
        for (int64_t g = 0; g < MB; ++g)
            if (bit(s, hh, 2 * t, g) || bit(s, hh, 2 * t + 1, g)) out.push_back((int)g);
        return out;
    };
    const int64_t tiles = heads * tph;
    std::vector<int64_t> base_q((size_t)tiles), base_kv((size_t)tiles);
    std::vector<int32_t> pre((size_t)(tiles * SW));
    int64_t aq = 0, ak = 0;
    for (int64_t t = 0; t < tiles; ++t) {
        const int64_t hh = t / tph, tt = t % tph;
        base_q[(size_t)t] = aq;
        base_kv[(size_t)t] = ak;
        aq += (int64_t)walk(gsel, hh, tt).size();
        ak += (int64_t)walk(gselT, hh, tt).size();
        int32_t c = 0;
        for (int64_t w = 0; w < SW; ++w) {
            pre[(size_t)(t * SW + w)] = c;
            c += ds::popc32(ds::union_word(gselT.data(), hh * MB + 2 * tt, SW, w));
        }
    }
    // key-stationary side: pieces as int64 values, 128 rows x 64 columns each
    std::vector<int64_t> pieces((size_t)((1 + ak) * 128 * 64), 0);
    for (int64_t t = 0; t < tiles; ++t) {
        const int64_t hh = t / tph, tk = t % tph;
        const std::vector<int> uk = walk(gselT, hh, tk);
        for (size_t u = 0; u < uk.size(); ++u) {
            const int gq = uk[u];
            for (int r = 0; r < 128; ++r) {
                const int64_t gk = 2 * tk + (r >> 6);
                if (!bit(gsel, hh, gq, gk)) continue;        // a half the look-up never reads
                const int64_t off = ds::piece_row_offset(base_kv[(size_t)t], (int64_t)u, r) / 128 * 64;
                for (int q = 0; q < 64; ++q) pieces[(size_t)(off + q)] = tag(hh, gk, r & 63, gq, q, MB);
            }
        }
    }
    // look-up side
    int64_t checked = 0, bad = 0;
    for (int64_t t = 0; t < tiles; ++t) {
        const int hh = (int)(t / tph);
        const int64_t tq = t % tph;
        const std::vector<int> uq = walk(gsel, hh, tq);
        for (size_t u = 0; u < uq.size(); ++u) {
            int32_t e[4];
            ds::make_entry(gsel.data(), gselT.data(), pre.data(), base_kv.data(), hh, MB, SW, tph, tq, uq[u], e);
            std::printf("E %lld %zu %d %d %d\n", (long long)t, u, e[0], e[1], e[2]);
            const int gk = e[0] / 64;
            for (int h = 0; h < 2; ++h) {
                const int64_t gq = 2 * tq + h;
                const bool sel = bit(gsel, hh, gq, gk);
                for (int kr = 0; kr < 64; ++kr)
                    for (int q = 0; q < 64; ++q) {
                        const int64_t idx = ((int64_t)e[1 + h] + kr) * 64 + q;
                        const int64_t got = idx < (int64_t)pieces.size() ? pieces[(size_t)idx] : -1;
                        const int64_t want = sel ? tag(hh, gk, kr, gq, q, MB) : 0;
                        ++checked;
                        if (got != want) ++bad;
                    }
            }
        }
    }
    std::printf("checked %lld mismatches %lld\n", (long long)checked, (long long)bad);
    return 0;
}
