// dS handoff of the bf16 backward: the key-stationary kernel stores the dS^T
// blocks it forms anyway, and the query-stationary kernel reads them back and
// does dQ += dS K alone, instead of forming S = Q K^T and dP = dO V^T a
// second time (7 GEMMs a selected block become 5).
//
// Pieces.  For every 128-key tile tk the key-stationary kernel walks the union
// U_k(tk) of the query granules that selected either of its two key granules,
// in ascending order; its u-th unit (tk, query granule U_k(tk)[u]) forms dS^T
// for 128 keys x 64 queries.  That block is piece 1 + base_kv[tk] + u:
// 128 rows (keys) of 64 bf16 (queries), 128 bytes a row, where base_kv is the
// exclusive prefix sum of |U_k| over the tiles in plan order (head-major).
// Piece 0 is all zeros.
//
// Entries.  For every 128-row query tile tq the query-stationary kernel walks
// the union U_q(tq) of the key granules its two query granules selected; its
// u-th unit reads entry base_q[tq] + u = (64 gk, y0, y1, 0) with
// gk = U_q(tq)[u] and y_h the first row, in the piece array, of the 64 x 64
// block that holds dS^T for key granule gk and query granule 2 tq + h:
// row 128 p + 64 (gk & 1) of piece p = 1 + base_kv[tile of gk] + the rank of
// 2 tq + h in U_k(tile of gk), or row 0 (the zero piece) when query granule
// 2 tq + h did not select gk.  The rank is a word prefix of the key tile's
// union (pre[w] = set bits of its words below w) plus one popcount.
//
// These helpers hold the index arithmetic only; they compile for the host as
// well, so that it can be checked against an independent enumeration.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define PRISM_HD __host__ __device__ __forceinline__
#else
#define PRISM_HD inline
#endif

namespace prism {
namespace ds {

constexpr int64_t kPieceRows = 128;                   // keys of a piece
constexpr int64_t kPieceBytes = kPieceRows * 64 * 2;  // 16 KB of bf16
constexpr int64_t kEntryBytes = 16;                   // one int4 entry
// TMA row coordinates are 32-bit: every piece row must stay below 2^31
constexpr int64_t kMaxPieces = (int64_t(1) << 31) / kPieceRows - 1;

PRISM_HD int popc32(uint32_t x) {
#if defined(__CUDA_ARCH__)
    return __popc(x);
#else
    return __builtin_popcount(x);
#endif
}

// word w of the union of the selection rows r and r + 1 (rows of SW words)
PRISM_HD uint32_t union_word(const uint32_t* sel, int64_t r, int64_t SW, int64_t w) {
    return sel[r * SW + w] | sel[(r + 1) * SW + w];
}

// position of granule q in the ascending union of rows r, r + 1 of `sel`,
// from that union's word prefix `pre_tile` (pre_tile[w] = set bits below word w)
PRISM_HD int64_t rank_in_union(const uint32_t* sel, const int32_t* pre_tile, int64_t r, int64_t SW, int q) {
    const int w = q >> 5;
    const uint32_t below = (1u << (q & 31)) - 1u;
    return (int64_t)pre_tile[w] + popc32(union_word(sel, r, SW, w) & below);
}

// Entry of key granule gk for query tile tq of head hh.
//   gsel   [heads][MB][SW] granule-level selection rows (query granule -> key granules)
//   gselT  [heads][MB][SW] its transpose (key granule -> query granules)
//   pre    [heads * tph][SW] word prefixes of the key tiles' unions of gselT rows
//   base_kv [heads * tph] exclusive prefix sums of the key tiles' union sizes
// out = (64 gk, y0, y1, 0), piece rows as described above.
PRISM_HD void make_entry(const uint32_t* gsel, const uint32_t* gselT, const int32_t* pre, const int64_t* base_kv,
                         int hh, int64_t MB, int64_t SW, int64_t tph, int64_t tq, int gk, int32_t out[4]) {
    const int64_t tk = (int64_t)hh * tph + (gk >> 1);          // the key tile, in plan order
    const int64_t rk = (int64_t)hh * MB + 2 * (gk >> 1);        // its first gselT row
    out[0] = 64 * gk;
    out[3] = 0;
    for (int h = 0; h < 2; ++h) {
        const int64_t gq = 2 * tq + h;
        const bool sel = (gsel[((int64_t)hh * MB + gq) * SW + (gk >> 5)] >> (gk & 31)) & 1u;
        int32_t y = 0;
        if (sel) {
            const int64_t p = 1 + base_kv[tk] + rank_in_union(gselT, pre + tk * SW, rk, SW, (int)gq);
            y = (int32_t)(kPieceRows * p + 64 * (gk & 1));
        }
        out[1 + h] = y;
    }
}

// byte offset of the dS^T row `key_row` (0..127) of piece 1 + base + u
PRISM_HD int64_t piece_row_offset(int64_t base, int64_t u, int key_row) {
    return ((1 + base + u) * kPieceRows + key_row) * 128;
}

}  // namespace ds
}  // namespace prism
