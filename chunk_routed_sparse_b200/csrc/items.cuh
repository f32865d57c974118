// Work items of the chunk-major attention kernels (the forward pass and the
// dQ part of the backward pass) and the walk over an item's key tiles.
//
// The attention over Omega(q) ("Mixture of Contexts for Long Video Generation
// | Summary" §3.1: the anchors and the selected chunks) is split into items:
//   anchor items - <= kItemRows consecutive queries of one query group against
//                  the group's anchor key ranges (partial slot 0);
//   routed items - <= kItemRows entries of one chunk's query list (query << 5 |
//                  slot) against that chunk's keys (partial slot 1 + slot).
// Anchor items come first, in the layout's anchor order (groups with the most
// keys first), each group's items for every (b, h); routed items follow in
// (b, h, chunk) order.
#pragma once

#include "common.cuh"

namespace moc {
namespace items {

constexpr int kKT = 128;  // keys per tile

struct Item {
    int bh, nq, slot_fixed, q0;
    const int32_t* entries;
    int r_beg, r_end, k0, k1;
};

// Item `item` of ROWS-row items: atab is the prefix of anchor items per group (in
// a_order), tile_off the prefix of routed items per (b, h, chunk) list.
template <int ROWS>
__device__ __forceinline__ bool decode_rows(const DevLayout& dv, const int32_t* atab, int BH, int64_t n_anchor,
                                            int64_t item, const int32_t* tile_off, const int32_t* qoff,
                                            const int32_t* qlist, Item& it) {
    if (item < n_anchor) {
        const int pos = upper_index(atab, dv.G + 1, item / BH);
        const int64_t local = item - int64_t(BH) * atab[pos];
        const int nt = atab[pos + 1] - atab[pos];
        const int g = dv.a_order[pos];
        it.bh = int(local / nt);
        it.q0 = dv.grp_q0[g] + int(local % nt) * ROWS;
        it.nq = min(ROWS, dv.grp_q1[g] - it.q0);
        it.slot_fixed = 0;
        it.entries = nullptr;
        it.r_beg = dv.ar_off[g];
        it.r_end = dv.ar_off[g + 1];
        it.k0 = it.k1 = 0;
        return true;
    }
    const int64_t r = item - n_anchor;
    const int64_t nlists = int64_t(BH) * dv.C;
    if (r >= tile_off[nlists]) return false;
    const int x = upper_index(tile_off, int(nlists + 1), r);
    const int c = x % dv.C;
    it.bh = x / dv.C;
    const int e0 = qoff[x] + int(r - tile_off[x]) * ROWS;
    it.nq = min(ROWS, qoff[x + 1] - e0);
    it.entries = qlist + e0;
    it.slot_fixed = -1;
    it.q0 = 0;
    it.r_beg = it.r_end = -1;
    it.k0 = dv.chunk_off[c];
    it.k1 = dv.chunk_off[c + 1];
    return true;
}

// Items of kItemRows rows (the layout's atile_off, the workspace's tile_off).
__device__ __forceinline__ bool decode(const DevLayout& dv, int BH, int64_t n_anchor, int64_t item,
                                       const int32_t* tile_off, const int32_t* qoff, const int32_t* qlist,
                                       Item& it) {
    return decode_rows<kItemRows>(dv, dv.atile_off, BH, n_anchor, item, tile_off, qoff, qlist, it);
}

// Key tiles of an item, in order: each range cut into 128-key tiles.
struct Cursor {
    const int32_t* ar;
    int r, r_end, pos, end;
    __device__ void init(const DevLayout& dv, const Item& it) {
        if (it.r_beg >= 0) {
            ar = dv.ar; r = it.r_beg; r_end = it.r_end;
            pos = ar[2 * r];
            end = ar[2 * r + 1];
        } else {
            ar = nullptr; r = 0; r_end = 1; pos = it.k0; end = it.k1;
        }
    }
    __device__ bool more() const { return r < r_end; }
    __device__ void next(int& key0, int& nvalid) {
        key0 = pos;
        nvalid = min(kKT, end - pos);
        pos += kKT;
        if (pos >= end) {
            ++r;
            if (ar && r < r_end) {
                pos = ar[2 * r];
                end = ar[2 * r + 1];
            }
        }
    }
};

__device__ __forceinline__ int count_tiles(const DevLayout& dv, const Item& it) {
    if (it.r_beg < 0) return (it.k1 - it.k0 + kKT - 1) / kKT;
    int t = 0;
    for (int r = it.r_beg; r < it.r_end; ++r) t += (dv.ar[2 * r + 1] - dv.ar[2 * r] + kKT - 1) / kKT;
    return t;
}

}  // namespace items
}  // namespace moc
