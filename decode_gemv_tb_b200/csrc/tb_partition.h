// tb_partition.h -- equal-cost split of a grouped GEMV into per-warp ranges
// (host and device).
//
// The work of a launch is the sequence of "tile-groups" (32 output rows x
// one 128-group of K) of every item, item by item, tile by tile, group by
// group.  A tile-group of item i costs c_i units (2 for the 2-bit container,
// 3 for 3 bits: its packed bytes / 512), so its cost position is
//     pos(tg) = cost_base_i + (tg - tg_base_i) * c_i.
// Warp w owns the tile-groups whose cost position lies in [w Q, (w+1) Q)
// with the quota Q = ceil(C / W) (C the total cost, W the warps): a
// contiguous range, and the owner of a tile-group is pos / Q.  Warps past
// the end get empty ranges.  Every quantity fits 32 bits (the launcher
// checks C < 2^31), and the ranges need no division.  (A launch may run
// two such partitions side by side, one per code width, each over its own
// items and warps.)
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define TB_HD __host__ __device__ __forceinline__
#else
#define TB_HD inline
#endif

namespace tb {

struct PartItem {
    int64_t tg_base, tg_count;  // first tile-group and count (tiles * groups)
    int64_t cost_base;          // cost position of the first tile-group
    int32_t unit_cost;          // cost of one tile-group (2 or 3)
};

// owner warp of the tile-group at cost position pos
TB_HD uint32_t part_owner(uint32_t pos, uint32_t Q) { return pos / Q; }

// first tile-group whose cost position is >= L (Item: any type with the
// PartItem fields)
template <class Item>
TB_HD uint32_t part_first_tg(const Item* it, int n, uint32_t L) {
    for (int i = 0; i < n; ++i) {
        const uint32_t cb = (uint32_t)it[i].cost_base, uc = (uint32_t)it[i].unit_cost;
        const uint32_t end = cb + (uint32_t)it[i].tg_count * uc;
        if (L < end) {
            const uint32_t d = L > cb ? L - cb : 0;
            const uint32_t k = uc == 2 ? (d + 1) >> 1 : (d + 2) / 3;
            return (uint32_t)it[i].tg_base + k;
        }
    }
    return n ? (uint32_t)(it[n - 1].tg_base + it[n - 1].tg_count) : 0;
}

// [begin, end) tile-groups of warp w (empty when w Q >= C)
template <class Item>
TB_HD void part_range(const Item* it, int n, uint32_t w, uint32_t Q, uint32_t C, uint32_t* begin, uint32_t* end) {
    const uint32_t lo = w * Q < C ? w * Q : C, hi = (w + 1) * Q < C ? (w + 1) * Q : C;
    *begin = part_first_tg(it, n, lo);
    *end = part_first_tg(it, n, hi);
}

// Chunked variant.  The work of item i is T_i tiles x G_i groups, read in
// chunks of C_i consecutive groups of one tile (a tile's last chunk may be
// shorter; chunks per tile cpt_i = ceil(G_i / C_i)), numbered item by item,
// tile by tile from chunk_base_i.  Chunk j of tile t starts at the cost
// position
//     pos = cost_base_i + (t G_i + j C_i) c_i,
// and a warp owns the chunks whose start position lies in its quota range
// [w Q, (w + 1) Q): whole chunks only, so no chunk is read by two warps.
struct ChunkItem {
    int64_t chunk_base, cost_base;
    int32_t T, G, C, cpt, unit_cost;
};

// first chunk whose start position is >= L (Item: any type with the
// ChunkItem fields)
template <class Item>
TB_HD uint32_t part_first_chunk(const Item* it, int n, uint32_t L) {
    for (int i = 0; i < n; ++i) {
        const uint32_t cb = (uint32_t)it[i].cost_base, uc = (uint32_t)it[i].unit_cost;
        const uint32_t tcost = (uint32_t)it[i].G * uc, end = cb + (uint32_t)it[i].T * tcost;
        if (L < end) {
            const uint32_t d = L > cb ? L - cb : 0, ccost = (uint32_t)it[i].C * uc;
            uint32_t t = d / tcost;
            const uint32_t r = d - t * tcost;
            uint32_t j = (r + ccost - 1) / ccost;
            if (j >= (uint32_t)it[i].cpt) {
                ++t;
                j = 0;
            }
            return (uint32_t)it[i].chunk_base + t * (uint32_t)it[i].cpt + j;
        }
    }
    return n ? (uint32_t)(it[n - 1].chunk_base + (int64_t)it[n - 1].T * it[n - 1].cpt) : 0;
}

// [begin, end) chunks of warp w (empty when w Q >= C)
template <class Item>
TB_HD void part_chunk_range(const Item* it, int n, uint32_t w, uint32_t Q, uint32_t C, uint32_t* begin,
                            uint32_t* end) {
    const uint32_t lo = w * Q < C ? w * Q : C, hi = (w + 1) * Q < C ? (w + 1) * Q : C;
    *begin = part_first_chunk(it, n, lo);
    *end = part_first_chunk(it, n, hi);
}

}  // namespace tb
