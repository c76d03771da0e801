// Host test of the per-warp work partitions (compiled with g++ by
// tests/test_partition.py): every tile-group (or chunk) is owned by exactly
// one warp, ranges are contiguous and cost-balanced to within one unit of
// work at each end, and part_owner() agrees with the ranges.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../decode_gemv_tb_b200/csrc/tb_partition.h"

using namespace tb;

static int check(const std::vector<PartItem>& items, uint32_t W) {
    const int n = (int)items.size();
    uint32_t C = 0, TG = 0;
    for (auto& it : items) {
        C += (uint32_t)(it.tg_count * it.unit_cost);
        TG += (uint32_t)it.tg_count;
    }
    const uint32_t Q = (C + W - 1) / W;
    std::vector<uint32_t> pos(TG), unit(TG);
    for (auto& it : items)
        for (int64_t k = 0; k < it.tg_count; ++k) {
            pos[it.tg_base + k] = (uint32_t)(it.cost_base + k * it.unit_cost);
            unit[it.tg_base + k] = (uint32_t)it.unit_cost;
        }
    uint32_t prev_end = 0;
    for (uint32_t w = 0; w < W; ++w) {
        uint32_t b, e;
        part_range(items.data(), n, w, Q, C, &b, &e);
        if (b != prev_end) { std::printf("gap at warp %u\n", w); return 1; }
        uint32_t cost = 0;
        for (uint32_t tg = b; tg < e; ++tg) {
            if (part_owner(pos[tg], Q) != w) { std::printf("owner mismatch tg %u\n", tg); return 1; }
            cost += unit[tg];
        }
        // a warp's cost is its quota up to the one tile-group that straddles each end of it
        if (cost > Q + 2 || (e < TG && cost + 3 < Q)) {
            std::printf("unbalanced warp %u: cost %u quota %u\n", w, cost, Q);
            return 1;
        }
        prev_end = e;
    }
    if (prev_end != TG) { std::printf("ranges end at %u of %u\n", prev_end, TG); return 1; }
    return 0;
}

static int check_chunks(const std::vector<ChunkItem>& items, uint32_t W) {
    const int n = (int)items.size();
    uint32_t C = 0, NC = 0, maxc = 0;
    std::vector<uint32_t> pos, cost;
    for (auto& it : items) {
        if ((uint32_t)it.chunk_base != NC || (uint32_t)it.cost_base != C) { std::printf("bad bases\n"); return 1; }
        for (int t = 0; t < it.T; ++t)
            for (int j = 0; j < it.cpt; ++j) {
                const int groups = (j + 1) * it.C <= it.G ? it.C : it.G - j * it.C;
                pos.push_back(C + (uint32_t)((t * it.G + j * it.C) * it.unit_cost));
                cost.push_back((uint32_t)(groups * it.unit_cost));
                if (cost.back() > maxc) maxc = cost.back();
            }
        C += (uint32_t)(it.T * it.G * it.unit_cost);
        NC += (uint32_t)(it.T * it.cpt);
    }
    const uint32_t Q = (C + W - 1) / W;
    uint32_t prev_end = 0;
    for (uint32_t w = 0; w < W; ++w) {
        uint32_t b, e;
        part_chunk_range(items.data(), n, w, Q, C, &b, &e);
        if (b != prev_end) { std::printf("chunk gap at warp %u\n", w); return 1; }
        uint32_t c = 0;
        for (uint32_t k = b; k < e; ++k) {
            if (part_owner(pos[k], Q) != w) { std::printf("chunk owner mismatch %u\n", k); return 1; }
            c += cost[k];
        }
        if (c > Q + maxc || (e < NC && c + maxc < Q)) {
            std::printf("unbalanced chunk warp %u: cost %u quota %u\n", w, c, Q);
            return 1;
        }
        prev_end = e;
    }
    if (prev_end != NC) { std::printf("chunk ranges end at %u of %u\n", prev_end, NC); return 1; }
    return 0;
}

int main() {
    std::srand(7);
    int fails = 0, cases = 0;
    for (int rep = 0; rep < 400; ++rep) {
        std::vector<PartItem> items;
        int n = 1 + std::rand() % 16;
        int64_t tg = 0, cost = 0;
        for (int i = 0; i < n; ++i) {
            PartItem it;
            it.tg_base = tg;
            it.tg_count = 1 + std::rand() % 3000;
            it.cost_base = cost;
            it.unit_cost = (std::rand() % 2) ? 2 : 3;
            tg += it.tg_count;
            cost += it.tg_count * it.unit_cost;
            items.push_back(it);
        }
        uint32_t W = 1 + std::rand() % 4000;
        fails += check(items, W);
        ++cases;
    }
    for (int rep = 0; rep < 400; ++rep) {
        std::vector<ChunkItem> items;
        int n = 1 + std::rand() % 16;
        int64_t nc = 0, cost = 0;
        for (int i = 0; i < n; ++i) {
            ChunkItem it;
            it.chunk_base = nc;
            it.cost_base = cost;
            it.T = 1 + std::rand() % 400;
            it.G = 1 + std::rand() % 140;
            it.unit_cost = (std::rand() % 2) ? 2 : 3;
            it.C = it.unit_cost == 2 ? 4 : 2;
            it.cpt = (it.G + it.C - 1) / it.C;
            nc += (int64_t)it.T * it.cpt;
            cost += (int64_t)it.T * it.G * it.unit_cost;
            items.push_back(it);
        }
        uint32_t W = 1 + std::rand() % 4000;
        fails += check_chunks(items, W);
        ++cases;
    }
    std::printf("%d cases, %d failures\n", cases, fails);
    return fails != 0;
}
