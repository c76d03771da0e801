// Host test of the per-warp work partition (compiled with g++ by
// tests/test_partition.py): every tile-group is owned by exactly one warp,
// ranges are contiguous and cost-balanced to within one tile-group, and
// part_owner() agrees with the ranges.
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
    std::printf("%d cases, %d failures\n", cases, fails);
    return fails != 0;
}
