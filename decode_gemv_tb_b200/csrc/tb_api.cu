// tb_api.cu -- the C interface declared in include/tb.h: argument checks,
// then one launch on the caller's stream.  No allocation, no
// synchronization, no host fallback: every computation runs in the kernels.
#include <algorithm>
#include <cstring>

#include "../../include/tb.h"
#include "tb_device.cuh"
#include "tb_internal.h"

using namespace tb;

namespace {

bool grid_ok(int g) { return g == TB_GRID_TERNARY || g == TB_GRID_INT2 || g == TB_GRID_INT3; }
bool dtype_ok(int d) { return d == TB_F32 || d == TB_BF16; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool shape_ok(int64_t N, int64_t K) { return N >= 1 && K >= kGroup && K % kGroup == 0; }

tb_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? TB_OK : TB_ERR_CUDA; }

// packed rows are read 8 bytes (2-bit) or 4 bytes (3-bit) at a time at
// offsets that are multiples of those sizes; the base must be 16-byte
// aligned (also required for TMA-style bulk copies).
tb_status_t check_weights(const void* packed, int grid, const uint16_t* scales, int64_t N, int64_t K) {
    if (!packed || !scales) return TB_ERR_ARG;
    if (!grid_ok(grid)) return TB_ERR_ARG;
    if (!shape_ok(N, K)) return TB_ERR_SHAPE;
    if (!aligned(packed, 16) || !aligned(scales, 2)) return TB_ERR_ALIGN;
    return TB_OK;
}

tb_status_t check_out(const void* y, int ydt) {
    if (!y) return TB_ERR_ARG;
    if (!dtype_ok(ydt)) return TB_ERR_ARG;
    if (!aligned(y, ydt == TB_F32 ? 4 : 2)) return TB_ERR_ALIGN;
    return TB_OK;
}

Item make_item(const void* packed, int grid, const uint16_t* scales, const uint16_t* X, int64_t ldx, void* Y,
               int ydt, int64_t ldy, int M, int64_t N, int64_t K) {
    Item it;
    it.packed = static_cast<const uint8_t*>(packed);
    it.scales = scales;
    it.X = X;
    it.Y = Y;
    it.N = N;
    it.K = K;
    it.ldx = ldx;
    it.ldy = ldy;
    it.grid = grid;
    it.ydt = ydt;
    it.M = M;
    it.unit_begin = 0;
    return it;
}

// Orders items by per-tile cost (descending) so that the expensive tiles
// are dispatched first, assigns CTA ranges and launches.
tb_status_t launch_items(Item* items, int n, int nt, cudaStream_t st) {
    Launch L;
    std::memset(&L, 0, sizeof(L));
    int order[kMaxItems];
    for (int i = 0; i < n; ++i) order[i] = i;
    auto cost = [&](int i) { return row_bytes(items[i].grid, items[i].K); };
    std::stable_sort(order, order + n, [&](int a, int b) { return cost(a) > cost(b); });
    int64_t ctas = 0;
    for (int j = 0; j < n; ++j) {
        L.it[j] = items[order[j]];
        L.it[j].unit_begin = (int32_t)ctas;
        ctas += (L.it[j].N + 15) / 16;
    }
    L.n_items = n;
    if (ctas > 0x7FFFFFFF) return TB_ERR_SHAPE;
    return cuda_status(launch_linear(L, nt, (int)ctas, st));
}

}  // namespace

extern "C" {

int tb_version(void) { return 100; }

const char* tb_status_string(tb_status_t s) {
    switch (s) {
        case TB_OK: return "ok";
        case TB_ERR_ARG: return "invalid argument (null pointer, unknown enum value or bad count)";
        case TB_ERR_SHAPE: return "invalid shape (N >= 1, K a positive multiple of 128, 1 <= M <= 64, ld >= extent)";
        case TB_ERR_ALIGN: return "misaligned pointer or leading dimension";
        case TB_ERR_UNSUPPORTED: return "unsupported request";
        case TB_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

size_t tb_packed_bytes(tb_grid_t grid, int64_t N, int64_t K) {
    if (!grid_ok(grid) || !shape_ok(N, K)) return 0;
    return (size_t)(N * row_bytes(grid, K));
}

size_t tb_scale_bytes(int64_t N, int64_t K) {
    if (!shape_ok(N, K)) return 0;
    return (size_t)(N * (K / kGroup) * 2);
}

tb_status_t tb_scales_absmax(const void* W, tb_dtype_t w_dtype, int64_t N, int64_t K, tb_grid_t grid,
                             uint16_t* scales, tb_stream_t stream) {
    if (!W || !scales || !dtype_ok(w_dtype) || !grid_ok(grid)) return TB_ERR_ARG;
    if (!shape_ok(N, K)) return TB_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(scales, 2)) return TB_ERR_ALIGN;
    return cuda_status(launch_scales(W, w_dtype, N, K, grid, scales, static_cast<cudaStream_t>(stream)));
}

tb_status_t tb_pack(const void* W, tb_dtype_t w_dtype, int64_t N, int64_t K, tb_grid_t grid,
                    const uint16_t* scales, void* packed, int32_t* bad_count, tb_stream_t stream) {
    if (!W || !scales || !packed || !dtype_ok(w_dtype) || !grid_ok(grid)) return TB_ERR_ARG;
    if (!shape_ok(N, K)) return TB_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(scales, 2) || !aligned(packed, 16) || (bad_count && !aligned(bad_count, 4)))
        return TB_ERR_ALIGN;
    return cuda_status(
        launch_pack(W, w_dtype, N, K, grid, scales, packed, bad_count, static_cast<cudaStream_t>(stream)));
}

tb_status_t tb_unpack(const void* packed, tb_grid_t grid, int64_t N, int64_t K, int8_t* codes,
                      tb_stream_t stream) {
    if (!packed || !codes || !grid_ok(grid)) return TB_ERR_ARG;
    if (!shape_ok(N, K)) return TB_ERR_SHAPE;
    if (!aligned(packed, 16) || !aligned(codes, 16)) return TB_ERR_ALIGN;
    return cuda_status(launch_unpack(packed, grid, N, K, codes, static_cast<cudaStream_t>(stream)));
}

tb_status_t tb_gemv(const void* packed, tb_grid_t grid, const uint16_t* scales, const uint16_t* x, void* y,
                    tb_dtype_t y_dtype, int64_t N, int64_t K, tb_stream_t stream) {
    tb_status_t s = check_weights(packed, grid, scales, N, K);
    if (s != TB_OK) return s;
    if (!x) return TB_ERR_ARG;
    if ((s = check_out(y, y_dtype)) != TB_OK) return s;
    if (!aligned(x, 16)) return TB_ERR_ALIGN;
    Item it = make_item(packed, grid, scales, x, K, y, y_dtype, N, 1, N, K);
    return launch_items(&it, 1, 1, static_cast<cudaStream_t>(stream));
}

tb_status_t tb_gemm(const void* packed, tb_grid_t grid, const uint16_t* scales, const uint16_t* X, int64_t ldx,
                    void* Y, tb_dtype_t y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                    tb_stream_t stream) {
    tb_status_t s = check_weights(packed, grid, scales, N, K);
    if (s != TB_OK) return s;
    if (!X) return TB_ERR_ARG;
    if ((s = check_out(Y, y_dtype)) != TB_OK) return s;
    if (M < 1 || M > 64 || ldx < K || ldy < N) return TB_ERR_SHAPE;
    if (!aligned(X, 16) || ldx % 8 != 0) return TB_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // column blocks of up to 16 batch rows per launch
    const size_t ysz = y_dtype == TB_F32 ? 4 : 2;
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int mb = (int)std::min<int64_t>(16, M - m0);
        Item it = make_item(packed, grid, scales, X + m0 * ldx, ldx, static_cast<char*>(Y) + m0 * ldy * ysz, y_dtype,
                            ldy, mb, N, K);
        if ((s = launch_items(&it, 1, mb > 8 ? 2 : 1, st)) != TB_OK) return s;
    }
    return TB_OK;
}

tb_status_t tb_layer_gemv(const tb_linear_t* items, int n_items, tb_stream_t stream) {
    if (!items || n_items < 1 || n_items > TB_MAX_LAYER_ITEMS) return TB_ERR_ARG;
    Item its[kMaxItems];
    for (int i = 0; i < n_items; ++i) {
        const tb_linear_t& l = items[i];
        tb_status_t s = check_weights(l.packed, l.grid, l.scales, l.N, l.K);
        if (s != TB_OK) return s;
        if (!l.x) return TB_ERR_ARG;
        if ((s = check_out(l.y, l.y_dtype)) != TB_OK) return s;
        if (!aligned(l.x, 16)) return TB_ERR_ALIGN;
        its[i] = make_item(l.packed, l.grid, l.scales, l.x, l.K, l.y, l.y_dtype, l.N, 1, l.N, l.K);
    }
    return launch_items(its, n_items, 1, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
