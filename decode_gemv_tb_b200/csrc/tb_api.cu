// tb_api.cu -- the C interface declared in include/tb.h: argument checks,
// then one launch on the caller's stream.  No allocation, no
// synchronization, no host fallback: every computation runs in the kernels.
#include <algorithm>
#include <climits>
#include <cstring>
#include <mutex>

#include "../../include/tb.h"
#include "tb_device.cuh"
#include "tb_internal.h"
#include "tb_partition.h"

using namespace tb;

namespace {

bool grid_ok(int g) {
    return g == TB_GRID_TERNARY || g == TB_GRID_INT2 || g == TB_GRID_INT3 || g == TB_GRID_TERNARY_B3;
}
bool is_b3(int g) { return g == TB_GRID_TERNARY_B3; }
bool dtype_ok(int d) { return d == TB_F32 || d == TB_BF16; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool shape_ok(int64_t N, int64_t K) { return N >= 1 && K >= kGroup && K % kGroup == 0; }

tb_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? TB_OK : TB_ERR_CUDA; }

// Packed rows and scales are read by tensor and bulk copies: both bases must
// be 16-byte aligned.
tb_status_t check_weights(const void* packed, int grid, const uint16_t* scales, int64_t N, int64_t K) {
    if (!packed || !scales) return TB_ERR_ARG;
    if (!grid_ok(grid)) return TB_ERR_ARG;
    if (!shape_ok(N, K)) return TB_ERR_SHAPE;
    if (!aligned(packed, 16) || !aligned(scales, 16)) return TB_ERR_ALIGN;
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
    std::memset(&it, 0, sizeof(it));
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
    return it;
}

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// The small-batch kernel (2 <= M < 32) reads the activations as they are and
// needs no workspace; its size is reported as this nominal minimum.
constexpr size_t kNoWorkspace = 256;

// tb_gemm's kernels by batch size: 2 <= M < 32 mma.sync; 32 <= M <= 64 the
// tcgen05 kernel with the decoded weights in tensor memory; larger (prefill)
// batches the tcgen05 kernel with both operands in shared memory, every batch
// row in one launch
constexpr int64_t kTCMinM = 32;
constexpr int64_t kSSMinM = 65;
constexpr long long kSSWaitCycles = 4000000000LL;  // about 2 s at 2 GHz

// Batch-1 products of at most this many weights run the single-launch row
// kernel (no split-tile combine, no workspace), as do all products in the
// 5-trits-per-byte layout; larger ones the integer tensor-path kernel.
constexpr int64_t kRowWarpMaxWeights = (int64_t)1 << 24;

// Largest batch of one tb_gemm call (prefill batches included: the
// tensor-core kernel takes every batch row in one launch).
constexpr int64_t kMaxGemmM = (int64_t)1 << 16;

bool use_rowwarp(int grid, int64_t N, int64_t K) {
    return is_b3(grid) || (N <= kRowWarpMaxWeights / K && gemv_rowwarp_supported(grid, K));
}

int device_sms() {
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        sms[dev] = v;
    }
    return sms[dev];
}

// Orders items by per-tile cost (descending) so that the expensive tiles
// are dispatched first, chooses how many warps share a 32-row tile (the
// K split) and launches.
tb_status_t launch_items(Item* items, int n, int nt, cudaStream_t st) {
    Launch L;
    std::memset(&L, 0, sizeof(L));
    int order[kMaxItems];
    for (int i = 0; i < n; ++i) order[i] = i;
    auto cost = [&](int i) { return row_bytes(items[i].grid, items[i].K); };
    std::stable_sort(order, order + n, [&](int a, int b) { return cost(a) > cost(b); });

    // K split per item: about 16 groups (2048 weights) per warp, then more
    // splits everywhere while the launch has too few warps to fill the GPU
    // (each split needs at least one group).
    int S[kMaxItems];
    for (int i = 0; i < n; ++i) {
        const int64_t G = items[i].K / kGroup;
        int s = 1;
        while (s < 8 && G / (2 * s) >= 16) s *= 2;
        S[i] = s;
    }
    const int64_t want = (int64_t)device_sms() * 16;
    for (;;) {
        int64_t warps = 0;
        bool grow = false;
        for (int i = 0; i < n; ++i) warps += (items[i].N + 31) / 32 * S[i];
        if (warps >= want) break;
        for (int i = 0; i < n; ++i)
            if (S[i] < 8 && items[i].K / kGroup >= 2 * S[i]) {
                S[i] *= 2;
                grow = true;
            }
        if (!grow) break;
    }
    int64_t gpw = 0;  // most groups any warp handles
    for (int i = 0; i < n; ++i) gpw = std::max<int64_t>(gpw, (items[i].K / kGroup + S[i] - 1) / S[i]);
    L.scl_stride = (int32_t)((gpw + 3) / 4 * 4 + 2);  // >= gpw, = 2 mod 4
    if (linear_smem_bytes(nt, L.scl_stride) > 227 * 1024) return TB_ERR_UNSUPPORTED;

    int64_t ctas = 0;
    for (int j = 0; j < n; ++j) {
        Item it = items[order[j]];
        it.ksplit = S[order[j]];
        it.cta_begin = (int32_t)ctas;
        const int64_t tiles_per_cta = 8 / it.ksplit;
        ctas += ((it.N + 31) / 32 + tiles_per_cta - 1) / tiles_per_cta;
        L.it[j] = it;
    }
    L.n_items = n;
    if (ctas > 0x7FFFFFFF) return TB_ERR_SHAPE;
    return cuda_status(launch_linear(L, nt, (int)ctas, st));
}

// Batch-1 (M == 1) launch on the integer tensor path: one kernel, k_gemv8
// (tb_gemv8.cu).  The items' tiles of 256 rows are cut into chunks of 4
// (2-bit container) or 2 (3 bits) groups, numbered item by item, and split
// into equal-cost contiguous ranges, one per CTA.
//
// Workspace.  The call's control words -- per CTA 256 flagged partial-sum
// words, and per row of a gate/up pair one flagged word -- are zero before
// and after every call and sit at the FRONT of the workspace; its data --
// the activation records of every distinct x and code width (1088 bytes per
// group), written by the record kernel -- are overwritten before they are
// read and sit at the BACK.  A call needs 2 max(control, data) bytes,
// so calls of different shapes can share one workspace sized for the
// largest: no call's data ever reaches another call's control words.
constexpr int64_t kMaxG8Ctas = 512;      // bound of the CTA count (partial-sum words)
constexpr int64_t kG8Rows = kG8TileRows;
// Cost of one 128-group of one 256-row tile in the equal-cost split: a
// 3-bit group takes about twice the consumer work of a 2-bit one (measured
// on the 8B-like stack), so every chunk (four 2-bit or two 3-bit groups)
// costs the same
constexpr int32_t kG8Cost2 = 2, kG8Cost3 = 4;
// chunks per SM from which a call runs two CTAs per SM: below it (single
// q/k/v, o, down or gate/up calls of an 8B-like layer) one CTA per SM with
// a deeper ring finishes first; from it (a whole layer in one call) two
// independent rings per SM stream faster
constexpr int64_t kG8TwoPerSm = 8;
constexpr long long kWaitCycles = 4000000000LL;      // about 2 s
constexpr long long kTestWaitCycles = 20000000LL;    // about 10 ms (TB_FLAG_TEST_STALL)

int64_t g8_tiles(int64_t N) { return (N + kG8Rows - 1) / kG8Rows; }
int64_t g8_chunks(int grid, int64_t N, int64_t K) {
    const int64_t C = g8_chunk_groups(grid);
    return g8_tiles(N) * ((K / kGroup + C - 1) / C);
}
bool same_records(const Item& a, const Item& b) {
    return a.X == b.X && a.K == b.K && (a.grid == TB_GRID_INT3) == (b.grid == TB_GRID_INT3);
}

struct G8Space {
    size_t control = 0, data = 0;
    size_t need() const { return 2 * std::max(control, data); }
};

// control and data bytes of a batch-1 launch over items[0 .. n)
// (`pair`: items 0 and 1 are a gate/up pair)
G8Space g8_space(const Item* items, int n, bool pair) {
    G8Space sp;
    int64_t chunks = 0;
    for (int j = 0; j < n; ++j) {
        chunks += g8_chunks(items[j].grid, items[j].N, items[j].K);
        bool shared = false;
        for (int i = 0; i < j && !shared; ++i) shared = same_records(items[i], items[j]);
        if (!shared) sp.data += align256((size_t)(items[j].K / kGroup * kG8RecBytes));
    }
    const int64_t ctas = std::min(kMaxG8Ctas, std::max<int64_t>(chunks, 1));
    sp.control = align256((size_t)(ctas * kG8Rows * 8));
    if (pair) sp.control += align256((size_t)(items[0].N * 8));
    return sp;
}

// `pair_first` >= 0 marks items pair_first (gate) and pair_first + 1 (up)
// of equal shape whose outputs also give h = bf16(silu(gate) * up) (only
// pair_first == 0 with two items is used).
tb_status_t launch_g8_items(const Item* items, int n, void* ws, size_t ws_bytes, bool overlap, bool stall,
                            cudaStream_t st, int pair_first = -1, uint16_t* h = nullptr) {
    G8Launch L;
    std::memset(&L, 0, sizeof(L));
    const G8Space sp = g8_space(items, n, pair_first >= 0);
    if (!ws || ws_bytes < sp.need()) return TB_ERR_ARG;
    char* ctl = static_cast<char*>(ws);                                        // control words: the front
    char* dat = static_cast<char*>(ws) + (ws_bytes & ~size_t(255)) - sp.data;  // data: the back
    int64_t chunk = 0, cost = 0;
    for (int j = 0; j < n; ++j) {
        const Item& it = items[j];
        G8Item& s = L.it[j];
        const int64_t G = it.K / kGroup;
        s.x = it.X;
        s.scales = it.scales;
        s.Y = it.Y;
        s.N = it.N;
        s.G = (int32_t)G;
        s.T = (int32_t)g8_tiles(it.N);
        s.C = g8_chunk_groups(it.grid);
        s.cpt = (s.G + s.C - 1) / s.C;
        s.unit_cost = it.grid == TB_GRID_INT3 ? kG8Cost3 : kG8Cost2;
        s.grid = it.grid;
        s.ydt = it.ydt;
        s.chunk_base = chunk;
        s.cost_base = cost;
        s.stage_scales = G % 8 != 0 ? 1 : 0;  // rows of 2 G bytes: a tensor copy needs multiples of 16
        chunk += (int64_t)s.T * s.cpt;
        cost += (int64_t)s.T * s.G * s.unit_cost;
    }
    if (cost >= ((int64_t)1 << 31) || chunk >= ((int64_t)1 << 31)) return TB_ERR_UNSUPPORTED;  // 32-bit partition
    const int64_t ctas_max = std::min(kMaxG8Ctas, std::max<int64_t>(chunk, 1));
    L.pslots = reinterpret_cast<uint64_t*>(ctl);
    ctl += align256((size_t)(ctas_max * kG8Rows * 8));
    // activation records: items reading the same x with the same code width share one set
    int32_t n_build = 0;
    for (int j = 0; j < n; ++j) {
        int owner = -1;
        for (int i = 0; i < j && owner < 0; ++i)
            if (same_records(items[i], items[j])) owner = L.it[i].owner;
        if (owner < 0) {
            owner = L.n_own++;
            G8Owner& o = L.own[owner];
            o.x = items[j].X;
            o.rec = reinterpret_cast<uint8_t*>(dat);
            o.G = L.it[j].G;
            o.three = items[j].grid == TB_GRID_INT3 ? 1 : 0;
            o.build_base = n_build;
            n_build += o.G;
            dat += align256((size_t)(o.G * kG8RecBytes));
        }
        L.it[j].owner = owner;
    }
    L.n_build = n_build;
    L.pair_first = -1;
    if (pair_first >= 0) {
        L.pair_first = pair_first;
        L.pair_slots = reinterpret_cast<uint64_t*>(ctl);
        L.h = h;
    }
    for (int j = 0; j < n; ++j) {
        const G8Item& s = L.it[j];
        if (!encode_g8_wmap(&L.wmap[j], items[j].packed, items[j].grid, s.N, items[j].K)) return TB_ERR_CUDA;
        if (!s.stage_scales && !encode_g8_smap(&L.smap[j], s.scales, s.N, s.G)) return TB_ERR_CUDA;
    }
    // many chunks per SM: two CTAs per SM (two independent rings); else one
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return TB_ERR_CUDA;
    const bool two = chunk >= (int64_t)kG8TwoPerSm * sms;
    const int resident = gemv8_ctas(two);
    if (resident <= 0) return TB_ERR_CUDA;
    // every quota at least one chunk's cost: then every CTA
    // between a tile's first and last owner owns a chunk of it, which the
    // split-tile combine relies on
    int64_t max_chunk_cost = 0;
    for (int j = 0; j < n; ++j) max_chunk_cost = std::max<int64_t>(max_chunk_cost, (int64_t)L.it[j].C * L.it[j].unit_cost);
    int64_t nctas =
        std::max<int64_t>(1, std::min<int64_t>({(int64_t)resident, chunk, kMaxG8Ctas, cost / max_chunk_cost}));
    const int64_t Q = (cost + nctas - 1) / nctas;
    nctas = (cost + Q - 1) / Q;
    L.n_items = n;
    L.nctas = (int32_t)nctas;
    L.Ctot = (uint32_t)cost;
    L.Q = (uint32_t)Q;
    // each CTA's range and its first chunk's place
    for (int64_t c = 0; c < nctas; ++c) {
        G8Range& r = L.range[c];
        part_chunk_range(L.it, n, (uint32_t)c, L.Q, L.Ctot, &r.cb, &r.ce);
        r.item = 0;
        for (int i = 1; i < n; ++i)
            if (r.cb >= (uint32_t)L.it[i].chunk_base) r.item = i;
        const uint32_t local = r.cb - (uint32_t)L.it[r.item].chunk_base, cpt = (uint32_t)L.it[r.item].cpt;
        r.tile = (int32_t)(local / cpt);
        r.j = (int32_t)(local - (uint32_t)r.tile * cpt);
    }
    L.stall = stall ? 1 : 0;
    L.wait_cycles = stall ? kTestWaitCycles : kWaitCycles;
    return cuda_status(launch_gemv8(L, two, overlap, st));
}

// the items of a layer call that run on the integer tensor path
int g8_layer_items(const tb_linear_t* items, int n_items, Item* its) {
    int n = 0;
    for (int i = 0; i < n_items; ++i) {
        const tb_linear_t& l = items[i];
        if (is_b3(l.grid)) continue;  // launched on their own, without workspace
        its[n++] = make_item(l.packed, l.grid, l.scales, l.x, l.K, l.y, l.y_dtype, l.N, 1, l.N, l.K);
    }
    return n;
}

}  // namespace

extern "C" {

int tb_version(void) { return 100; }

unsigned int tb_wait_timeouts(void) {
    const unsigned int a = take_wait_timeouts(), b = take_g8_timeouts(), c = take_ss_timeouts();
    return (a == 0xFFFFFFFFu || b == 0xFFFFFFFFu || c == 0xFFFFFFFFu) ? 0xFFFFFFFFu : a + b + c;
}

tb_status_t tb_sync_status(tb_stream_t stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TB_ERR_CUDA;
    const unsigned int n = tb_wait_timeouts();
    if (n == 0xFFFFFFFFu) return TB_ERR_CUDA;
    return n ? TB_ERR_TIMEOUT : TB_OK;
}

const char* tb_status_string(tb_status_t s) {
    switch (s) {
        case TB_OK: return "ok";
        case TB_ERR_ARG: return "invalid argument (null pointer, unknown enum value or bad count)";
        case TB_ERR_SHAPE: return "invalid shape (N >= 1, K a positive multiple of 128, 1 <= M <= 65536, ld >= extent)";
        case TB_ERR_ALIGN: return "misaligned pointer or leading dimension";
        case TB_ERR_UNSUPPORTED: return "unsupported request";
        case TB_ERR_CUDA: return "CUDA error";
        case TB_ERR_TIMEOUT: return "a bounded device-side wait gave up: the calls since the last check have no result";
    }
    return "unknown status";
}

size_t tb_packed_bytes(tb_grid_t grid, int64_t N, int64_t K) {
    if (!grid_ok(grid) || !shape_ok(N, K)) return 0;
    return (size_t)(N * (is_b3(grid) ? b3_row_bytes(K) : row_bytes(grid, K)));
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
    // the 5-trits-per-byte layout stores the ternary grid: same scale rule
    return cuda_status(launch_scales(W, w_dtype, N, K, is_b3(grid) ? (int)TB_GRID_TERNARY : (int)grid, scales,
                                     static_cast<cudaStream_t>(stream)));
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

size_t tb_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || M > kMaxGemmM || !shape_ok(N, K)) return 0;
    if (M == 1) {  // the 3-bit chunking (more chunks) bounds both widths
        const Item it = make_item(nullptr, TB_GRID_INT3, nullptr, nullptr, K, nullptr, TB_F32, N, 1, N, K);
        return g8_space(&it, 1, false).need();
    }
    if (M >= kSSMinM) {
        const SSSpace sp = gemm_ss_space(M, N, K);
        return 2 * std::max(sp.control, sp.data);
    }
    if (M >= kTCMinM) return 2 * gemm_tc_workspace_bytes(M, N, K);  // data only
    return kNoWorkspace;
}

size_t tb_layer_workspace_bytes(const tb_linear_t* items, int n_items) {
    if (!items || n_items < 1 || n_items > TB_MAX_LAYER_ITEMS) return 0;
    for (int i = 0; i < n_items; ++i)
        if (!shape_ok(items[i].N, items[i].K) || !grid_ok(items[i].grid)) return 0;
    Item its[kMaxItems];
    const int n = g8_layer_items(items, n_items, its);
    return n ? g8_space(its, n, false).need() : kNoWorkspace;
}

tb_status_t tb_gemv(const void* packed, tb_grid_t grid, const uint16_t* scales, const uint16_t* x, void* y,
                    tb_dtype_t y_dtype, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                    tb_stream_t stream) {
    tb_status_t s = check_weights(packed, grid, scales, N, K);
    if (s != TB_OK) return s;
    if (!x) return TB_ERR_ARG;
    if ((s = check_out(y, y_dtype)) != TB_OK) return s;
    if (!workspace) return TB_ERR_ARG;
    if (!aligned(x, 16) || !aligned(workspace, 256)) return TB_ERR_ALIGN;
    if (workspace_bytes < tb_workspace_bytes(1, N, K)) return TB_ERR_ARG;  // the contract, whichever kernel runs
    if (use_rowwarp(grid, N, K)) {
        if (!gemv_rowwarp_supported(grid, K)) return TB_ERR_UNSUPPORTED;  // 5-trit layout only
        return cuda_status(
            launch_gemv_rowwarp(packed, grid, scales, x, y, y_dtype, N, K, static_cast<cudaStream_t>(stream)));
    }
    Item it = make_item(packed, grid, scales, x, K, y, y_dtype, N, 1, N, K);
    return launch_g8_items(&it, 1, workspace, workspace_bytes, false, false, static_cast<cudaStream_t>(stream));
}

tb_status_t tb_gemm(const void* packed, tb_grid_t grid, const uint16_t* scales, const uint16_t* X, int64_t ldx,
                    void* Y, tb_dtype_t y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                    void* workspace, size_t workspace_bytes, tb_stream_t stream) {
    tb_status_t s = check_weights(packed, grid, scales, N, K);
    if (s != TB_OK) return s;
    if (!X) return TB_ERR_ARG;
    if ((s = check_out(Y, y_dtype)) != TB_OK) return s;
    if (M < 1 || M > kMaxGemmM || ldx < K || ldy < N) return TB_ERR_SHAPE;
    if (!workspace) return TB_ERR_ARG;
    if (!aligned(X, 16) || ldx % 8 != 0 || !aligned(workspace, 256)) return TB_ERR_ALIGN;
    if (workspace_bytes < tb_workspace_bytes(M, N, K)) return TB_ERR_ARG;  // the contract, whichever kernel runs
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the row kernel: the 5-trit layout (one launch per batch row) and small batch-1 products
    if (is_b3(grid) || (M == 1 && use_rowwarp(grid, N, K))) {
        if (!gemv_rowwarp_supported(grid, K)) return TB_ERR_UNSUPPORTED;
        const size_t ysz = y_dtype == TB_F32 ? 4 : 2;
        for (int64_t m = 0; m < M; ++m) {
            const cudaError_t e = launch_gemv_rowwarp(packed, grid, scales, X + m * ldx,
                                                      static_cast<char*>(Y) + m * ldy * ysz, y_dtype, N, K, st);
            if (e != cudaSuccess) return TB_ERR_CUDA;
        }
        return TB_OK;
    }
    if (M == 1) {
        Item it = make_item(packed, grid, scales, X, ldx, Y, y_dtype, N, 1, N, K);
        return launch_g8_items(&it, 1, workspace, workspace_bytes, false, false, st);
    }
    if (M >= kSSMinM) {
        // tiles, batch blocks and groups index 32-bit cursors; chunks are counted in 64 bits
        if ((N + 127) / 128 * ((M + 63) / 64) >= ((int64_t)1 << 31)) return TB_ERR_SHAPE;
        return cuda_status(launch_gemm_ss(packed, grid, scales, X, ldx, Y, y_dtype, ldy, M, N, K, workspace,
                                          workspace_bytes, kSSWaitCycles, st));
    }
    if (M >= kTCMinM) {
        if (K / kGroup * 64 > INT_MAX || (N + 127) / 128 > INT_MAX / 16 ||
            (N + 127) / 128 * (K / kGroup) >= ((int64_t)1 << 32))
            return TB_ERR_SHAPE;
        // all of its workspace is data (it clears its own counters): the back
        char* back = static_cast<char*>(workspace) + (workspace_bytes & ~size_t(255)) - gemm_tc_workspace_bytes(M, N, K);
        return cuda_status(launch_gemm_tc(packed, grid, scales, X, ldx, Y, y_dtype, ldy, (int)M, N, K, back, st));
    }
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

tb_status_t tb_layer_gemv(const tb_linear_t* items, int n_items, unsigned flags, void* workspace,
                          size_t workspace_bytes, tb_stream_t stream) {
    if (!items || n_items < 1 || n_items > TB_MAX_LAYER_ITEMS) return TB_ERR_ARG;
    if ((flags & ~(unsigned)(TB_FLAG_OVERLAP_PREVIOUS | TB_FLAG_TEST_STALL)) != 0 || !workspace) return TB_ERR_ARG;
    if (!aligned(workspace, 256)) return TB_ERR_ALIGN;
    Item its[kMaxItems];
    int n_main = 0;
    for (int i = 0; i < n_items; ++i) {
        const tb_linear_t& l = items[i];
        tb_status_t s = check_weights(l.packed, l.grid, l.scales, l.N, l.K);
        if (s != TB_OK) return s;
        if (!l.x) return TB_ERR_ARG;
        if ((s = check_out(l.y, l.y_dtype)) != TB_OK) return s;
        if (!aligned(l.x, 16)) return TB_ERR_ALIGN;
        if (is_b3(l.grid)) {
            if (!gemv_rowwarp_supported(l.grid, l.K)) return TB_ERR_UNSUPPORTED;
            continue;
        }
        its[n_main++] = make_item(l.packed, l.grid, l.scales, l.x, l.K, l.y, l.y_dtype, l.N, 1, l.N, l.K);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_main > 0) {
        const tb_status_t s = launch_g8_items(its, n_main, workspace, workspace_bytes,
                                              (flags & TB_FLAG_OVERLAP_PREVIOUS) != 0,
                                              (flags & TB_FLAG_TEST_STALL) != 0, st);
        if (s != TB_OK) return s;
    }
    // items in the 5-trits-per-byte layout: one launch each, after the grouped launch
    for (int i = 0; i < n_items; ++i) {
        const tb_linear_t& l = items[i];
        if (!is_b3(l.grid)) continue;
        if (launch_gemv_rowwarp(l.packed, l.grid, l.scales, l.x, l.y, l.y_dtype, l.N, l.K, st) != cudaSuccess)
            return TB_ERR_CUDA;
    }
    return TB_OK;
}

size_t tb_gate_up_workspace_bytes(const tb_linear_t* gate, const tb_linear_t* up) {
    if (!gate || !up || gate->N != up->N || gate->K != up->K) return 0;
    if (!shape_ok(gate->N, gate->K) || !grid_ok(gate->grid) || !grid_ok(up->grid)) return 0;
    if (is_b3(gate->grid) || is_b3(up->grid)) return 0;
    const tb_linear_t two[2] = {*gate, *up};
    Item its[2];
    g8_layer_items(two, 2, its);
    return g8_space(its, 2, true).need();
}

tb_status_t tb_gate_up_silu(const tb_linear_t* gate, const tb_linear_t* up, uint16_t* h, unsigned flags,
                            void* workspace, size_t workspace_bytes, tb_stream_t stream) {
    if (!gate || !up || !h || !workspace) return TB_ERR_ARG;
    if ((flags & ~(unsigned)TB_FLAG_OVERLAP_PREVIOUS) != 0) return TB_ERR_ARG;
    if (gate->N != up->N || gate->K != up->K) return TB_ERR_SHAPE;
    if (!aligned(workspace, 256) || !aligned(h, 2)) return TB_ERR_ALIGN;
    Item its[2];
    const tb_linear_t* l2[2] = {gate, up};
    for (int i = 0; i < 2; ++i) {
        const tb_linear_t& l = *l2[i];
        tb_status_t s = check_weights(l.packed, l.grid, l.scales, l.N, l.K);
        if (s != TB_OK) return s;
        if (!l.x) return TB_ERR_ARG;
        if ((s = check_out(l.y, l.y_dtype)) != TB_OK) return s;
        if (!aligned(l.x, 16)) return TB_ERR_ALIGN;
        if (is_b3(l.grid)) return TB_ERR_UNSUPPORTED;  // the 5-trit layout runs its own kernel
        its[i] = make_item(l.packed, l.grid, l.scales, l.x, l.K, l.y, l.y_dtype, l.N, 1, l.N, l.K);
    }
    if (workspace_bytes < tb_gate_up_workspace_bytes(gate, up)) return TB_ERR_ARG;
    return launch_g8_items(its, 2, workspace, workspace_bytes, (flags & TB_FLAG_OVERLAP_PREVIOUS) != 0, false,
                           static_cast<cudaStream_t>(stream), 0, h);
}

}  // extern "C"

// ---- tb_gemv_noalloc: tb_gemv over a fixed, statically allocated scratch ----
//
// Same kernels and results as tb_gemv; the workspace is this file-scope
// device array instead of caller memory, so the call allocates nothing.
// The only state that must start at zero (the per-tile arrival counters)
// starts zeroed (static storage) and every call leaves it zero again, so
// the array needs no clearing; every call rewrites what else it reads.  All
// calls on a device
// share the one array: calls that may run at the same time (different
// streams, or different host threads without stream ordering) race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TB_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Address of the array on the current device, looked up once per device
// (with that device current) and cached; nullptr if the lookup fails.
void* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

tb_status_t tb_gemv_noalloc(const void* packed, tb_grid_t grid, const uint16_t* scales, const uint16_t* x, void* y,
                            tb_dtype_t y_dtype, int64_t N, int64_t K, tb_stream_t stream) {
    tb_status_t s = check_weights(packed, grid, scales, N, K);
    if (s != TB_OK) return s;
    if (!x) return TB_ERR_ARG;
    if ((s = check_out(y, y_dtype)) != TB_OK) return s;
    if (!aligned(x, 16)) return TB_ERR_ALIGN;
    if (use_rowwarp(grid, N, K)) {  // needs no scratch
        if (!gemv_rowwarp_supported(grid, K)) return TB_ERR_UNSUPPORTED;
        return cuda_status(
            launch_gemv_rowwarp(packed, grid, scales, x, y, y_dtype, N, K, static_cast<cudaStream_t>(stream)));
    }
    // the size rule is checked before any CUDA call
    if (tb_workspace_bytes(1, N, K) > (size_t)TB_NOALLOC_SCRATCH_BYTES) return TB_ERR_UNSUPPORTED;
    void* scratch = noalloc_scratch();
    if (!scratch) return TB_ERR_CUDA;
    Item it = make_item(packed, grid, scales, x, K, y, y_dtype, N, 1, N, K);
    return launch_g8_items(&it, 1, scratch, TB_NOALLOC_SCRATCH_BYTES, false, false, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
