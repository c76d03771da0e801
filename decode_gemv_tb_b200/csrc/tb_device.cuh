// tb_device.cuh -- device-side pieces shared by the sm_100a kernels:
// grid constants, the packed layout, bf16 helpers and launch descriptors.
//
// Format (declared in include/tb.h): w = c * s, one bf16 scale per 128
// weights along K, per-layer grid ternary / 2-bit / 3-bit (ThinkBit page
// "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로 검증한다",
// onedev.kr/papers/1416, section 어떻게 동작하나).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tb {

constexpr int kGroup = 128;      // weights per scale
constexpr int kMaxItems = 16;    // grouped-launch capacity

enum Grid : int { kTernary = 0, kInt2 = 1, kInt3 = 2 };
enum DType : int { kF32 = 0, kBF16 = 1 };

__host__ __device__ inline int grid_qmin(int g) { return g == kTernary ? -1 : (g == kInt2 ? -2 : -4); }
__host__ __device__ inline int grid_qmax(int g) { return g == kInt3 ? 3 : 1; }
__host__ __device__ inline int grid_offset(int g) { return g == kInt3 ? 4 : 2; }
// bytes of one packed row of K weights
__host__ __device__ inline int64_t row_bytes(int g, int64_t K) { return g == kInt3 ? 3 * K / 8 : K / 4; }

// ---- one linear layer inside a launch ------------------------------------
struct Item {
    const uint8_t* packed;
    const uint16_t* scales;
    const uint16_t* X;   // [M][ldx] bf16 activations
    void* Y;             // [M][ldy] outputs
    uint16_t* xs;        // workspace: [M][K] prepared activations (see tb_linear.cu)
    float2* cf;          // workspace: [K/128][M] per-group (offset * sum x, 2^S)
    int64_t N, K, ldx, ldy;
    int32_t grid, ydt, M;
    int32_t cta_begin;   // first CTA of this item in the main launch
    int32_t prep_begin;  // first warp of this item in the preparation launch
    int32_t ksplit;      // warps sharing one 32-row tile (1, 2, 4 or 8)
    uint8_t* rec;        // batch-1 TMA path: per-group records (see kRecBytes) instead of xs / cf
};

// Prepared activations of one 128-group for the batch-1 TMA kernel, one
// contiguous record: the 128 scaled activations in MMA order, first half at
// bytes 0..127, (offset * sum x, 2^S) at 128..135, zero at 136..143, second
// half at 144..271 (the 16-byte gap keeps the fragment loads free of bank
// conflicts).  A chunk of consecutive groups is one bulk copy.
constexpr int kRecBytes = 272;

struct Launch {
    Item it[kMaxItems];
    int32_t n_items;
    int32_t scl_stride;  // scales staged per row per warp (>= groups per warp)
    int32_t* zero;       // int32 words the preparation kernel clears (stream-K tile counters)
    int32_t n_zero;
};

// ---- stream-K batch-1 launch (see tb_linear.cu) ----------------------------
// Two partitions side by side: the 3-bit items (it[0 .. n3)) on warps
// [0, W3), the 2-bit items (it[n3 .. n_items)) on warps [W3, W); tile-group
// and cost positions of the 2-bit items start again at 0.
struct SKPart {
    int32_t first, count;  // items
    int32_t W0, W;         // first warp, warps
    uint32_t C, Q;         // total cost, cost quota per warp (tb_partition.h)
};

// Batch-1 TMA kernel (tb_linear.cu): items read in chunks of C groups x 32
// rows through one 2-D tensor map each (see tb_partition.h, ChunkItem).
struct TMItem {
    const uint16_t* scales;
    const uint8_t* rec;  // G records of kRecBytes
    void* Y;
    int64_t N;
    int64_t chunk_base, cost_base;  // ChunkItem fields
    int32_t T, G, C, cpt, unit_cost;
    int32_t grid, ydt, tile_base;
};

struct TMLaunch {
    CUtensorMap maps[kMaxItems];  // packed weights of item i: bytes x rows, box (C group bytes) x 32
    TMItem it[kMaxItems];
    int32_t n_items, W;
    SKPart part[2];  // 3-bit items first, then the 2-bit container
    int32_t* counters;
    float* partials;
};

// ---- cache-controlled loads ----------------------------------------------
// Streamed weights: read once, keep them out of L1.
__device__ __forceinline__ uint2 ld_stream_u2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint16_t ld_stream_u16(const void* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
// Activations: small, re-read by every CTA: cache in L1.
__device__ __forceinline__ uint4 ld_act_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ float2 ld_act_f2(const void* p) {
    float2 v;
    asm volatile("ld.global.nc.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}

// Programmatic dependent launch (sm_90+): wait for the grids this one
// depends on / let the dependent grid start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// bf16x2 a*b+c, one rounding (exact whenever the true result is a bf16)
__device__ __forceinline__ uint32_t hfma2_bf16(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// (a & b) | c  in one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// bitwise select: (a & ~m) | (b & m); LOP3 table 0xCA is "x ? y : z"
__device__ __forceinline__ uint32_t bit_mux(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xCA;" : "=r"(d) : "r"(m), "r"(b), "r"(a));
    return d;
}

}  // namespace tb
