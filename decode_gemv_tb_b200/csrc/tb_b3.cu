// tb_b3.cu -- batch-1 GEMV over the optional 5-trits-per-byte ternary
// layout (include/tb.h): y[n] = sum_j s[n][j] * sum_{k in group j} c[n][k] x[k].
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416), section 어떻게 동작하나: w = c * s, the
// ternary grid {-1,0,1}, one bf16 scale per 128 weights.  The base-3 byte
// layout is the library's.
//
// One warp per output row, one lane per 128-group (Z lanes per row, Z the
// smallest power of two >= the group count, at most 32; a warp serves
// 32 / Z rows at once when a row has fewer than 32 groups).  A lane reads
// its group's 26 bytes as 13 half-words (the warp's loads of one row are
// contiguous), splits each byte into base-3 digits with multiply-high
// divisions, turns digit d into the code c = d - 1 as an exact float and
// accumulates c * x in fp32 against the activations, which every CTA
// stages in shared memory as fp32 with 129 floats per group (lanes on
// consecutive groups then read consecutive banks).  The group sum is
// scaled once; lanes of a row are combined by a fixed butterfly, so results
// are deterministic.
#include <algorithm>

#include "tb_device.cuh"
#include "tb_internal.h"

namespace tb {
namespace {

constexpr int kB3Threads = 256;
constexpr int kB3Warps = kB3Threads / 32;
constexpr int kB3Stride = 129;  // floats per staged activation group

// largest dynamic shared memory a CTA may use on sm_100a
constexpr size_t kB3MaxSmem = 227 * 1024;

size_t b3_smem_bytes(int64_t K) { return (size_t)(K / kGroup) * kB3Stride * sizeof(float); }

// d - 1 as a float, exact for small d: 2^23 + d is exact, minus (2^23 + 1)
__device__ __forceinline__ float b3_code(uint32_t d) { return __uint_as_float(0x4B000000u | d) - 8388609.0f; }

__global__ void __launch_bounds__(kB3Threads) k_gemv_b3(const uint8_t* __restrict__ P,
                                                        const uint16_t* __restrict__ S,
                                                        const uint16_t* __restrict__ x, void* __restrict__ Y,
                                                        int ydt, int64_t N, int64_t K, int zlog) {
    extern __shared__ float xs[];  // [G][kB3Stride]
    const int G = (int)(K / kGroup);
    const int64_t RB = b3_row_bytes(K);
    for (int64_t i = threadIdx.x; i < K; i += kB3Threads)
        xs[(i >> 7) * kB3Stride + (i & 127)] = bf16_bits_to_float(__ldg(x + i));
    __syncthreads();

    const int lane = threadIdx.x & 31, Z = 1 << zlog, R = 32 >> zlog;
    const int r = lane >> zlog, jl = lane & (Z - 1);
    const int64_t wg = (int64_t)blockIdx.x * kB3Warps + (threadIdx.x >> 5);
    const int64_t stride = (int64_t)gridDim.x * kB3Warps * R;
    for (int64_t n0 = wg * R; n0 < N; n0 += stride) {  // warp-uniform
        const int64_t n = n0 + r;
        float acc = 0.f;
        if (n < N) {
            const uint8_t* row = P + n * RB;
            const uint16_t* srow = S + n * G;
            for (int j = jl; j < G; j += Z) {
                // 26 j is even and rows start on 16 bytes: half-word loads are aligned
                const uint16_t* gp = reinterpret_cast<const uint16_t*>(row + kB3GroupBytes * j);
                const float* xg = xs + j * kB3Stride;
                float part = 0.f;
#pragma unroll
                for (int h = 0; h < 13; ++h) {
                    const uint32_t w = __ldg(gp + h);  // group bytes 2h (low) and 2h + 1 (high)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int b = 2 * h + e;
                        uint32_t v = e ? (w >> 8) : (w & 0xFFu);
#pragma unroll
                        for (int i = 0; i < 5; ++i) {
                            if (i < 3 || b < 25) {  // byte 25 holds three codes
                                const uint32_t q = __umulhi(v, 0x55555556u);  // floor(v / 3), v < 2^31
                                part = fmaf(b3_code(v - 3u * q), xg[5 * b + i], part);
                                v = q;
                            }
                        }
                    }
                }
                acc = fmaf(bf16_bits_to_float(__ldg(srow + j)), part, acc);
            }
        }
        for (int o = Z >> 1; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (jl == 0 && n < N) {
            if (ydt == kF32) static_cast<float*>(Y)[n] = acc;
            else static_cast<__nv_bfloat16*>(Y)[n] = __float2bfloat16_rn(acc);
        }
    }
}

// CTAs of k_gemv_b3 resident per SM at this K (0 on error)
int b3_ctas_per_sm(size_t smem) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv_b3, kB3Threads, smem) != cudaSuccess)
        return 0;
    return per_sm;
}

}  // namespace

bool gemv_b3_supported(int64_t K) { return b3_smem_bytes(K) <= kB3MaxSmem; }

cudaError_t launch_gemv_b3(const void* packed, const uint16_t* scales, const uint16_t* x, void* y, int ydt,
                           int64_t N, int64_t K, cudaStream_t st) {
    static bool ready[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!ready[dev]) {
        e = cudaFuncSetAttribute((const void*)k_gemv_b3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kB3MaxSmem);
        if (e != cudaSuccess) return e;
        ready[dev] = true;
    }
    const size_t smem = b3_smem_bytes(K);
    const int64_t G = K / kGroup;
    int zlog = 0;
    while ((1 << zlog) < G && zlog < 5) ++zlog;
    const int64_t rows_per_warp_step = 32 >> zlog;
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int per_sm = b3_ctas_per_sm(smem);
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t want = (N + kB3Warps * rows_per_warp_step - 1) / (kB3Warps * rows_per_warp_step);
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * per_sm));
    k_gemv_b3<<<(unsigned)ctas, kB3Threads, smem, st>>>(static_cast<const uint8_t*>(packed), scales, x, y, ydt, N, K,
                                                          zlog);
    return cudaGetLastError();
}

}  // namespace tb
