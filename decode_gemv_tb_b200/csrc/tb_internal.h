// tb_internal.h -- launchers behind the C interface (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tb {

struct Launch;

// The ternary grid in the optional 5-trits-per-byte layout (include/tb.h):
// 26 bytes per 128-group, rows padded to 16 bytes.
constexpr int kTernaryB3 = 3;
constexpr int64_t kB3GroupBytes = 26;
__host__ __device__ inline int64_t b3_row_bytes(int64_t K) { return 16 * ((kB3GroupBytes * (K / 128) + 15) / 16); }

cudaError_t launch_scales(const void* W, int w_dtype, int64_t N, int64_t K, int grid, uint16_t* scales,
                          cudaStream_t st);
cudaError_t launch_pack(const void* W, int w_dtype, int64_t N, int64_t K, int grid, const uint16_t* scales,
                        void* packed, int32_t* bad_count, cudaStream_t st);
cudaError_t launch_unpack(const void* packed, int grid, int64_t N, int64_t K, int8_t* codes, cudaStream_t st);

// Small-batch launch (2 <= M <= 16 batch rows per item): one kernel, no
// workspace.  `nt` is the number of 8-wide column tiles (1 or 2), `ctas`
// the grid.
cudaError_t launch_linear(const Launch& L, int nt, int ctas, cudaStream_t st);
// dynamic shared memory of the main kernel
size_t linear_smem_bytes(int nt, int scl_stride);

struct G8Launch;
// Batch-1 GEMV on the integer tensor path (tb_gemv8.cu): one kernel,
// k_gemv8.  `overlap` launches it as a programmatic dependent of the
// previous work (it streams weights before that work has finished).
// `two`: the layout of two CTAs per SM (calls of many chunks per SM), else
// one CTA per SM.
cudaError_t launch_gemv8(const G8Launch& L, bool two, bool overlap, cudaStream_t st);
// weights of one matrix (box: one chunk x 256 rows) / its scales [N][G] (G % 8 == 0)
bool encode_g8_wmap(CUtensorMap* map, const void* packed, int grid, int64_t N, int64_t K);
bool encode_g8_smap(CUtensorMap* map, const uint16_t* scales, int64_t N, int64_t Gp);
// groups per chunk (4 for the 2-bit container, 2 for 3 bits)
int g8_chunk_groups(int grid);
// CTAs of k_gemv8 resident at once on the current device in the layout
// `two` (0 on error)
int gemv8_ctas(bool two);
// bounded waits of k_gemv8 that gave up since the last call (clears)
unsigned int take_g8_timeouts();

// Batch-1 GEMV in one launch, one warp per output row, no workspace: the
// 5-trits-per-byte layout, and small problems in the other layouts.  The
// activations are staged in shared memory, which bounds K
// (gemv_rowwarp_supported).
bool gemv_rowwarp_supported(int grid, int64_t K);
cudaError_t launch_gemv_rowwarp(const void* packed, int grid, const uint16_t* scales, const uint16_t* x, void* y,
                                int ydt, int64_t N, int64_t K, cudaStream_t st);

// Small-batch GEMM on the tcgen05 tensor cores (2 <= M <= 64): preparation
// kernel + main kernel.  Workspace: gemm_tc_workspace_bytes(M, N, K) bytes,
// 256-byte aligned (device independent).
size_t gemm_tc_workspace_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_tc(const void* packed, int grid, const uint16_t* scales, const uint16_t* X, int64_t ldx,
                           void* Y, int ydt, int64_t ldy, int M, int64_t N, int64_t K, void* ws, cudaStream_t st);
// Prefill GEMM with both MMA operands in shared memory (tb_gemm_ss.cu): one
// kernel, M > 64 batch rows in blocks of 128.  Its workspace (ws_bytes,
// 256-byte aligned) holds space.control bytes of flags at the front (zero
// before the call and left zero by it) and space.data bytes of partial sums
// at the back.
struct SSSpace {
    size_t control, data;
};
int gemm_ss_np(int64_t M);
SSSpace gemm_ss_space(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_ss(const void* packed, int grid, const uint16_t* scales, const uint16_t* X, int64_t ldx,
                           void* Y, int ydt, int64_t ldy, int64_t M, int64_t N, int64_t K, void* ws,
                           size_t ws_bytes, long long wait_cycles, cudaStream_t st);
unsigned int take_ss_timeouts();
// bounded device waits that gave up since the last call (clears the count;
// synchronous); 0xFFFFFFFF if the count cannot be read
unsigned int take_wait_timeouts();

}  // namespace tb
