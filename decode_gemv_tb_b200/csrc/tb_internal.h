// tb_internal.h -- launchers behind the C interface (host side).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tb {

struct Launch;

cudaError_t launch_scales(const void* W, int w_dtype, int64_t N, int64_t K, int grid, uint16_t* scales,
                          cudaStream_t st);
cudaError_t launch_pack(const void* W, int w_dtype, int64_t N, int64_t K, int grid, const uint16_t* scales,
                        void* packed, int32_t* bad_count, cudaStream_t st);
cudaError_t launch_unpack(const void* packed, int grid, int64_t N, int64_t K, int8_t* codes, cudaStream_t st);

// Grouped linear launch (GEMV when every item has M == 1).  `nt` is the
// number of 8-wide column tiles (1 or 2), `ctas` the total CTA count.
cudaError_t launch_linear(const Launch& L, int nt, int ctas, cudaStream_t st);

}  // namespace tb
