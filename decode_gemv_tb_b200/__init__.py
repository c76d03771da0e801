"""ThinkBit scalar low-bit weights on B200: pack, GEMV, small-batch GEMM."""
