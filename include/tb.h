/*
 * tb.h -- C interface of libtb_b200: ThinkBit scalar low-bit weights on
 * NVIDIA B200 (sm_100a).  Quantize/pack, unpack, batch-1 GEMV, GEMM
 * (small batches up to 64 rows, prefill batches up to 65536 rows in one
 * launch), a grouped launcher for a decoder layer's projections and the
 * gate/up pair with its SiLU-gated output.
 *
 * What the method fixes -- ThinkBit page, "ThinkBit은 2비트 양자화에서 추론
 * 능력 보존을 추론 평가로 검증한다" (onedev.kr/papers/1416):
 *   section 어떻게 동작하나 ("how it works"): the storage format is strictly
 *     scalar.  A weight is w = c * s, an integer codeword c times a bf16
 *     scale s; one scale serves 128 consecutive weights; the codeword grid
 *     is chosen per layer among ternary {-1,0,1}, 2-bit {-2,-1,0,1} and
 *     3-bit {-4,...,3}; dequantization is one multiplication (no codebook,
 *     no rotation, no zero point).
 *   section 무엇과 다른가 ("what is different"): the per-layer grids are
 *     mixed within one model (75.3% ternary, 6.0% 2-bit, 18.7% 3-bit on
 *     Qwen3-1.7B), codewords come out of a rounding step.
 *   section 무엇인가 ("what it is"): decoding a token reads every weight,
 *     so decode speed is bound by memory bandwidth.
 *   section 전제와 한계 ("assumptions and limits"): released checkpoints
 *     keep the 2- and 3-bit codewords in 4-bit containers because no kernel
 *     reads them directly; this library is such a reader.
 *
 * ------------------------------------------------------------------------
 * FORMAT (this library's definition; the pages give no bit layout)
 *
 *   W is [N][K] row-major: N outputs, K inputs (y = W x), K % 128 == 0.
 *   Scales: bf16, [N][K/128]; scale (n, j) covers k in [128 j, 128 j + 128).
 *   Stored code u = c + offset (offset 2 for the 2-bit container, 4 for
 *   3 bits), so every stored code is an unsigned bit pattern.
 *
 *   TB_GRID_TERNARY, TB_GRID_INT2 -- 2 bits per code, 16 codes per uint32:
 *     row n: K/16 little-endian uint32 words (K/4 bytes); word i holds codes
 *     k = 16i .. 16i+15; code 16i+2m is at bits [2m, 2m+1] and code
 *     16i+2m+1 at bits [16+2m, 17+2m], m = 0..7 (even codes in the low
 *     half-word, odd codes in the high one).  Ternary codes use u in
 *     {1,2,3}; a stored 0 in a ternary row decodes as -2.
 *   TB_GRID_INT3 -- 3 bits per code, 32 codes per three uint32 bit-planes:
 *     row n: K/32 blocks of three uint32 (3K/8 bytes); block j holds codes
 *     k = 32j .. 32j+31 in planes p = 0, 1, 2 (consecutive words); bit m of
 *     plane p is bit p of u for code 32j+2m, bit 16+m of plane p is bit p of
 *     u for code 32j+2m+1, m = 0..15.
 *   TB_GRID_TERNARY_B3 -- the ternary grid, 5 codes per byte: digit
 *     d = c + 1 in {0,1,2}; row n is 16 * ceil(26 K/128 / 16) bytes; group j
 *     takes the 26 bytes from byte 26 j: group byte b < 25 is
 *     sum_{i<5} d(128 j + 5 b + i) 3^i, byte 25 is sum_{i<3} d(128 j + 125 +
 *     i) 3^i; the row's remaining bytes are zero.  Any byte value v decodes
 *     digit i as floor(v / 3^i) mod 3 (243..255 are never written).  No byte
 *     holds codes of two groups.
 *   Bytes per weight including the scales: 2.125 / 8 (ternary, 2-bit),
 *   3.125 / 8 (3-bit) and 1.75 / 8 (5 trits per byte, when K/128 is a
 *   multiple of 8; the row padding adds at most 15 bytes otherwise).
 *
 * QUANTIZATION RULES (readings where the pages are silent)
 *   scale  s = bf16_rne(absmax / d), d = |qmin| = 1, 2, 4 for ternary,
 *          2-bit, 3-bit; absmax over the finite weights of the group; a
 *          scale that rounds to 0 becomes 1.0, one that rounds to infinity
 *          becomes the largest finite bf16.
 *   code   c = clamp(round_half_even(w / s), qmin, qmax), decided exactly
 *          (the exact quotient, not a rounded one, is rounded).
 *   NaN w gives code 0, +-Inf gives qmax / qmin, a scale that is not a
 *   positive finite number gives code 0; every such weight is counted.
 *
 * PRODUCTS
 *   y[n] = sum_k x[k] * c[n][k] * s[n][k/128], every product x * c formed
 *   exactly from the signed codeword (a zero codeword contributes nothing),
 *   summed per 128-group, scaled once per group, accumulated in fp32; fp32
 *   output, or bf16 rounded half to even from the fp32 result.  Error
 *   bound: |y - y_exact| <= 1e-5 * sum_k |x[k] c[n][k] s[n][k/128]| (plus
 *   4e-3 |y| for bf16 outputs).  Results are bitwise deterministic from run
 *   to run (no atomics in any reduction).
 *   ACTIVATION RANGE: x must be finite with |x| < 2^120.  The batch-1
 *   products (M = 1) form each group's sum in integers on a fixed-point
 *   grid 2^55 below the group's largest |x|: an activation more than 2^42
 *   below its group's largest one loses its low bits, by less than 2^-48
 *   of that largest |x| each (the bound above holds whenever such tiny
 *   activations are not the group's only ones meeting nonzero codes).
 *
 * ------------------------------------------------------------------------
 * CONVENTIONS
 *   - Every pointer argument is DEVICE memory on the current CUDA device
 *     unless the argument says otherwise.  The caller owns all buffers,
 *     including the products' scratch workspace; the library allocates
 *     nothing and keeps no allocation between calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All calls
 *     are asynchronous on `stream`; none synchronizes.
 *   - Alignment: packed, W, x / X rows: 16 bytes; scales: 16 bytes for the
 *     products (they are read by tensor copies), 2 bytes for
 *     tb_scales_absmax and tb_pack; y / Y: 4 bytes (fp32) or 2 bytes (bf16).
 *   - Argument errors are reported before anything is launched; a launch
 *     failure is reported as TB_ERR_CUDA (cudaGetLastError is consumed).
 *   - Outputs must not overlap inputs.
 */
#ifndef TB_B200_H
#define TB_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TB_API __attribute__((visibility("default")))
#else
#define TB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef void *tb_stream_t; /* a cudaStream_t */

typedef enum {
    TB_GRID_TERNARY = 0, /* {-1, 0, 1}, 2-bit container, offset 2 */
    TB_GRID_INT2 = 1,    /* {-2, -1, 0, 1}, offset 2 */
    TB_GRID_INT3 = 2,    /* {-4, ..., 3}, three bit-planes, offset 4 */
    TB_GRID_TERNARY_B3 = 3 /* {-1, 0, 1}, 5 trits per byte (optional denser ternary layout) */
} tb_grid_t;

typedef enum { TB_F32 = 0, TB_BF16 = 1 } tb_dtype_t;

typedef enum {
    TB_OK = 0,
    TB_ERR_ARG = 1,         /* null pointer, unknown enum value, bad count */
    TB_ERR_SHAPE = 2,       /* N < 1, K < 128, K % 128 != 0, M outside 1..65536, ld too small */
    TB_ERR_ALIGN = 3,       /* a pointer or leading dimension breaks the alignment rules */
    TB_ERR_UNSUPPORTED = 4, /* valid request this build does not implement */
    TB_ERR_CUDA = 5,        /* a CUDA call or launch failed */
    TB_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (tb_sync_status only) */
} tb_status_t;

/* Library version as 10000*major + 100*minor + patch. */
TB_API int tb_version(void);

/* Static text for a status code (never NULL). */
TB_API const char *tb_status_string(tb_status_t status);

/* Bytes of the packed codes of an N x K matrix (scales not included):
 * N*K/4 for ternary and 2-bit, 3*N*K/8 for 3-bit, N * 16 * ceil(26 K/128 /
 * 16) for 5 trits per byte; 0 for bad arguments. */
TB_API size_t tb_packed_bytes(tb_grid_t grid, int64_t N, int64_t K);

/* Bytes of the bf16 scales of an N x K matrix: N * (K/128) * 2; 0 for bad
 * arguments. */
TB_API size_t tb_scale_bytes(int64_t N, int64_t K);

/* Group scales by absmax (rule above; ThinkBit page, 어떻게 동작하나, one
 * bf16 scale per 128 weights).  TB_GRID_TERNARY_B3 uses the ternary rule.
 *   W       [N][K] fp32 or bf16 (w_dtype), device.
 *   scales  [N][K/128] bf16 bit patterns, device, written. */
TB_API tb_status_t tb_scales_absmax(const void *W, tb_dtype_t w_dtype, int64_t N, int64_t K, tb_grid_t grid,
                             uint16_t *scales, tb_stream_t stream);

/* Round-to-nearest quantize and bit-pack (rules and layout above;
 * ThinkBit page, 어떻게 동작하나 and 무엇과 다른가).
 *   W          [N][K] fp32 or bf16 (w_dtype), device.
 *   scales     [N][K/128] bf16, device (e.g. from tb_scales_absmax).
 *   packed     tb_packed_bytes(grid, N, K) bytes, device, fully written.
 *   bad_count  device int32, or NULL; when given, it is OVERWRITTEN with
 *              the number of weights that met a NaN/Inf weight or an
 *              invalid scale. */
TB_API tb_status_t tb_pack(const void *W, tb_dtype_t w_dtype, int64_t N, int64_t K, tb_grid_t grid,
                    const uint16_t *scales, void *packed, int32_t *bad_count, tb_stream_t stream);

/* Inverse of the bit layout: codes[n][k] = c (int8), device, [N][K] -- the
 * integer codewords of the format (ThinkBit page, 어떻게 동작하나: w = c * s,
 * c on the layer's grid), for inspection and tests.
 *   packed  as produced by tb_pack, 16-byte aligned.
 *   codes   [N][K] int8, device, 16-byte aligned, fully written. */
TB_API tb_status_t tb_unpack(const void *packed, tb_grid_t grid, int64_t N, int64_t K, int8_t *codes,
                      tb_stream_t stream);

/* Scratch ("workspace") of the products below.  A call's scratch is of two
 * kinds: CONTROL words (arrival and completion counters), which must be
 * zero when a call starts and which every completed call leaves zero; and
 * DATA, which a call overwrites before it reads it.  Control words sit at
 * the front of the workspace, data at its back (ending at
 * workspace_bytes rounded down to 256), and each call asks for
 *       2 * max(control bytes, data bytes),
 * so that calls of any shapes and paths can share one workspace sized for
 * the largest of them: no call's data reaches another call's control words.
 * By path:
 *   M = 1 (tb_gemv above 2^24 weights, tb_layer_gemv, tb_gate_up_silu):
 *     control: per CTA 256 flagged partial-sum words (tiles whose K range
 *       is split between CTAs are combined in a fixed order by the CTA that
 *       reads the tile's start):
 *         ceil256(2048 * min(512, T1 * ceil(G / 2)));
 *     data: the activation records of x (1088 bytes per 128-group, built
 *       once per call by the call's first kernel):
 *         ceil256(1088 * G);
 *     with G = K/128 and T1 = ceil(N / 256).  tb_layer_workspace_bytes: the
 *     chunks of all items, the records of each distinct (x, code width);
 *     tb_gate_up_workspace_bytes adds ceil256(8 N) to the control words.
 *     (The row kernel behind small tb_gemv calls uses none of it.)
 *   2 <= M < 32: none (the kernel reads X as it is); the size is reported
 *     as 256.
 *   32 <= M <= 64 (the tensor-core path with the decoded weights in tensor
 *     memory), data only: X copied per group into the MMA's layout, the
 *     scales transposed per 128-row tile, a counter per tile (cleared by the
 *     call itself) and the K-split partial sums,
 *       D = ceil256(G * NP * 256) + ceil256(T * G * 256) + ceil256(4 * T)
 *         + [S > 1] ceil256(T * S * NP * 512),
 *     size 2 D, with NP = M rounded up to 16, T = ceil(N / 128) and S = the
 *     K split, max(1, min(floor((296 + T/2) / T), 16, G)).
 *   M > 64 (prefill: the tensor-core path with both operands in shared
 *     memory): per CTA (at most 256, at most one per chunk) a flag (control)
 *     and 128 x 128 fp32 partial sums (data; units whose groups are split
 *     between CTAs are combined in a fixed order by the CTA that reads the
 *     unit's first group):
 *       control ceil256(4 C), data ceil256(65536 C),
 *       C = min(256, T * ceil(M / 128) * G),
 *     size 2 max(control, data).
 * The workspace is
 *   - device memory, 256-byte aligned, at least the size returned here (for
 *     every call that uses it), ZERO-FILLED ONCE when allocated, and again
 *     after a call that reported TB_ERR_TIMEOUT;
 *   - owned by the caller, written by every call: two calls that share a
 *     workspace must be ordered (e.g. the same stream);
 *   - no other state is kept between calls.
 * Returns 0 for bad arguments. */
TB_API size_t tb_workspace_bytes(int64_t M, int64_t N, int64_t K); /* tb_gemv: M = 1; tb_gemm: its M */

/* Batch-1 GEMV y = W x over packed W (ThinkBit page, 무엇인가: one read of
 * every weight per decoded token; 전제와 한계: the direct 2/3-bit reader).
 *   packed, scales  as produced by tb_pack.
 *   x               [K] bf16, device, 16-byte aligned; finite, |x| < 2^120.
 *   y               [N] fp32 or bf16 (y_dtype), device, written.
 *   workspace       tb_workspace_bytes(1, N, K) bytes (see above), whichever
 *                   kernel runs.
 * Two kernels serve it.  Products of at most 2^24 weights (N * K), and every
 * TB_GRID_TERNARY_B3 product, run a single-launch kernel with one warp per
 * output row that stages x in shared memory and uses no workspace (for
 * TB_GRID_TERNARY_B3, K <= 57600, else TB_ERR_UNSUPPORTED).  Larger ones
 * run the integer tensor-path kernel of tb_layer_gemv.  Both meet the
 * error bound above; the same product through tb_gemv and tb_layer_gemv
 * may differ in rounding. */
TB_API tb_status_t tb_gemv(const void *packed, tb_grid_t grid, const uint16_t *scales, const uint16_t *x, void *y,
                           tb_dtype_t y_dtype, int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                           tb_stream_t stream);

/* GEMM Y = X W^T, 1 <= M <= 65536 (ThinkBit page, 무엇인가: the
 * weights are read once for all M activation rows; 어떻게 동작하나: w = c * s,
 * so every row is the GEMV above on its own activations).  M = 1 runs as
 * tb_gemv; 2 <= M < 32 on mma.sync, 32 <= M <= 64 on the tcgen05 tensor
 * cores with the decoded weights in tensor memory; prefill batches,
 * 64 < M <= 65536, in ONE launch on the tcgen05 tensor cores with both
 * operands in shared memory, 128 weight rows by blocks of 128 batch rows per
 * MMA unit (the weights are read from HBM once and decoded once per block);
 * all with the codewords decoded exactly to bf16.  TB_GRID_TERNARY_B3: one
 * GEMV launch per batch row, K <= 57600.
 *   X          [M][ldx] bf16, ldx >= K, ldx % 8 == 0, device; finite, |x| < 2^120.
 *   Y          [M][ldy] fp32 or bf16, ldy >= N, device; Y[m][n] for n < N written.
 *   workspace  tb_workspace_bytes(M, N, K) bytes. */
TB_API tb_status_t tb_gemm(const void *packed, tb_grid_t grid, const uint16_t *scales, const uint16_t *X,
                           int64_t ldx, void *Y, tb_dtype_t y_dtype, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           void *workspace, size_t workspace_bytes, tb_stream_t stream);

/* Diagnostic: how many bounded device-side waits gave up since the last
 * call, on the current device (the count is then cleared).  Every kernel
 * that waits on a copy or on the tensor-core pipeline gives up after about
 * two seconds, writes NaN to the outputs it has not finished and returns;
 * a nonzero count means such a launch produced no result.  Synchronizes
 * with the device; returns 0xFFFFFFFF if the count cannot be read. */
TB_API unsigned int tb_wait_timeouts(void);

/* Status of the work issued so far.  Every call above returns as soon as
 * its kernels are queued, so a wait that gives up on the device (a copy
 * that never lands, a tensor-core hand-off that never completes) can only
 * be reported afterwards: this call synchronizes `stream`, then returns
 * TB_ERR_TIMEOUT if any bounded wait on the current device gave up since
 * the last check (and clears the count), TB_ERR_CUDA if the stream or the
 * count reports a CUDA error, TB_OK otherwise. */
TB_API tb_status_t tb_sync_status(tb_stream_t stream);

/* One linear layer of a grouped launch. */
typedef struct {
    const void *packed;     /* device */
    const uint16_t *scales; /* device */
    const uint16_t *x;      /* [K] bf16, device, 16-byte aligned */
    void *y;                /* [N], device */
    int64_t N, K;
    int32_t grid;    /* tb_grid_t */
    int32_t y_dtype; /* tb_dtype_t */
} tb_linear_t;

#define TB_MAX_LAYER_ITEMS 16

/* Allow the call's kernels to start before earlier work in the stream has
 * finished (programmatic dependent launch): they begin streaming the packed
 * weights and scales at once and wait for the earlier work only before
 * touching activations, outputs or the workspace.  The caller promises that
 * no earlier work still in flight writes the packed weights or scales of
 * this call (true for resident model weights during decode). */
#define TB_FLAG_OVERLAP_PREVIOUS 1u

/* Test hook for the failure path of the batch-1 kernel: its copies are
 * never issued, every bounded wait gives up after about 10 ms instead of
 * 2 s, the outputs of the call are NaN, and the next tb_sync_status
 * returns TB_ERR_TIMEOUT.  Nothing faults and the context stays usable. */
#define TB_FLAG_TEST_STALL 0x80000000u

/* Workspace bytes of tb_layer_gemv for these items (0 for bad arguments):
 * the batch-1 rule above over all items together -- the tiles and chunks of
 * every item, the records of each distinct (x, code width) -- or 256 when
 * every item is in TB_GRID_TERNARY_B3. */
TB_API size_t tb_layer_workspace_bytes(const tb_linear_t *items, int n_items);

/* Mixed-grid grouped GEMV: every item is an independent y = W x with its
 * own grid, shape, input and output, all run by ONE main kernel launch (e.g.
 * a decoder layer's q, k, v, o, gate, up and down projections, each on its
 * own grid; ThinkBit page, 무엇과 다른가: grids chosen per layer).
 *   items      HOST array of n_items descriptors (read before returning).
 *   n_items    1 .. TB_MAX_LAYER_ITEMS.
 *   flags      0 or TB_FLAG_OVERLAP_PREVIOUS (test hook: TB_FLAG_TEST_STALL).
 *   workspace  tb_layer_workspace_bytes(items, n_items) bytes.
 * Items in TB_GRID_TERNARY_B3 are not part of the grouped launch: each runs
 * its own GEMV launch after it, in the same stream (K <= 57600), and needs
 * no workspace.
 * Outputs of different items must not overlap. */
TB_API tb_status_t tb_layer_gemv(const tb_linear_t *items, int n_items, unsigned flags, void *workspace,
                                 size_t workspace_bytes, tb_stream_t stream);

/* Workspace bytes of tb_gate_up_silu: the batch-1 rule above for the two
 * items, with ceil256(8 N) more control bytes for the pair; 0 for bad
 * arguments. */
TB_API size_t tb_gate_up_workspace_bytes(const tb_linear_t *gate, const tb_linear_t *up);

/* The gate and up projections of a decoder layer's MLP in one launch, and
 * the down projection's input from them:
 *     gate->y = W_gate x,  up->y = W_up x,  h[n] = bf16(silu(gate[n]) * up[n]),
 *     silu(g) = g / (1 + e^-g),
 * (ThinkBit page, 무엇인가: decoding a token runs every projection of every
 * layer; the SiLU-gated MLP is that of the Qwen3 layers the page quantizes).
 * The two products are those of tb_layer_gemv (same kernel, same bound);
 * h is formed in fp32 from the fp32 results and rounded half to even.
 *   gate, up   HOST descriptors of equal N and K, each on its own grid (not
 *              TB_GRID_TERNARY_B3); x is normally the same buffer, and then
 *              its activation records are prepared once for both when the
 *              grids have the same code width; y of each is written as for
 *              tb_layer_gemv.
 *   h          [N] bf16, device, written.
 *   flags      0 or TB_FLAG_OVERLAP_PREVIOUS.
 *   workspace  tb_gate_up_workspace_bytes(gate, up) bytes. */
TB_API tb_status_t tb_gate_up_silu(const tb_linear_t *gate, const tb_linear_t *up, uint16_t *h, unsigned flags,
                                   void *workspace, size_t workspace_bytes, tb_stream_t stream);

/* Size of the fixed device scratch behind tb_gemv_noalloc (4 MiB). */
#define TB_NOALLOC_SCRATCH_BYTES (4u << 20)

/* tb_gemv without a workspace argument and without allocating anything.
 * The ThinkBit pages have no counterpart: this is an interface variant of
 * tb_gemv for callers that cannot hand over device scratch -- a plain C
 * host with no device allocator of its own, or a decode loop that must not
 * call cudaMalloc/cudaFree (or an allocator that may call them) because
 * those calls can synchronize the device and stall other streams.
 * Arguments and results are those of tb_gemv; x and y still belong to the
 * caller.
 *   scratch  one statically allocated device array of
 *            TB_NOALLOC_SCRATCH_BYTES per device, inside this library.  A
 *            problem whose tb_workspace_bytes(1, N, K) exceeds that size is
 *            rejected with TB_ERR_UNSUPPORTED before any CUDA call (every
 *            K <= 2^17 fits, whatever N: the size does not grow with N).
 *            Nothing has to be cleared by the caller: the array starts
 *            zeroed (static storage) and every call leaves its control
 *            words zero again.
 *   setup    the first call on each device (with that device current) looks
 *            up the array's address with cudaGetSymbolAddress and caches it;
 *            make that first call before any stream capture.  A failed
 *            lookup returns TB_ERR_CUDA and is retried on the next call.
 *            The cached address belongs to the device's current context: a
 *            cudaDeviceReset (or any other end of that context) makes it
 *            stale, so do not call this entry point again in the same
 *            process after resetting the device.
 *   sharing  every call on a device uses the same array: calls on one stream
 *            are ordered and safe; calls that can overlap (other streams,
 *            other host threads) race and give wrong results -- use tb_gemv
 *            with separate workspaces for those. */
TB_API tb_status_t tb_gemv_noalloc(const void *packed, tb_grid_t grid, const uint16_t *scales, const uint16_t *x,
                                   void *y, tb_dtype_t y_dtype, int64_t N, int64_t K, tb_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TB_B200_H */
