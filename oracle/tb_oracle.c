/*
 * tb_oracle.c -- plain, single-threaded, fp64 CPU oracle for the ThinkBit
 * scalar low-bit weight format and the decode-time products over it.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library links, loads or calls
 * this file; only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with
 * the CUDA implementation: every rule below is restated here from its
 * source.
 *
 * Sources (cited by page title and section):
 *  [TB-how]  ThinkBit page, "ThinkBit은 2비트 양자화에서 추론 능력 보존을
 *            추론 평가로 검증한다" (onedev.kr/papers/1416), section
 *            어떻게 동작하나 ("how it works"): every weight is an integer
 *            codeword c times a bf16 scale s shared by 128 weights; the
 *            codeword grid is per layer, ternary {-1,0,1}, 2-bit
 *            {-2,-1,0,1} or 3-bit {-4,...,3}; dequantization is a single
 *            multiplication; no codebook, rotation or zero point.
 *  [TB-diff] same page, section 무엇과 다른가 ("what is different"):
 *            the codewords come out of a rounding step (QAT rounds fp32
 *            latents; the allocator compares per-grid rounding noise).
 *  [TB-lim]  same page, section 전제와 한계 ("assumptions and limits"):
 *            no kernel reads 2- and 3-bit codewords directly yet.
 *
 * Readings taken where the pages are silent (each one is listed in the
 * design notes of the repository):
 *  R1  scale = bf16_rne(fp32(absmax / d)) with d = |qmin| (1, 2, 4), so
 *      every grid point is reachable; a group whose scale would be zero
 *      (all-zero group, or underflow) gets scale 1.0; a scale that would
 *      round to infinity gets the largest finite bf16.  absmax is taken
 *      over the finite entries only.
 *  R2  rounding is round-half-to-even, then clamp to [qmin, qmax].
 *  R3  NaN weight -> code 0; +-Inf weight -> qmax / qmin; a scale that is
 *      not a positive finite number -> code 0.  Each such weight is
 *      counted.
 *  R4  groups are 128 consecutive weights along the input dimension K,
 *      starting at k = 0; K must be a multiple of 128.
 *  R5  stored code u = c + offset: offset 2 for the 2-bit container
 *      (ternary and 2-bit grids share it), offset 4 for 3-bit.
 *  R6  bit layout (the packing densities 16 codes per uint32 and 32 codes
 *      per three uint32 bit-planes are given; the order inside a word is
 *      this library's choice):
 *        2-bit: row n is K/16 uint32 words; word i holds codes
 *               k = 16i .. 16i+15.  Code 16i+2m sits at bits [2m, 2m+1],
 *               code 16i+2m+1 at bits [16+2m, 17+2m]  (m = 0..7): even
 *               codes in the low half-word, odd codes in the high one.
 *        3-bit: row n is K/32 blocks of three uint32 words (planes
 *               p = 0, 1, 2, in that order); block j holds codes
 *               k = 32j .. 32j+31.  In plane p, bit m holds bit p of code
 *               32j+2m and bit 16+m holds bit p of code 32j+2m+1
 *               (m = 0..15).
 *        ternary, 5 trits per byte ("b3", grid id 3; the 2-bit container is
 *               the default ternary layout, this one is the optional denser
 *               variant): digit d = c + 1 in {0,1,2}.  Row n is RB =
 *               16 * ceil(26 G / 16) bytes (G = K/128); group j takes the
 *               26 bytes from byte 26 j.  Group byte b < 25 holds codes
 *               128 j + 5 b + i (i = 0..4) as sum_i d_i 3^i; byte 25 holds
 *               codes 128 j + 125 + i (i = 0..2) the same way; bytes from
 *               26 G on are zero.  Any byte value v decodes digit i as
 *               floor(v / 3^i) mod 3, so the values 243..255 (never
 *               written) still decode to ternary codes.  Byte a of a row is
 *               bits [8 (a mod 4), 8 (a mod 4) + 7] of uint32 word a / 4
 *               (the bytes' memory order).
 *  R7  W is [N out][K in] row-major, y = W x, no bias.
 *  R8  products are summed in k order in fp64; fp32 output is the RNE
 *      rounding of that sum; bf16 output is the RNE rounding of the fp32.
 *  R9  the down projection's input is silu(gate) * up of the layer's gate
 *      and up projections (the Qwen3 MLP; the pages name the model family,
 *      not its layer), computed from the exact projections in fp64.
 *
 * Why the fp64 quotient gives the exact round-half-even of w/s (R2):
 * write w = W 2^a, s = S 2^b with integers |W|, S < 2^24.  If q = w/s is
 * not a half-integer h+1/2, then |q - (h+1/2)| = |2w - (2h+1)s| / (2s) is
 * at least 2^min(a+1,b) / (2 S 2^b).  When a+1 >= b this is >= 2^-25, which
 * exceeds the fp64 rounding error 2^-53 |q| unless |q| >= 2^28 (such q is
 * clamped anyway).  When a+1 < b, |q| < 2^(a-b+1) and the bound
 * 2^(a+1-b-25) again exceeds 2^-53 |q|.  So fl64(q) never lands on or
 * crosses a half-integer that q itself is not, and nearbyint(fl64(q)) is
 * the exact round-half-even of q.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#define TBO_GROUP 128

/* grid ids, same numbering the public interface uses */
enum { TBO_TERNARY = 0, TBO_INT2 = 1, TBO_INT3 = 2, TBO_TERNARY_B3 = 3 };

static int grid_ok(int g) { return g == TBO_TERNARY || g == TBO_INT2 || g == TBO_INT3 || g == TBO_TERNARY_B3; }

/* [TB-how]: the three grids (the 5-trits-per-byte layout stores the ternary grid) */
static int grid_qmin(int g) { return (g == TBO_TERNARY || g == TBO_TERNARY_B3) ? -1 : (g == TBO_INT2 ? -2 : -4); }
static int grid_qmax(int g) { return g == TBO_INT3 ? 3 : 1; }
/* R5; R6 for the base-3 digit */
static int grid_offset(int g) { return g == TBO_INT3 ? 4 : (g == TBO_TERNARY_B3 ? 1 : 2); }
/* R1: divisor d = |qmin| */
static int grid_scale_div(int g) { return -grid_qmin(g); }

/* ---- bf16 <-> binary floating point ------------------------------------ */

double tbo_bf16_to_double(uint16_t h)
{
    uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, 4);
    return (double)f;
}

/* Round an fp32 value to bf16, round-half-to-even.  bf16 is the top half
 * of the fp32 bit pattern, so the bf16 candidates around f are the
 * truncated pattern and the next pattern away from zero; the discarded 16
 * bits decide between them (sign-magnitude: rounding the magnitude to
 * nearest-even is round-to-nearest-even on the value). */
uint16_t tbo_bf16_round(float f)
{
    if (isnan(f)) return (uint16_t)0x7FC0;
    uint32_t b;
    memcpy(&b, &f, 4);
    uint16_t hi = (uint16_t)(b >> 16);
    uint32_t rest = b & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (hi & 1u))) hi = (uint16_t)(hi + 1u);
    return hi;
}

/* ---- group scale (R1) --------------------------------------------------- */

uint16_t tbo_scale_of_group(const float *w, int64_t len, int grid)
{
    double absmax = 0.0;
    for (int64_t i = 0; i < len; ++i) {
        double a = fabs((double)w[i]);
        if (isfinite(a) && a > absmax) absmax = a;
    }
    float q = (float)(absmax / (double)grid_scale_div(grid)); /* exact: d is a power of two */
    uint16_t s = tbo_bf16_round(q);
    if ((s & 0x7FFFu) == 0) s = 0x3F80;      /* zero scale -> 1.0 */
    if ((s & 0x7FFFu) == 0x7F80u) s = 0x7F7F; /* infinite scale -> largest finite */
    return s;
}

/* scales[n*(K/128) + j] for rows n < N, groups j < K/128.  Returns 0, or -1
 * on bad arguments. */
int tbo_scales_absmax(const float *W, int64_t N, int64_t K, int grid, uint16_t *scales)
{
    if (!grid_ok(grid) || N < 0 || K < 0 || K % TBO_GROUP) return -1;
    int64_t G = K / TBO_GROUP;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < G; ++j)
            scales[n * G + j] = tbo_scale_of_group(W + n * K + j * TBO_GROUP, TBO_GROUP, grid);
    return 0;
}

/* ---- round-to-nearest quantization (R2, R3) ----------------------------- */

int tbo_quantize(float w, uint16_t scale_bf16, int grid, int *bad)
{
    double s = tbo_bf16_to_double(scale_bf16);
    int qmin = grid_qmin(grid), qmax = grid_qmax(grid);
    *bad = 0;
    if (!(s > 0.0) || isinf(s)) { *bad = 1; return 0; }
    if (isnan(w)) { *bad = 1; return 0; }
    if (isinf(w)) { *bad = 1; return w > 0 ? qmax : qmin; }
    double q = (double)w / s;   /* see the header for why this is enough */
    double r = nearbyint(q);    /* default rounding mode: half to even */
    if (r < (double)qmin) r = (double)qmin;
    if (r > (double)qmax) r = (double)qmax;
    return (int)r;
}

/* ---- bit layout (R6) ----------------------------------------------------- */

/* R6, 5-trits-per-byte layout: bytes per group and per row */
#define TBO_B3_GROUP_BYTES 26
static int64_t b3_row_bytes(int64_t K) { return 16 * ((TBO_B3_GROUP_BYTES * (K / TBO_GROUP) + 15) / 16); }

int64_t tbo_row_words(int grid, int64_t K)
{
    if (grid == TBO_TERNARY_B3) return b3_row_bytes(K) / 4;
    return grid == TBO_INT3 ? 3 * (K / 32) : K / 16;
}

/* byte of row position k and its base-3 digit index */
static void b3_place(int64_t k, int64_t *byte, int *digit)
{
    int64_t j = k / TBO_GROUP, r = k % TBO_GROUP;
    *byte = TBO_B3_GROUP_BYTES * j + r / 5;
    *digit = (int)(r % 5);
}

static unsigned pow3(int i)
{
    unsigned p = 1;
    while (i-- > 0) p *= 3;
    return p;
}

static void put_code(uint32_t *row, int grid, int64_t k, unsigned u)
{
    if (grid == TBO_TERNARY_B3) {
        int64_t a;
        int i;
        b3_place(k, &a, &i);
        /* the row starts zeroed and a byte's digits never exceed 242 in total: no carry */
        row[a / 4] += (uint32_t)(u * pow3(i)) << (8 * (a % 4));
    } else if (grid == TBO_INT3) {
        int64_t block = k / 32;
        int i = (int)(k % 32);
        int bitpos = (i % 2 == 0) ? i / 2 : 16 + i / 2;
        for (int p = 0; p < 3; ++p)
            row[3 * block + p] |= (uint32_t)((u >> p) & 1u) << bitpos;
    } else {
        int64_t word = k / 16;
        int i = (int)(k % 16);
        int shift = (i % 2 == 0) ? 2 * (i / 2) : 16 + 2 * (i / 2);
        row[word] |= (uint32_t)(u & 3u) << shift;
    }
}

static unsigned get_code(const uint32_t *row, int grid, int64_t k)
{
    if (grid == TBO_TERNARY_B3) {
        int64_t a;
        int i;
        b3_place(k, &a, &i);
        unsigned v = (row[a / 4] >> (8 * (a % 4))) & 0xFFu;
        return (v / pow3(i)) % 3u;
    } else if (grid == TBO_INT3) {
        int64_t block = k / 32;
        int i = (int)(k % 32);
        int bitpos = (i % 2 == 0) ? i / 2 : 16 + i / 2;
        unsigned u = 0;
        for (int p = 0; p < 3; ++p)
            u |= ((row[3 * block + p] >> bitpos) & 1u) << p;
        return u;
    } else {
        int64_t word = k / 16;
        int i = (int)(k % 16);
        int shift = (i % 2 == 0) ? 2 * (i / 2) : 16 + 2 * (i / 2);
        return (row[word] >> shift) & 3u;
    }
}

/* ---- pack / unpack ------------------------------------------------------- */

/* W fp32 [N][K] (a bf16 W is widened exactly by the caller), scales as
 * produced by the caller; writes N * row_words uint32.  *bad_count (if not
 * NULL) receives the number of weights covered by R3. */
int tbo_pack(const float *W, int64_t N, int64_t K, int grid, const uint16_t *scales,
             uint32_t *packed, int64_t *bad_count)
{
    if (!grid_ok(grid) || N < 0 || K < 0 || K % TBO_GROUP) return -1;
    int64_t G = K / TBO_GROUP, RW = tbo_row_words(grid, K), nbad = 0;
    memset(packed, 0, (size_t)(N * RW) * sizeof(uint32_t));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int bad;
            int c = tbo_quantize(W[n * K + k], scales[n * G + k / TBO_GROUP], grid, &bad);
            nbad += bad;
            put_code(packed + n * RW, grid, k, (unsigned)(c + grid_offset(grid)));
        }
    }
    if (bad_count) *bad_count = nbad;
    return 0;
}

/* codes[n*K + k] = stored code minus offset.  (Ternary rows never hold a
 * stored 0; if one does, it decodes to -2, like the 2-bit grid.) */
int tbo_unpack(const uint32_t *packed, int grid, int64_t N, int64_t K, int8_t *codes)
{
    if (!grid_ok(grid) || N < 0 || K < 0 || K % TBO_GROUP) return -1;
    int64_t RW = tbo_row_words(grid, K);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            codes[n * K + k] = (int8_t)((int)get_code(packed + n * RW, grid, k) - grid_offset(grid));
    return 0;
}

/* ---- dequantized products (R7, R8) -------------------------------------- */

/* One output row: y = sum_k x_k * (c_k * s_{k/128}) in k order, fp64.
 * *yabs = sum_k |x_k * c_k * s|, the scale of the error bound.  Every
 * product is exact in fp64 (8-bit x times 3-bit c times 8-bit s). */
static void dot_row(const uint32_t *row, int grid, const uint16_t *srow, const uint16_t *x,
                    int64_t K, double *y, double *yabs)
{
    double acc = 0.0, aabs = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        int c = (int)get_code(row, grid, k) - grid_offset(grid);
        double w = (double)c * tbo_bf16_to_double(srow[k / TBO_GROUP]); /* dequantize: one multiply */
        double p = tbo_bf16_to_double(x[k]) * w;
        acc += p;
        aabs += fabs(p);
    }
    *y = acc;
    *yabs = aabs;
}

/* y[n], yabs[n] for n < N; x is K bf16 values. */
int tbo_gemv(const uint32_t *packed, int grid, const uint16_t *scales, const uint16_t *x,
             int64_t N, int64_t K, double *y, double *yabs)
{
    if (!grid_ok(grid) || N < 0 || K < 0 || K % TBO_GROUP) return -1;
    int64_t G = K / TBO_GROUP, RW = tbo_row_words(grid, K);
    for (int64_t n = 0; n < N; ++n)
        dot_row(packed + n * RW, grid, scales + n * G, x, K, y + n, yabs + n);
    return 0;
}

/* Y[m*N + n] for m < M: row m of X (stride ldx elements) times W^T. */
int tbo_gemm(const uint32_t *packed, int grid, const uint16_t *scales, const uint16_t *X,
             int64_t ldx, int64_t M, int64_t N, int64_t K, double *Y, double *Yabs)
{
    if (!grid_ok(grid) || M < 0 || N < 0 || K < 0 || K % TBO_GROUP || ldx < K) return -1;
    for (int64_t m = 0; m < M; ++m)
        if (tbo_gemv(packed, grid, scales, X + m * ldx, N, K, Y + m * N, Yabs + m * N)) return -1;
    return 0;
}

/* Single output element (n) of a GEMV: used to check sampled rows of
 * full-size problems without computing every row. */
int tbo_gemv_rows(const uint32_t *packed, int grid, const uint16_t *scales, const uint16_t *x,
                  int64_t K, const int64_t *rows, int64_t nrows, double *y, double *yabs)
{
    if (!grid_ok(grid) || K < 0 || K % TBO_GROUP) return -1;
    int64_t G = K / TBO_GROUP, RW = tbo_row_words(grid, K);
    for (int64_t i = 0; i < nrows; ++i)
        dot_row(packed + rows[i] * RW, grid, scales + rows[i] * G, x, K, y + i, yabs + i);
    return 0;
}

/* ---- the step between a decoder layer's gate/up and down projections ------
 * [TB-what] (section 무엇인가): decode runs every projection of every layer
 * for each token; in the Qwen3 layers the pages quantize, the down
 * projection's input is the SiLU-gated product of the gate and up
 * projections of the same input (reading R9):
 *     h[n] = silu(g[n]) * u[n],   silu(g) = g / (1 + e^-g).
 * Plain fp64 with libm's exp. */
double tbo_silu(double g) { return g / (1.0 + exp(-g)); }

int tbo_swiglu(const double *g, const double *u, int64_t n, double *h)
{
    if (n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) h[i] = tbo_silu(g[i]) * u[i];
    return 0;
}

/* Make sure the default rounding mode is in force (nearbyint relies on it). */
int tbo_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }
