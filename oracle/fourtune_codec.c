/*
 * FourTune oracle: the 4-bit block codec, written out plainly for the CPU.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, __graft_entry__.smoke()
 * and bench.py's cpu_baseline / reference arms may load this library.  It shares
 * no code, header, table or helper with the CUDA library under
 * diffusion_dit_b200/csrc/, and neither side includes the other.
 *
 * What it computes (FourTune: Towards Fully 4-Bit Efficient Post-Training for
 * Diffusion Models, arXiv 2607.05711):
 *   - section 2.3 "Model Quantization": W~ = Round(W / s) with a scale s;
 *   - section 3.1: the residual R and the activations X are quantized to NVFP4
 *     (E2M1 elements with a scale per block);
 *   - section 3.2 and Table 5: the blocks are 16x16 tiles of the stored matrix, so
 *     the transpose of a quantized matrix reuses the same codes and scales.
 *
 * Readings taken where the pages are silent:
 *   - NVFP4 two-level scaling: one fp32 factor g per tensor, g = 2688 / amax_t
 *     (2688 = 6 * 448 maps the tensor max to the largest E2M1 value times the
 *     largest UE4M3 value), and one UE4M3 scale per 16x16 block;
 *   - block scale sb = UE4M3( (amax_b / 6) * g ), both operations fp32 round-to-
 *     nearest-even; element code = E2M1( x * (g / val(sb)) ), the quotient and the
 *     product each rounded to fp32;
 *   - both conversions round to nearest, ties to the even code, and saturate to
 *     the largest finite value; the code keeps the sign bit of x (so -0.1 may
 *     give code 0x8); a block whose scale is 0 gets all-zero codes;
 *   - amax_t == 0, or a g that is not finite, gives g = 1 and all-zero output.
 *
 * Both conversions are written as a brute-force search for the nearest member of
 * the format's value set, with an explicit even-code tie-break, not as bit
 * manipulation.  Compile with -ffp-contract=off so every fp32 multiply and divide
 * is rounded on its own.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* E2M1 magnitudes for codes 0..7: sign bit 3, exponent bits 2..1 (bias 1),
 * mantissa bit 0; exponent 0 is subnormal (0 and 0.5). */
static double e2m1_magnitude(int code3) {
    int e = (code3 >> 1) & 3, m = code3 & 1;
    if (e == 0) return 0.5 * m;
    return ldexp(1.0 + 0.5 * m, e - 1);
}

/* UE4M3 value of code 0..126 (0x7F is NaN and never produced): exponent bits
 * 6..3 (bias 7), mantissa bits 2..0; exponent 0 is subnormal. */
static double ue4m3_value(int code) {
    int e = (code >> 3) & 15, m = code & 7;
    if (e == 0) return ldexp(m / 8.0, -6);
    return ldexp(1.0 + m / 8.0, e - 7);
}

double ora_e2m1_value(int code) {
    double v = e2m1_magnitude(code & 7);
    return (code & 8) ? -v : v;
}

double ora_ue4m3_value(int code) { return ue4m3_value(code); }

/* Nearest E2M1 code to v: search all 8 magnitudes, ties to the even code.
 * Magnitudes above 6 fall back to 6 (saturation) because 6 is then nearest. */
int ora_e2m1_encode(float v) {
    double a = fabs((double)v);
    /* saturation: at or above the largest value the answer is the largest value
     * (stated outright: for huge a every distance rounds to the same double) */
    if (a >= e2m1_magnitude(7)) return (signbit(v) ? 8 : 0) | 7;
    int best = 0;
    double bestd = fabs(a - e2m1_magnitude(0));
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - e2m1_magnitude(c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return (signbit(v) ? 8 : 0) | best;
}

/* Nearest UE4M3 code to a non-negative v: search all 127 finite values, ties to
 * the even code; anything above 448 saturates to 448 (code 0x7E). */
int ora_ue4m3_encode(float v) {
    double a = (double)v;
    if (!(a > 0.0)) return 0;
    if (a >= ue4m3_value(126)) return 126; /* saturate to 448 */
    int best = 0;
    double bestd = fabs(a - ue4m3_value(0));
    for (int c = 1; c < 127; ++c) {
        double d = fabs(a - ue4m3_value(c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Element (i) of an input matrix stored as bf16 (is_f32 == 0) or fp32. */
static float load_elem(const void* x, int is_f32, int64_t idx) {
    if (is_f32) return ((const float*)x)[idx];
    return bf16_to_f32(((const uint16_t*)x)[idx]);
}

/* max |x| over a matrix (exact). */
static float amax_any(const void* x, int is_f32, int64_t rows, int64_t cols, int64_t ld) {
    float m = 0.0f;
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j) {
            float a = fabsf(load_elem(x, is_f32, i * ld + j));
            if (a > m) m = a;
        }
    return m;
}

float ora_amax_bf16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
    return amax_any(x, 0, rows, cols, ld);
}

float ora_amax_f32(const float* x, int64_t rows, int64_t cols, int64_t ld) {
    return amax_any(x, 1, rows, cols, ld);
}

/* The tensor-level factor g (second-level scale). */
float ora_global_scale(float amax_t) {
    if (!(amax_t > 0.0f)) return 1.0f;
    volatile float num = 2688.0f;
    float g = num / amax_t;
    if (!isfinite(g) || !(g > 0.0f)) return 1.0f;
    return g;
}

/*
 * Quantize a matrix x[rows, cols] (bf16 or fp32, row stride ld elements) in blocks of
 * bh rows x 16 columns: bh = 16 is FourTune's block-wise 16x16 (section 3.1), bh = 1 the
 * group-wise 1x16 it is compared with (section 4.3, "Impact of Quantization Granularity",
 * Table 5).  The same two-level scaling either way.
 * amax_t < 0 means "compute it here"; otherwise it is used as given.
 * Outputs (caller-allocated):
 *   codes  [rows, cols/2]  element (i, 2j) in the low nibble of byte (i, j)
 *   scales [rows/bh, cols/16]  one UE4M3 byte per block
 *   *g_out                 the tensor factor g
 * rows must be a multiple of bh, cols of 16.  Returns 0, or -1 on bad shape.
 */
static int quantize_blocks(const void* x, int is_f32, int64_t rows, int64_t cols, int64_t ld, int bh,
                           float amax_t, uint8_t* codes, uint8_t* scales, float* g_out) {
    if (bh < 1 || rows % bh || cols % 16 || rows < 0 || cols < 0) return -1;
    if (amax_t < 0.0f) amax_t = amax_any(x, is_f32, rows, cols, ld);
    int degenerate = 1;
    float g = 1.0f;
    if (amax_t > 0.0f) {
        volatile float num = 2688.0f;
        float gg = num / amax_t;
        if (isfinite(gg) && gg > 0.0f) {
            g = gg;
            degenerate = 0;
        }
    }
    *g_out = g;
    memset(codes, 0, (size_t)(rows * (cols / 2)));
    memset(scales, 0, (size_t)((rows / bh) * (cols / 16)));
    if (degenerate) return 0;
    for (int64_t bi = 0; bi < rows / bh; ++bi) {
        for (int64_t bj = 0; bj < cols / 16; ++bj) {
            float amax_b = 0.0f;
            for (int r = 0; r < bh; ++r)
                for (int c = 0; c < 16; ++c) {
                    float a = fabsf(load_elem(x, is_f32, (bi * bh + r) * ld + bj * 16 + c));
                    if (a > amax_b) amax_b = a;
                }
            volatile float six = 6.0f;
            float q = amax_b / six;  /* fp32 quotient */
            float s = q * g;         /* fp32 product  */
            int sb = ora_ue4m3_encode(s);
            scales[bi * (cols / 16) + bj] = (uint8_t)sb;
            if (sb == 0) continue; /* codes stay 0 */
            float inv = g / (float)ue4m3_value(sb);
            for (int r = 0; r < bh; ++r) {
                for (int c = 0; c < 16; ++c) {
                    int64_t i = bi * bh + r, j = bj * 16 + c;
                    float v = load_elem(x, is_f32, i * ld + j) * inv;
                    int code = ora_e2m1_encode(v);
                    uint8_t* byte = &codes[i * (cols / 2) + j / 2];
                    if (j & 1) *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
                    else *byte = (uint8_t)((*byte & 0xF0) | code);
                }
            }
        }
    }
    return 0;
}

int ora_quantize_block16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                         float amax_t, uint8_t* codes, uint8_t* scales, float* g_out) {
    return quantize_blocks(x, 0, rows, cols, ld, 16, amax_t, codes, scales, g_out);
}

int ora_quantize_block16_f32(const float* x, int64_t rows, int64_t cols, int64_t ld,
                             float amax_t, uint8_t* codes, uint8_t* scales, float* g_out) {
    return quantize_blocks(x, 1, rows, cols, ld, 16, amax_t, codes, scales, g_out);
}

/* Group-wise 1x16 (bf16 input): scales [rows, cols/16]. */
int ora_quantize_1x16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                      float amax_t, uint8_t* codes, uint8_t* scales, float* g_out) {
    return quantize_blocks(x, 0, rows, cols, ld, 1, amax_t, codes, scales, g_out);
}

/* Dequantize blocks of bh rows x 16: xhat = val(code) * val(sb) / g, in double. */
void ora_dequantize_blocks(const uint8_t* codes, const uint8_t* scales, float g, int64_t rows,
                           int64_t cols, int bh, double* out) {
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j) {
            uint8_t byte = codes[i * (cols / 2) + j / 2];
            int code = (j & 1) ? (byte >> 4) : (byte & 15);
            double sb = ue4m3_value(scales[(i / bh) * (cols / 16) + j / 16]);
            out[i * cols + j] = ora_e2m1_value(code) * sb / (double)g;
        }
}

void ora_dequantize_block16(const uint8_t* codes, const uint8_t* scales, float g,
                            int64_t rows, int64_t cols, double* out) {
    ora_dequantize_blocks(codes, scales, g, rows, cols, 16, out);
}

/* Transpose of a quantized matrix without requantization (section 3.2): the codes
 * of element (i, j) move to (j, i) and the block scale of block (a, b) to (b, a). */
void ora_transpose_block16(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                           int64_t cols, uint8_t* codes_t, uint8_t* scales_t) {
    memset(codes_t, 0, (size_t)(cols * (rows / 2)));
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j) {
            uint8_t byte = codes[i * (cols / 2) + j / 2];
            int code = (j & 1) ? (byte >> 4) : (byte & 15);
            uint8_t* dst = &codes_t[j * (rows / 2) + i / 2];
            if (i & 1) *dst = (uint8_t)((*dst & 0x0F) | (code << 4));
            else *dst = (uint8_t)((*dst & 0xF0) | code);
        }
    for (int64_t a = 0; a < rows / 16; ++a)
        for (int64_t b = 0; b < cols / 16; ++b)
            scales_t[b * (rows / 16) + a] = scales[a * (cols / 16) + b];
}

/* Encode an array of fp32 values (used by the codec tests). */
void ora_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)ora_e2m1_encode(v[i]);
}

void ora_ue4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)ora_ue4m3_encode(v[i]);
}
