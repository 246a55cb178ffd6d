/*
 * csld_oracle.c -- plain, slow, float64 CPU oracle for the hybrid compressed-attention
 * decode path (CSA + HCA compressors, lightning indexer + top-k, hybrid decode attention,
 * KV-cache append).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this file:
 * only the tests, the smoke check and the bench's CPU-baseline / reference leg use it.  It
 * shares no code, header, table or constant generator with the CUDA library; every codec
 * below is written out from the published number-format definitions (OCP 8-bit floating
 * point E4M3, bfloat16, OCP microscaling E2M1), not from any GPU header.
 *
 * Sources (web pages about DeepSeek-V4; cited by title and section):
 *  [HF]   "DeepSeek-V4: a million-token context that agents can actually use" (Korean
 *         rendering of the Hugging Face blog): CSA paragraph, Figure 3 caption, HCA paragraph,
 *         Figure 4 caption, layer-pattern paragraph, storage paragraph.
 *  [VEL]  velog.io "DeepSeek V4 paper review": sections "core technique 1: CSA",
 *         "core technique 2: HCA", "KV cache layout handled separately".
 *  [AXB]  axbrief.com summary, section "1M context, 27% FLOPs, 2% KV cache".
 *
 * Readings where the pages are silent (listed with reasons in the design notes):
 *  - one scalar gate logit per token, one positional-bias scalar per slot of the block;
 *  - one shared 512-d entry is both key and value; dims 0..447 are stored E4M3 (scale 1),
 *    dims 448..511 (the RoPE dims) bf16;
 *  - the indexer key of an entry is FP4(c_s . W_I) with c_s the pooled vector before FP8
 *    rounding; FP4 = E2M1 codes with one power-of-two fp32 scale per 32 values;
 *  - the indexer score is computed in fp32 in a fixed operation order (see
 *    orc_indexer_scores); selection is by (score desc, index asc);
 *  - attention is one joint softmax over {selected or all visible compressed entries} and
 *    {the last W raw tokens}; a compressed entry is visible once its last token arrived;
 *  - layout variants: per-channel gating (orc_pool_block_channel), RoPE applied at
 *    compressed positions (orc_rope_rotate: RoFormer pairs (448+2i, 449+2i), angle
 *    pos * base^(-i/32); an entry at its block's last token, a window entry at its token) and
 *    scaled FP8 entries (one scale per layer cache: E4M3(x / sigma), RoPE dims unscaled) and
 *    per-head indexer keys (orc_indexer_key_raw_perhead: head h projected by its own W_h and
 *    scored against its own key).
 *
 * parity unpinned: the real model's gate form, indexer projection and FP4 scale rule are not
 * given by the pages (no weights); what is pinned is listed in the tests.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 512
#define ORC_D_NOPE 448
#define ORC_D_ROPE 64
#define ORC_ENTRY_BYTES 576
#define ORC_IDX_HEADS 4
#define ORC_IDX_DIM 64
#define ORC_IDX_GROUP 32
#define ORC_IKEY_BYTES 32

/* ------------------------------------------------------------------------------------------
 * Number formats ([HF] storage paragraph: most KV dims FP8, RoPE dims BF16, indexer FP4).
 * ---------------------------------------------------------------------------------------- */

/* E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * S.1111.111 is NaN; largest finite 448; smallest subnormal 2^-9. */
double orc_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);              /* 0.mmm x 2^-6 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round-to-nearest-even onto the E4M3 grid, saturating to +-448 (no infinities exist). */
uint8_t orc_e4m3_encode(double x) {
    uint8_t s = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return s | 0x7E;
    int e2;
    frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5,1)  =>  floor(log2 a) = e2-1 */
    int E = (a == 0.0) ? -6 : e2 - 1;
    if (E < -6) E = -6;            /* below the normal range the spacing stays 2^-9 */
    double q = ldexp(1.0, E - 3);  /* spacing of representable values in this binade */
    double r = nearbyint(a / q) * q;   /* a/q is exact; nearbyint = ties-to-even */
    if (r >= 448.0) return s | 0x7E;
    if (r == 0.0) return s;
    int er;
    frexp(r, &er);
    int Er = er - 1;
    if (Er < -6) {                 /* subnormal: r = m * 2^-9 */
        int m = (int)ldexp(r, 9);
        return s | (uint8_t)m;
    }
    int m = (int)((ldexp(r, -Er) - 1.0) * 8.0);
    return s | (uint8_t)(((Er + 7) << 3) | m);
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 mantissa bits. */
double orc_bf16_decode(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 7) & 0xFF, m = h & 0x7F;
    double v;
    if (e == 0xFF) return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0) v = ldexp((double)m, -133);
    else v = ldexp(1.0 + m / 128.0, e - 127);
    return s ? -v : v;
}

/* Round-to-nearest-even onto the bf16 grid (overflow to infinity). */
uint16_t orc_bf16_encode(double x) {
    uint16_t s = signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    if (isnan(x)) return 0x7FC0;
    int e2;
    frexp(a, &e2);
    int E = (a == 0.0) ? -126 : e2 - 1;
    if (E < -126) E = -126;
    double q = ldexp(1.0, E - 7);
    double r = nearbyint(a / q) * q;
    if (r >= ldexp(1.0, 128)) return s | 0x7F80;
    if (r == 0.0) return s;
    int er;
    frexp(r, &er);
    int Er = er - 1;
    if (Er < -126) return s | (uint16_t)(int)ldexp(r, 133);
    int m = (int)((ldexp(r, -Er) - 1.0) * 128.0);
    return s | (uint16_t)(((Er + 127) << 7) | m);
}

/* E2M1 (4-bit): bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * Magnitudes of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double orc_e2m1_decode(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* Round-to-nearest-even onto the E2M1 grid; magnitudes above 6 saturate to 6. */
uint8_t orc_e2m1_encode(double v) {
    uint8_t s = signbit(v) ? 8 : 0;
    double a = fabs(v);
    if (a >= 6.0) return s | 7;
    double q = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);   /* grid spacing in each range */
    double r = nearbyint(a / q) * q;                       /* ties go to the even multiple */
    /* r is now one of the grid values */
    uint8_t m;
    if (r == 0.0) m = 0;
    else if (r == 0.5) m = 1;
    else if (r == 1.0) m = 2;
    else if (r == 1.5) m = 3;
    else if (r == 2.0) m = 4;
    else if (r == 3.0) m = 5;
    else if (r == 4.0) m = 6;
    else m = 7;
    return s | m;
}

/* Group scale: the smallest power of two sigma with amax <= 6*sigma (so the scaled group
 * fits the E2M1 range), i.e. 2^ceil(log2(amax/6)); 1 when amax == 0.  Found by exact
 * comparisons rather than a floating-point log. */
double orc_fp4_group_scale(double amax) {
    if (!(amax > 0.0)) return 1.0;
    int e2;
    frexp(amax / 6.0, &e2);
    int e = e2;                                  /* start near the answer, then fix exactly */
    while (6.0 * ldexp(1.0, e - 1) >= amax) --e;
    while (6.0 * ldexp(1.0, e) < amax) ++e;
    return ldexp(1.0, e);
}

/* FP4 quantisation of a 64-vector: two groups of 32, each with its scale (an fp32 power of
 * two) and E2M1 codes of x/scale.  Codes are packed two per byte, element 2i in the low
 * nibble of byte i. */
void orc_fp4_quantize64(const double* u, uint8_t* codes, float* scales) {
    memset(codes, 0, ORC_IKEY_BYTES);
    for (int g = 0; g < 2; ++g) {
        double amax = 0.0;
        for (int i = 0; i < ORC_IDX_GROUP; ++i) {
            double a = fabs(u[g * ORC_IDX_GROUP + i]);
            if (a > amax) amax = a;
        }
        double sc = orc_fp4_group_scale(amax);
        scales[g] = (float)sc;
        for (int i = 0; i < ORC_IDX_GROUP; ++i) {
            int d = g * ORC_IDX_GROUP + i;
            uint8_t c = orc_e2m1_encode(u[d] / sc);
            codes[d / 2] |= (uint8_t)((d & 1) ? (c << 4) : c);
        }
    }
}

static uint8_t orc_nibble(const uint8_t* codes, int d) {
    return (d & 1) ? (codes[d / 2] >> 4) & 0xF : codes[d / 2] & 0xF;
}

void orc_fp4_dequantize64(const uint8_t* codes, const float* scales, double* u) {
    for (int d = 0; d < ORC_IDX_DIM; ++d)
        u[d] = orc_e2m1_decode(orc_nibble(codes, d)) * (double)scales[d / ORC_IDX_GROUP];
}

/* Entry layout: bytes 0..447 = E4M3 codes of dims 0..447; bytes 448..575 = 64 bf16
 * (little-endian) of dims 448..511 ([HF] storage paragraph; [AXB]). */
void orc_entry_encode(const double* x, uint8_t* entry) {
    for (int d = 0; d < ORC_D_NOPE; ++d) entry[d] = orc_e4m3_encode(x[d]);
    for (int r = 0; r < ORC_D_ROPE; ++r) {
        uint16_t h = orc_bf16_encode(x[ORC_D_NOPE + r]);
        entry[ORC_D_NOPE + 2 * r] = (uint8_t)(h & 0xFF);
        entry[ORC_D_NOPE + 2 * r + 1] = (uint8_t)(h >> 8);
    }
}

void orc_entry_decode(const uint8_t* entry, double* x) {
    for (int d = 0; d < ORC_D_NOPE; ++d) x[d] = orc_e4m3_decode(entry[d]);
    for (int r = 0; r < ORC_D_ROPE; ++r) {
        uint16_t h = (uint16_t)(entry[ORC_D_NOPE + 2 * r] | (entry[ORC_D_NOPE + 2 * r + 1] << 8));
        x[ORC_D_NOPE + r] = orc_bf16_decode(h);
    }
}

/* Scaled FP8 entries (a layout variant of the storage paragraph's FP8 entries): one positive
 * scale sigma per layer cache; the E4M3 dims hold E4M3(x / sigma) and stand for sigma times
 * their code value, the bf16 RoPE dims are unscaled.  sigma = 1 is the base layout. */
void orc_entry_encode_scaled(const double* x, double kv_scale, uint8_t* entry) {
    double y[ORC_D];
    for (int d = 0; d < ORC_D; ++d) y[d] = d < ORC_D_NOPE ? x[d] / kv_scale : x[d];
    orc_entry_encode(y, entry);
}

void orc_entry_decode_scaled(const uint8_t* entry, double kv_scale, double* x) {
    orc_entry_decode(entry, x);
    for (int d = 0; d < ORC_D_NOPE; ++d) x[d] *= kv_scale;
}

/* ------------------------------------------------------------------------------------------
 * O1 -- softmax-gated pooling with a learned positional bias ([HF] CSA paragraph: "compresses
 * KV entries 4x along the sequence with softmax-gated pooling and a learned positional bias";
 * Figure 3 caption: every 4 tokens -> one entry; HCA paragraph / Figure 4: the same with 128).
 * For block s of m tokens t = s*m + j:  a_j = z_t + b_j,  w = softmax(a),  c = sum_j w_j x_t.
 * ---------------------------------------------------------------------------------------- */
void orc_pool_block(const uint16_t* raw, const float* gate, const float* bias, int m, double* c) {
    double amax = -INFINITY;
    for (int j = 0; j < m; ++j) {
        double a = (double)gate[j] + (double)bias[j];
        if (a > amax) amax = a;
    }
    double wsum = 0.0;
    double* w = (double*)malloc(sizeof(double) * (size_t)m);
    for (int j = 0; j < m; ++j) {
        w[j] = exp((double)gate[j] + (double)bias[j] - amax);
        wsum += w[j];
    }
    for (int d = 0; d < ORC_D; ++d) c[d] = 0.0;
    for (int j = 0; j < m; ++j) {
        double wj = w[j] / wsum;
        for (int d = 0; d < ORC_D; ++d) c[d] += wj * orc_bf16_decode(raw[(size_t)j * ORC_D + d]);
    }
    free(w);
}

/* O1, per-channel variant (the other plain reading of "softmax-gated pooling with a learned
 * positional bias", [HF] CSA paragraph): one gate logit per token AND dimension, one bias per
 * block slot and dimension.  For every dimension d separately:
 *   a_j = z[j][d] + b[j][d],  w = softmax_j(a),  c_d = sum_j w_j x[j][d].
 * gate [m][512] and bias [m][512] f32; with z[j][d] = z_j and b[j][d] = b_j for every d it is
 * orc_pool_block. */
void orc_pool_block_channel(const uint16_t* raw, const float* gate, const float* bias, int m, double* c) {
    for (int d = 0; d < ORC_D; ++d) {
        double amax = -INFINITY;
        for (int j = 0; j < m; ++j) {
            double a = (double)gate[(size_t)j * ORC_D + d] + (double)bias[(size_t)j * ORC_D + d];
            if (a > amax) amax = a;
        }
        double wsum = 0.0;
        for (int j = 0; j < m; ++j)
            wsum += exp((double)gate[(size_t)j * ORC_D + d] + (double)bias[(size_t)j * ORC_D + d] - amax);
        double acc = 0.0;
        for (int j = 0; j < m; ++j) {
            double wj = exp((double)gate[(size_t)j * ORC_D + d] + (double)bias[(size_t)j * ORC_D + d] - amax) / wsum;
            acc += wj * orc_bf16_decode(raw[(size_t)j * ORC_D + d]);
        }
        c[d] = acc;
    }
}

/* O2 -- indexer key before quantisation: u = c . W_I with W_I [512][64] row-major. */
void orc_indexer_key_raw(const double* c, const float* w_idx, double* u) {
    for (int j = 0; j < ORC_IDX_DIM; ++j) {
        double acc = 0.0;
        for (int d = 0; d < ORC_D; ++d) acc += c[d] * (double)w_idx[(size_t)d * ORC_IDX_DIM + j];
        u[j] = acc;
    }
}

/* ------------------------------------------------------------------------------------------
 * O1r -- RoPE at compressed positions (a layout variant.  [HF] storage paragraph: each entry
 * keeps its RoPE dims in bf16; in the base reading those dims are stored as given.  In this
 * variant the raw tokens' dims 448..511 arrive before rotary position encoding and the
 * compressor rotates them itself, at the entry's own position).  Readings: the rotation is
 * RoFormer's -- consecutive pairs, pair i = dims (448 + 2i, 449 + 2i) for i = 0..31, turned by
 * the angle pos * base^(-i/32); a compressed entry s of ratio m stands at its block's last
 * token, pos0 + (s+1) m - 1 (where it becomes visible), a window entry at its own token; the
 * indexer key is projected from the rotated pooled vector.
 * ---------------------------------------------------------------------------------------- */
void orc_rope_rotate(double* x, double pos, double base) {
    for (int i = 0; i < ORC_D_ROPE / 2; ++i) {
        double theta = pow(base, -(double)i / (double)(ORC_D_ROPE / 2));
        double a = pos * theta;
        double c = cos(a), s = sin(a);
        double x0 = x[ORC_D_NOPE + 2 * i], x1 = x[ORC_D_NOPE + 2 * i + 1];
        x[ORC_D_NOPE + 2 * i] = x0 * c - x1 * s;
        x[ORC_D_NOPE + 2 * i + 1] = x0 * s + x1 * c;
    }
}

/* O2, per-head variant (a layout variant of the indexer key: [HF] CSA paragraph scores "a
 * multi-head dot product" against the compressed entries; in the base reading the 4 indexer
 * heads share one 64-d key per entry).  Here every head h has its own projection W_h and its
 * own key: u_h = c . W_h, with w_idx [512][4][64] row-major (W_h[d][j] = w_idx[d*256 + h*64 + j]),
 * each head's key FP4-quantised as in the base (two groups of 32, power-of-two scales). */
void orc_indexer_key_raw_perhead(const double* c, const float* w_idx, double* u) {
    for (int h = 0; h < ORC_IDX_HEADS; ++h)
        for (int j = 0; j < ORC_IDX_DIM; ++j) {
            double acc = 0.0;
            for (int d = 0; d < ORC_D; ++d)
                acc += c[d] * (double)w_idx[(size_t)d * ORC_IDX_HEADS * ORC_IDX_DIM + h * ORC_IDX_DIM + j];
            u[h * ORC_IDX_DIM + j] = acc;
        }
}

/* O1 + O2 over a whole prefill: T tokens of one sequence -> floor(T/m) entries; the trailing
 * T mod m tokens form no entry.  ikey_out / iscale_out are written only when w_idx != NULL
 * (CSA; [HF] CSA paragraph: the lightning indexer runs over the 4x-compressed entries).
 * rope_base > 0: O1r, entry s rotated at position pos0 + (s+1) m - 1 after pooling. */
static void orc_compress_impl(const uint16_t* raw, const float* gate, const float* bias, const float* w_idx,
                              int64_t T, int m, int64_t pos0, double rope_base, double kv_scale, int key_heads,
                              uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out) {
    int64_t E = T / m;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < E; ++s) {
        double c[ORC_D], u[ORC_IDX_HEADS * ORC_IDX_DIM];
        orc_pool_block(raw + (size_t)s * m * ORC_D, gate + (size_t)s * m, bias, m, c);
        if (rope_base > 0.0) orc_rope_rotate(c, (double)(pos0 + (s + 1) * (int64_t)m - 1), rope_base);
        if (kv_scale != 1.0)
            orc_entry_encode_scaled(c, kv_scale, kv_out + (size_t)s * ORC_ENTRY_BYTES);
        else
            orc_entry_encode(c, kv_out + (size_t)s * ORC_ENTRY_BYTES);
        if (w_idx && key_heads == 1) {
            orc_indexer_key_raw(c, w_idx, u);
            orc_fp4_quantize64(u, ikey_out + (size_t)s * ORC_IKEY_BYTES, iscale_out + (size_t)s * 2);
        } else if (w_idx) {
            orc_indexer_key_raw_perhead(c, w_idx, u);
            for (int h = 0; h < ORC_IDX_HEADS; ++h)
                orc_fp4_quantize64(u + h * ORC_IDX_DIM, ikey_out + ((size_t)s * ORC_IDX_HEADS + h) * ORC_IKEY_BYTES,
                                   iscale_out + ((size_t)s * ORC_IDX_HEADS + h) * 2);
        }
    }
}

void orc_compress(const uint16_t* raw, const float* gate, const float* bias, const float* w_idx,
                  int64_t T, int m, uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out) {
    orc_compress_impl(raw, gate, bias, w_idx, T, m, 0, 0.0, 1.0, 1, kv_out, ikey_out, iscale_out);
}

/* O1r + O1 + O2: raw token 0 at position pos0, rotation base rope_base > 0. */
void orc_compress_rope(const uint16_t* raw, const float* gate, const float* bias, const float* w_idx,
                       int64_t T, int m, int64_t pos0, double rope_base, uint8_t* kv_out,
                       uint8_t* ikey_out, float* iscale_out) {
    orc_compress_impl(raw, gate, bias, w_idx, T, m, pos0, rope_base, 1.0, 1, kv_out, ikey_out, iscale_out);
}

/* Scaled FP8 entries: as orc_compress with entries encoded by orc_entry_encode_scaled (the
 * indexer key is projected from the unscaled pooled vector). */
void orc_compress_scaled(const uint16_t* raw, const float* gate, const float* bias, const float* w_idx,
                         int64_t T, int m, double kv_scale, uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out) {
    orc_compress_impl(raw, gate, bias, w_idx, T, m, 0, 0.0, kv_scale, 1, kv_out, ikey_out, iscale_out);
}

/* Per-head indexer keys: as orc_compress with w_idx [512][4][64]; ikey_out [E][4][32] (each
 * head's 32 code bytes as in the base), iscale_out [E][4][2]. */
void orc_compress_perhead(const uint16_t* raw, const float* gate, const float* bias, const float* w_idx,
                          int64_t T, int m, uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out) {
    orc_compress_impl(raw, gate, bias, w_idx, T, m, 0, 0.0, 1.0, ORC_IDX_HEADS, kv_out, ikey_out, iscale_out);
}

/* O1 (per-channel) + O2 over a whole prefill: gate [T][512], bias [m][512]. */
void orc_compress_channel(const uint16_t* raw, const float* gate, const float* bias, const float* w_idx,
                          int64_t T, int m, uint8_t* kv_out, uint8_t* ikey_out, float* iscale_out) {
    int64_t E = T / m;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < E; ++s) {
        double c[ORC_D], u[ORC_IDX_DIM];
        orc_pool_block_channel(raw + (size_t)s * m * ORC_D, gate + (size_t)s * m * ORC_D, bias, m, c);
        orc_entry_encode(c, kv_out + (size_t)s * ORC_ENTRY_BYTES);
        if (w_idx) {
            orc_indexer_key_raw(c, w_idx, u);
            orc_fp4_quantize64(u, ikey_out + (size_t)s * ORC_IKEY_BYTES, iscale_out + (size_t)s * 2);
        }
    }
}

/* ------------------------------------------------------------------------------------------
 * O3 -- lightning indexer score ([HF] CSA paragraph: "FP4, ReLU-scored multi-head dot
 * product"; [VEL] core technique 1: the indexer scores each compressed entry for the query).
 *   e_s = sum_h w_h * ReLU(q_h . k_s), over the 4 indexer heads, q and k both FP4.
 * The per-group dot of two E2M1 vectors is an exact integer multiple of 1/4 times the two
 * scales.  The fp32 score (the precision that decides the selection) is formed in this fixed
 * order, each step one IEEE fp32 operation:
 *   I_g   = sum over the group of (2*q_code_value)*(2*k_code_value)       (exact integer)
 *   s_g   = (qscale_g * kscale_g) * 0.25f
 *   d     = fmaf((float)I_1, s_1, (float)I_0 * s_0)
 *   r     = d > 0 ? d : 0
 *   e     = w_0*r_0;  e = fmaf(w_1, r_1, e);  e = fmaf(w_2, r_2, e);  e = fmaf(w_3, r_3, e)
 * score64 is the same quantity in float64 without intermediate rounding.
 * ---------------------------------------------------------------------------------------- */
static int orc_twice_e2m1(uint8_t c) {       /* 2 * value of an E2M1 code: an integer */
    return (int)lrint(2.0 * orc_e2m1_decode(c));
}

static void orc_indexer_scores_impl(const uint8_t* ikeys, const float* iscales, int64_t n, int key_heads,
                                    const float* q_idx, const float* head_w, float* score32, double* score64) {
    uint8_t qc[ORC_IDX_HEADS][ORC_IKEY_BYTES];
    float qs[ORC_IDX_HEADS][2];
    double qd[ORC_IDX_HEADS][ORC_IDX_DIM];
    for (int h = 0; h < ORC_IDX_HEADS; ++h) {
        double qv[ORC_IDX_DIM];
        for (int d = 0; d < ORC_IDX_DIM; ++d) qv[d] = (double)q_idx[h * ORC_IDX_DIM + d];
        orc_fp4_quantize64(qv, qc[h], qs[h]);
        orc_fp4_dequantize64(qc[h], qs[h], qd[h]);
    }
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < n; ++s) {
        float r32[ORC_IDX_HEADS];
        double e64 = 0.0;
        for (int h = 0; h < ORC_IDX_HEADS; ++h) {
            /* the head's key: the entry's one key, or (per-head keys) key h of the entry */
            const int kh = key_heads == 1 ? 0 : h;
            const uint8_t* kc = ikeys + ((size_t)s * key_heads + kh) * ORC_IKEY_BYTES;
            const float* ks = iscales + ((size_t)s * key_heads + kh) * 2;
            double kd[ORC_IDX_DIM];
            orc_fp4_dequantize64(kc, ks, kd);
            long I[2] = {0, 0};
            double dot = 0.0;
            for (int d = 0; d < ORC_IDX_DIM; ++d) {
                I[d / ORC_IDX_GROUP] += (long)orc_twice_e2m1(orc_nibble(qc[h], d)) *
                                        (long)orc_twice_e2m1(orc_nibble(kc, d));
                dot += qd[h][d] * kd[d];
            }
            float s0 = (qs[h][0] * ks[0]) * 0.25f;
            float s1 = (qs[h][1] * ks[1]) * 0.25f;
            float p0 = (float)I[0] * s0;
            float d32 = fmaf((float)I[1], s1, p0);
            r32[h] = d32 > 0.0f ? d32 : 0.0f;
            e64 += (double)head_w[h] * (dot > 0.0 ? dot : 0.0);
        }
        float e = head_w[0] * r32[0];
        e = fmaf(head_w[1], r32[1], e);
        e = fmaf(head_w[2], r32[2], e);
        e = fmaf(head_w[3], r32[3], e);
        if (score32) score32[s] = e;
        if (score64) score64[s] = e64;
    }
}

void orc_indexer_scores(const uint8_t* ikeys, const float* iscales, int64_t n,
                        const float* q_idx, const float* head_w, float* score32, double* score64) {
    orc_indexer_scores_impl(ikeys, iscales, n, 1, q_idx, head_w, score32, score64);
}

/* O3 with per-head keys: ikeys [n][4][32], iscales [n][4][2]; head h scores against key h,
 * in the same fp32 operation order. */
void orc_indexer_scores_perhead(const uint8_t* ikeys, const float* iscales, int64_t n,
                                const float* q_idx, const float* head_w, float* score32, double* score64) {
    orc_indexer_scores_impl(ikeys, iscales, n, ORC_IDX_HEADS, q_idx, head_w, score32, score64);
}

/* ------------------------------------------------------------------------------------------
 * O4 -- top-k ([HF] CSA paragraph / Figure 3: the indexer picks the top-k compressed blocks
 * per query).  Order by (score desc, index asc); keep the first min(k, n); return them in
 * ascending index order, padded with -1.
 * ---------------------------------------------------------------------------------------- */
typedef struct { double score; int64_t idx; } orc_pair;

static int orc_pair_cmp(const void* a, const void* b) {
    const orc_pair* x = (const orc_pair*)a;
    const orc_pair* y = (const orc_pair*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

static int orc_i32_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

static void orc_topk_pairs(orc_pair* p, int64_t n, int k, int32_t* out) {
    qsort(p, (size_t)n, sizeof(orc_pair), orc_pair_cmp);
    int64_t take = n < k ? n : k;
    for (int64_t i = 0; i < take; ++i) out[i] = (int32_t)p[i].idx;
    qsort(out, (size_t)take, sizeof(int32_t), orc_i32_cmp);
    for (int64_t i = take; i < k; ++i) out[i] = -1;
}

void orc_topk(const float* score32, int64_t n, int k, int32_t* out) {
    orc_pair* p = (orc_pair*)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) { p[i].score = (double)score32[i]; p[i].idx = i; }
    orc_topk_pairs(p, n, k, out);
    free(p);
}

void orc_topk64(const double* score64, int64_t n, int k, int32_t* out) {
    orc_pair* p = (orc_pair*)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) { p[i].score = score64[i]; p[i].idx = i; }
    orc_topk_pairs(p, n, k, out);
    free(p);
}

/* Batched indexer + top-k for B sequences: keys [B][cap], the visible count of sequence b is
 * min(seq_len[b] / ratio, cap). */
static void orc_indexer_topk_batch_impl(const uint8_t* ikeys, const float* iscales, int64_t cap, int key_heads,
                                        const int32_t* seq_len, int ratio, const float* q_idx,
                                        const float* head_w, int B, int k, int32_t* out) {
    for (int b = 0; b < B; ++b) {
        int64_t n = seq_len[b] / ratio;
        if (n > cap) n = cap;
        float* sc = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
        orc_indexer_scores_impl(ikeys + (size_t)b * cap * key_heads * ORC_IKEY_BYTES,
                                iscales + (size_t)b * cap * key_heads * 2, n, key_heads,
                                q_idx + (size_t)b * ORC_IDX_HEADS * ORC_IDX_DIM,
                                head_w + (size_t)b * ORC_IDX_HEADS, sc, NULL);
        orc_topk(sc, n, k, out + (size_t)b * k);
        free(sc);
    }
}
void orc_indexer_topk_batch(const uint8_t* ikeys, const float* iscales, int64_t cap,
                            const int32_t* seq_len, int ratio, const float* q_idx,
                            const float* head_w, int B, int k, int32_t* out) {
    orc_indexer_topk_batch_impl(ikeys, iscales, cap, 1, seq_len, ratio, q_idx, head_w, B, k, out);
}
/* Per-head keys: ikeys [B][cap][4][32], iscales [B][cap][4][2]. */
void orc_indexer_topk_batch_perhead(const uint8_t* ikeys, const float* iscales, int64_t cap,
                                    const int32_t* seq_len, int ratio, const float* q_idx,
                                    const float* head_w, int B, int k, int32_t* out) {
    orc_indexer_topk_batch_impl(ikeys, iscales, cap, ORC_IDX_HEADS, seq_len, ratio, q_idx, head_w, B, k, out);
}

/* ------------------------------------------------------------------------------------------
 * O5 -- hybrid decode attention for one query token of one sequence ([HF] CSA paragraph and
 * Figure 3: attention over the selected compressed entries plus a sliding-window branch over
 * the most recent uncompressed tokens; HCA paragraph and Figure 4: dense attention over every
 * compressed entry, same window branch; [VEL] core techniques 1-2).
 * Keys = values = the decoded 512-vectors of:
 *   - sparse mode (sel != NULL): the entries listed in sel[0..k) that are >= 0;
 *   - dense mode  (sel == NULL): every visible entry s < min(seq_len / ratio, cap);
 *   - plus the window: raw tokens t in [max(0, seq_len - W), seq_len), ring slot t mod W.
 * For each head h: l_j = scale * q_h . K_j; out_h = sum_j softmax(l)_j V_j; lse_h = log sum exp.
 * Returns 0, or -1 when a selected index is not a visible entry.
 * An empty key set gives out = 0 and lse = -inf.
 * ---------------------------------------------------------------------------------------- */
static int orc_attention_impl(const uint16_t* q, int H, const uint8_t* comp_kv, int64_t cap, int ratio,
                              const int32_t* sel, int k, const uint8_t* win_kv, int W, int32_t seq_len,
                              double scale, double kv_scale, double* out, double* lse) {
    int64_t n_vis = seq_len / ratio;
    if (n_vis > cap) n_vis = cap;
    int64_t n_comp = 0;
    if (sel) {
        for (int i = 0; i < k; ++i) {
            if (sel[i] < 0) continue;
            if (sel[i] >= n_vis) return -1;
            ++n_comp;
        }
    } else {
        n_comp = n_vis;
    }
    int64_t w0 = seq_len - W > 0 ? seq_len - W : 0;
    int64_t n_win = W > 0 ? seq_len - w0 : 0;
    int64_t L = n_comp + n_win;
    double* kv = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * ORC_D);
    int64_t j = 0;
    if (sel) {
        for (int i = 0; i < k; ++i)
            if (sel[i] >= 0)
                orc_entry_decode_scaled(comp_kv + (size_t)sel[i] * ORC_ENTRY_BYTES, kv_scale, kv + (size_t)(j++) * ORC_D);
    } else {
        for (int64_t s = 0; s < n_vis; ++s)
            orc_entry_decode_scaled(comp_kv + (size_t)s * ORC_ENTRY_BYTES, kv_scale, kv + (size_t)(j++) * ORC_D);
    }
    for (int64_t t = w0; t < seq_len && W > 0; ++t)
        orc_entry_decode_scaled(win_kv + (size_t)(t % W) * ORC_ENTRY_BYTES, kv_scale, kv + (size_t)(j++) * ORC_D);

    double* logit = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int h = 0; h < H; ++h) {
        double qd[ORC_D];
        for (int d = 0; d < ORC_D; ++d) qd[d] = orc_bf16_decode(q[(size_t)h * ORC_D + d]);
        double* o = out + (size_t)h * ORC_D;
        for (int d = 0; d < ORC_D; ++d) o[d] = 0.0;
        if (L == 0) { lse[h] = -INFINITY; continue; }
        double mx = -INFINITY;
        for (int64_t i = 0; i < L; ++i) {
            double acc = 0.0;
            const double* kr = kv + (size_t)i * ORC_D;
            for (int d = 0; d < ORC_D; ++d) acc += qd[d] * kr[d];
            logit[i] = scale * acc;
            if (logit[i] > mx) mx = logit[i];
        }
        double l = 0.0;
        for (int64_t i = 0; i < L; ++i) {
            double p = exp(logit[i] - mx);
            l += p;
            const double* vr = kv + (size_t)i * ORC_D;
            for (int d = 0; d < ORC_D; ++d) o[d] += p * vr[d];
        }
        for (int d = 0; d < ORC_D; ++d) o[d] /= l;
        lse[h] = mx + log(l);
    }
    free(logit);
    free(kv);
    return 0;
}

int orc_attention(const uint16_t* q, int H, const uint8_t* comp_kv, int64_t cap, int ratio,
                  const int32_t* sel, int k, const uint8_t* win_kv, int W, int32_t seq_len,
                  double scale, double* out, double* lse) {
    return orc_attention_impl(q, H, comp_kv, cap, ratio, sel, k, win_kv, W, seq_len, scale, 1.0, out, lse);
}

/* Batched attention: q [B][H][512]; caches [B][cap] and [B][W]; sel [B][k] or NULL;
 * kv_scale: scaled FP8 entries (1: the base layout). */
int orc_attention_batch_scaled(const uint16_t* q, int H, const uint8_t* comp_kv, int64_t cap, int ratio,
                               const int32_t* sel, int k, const uint8_t* win_kv, int W,
                               const int32_t* seq_len, int B, double scale, double kv_scale, double* out,
                               double* lse) {
    int rc = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        rc |= orc_attention_impl(q + (size_t)b * H * ORC_D, H, comp_kv + (size_t)b * cap * ORC_ENTRY_BYTES,
                                 cap, ratio, sel ? sel + (size_t)b * k : NULL, k,
                                 win_kv + (size_t)b * (W > 0 ? W : 0) * ORC_ENTRY_BYTES, W, seq_len[b],
                                 scale, kv_scale, out + (size_t)b * H * ORC_D, lse + (size_t)b * H);
    }
    return rc;
}

int orc_attention_batch(const uint16_t* q, int H, const uint8_t* comp_kv, int64_t cap, int ratio,
                        const int32_t* sel, int k, const uint8_t* win_kv, int W,
                        const int32_t* seq_len, int B, double scale, double* out, double* lse) {
    return orc_attention_batch_scaled(q, H, comp_kv, cap, ratio, sel, k, win_kv, W, seq_len, B, scale, 1.0, out, lse);
}

/* ------------------------------------------------------------------------------------------
 * O6 -- appending one token to a layer's cache state ([VEL] "KV cache layout handled
 * separately": compressed CSA/HCA caches, a separate sliding-window state for recent tokens,
 * and a separately kept uncompressed tail).
 * State of one sequence: comp_kv [cap][576], ikeys [cap][32] + iscales [cap][2] (CSA only),
 * win_kv [W][576] ring, tail_kv [m][512] bf16 + tail_gate [m], *seq_len.
 * Token t = *seq_len:  window slot t mod W <- entry(x); tail slot t mod m <- (x, gate);
 * when (t+1) mod m == 0 the tail (slot j = token s*m + j) is pooled into entry s = t / m
 * (plus its indexer key when w_idx != NULL).  Returns -1 and changes nothing when entry s
 * would not fit in cap.
 * ---------------------------------------------------------------------------------------- */
/* rope_base > 0: O1r -- the window entry of token t rotated at position t, the completed
 * entry s at position t = (s+1) m - 1, its block's last token. */
static int orc_append_impl(int m, int W, int64_t cap, uint8_t* comp_kv, uint8_t* ikeys, float* iscales,
                           uint8_t* win_kv, uint16_t* tail_kv, float* tail_gate, int32_t* seq_len,
                           const float* bias, const float* w_idx, const uint16_t* x, float gate,
                           double rope_base, double kv_scale, int key_heads) {
    int32_t t = *seq_len;
    int complete = ((t + 1) % m) == 0;
    int64_t s = t / m;
    if (complete && s >= cap) return -1;
    if (W > 0) {
        double xd[ORC_D];
        for (int d = 0; d < ORC_D; ++d) xd[d] = orc_bf16_decode(x[d]);
        if (rope_base > 0.0) orc_rope_rotate(xd, (double)t, rope_base);
        orc_entry_encode_scaled(xd, kv_scale, win_kv + (size_t)(t % W) * ORC_ENTRY_BYTES);
    }
    memcpy(tail_kv + (size_t)(t % m) * ORC_D, x, sizeof(uint16_t) * ORC_D);
    tail_gate[t % m] = gate;
    if (complete) {
        double c[ORC_D], u[ORC_IDX_HEADS * ORC_IDX_DIM];
        orc_pool_block(tail_kv, tail_gate, bias, m, c);
        if (rope_base > 0.0) orc_rope_rotate(c, (double)t, rope_base);
        orc_entry_encode_scaled(c, kv_scale, comp_kv + (size_t)s * ORC_ENTRY_BYTES);
        if (w_idx && key_heads == 1) {
            orc_indexer_key_raw(c, w_idx, u);
            orc_fp4_quantize64(u, ikeys + (size_t)s * ORC_IKEY_BYTES, iscales + (size_t)s * 2);
        } else if (w_idx) {
            orc_indexer_key_raw_perhead(c, w_idx, u);
            for (int h = 0; h < ORC_IDX_HEADS; ++h)
                orc_fp4_quantize64(u + h * ORC_IDX_DIM, ikeys + ((size_t)s * ORC_IDX_HEADS + h) * ORC_IKEY_BYTES,
                                   iscales + ((size_t)s * ORC_IDX_HEADS + h) * 2);
        }
    }
    *seq_len = t + 1;
    return 0;
}

int orc_append(int m, int W, int64_t cap, uint8_t* comp_kv, uint8_t* ikeys, float* iscales,
               uint8_t* win_kv, uint16_t* tail_kv, float* tail_gate, int32_t* seq_len,
               const float* bias, const float* w_idx, const uint16_t* x, float gate) {
    return orc_append_impl(m, W, cap, comp_kv, ikeys, iscales, win_kv, tail_kv, tail_gate, seq_len, bias,
                           w_idx, x, gate, 0.0, 1.0, 1);
}

/* The same for B sequences, one token each: x [B][512], gate [B]; rope_base as above (0: none);
 * kv_scale: scaled FP8 entries (1: the base layout); key_heads: 1 (one shared indexer key) or 4
 * (per-head keys, w_idx [512][4][64], ikeys [B][cap][4][32], iscales [B][cap][4][2]). */
int orc_append_batch_variant(int m, int W, int64_t cap, int B, uint8_t* comp_kv, uint8_t* ikeys,
                             float* iscales, uint8_t* win_kv, uint16_t* tail_kv, float* tail_gate,
                             int32_t* seq_len, const float* bias, const float* w_idx, const uint16_t* x,
                             const float* gate, double rope_base, double kv_scale, int key_heads) {
    int rc = 0;
    for (int b = 0; b < B; ++b) {
        rc |= orc_append_impl(m, W, cap, comp_kv + (size_t)b * cap * ORC_ENTRY_BYTES,
                              ikeys ? ikeys + (size_t)b * cap * key_heads * ORC_IKEY_BYTES : NULL,
                              iscales ? iscales + (size_t)b * cap * key_heads * 2 : NULL,
                              win_kv + (size_t)b * (W > 0 ? W : 0) * ORC_ENTRY_BYTES,
                              tail_kv + (size_t)b * m * ORC_D, tail_gate + (size_t)b * m, seq_len + b,
                              bias, w_idx, x + (size_t)b * ORC_D, gate[b], rope_base, kv_scale, key_heads);
    }
    return rc;
}

int orc_append_batch(int m, int W, int64_t cap, int B, uint8_t* comp_kv, uint8_t* ikeys,
                     float* iscales, uint8_t* win_kv, uint16_t* tail_kv, float* tail_gate,
                     int32_t* seq_len, const float* bias, const float* w_idx, const uint16_t* x,
                     const float* gate) {
    return orc_append_batch_variant(m, W, cap, B, comp_kv, ikeys, iscales, win_kv, tail_kv, tail_gate, seq_len,
                                    bias, w_idx, x, gate, 0.0, 1.0, 1);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
