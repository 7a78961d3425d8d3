/*
 * nvkv_oracle.c -- plain, slow float64 CPU oracle for the NVFP4 paged KV path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, table, header or constant generator
 * with the CUDA path.
 *
 * What it computes, and where the statement comes from:
 *
 *   NVFP4 KV storage -- "gzenz/ninfer" README, "Fork changes vs upstream",
 *   subsection "Context and model", NVFP4 KV cache bullet: each KV element is
 *   a 4-bit E2M1 code and every group of 16 elements shares one E4M3 scale.
 *   The groups run along head_dim.  The scale of a group is the E4M3 value
 *   nearest to amax/6 (amax = max |x| over the 16 inputs, 6 = the largest
 *   E2M1 magnitude); each element's code is the E2M1 value nearest to
 *   x/scale.  The pages fix none of the rounding details; the readings used
 *   here are:
 *     - both roundings are round-to-nearest with ties to the even encoding;
 *     - a scale above the E4M3 maximum (448) saturates to 448;
 *     - an x/scale above 6 saturates to 6;
 *     - a group whose scale rounds to 0 (including an all-zero group) has all
 *       codes 0;
 *     - a magnitude that rounds to 0 is stored as code 0 (no negative zero);
 *     - there is no second, per-tensor scale.
 *
 *   Paged pool -- "knoopx/ninfer" README, "Quick start" and "Capabilities and
 *   limits" (a single KV pool, sized at startup, serves all active requests).
 *   Pages hold 16 token slots; the byte layout of a page is this project's
 *   own (the pages are silent), written out in pool_offset_* below.
 *
 *   Attention -- "knoopx/ninfer" README, "Capabilities and limits" (batched
 *   decode, MTP verify with one to five drafts, chunked prefill): for query
 *   row q at absolute position pos, attending kv-head h,
 *       s_j = sm_scale * sum_d q[d] * Khat[j][d]          for j <= pos
 *       p_j = exp(s_j - max s) / sum_i exp(s_i - max s)
 *       out = sum_j p_j * Vhat[j]
 *   with Khat, Vhat the dequantised cache (code value times scale).  Query
 *   head hq reads kv-head hq / (Hq / Hkv) (consecutive grouping).
 *
 * Everything is computed in IEEE double with the default rounding mode.
 * Build with plain -O2 (never -ffast-math: it would change rounding and NaN
 * handling).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16: the top 16 bits of an IEEE binary32. */
double oracle_bf16_value(uint16_t bits) {
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* E2M1: sign bit, 2 exponent bits (bias 1), 1 mantissa bit; no inf, no NaN.
 *   exponent field 0:  (-1)^s * (m/2)                (subnormal)
 *   exponent field e:  (-1)^s * 2^(e-1) * (1 + m/2)                        */
double oracle_e2m1_value(int code) {
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? (m / 2.0) : ldexp(1.0 + m / 2.0, e - 1);
    return s ? -mag : mag;
}

/* E4M3, "FN" flavour: sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
 * no infinity; exponent field 15 with mantissa 7 is NaN.
 *   exponent field 0:  (-1)^s * 2^-6 * (m/8)         (subnormal)
 *   exponent field e:  (-1)^s * 2^(e-7) * (1 + m/8)                        */
double oracle_e4m3_value(int byte) {
    int s = (byte >> 7) & 1;
    int e = (byte >> 3) & 15;
    int m = byte & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round a non-negative real k to an integer, ties to the even integer. */
static double round_half_even(double k) {
    double f = floor(k);
    double frac = k - f; /* exact: k and f share an exponent range */
    if (frac > 0.5) return f + 1.0;
    if (frac < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Encode an exactly representable, non-negative, finite E4M3 value. */
static uint8_t e4m3_encode(double v) {
    if (v == 0.0) return 0;
    if (v < ldexp(1.0, -6)) { /* subnormal: v = m * 2^-9 */
        return (uint8_t)(int)(v / ldexp(1.0, -9));
    }
    int e2;
    frexp(v, &e2); /* v = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1; /* v = (1 + m/8) * 2^E */
    int m = (int)((v / ldexp(1.0, E) - 1.0) * 8.0);
    return (uint8_t)(((E + 7) << 3) | m);
}

/* Nearest E4M3 value to x >= 0, ties to even mantissa, saturating at 448.
 *
 * Within the binade [2^E, 2^(E+1)) the E4M3 values are spaced 2^(E-3); the
 * subnormal range [0, 2^-6) uses the spacing of the smallest binade, 2^-9.
 * Dividing by the spacing is exact (power of two); rounding the quotient
 * half-to-even picks the even mantissa on a tie, because the integer
 * quotient of a representable value has the mantissa as its low bits. */
uint8_t oracle_e4m3_round(double x) {
    if (!(x > 0.0)) return 0;
    if (x >= 448.0) return 0x7E; /* 448 = largest finite E4M3 */
    int e2;
    frexp(x, &e2);
    int E = e2 - 1; /* 2^E <= x < 2^(E+1) */
    if (E < -6) E = -6;
    double spacing = ldexp(1.0, E - 3);
    double v = round_half_even(x / spacing) * spacing;
    return e4m3_encode(v);
}

/* Index 0..7 of the E2M1 magnitude nearest to r >= 0, ties to the even
 * index (even mantissa bit), saturating at 6.
 *   magnitudes by index: 0, 0.5, 1, 1.5, 2, 3, 4, 6
 * Spacing is 0.5 below 2, 1 in [2, 4) and 2 in [4, 8). */
int oracle_e2m1_round_index(double r) {
    if (r >= 6.0) return 7;
    double spacing = (r < 2.0) ? 0.5 : (r < 4.0 ? 1.0 : 2.0);
    double v = round_half_even(r / spacing) * spacing;
    if (v == 0.0) return 0;
    if (v == 0.5) return 1;
    int e2;
    frexp(v, &e2);
    int E = e2 - 1;                                 /* 0, 1 or 2 */
    int m = (v / ldexp(1.0, E) - 1.0) == 0.5 ? 1 : 0; /* mantissa bit */
    return ((E + 1) << 1) | m;
}

/* Quantise one group of 16 bf16 values (given as raw bits) into 16 E2M1
 * codes (one per byte, low nibble) and one E4M3 scale byte.
 *
 * amax / 6 and x / scale are computed in double.  Neither quotient can land
 * on a rounding midpoint unless it equals it exactly: a midpoint times the
 * divisor has at most 7 significant bits while the dividend has at most 8,
 * so an inexact quotient is at least 2^-9 (relative) away from any midpoint,
 * far more than the 2^-53 double rounding error.  The decisions are
 * therefore those of exact arithmetic. */
void oracle_quantize_group(const uint16_t x[16], uint8_t codes[16], uint8_t *scale_byte) {
    double amax = 0.0;
    for (int i = 0; i < 16; ++i) {
        double a = fabs(oracle_bf16_value(x[i]));
        if (a > amax) amax = a;
    }
    uint8_t sb = oracle_e4m3_round(amax / 6.0);
    double scale = oracle_e4m3_value(sb);
    *scale_byte = sb;
    for (int i = 0; i < 16; ++i) {
        if (scale == 0.0) {
            codes[i] = 0;
            continue;
        }
        double xv = oracle_bf16_value(x[i]);
        int idx = oracle_e2m1_round_index(fabs(xv) / scale);
        int neg = (x[i] >> 15) & 1;
        codes[i] = (uint8_t)((idx == 0) ? 0 : ((neg << 3) | idx));
    }
}

/* Quantise ngroups consecutive groups of 16 (x: [ngroups][16] bf16 bits)
 * into codes [ngroups][16] and scales [ngroups]. */
void oracle_quantize_groups(const uint16_t *x, long ngroups, uint8_t *codes, uint8_t *scales) {
    for (long g = 0; g < ngroups; ++g) oracle_quantize_group(x + 16 * g, codes + 16 * g, scales + g);
}

/* Dequantise: code value times scale value (exact in double). */
double oracle_dequant(int code, int scale_byte) {
    return oracle_e2m1_value(code) * oracle_e4m3_value(scale_byte);
}

/* Quantise then dequantise one row of D elements (D a multiple of 16). */
void oracle_qdq_row(const uint16_t *x, int D, double *out) {
    uint8_t codes[16], sb;
    for (int g = 0; g < D / 16; ++g) {
        oracle_quantize_group(x + 16 * g, codes, &sb);
        for (int i = 0; i < 16; ++i) out[16 * g + i] = oracle_dequant(codes[i], sb);
    }
}

/* oracle_qdq_row over n consecutive rows of D elements. */
void oracle_qdq_rows(const uint16_t *x, long n, int D, double *out) {
    for (long r = 0; r < n; ++r) oracle_qdq_row(x + (size_t)r * D, D, out + (size_t)r * D);
}

/* ------------------------------------------------------------------------ */
/* Page layout                                                               */
/* ------------------------------------------------------------------------ */
/*
 * A page holds 16 token slots for every kv-head.  Page p starts at byte
 * p * page_bytes, page_bytes = 18 * Hkv * D.  Inside the page, kv-head h
 * owns the block starting at h * 18 * D, laid out as:
 *
 *   K codes   [16 slots][D/2]  at  0       byte (slot, i): element 2i in the
 *                                          low nibble, 2i+1 in the high one
 *   K scales  [16 slots][D/16] at  8*D     byte (slot, g): group g of the row
 *   V codes   [D][8]           at  9*D     byte (d, i): slot 2i in the low
 *                                          nibble, slot 2i+1 in the high one
 *   V scales  [D/16][16 slots] at 17*D     byte (g, slot)
 */
size_t oracle_page_bytes(int Hkv, int D) { return (size_t)18 * Hkv * D; }

static size_t head_base(int page, int h, int Hkv, int D) {
    return (size_t)page * oracle_page_bytes(Hkv, D) + (size_t)h * 18 * D;
}

/* Byte and nibble (0 = low, 1 = high) holding element d of slot s. */
static size_t pool_offset_kcode(int page, int h, int s, int d, int Hkv, int D, int *nib) {
    *nib = d & 1;
    return head_base(page, h, Hkv, D) + (size_t)s * (D / 2) + d / 2;
}
static size_t pool_offset_kscale(int page, int h, int s, int g, int Hkv, int D) {
    return head_base(page, h, Hkv, D) + (size_t)8 * D + (size_t)s * (D / 16) + g;
}
static size_t pool_offset_vcode(int page, int h, int s, int d, int Hkv, int D, int *nib) {
    *nib = s & 1;
    return head_base(page, h, Hkv, D) + (size_t)9 * D + (size_t)d * 8 + s / 2;
}
static size_t pool_offset_vscale(int page, int h, int s, int g, int Hkv, int D) {
    return head_base(page, h, Hkv, D) + (size_t)17 * D + (size_t)g * 16 + s;
}

static void put_nibble(uint8_t *pool, size_t off, int nib, uint8_t code) {
    if (nib)
        pool[off] = (uint8_t)((pool[off] & 0x0F) | (code << 4));
    else
        pool[off] = (uint8_t)((pool[off] & 0xF0) | (code & 0x0F));
}
static int get_nibble(const uint8_t *pool, size_t off, int nib) {
    return nib ? (pool[off] >> 4) : (pool[off] & 0x0F);
}

/* Quantise one K or V row (all kv-heads) into the slot for absolute
 * position pos of a sequence whose page table row is page_row. */
static void write_row(uint8_t *pool, int Hkv, int D, const int32_t *page_row, int pos,
                      const uint16_t *k_row, const uint16_t *v_row) {
    int page = page_row[pos / 16];
    int s = pos % 16;
    uint8_t codes[16], sb;
    int nib;
    for (int h = 0; h < Hkv; ++h) {
        for (int g = 0; g < D / 16; ++g) {
            oracle_quantize_group(k_row + (size_t)h * D + 16 * g, codes, &sb);
            for (int i = 0; i < 16; ++i) {
                size_t off = pool_offset_kcode(page, h, s, 16 * g + i, Hkv, D, &nib);
                put_nibble(pool, off, nib, codes[i]);
            }
            pool[pool_offset_kscale(page, h, s, g, Hkv, D)] = sb;

            oracle_quantize_group(v_row + (size_t)h * D + 16 * g, codes, &sb);
            for (int i = 0; i < 16; ++i) {
                size_t off = pool_offset_vcode(page, h, s, 16 * g + i, Hkv, D, &nib);
                put_nibble(pool, off, nib, codes[i]);
            }
            pool[pool_offset_vscale(page, h, s, g, Hkv, D)] = sb;
        }
    }
}

/* Append: rows cu_new[b] .. cu_new[b+1]-1 of k_new / v_new ([rows][Hkv][D]
 * bf16 bits) belong to sequence b and land at positions
 * kv_lens[b] - n_b .. kv_lens[b] - 1 (n_b = cu_new[b+1] - cu_new[b]), i.e.
 * kv_lens holds the lengths after the append. */
void oracle_append(uint8_t *pool, int Hkv, int D, const int32_t *page_table,
                   int max_pages_per_seq, const int32_t *kv_lens, int batch,
                   const uint16_t *k_new, const uint16_t *v_new, const int32_t *cu_new) {
    for (int b = 0; b < batch; ++b) {
        int n = cu_new[b + 1] - cu_new[b];
        for (int i = 0; i < n; ++i) {
            int row = cu_new[b] + i;
            int pos = kv_lens[b] - n + i;
            write_row(pool, Hkv, D, page_table + (size_t)b * max_pages_per_seq, pos,
                      k_new + (size_t)row * Hkv * D, v_new + (size_t)row * Hkv * D);
        }
    }
}

/* Read back one dequantised row (kv-head h, absolute position pos) from a
 * pool image.  is_v selects V (1) or K (0). */
void oracle_pool_read_row(const uint8_t *pool, int Hkv, int D, const int32_t *page_row,
                          int pos, int h, int is_v, double *out) {
    int page = page_row[pos / 16];
    int s = pos % 16;
    int nib;
    for (int d = 0; d < D; ++d) {
        int g = d / 16, code, sb;
        if (is_v) {
            size_t off = pool_offset_vcode(page, h, s, d, Hkv, D, &nib);
            code = get_nibble(pool, off, nib);
            sb = pool[pool_offset_vscale(page, h, s, g, Hkv, D)];
        } else {
            size_t off = pool_offset_kcode(page, h, s, d, Hkv, D, &nib);
            code = get_nibble(pool, off, nib);
            sb = pool[pool_offset_kscale(page, h, s, g, Hkv, D)];
        }
        out[d] = oracle_dequant(code, sb);
    }
}

/* ------------------------------------------------------------------------ */
/* Rotary position embedding of K, fused with quantise-append               */
/* ------------------------------------------------------------------------ */
/* "gzenz/ninfer" README, "Fork changes vs upstream" -> "Context and model":
 * YaRN context extension, stated there as linear RoPE scaling (positions
 * divided by a scaling factor).  The pages fix nothing else; the readings:
 * the first rotary_dim elements of a head rotate, element i paired with
 * element i + rotary_dim/2 (i < rotary_dim/2), by the angle
 * (pos / scale) * base^(-2i / rotary_dim); the remaining elements pass
 * through.  V is not rotated. */

/* (cos, sin) of the angle for positions 0 .. max_pos-1 and pairs
 * 0 .. rotary_dim/2-1, computed in double and rounded once to float:
 * cs[(pos * rotary_dim/2 + i) * 2 + {0, 1}]. */
void oracle_rope_table(int max_pos, int rotary_dim, double base, double scale, float *cs) {
    int h = rotary_dim / 2;
    for (int p = 0; p < max_pos; ++p)
        for (int i = 0; i < h; ++i) {
            double inv_freq = pow(base, -2.0 * i / rotary_dim);
            double a = ((double)p / scale) * inv_freq;
            cs[((size_t)p * h + i) * 2 + 0] = (float)cos(a);
            cs[((size_t)p * h + i) * 2 + 1] = (float)sin(a);
        }
}

/* Rotate one bf16 row of D elements in float, in the stated operation
 * order (the fused append kernel's): with c, s the float table entries,
 *   x' = fma(x, c, -(y * s)),   y' = fma(y, c, x * s),
 * each product y*s and x*s rounded to float, fma rounded once. */
void oracle_rope_rotate_f32(const uint16_t *row, int D, int rotary_dim, const float *cs_pos,
                            float *out) {
    int h = rotary_dim / 2;
    for (int d = 0; d < D; ++d) out[d] = (float)oracle_bf16_value(row[d]);
    for (int i = 0; i < h; ++i) {
        float c = cs_pos[2 * i], sn = cs_pos[2 * i + 1];
        float x = (float)oracle_bf16_value(row[i]), y = (float)oracle_bf16_value(row[i + h]);
        float ys = y * sn, xs = x * sn;
        out[i] = fmaf(x, c, -ys);
        out[i + h] = fmaf(y, c, xs);
    }
}

/* Quantise one group of 16 float values.  The scale is taken from the
 * float quotient amax / 6 rounded to E4M3 (what the kernel computes); for
 * normal values this is the decision of the exact quotient too (amax lies on
 * a grid 4-8 float ulps of amax/6 wide, so an inexact float quotient is at
 * least 2/3 ulp away from any E4M3 midpoint).  Codes: as for bf16 groups; an
 * inexact x / scale is at least 2^-24 (relative) away from an E2M1
 * midpoint, far more than the double rounding error. */
void oracle_quantize_group_f32(const float x[16], uint8_t codes[16], uint8_t *scale_byte) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float q = amax / 6.0f;
    uint8_t sb = oracle_e4m3_round((double)q);
    double scale = oracle_e4m3_value(sb);
    *scale_byte = sb;
    for (int i = 0; i < 16; ++i) {
        if (scale == 0.0) {
            codes[i] = 0;
            continue;
        }
        int idx = oracle_e2m1_round_index(fabs((double)x[i]) / scale);
        int neg = signbit(x[i]) ? 1 : 0;
        codes[i] = (uint8_t)((idx == 0) ? 0 : ((neg << 3) | idx));
    }
}

/* Append with K rotated at its position (table cs as from
 * oracle_rope_table, max_pos rows); V as oracle_append. */
void oracle_append_rope(uint8_t *pool, int Hkv, int D, const int32_t *page_table,
                        int max_pages_per_seq, const int32_t *kv_lens, int batch,
                        const uint16_t *k_new, const uint16_t *v_new, const int32_t *cu_new,
                        int rotary_dim, const float *cs, int max_pos) {
    float krot[512];
    uint8_t codes[16], sb;
    int nib;
    for (int b = 0; b < batch; ++b) {
        int n = cu_new[b + 1] - cu_new[b];
        const int32_t *page_row = page_table + (size_t)b * max_pages_per_seq;
        for (int i = 0; i < n; ++i) {
            int row = cu_new[b] + i;
            int pos = kv_lens[b] - n + i;
            if (pos >= max_pos) continue;  /* no table row: the kernel skips it too */
            int page = page_row[pos / 16], s = pos % 16;
            for (int hh = 0; hh < Hkv; ++hh) {
                const uint16_t *kr = k_new + ((size_t)row * Hkv + hh) * D;
                const uint16_t *vr = v_new + ((size_t)row * Hkv + hh) * D;
                oracle_rope_rotate_f32(kr, D, rotary_dim, cs + (size_t)pos * (rotary_dim / 2) * 2,
                                       krot);
                for (int g = 0; g < D / 16; ++g) {
                    oracle_quantize_group_f32(krot + 16 * g, codes, &sb);
                    for (int e = 0; e < 16; ++e) {
                        size_t off = pool_offset_kcode(page, hh, s, 16 * g + e, Hkv, D, &nib);
                        put_nibble(pool, off, nib, codes[e]);
                    }
                    pool[pool_offset_kscale(page, hh, s, g, Hkv, D)] = sb;
                    oracle_quantize_group(vr + 16 * g, codes, &sb);
                    for (int e = 0; e < 16; ++e) {
                        size_t off = pool_offset_vcode(page, hh, s, 16 * g + e, Hkv, D, &nib);
                        put_nibble(pool, off, nib, codes[e]);
                    }
                    pool[pool_offset_vscale(page, hh, s, g, Hkv, D)] = sb;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/* One output row.  The cache is taken from bf16 rows in position order
 * (k_rows / v_rows: [n_rows][Hkv][D]) and quantised-dequantised on the fly,
 * or, when pool != NULL, read from a pool image through page_row. */
typedef struct {
    const uint16_t *k_rows, *v_rows; /* logical source (pool == NULL) */
    const uint8_t *pool;             /* pool source */
    const int32_t *page_row;
    int Hkv, D, h;
    int n_visible; /* keys 0 .. n_visible-1 are visible */
    const uint16_t *q; /* [D] bf16 bits */
    double sm_scale;
    double *out;   /* [D] */
    double *lse;   /* natural-log sum of exp of the scores, may be NULL */
    double *psum;  /* sum of the normalised weights, may be NULL */
    int k8;        /* K8V4 cache: K in the 8-bit row format (0: NVFP4 K) */
} oracle_job;

void oracle_k8v4_read_row(const uint8_t *pool, int Hkv, int D, const int32_t *page_row, int pos,
                          int h, int is_v, double *out);
void oracle_k8_qdq_row(const uint16_t *x, int D, double *out);

static void load_row(const oracle_job *jb, int j, int is_v, double *dst) {
    if (jb->pool) {
        if (jb->k8)
            oracle_k8v4_read_row(jb->pool, jb->Hkv, jb->D, jb->page_row, j, jb->h, is_v, dst);
        else
            oracle_pool_read_row(jb->pool, jb->Hkv, jb->D, jb->page_row, j, jb->h, is_v, dst);
    } else {
        const uint16_t *src = (is_v ? jb->v_rows : jb->k_rows) + ((size_t)j * jb->Hkv + jb->h) * jb->D;
        if (jb->k8 && !is_v)
            oracle_k8_qdq_row(src, jb->D, dst);
        else
            oracle_qdq_row(src, jb->D, dst);
    }
}

static void run_job(const oracle_job *jb) {
    int D = jb->D, n = jb->n_visible;
    for (int d = 0; d < D; ++d) jb->out[d] = 0.0;
    if (jb->lse) *jb->lse = -INFINITY;
    if (jb->psum) *jb->psum = 0.0;
    if (n <= 0) return;
    double *row = (double *)malloc(sizeof(double) * D);
    double *s = (double *)malloc(sizeof(double) * n);
    double *qd = (double *)malloc(sizeof(double) * D);
    for (int d = 0; d < D; ++d) qd[d] = oracle_bf16_value(jb->q[d]);
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        load_row(jb, j, 0, row);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qd[d] * row[d];
        s[j] = jb->sm_scale * dot;
        if (s[j] > m) m = s[j];
    }
    double denom = 0.0;
    for (int j = 0; j < n; ++j) denom += exp(s[j] - m);
    double psum = 0.0;
    for (int j = 0; j < n; ++j) {
        double p = exp(s[j] - m) / denom;
        psum += p;
        load_row(jb, j, 1, row);
        for (int d = 0; d < D; ++d) jb->out[d] += p * row[d];
    }
    if (jb->lse) *jb->lse = m + log(denom);
    if (jb->psum) *jb->psum = psum;
    free(row);
    free(s);
    free(qd);
}

typedef struct {
    oracle_job *jobs;
    int njobs, stride, first;
} worker_arg;

static void *worker(void *p) {
    worker_arg *a = (worker_arg *)p;
    for (int i = a->first; i < a->njobs; i += a->stride) run_job(&a->jobs[i]);
    return NULL;
}

static void run_jobs(oracle_job *jobs, int njobs, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > njobs) nthreads = njobs;
    if (nthreads <= 1) {
        for (int i = 0; i < njobs; ++i) run_job(&jobs[i]);
        return;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    worker_arg *args = (worker_arg *)malloc(sizeof(worker_arg) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        args[t].jobs = jobs;
        args[t].njobs = njobs;
        args[t].stride = nthreads;
        args[t].first = t;
        pthread_create(&th[t], NULL, worker, &args[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(args);
}

/* Attention for njobs output rows, over the logical (bf16 row) cache.
 * Job i: sequence rows k_seq[i] / v_seq[i] ([rows][Hkv][D]), kv-head h[i],
 * visible keys 0 .. n_visible[i]-1, query q[i] ([D] bf16).  Writes
 * out[i*D .. i*D+D-1], lse[i] and psum[i] (either may be NULL). */
void oracle_attention_rows(int njobs, const uint16_t *const *k_seq, const uint16_t *const *v_seq,
                           int Hkv, int D, const int32_t *h, const int32_t *n_visible,
                           const uint16_t *const *q, double sm_scale, double *out, double *lse,
                           double *psum, int nthreads) {
    oracle_job *jobs = (oracle_job *)calloc((size_t)njobs, sizeof(oracle_job));
    for (int i = 0; i < njobs; ++i) {
        jobs[i].k_rows = k_seq[i];
        jobs[i].v_rows = v_seq[i];
        jobs[i].Hkv = Hkv;
        jobs[i].D = D;
        jobs[i].h = h[i];
        jobs[i].n_visible = n_visible[i];
        jobs[i].q = q[i];
        jobs[i].sm_scale = sm_scale;
        jobs[i].out = out + (size_t)i * D;
        jobs[i].lse = lse ? lse + i : NULL;
        jobs[i].psum = psum ? psum + i : NULL;
    }
    run_jobs(jobs, njobs, nthreads);
    free(jobs);
}

/* The same over a pool image: job i reads sequence page-table row
 * page_rows[i] ([max_pages] page ids). */
void oracle_attention_pool(int njobs, const uint8_t *pool, int Hkv, int D,
                           const int32_t *const *page_rows, const int32_t *h,
                           const int32_t *n_visible, const uint16_t *const *q, double sm_scale,
                           double *out, double *lse, double *psum, int nthreads) {
    oracle_job *jobs = (oracle_job *)calloc((size_t)njobs, sizeof(oracle_job));
    for (int i = 0; i < njobs; ++i) {
        jobs[i].pool = pool;
        jobs[i].page_row = page_rows[i];
        jobs[i].Hkv = Hkv;
        jobs[i].D = D;
        jobs[i].h = h[i];
        jobs[i].n_visible = n_visible[i];
        jobs[i].q = q[i];
        jobs[i].sm_scale = sm_scale;
        jobs[i].out = out + (size_t)i * D;
        jobs[i].lse = lse ? lse + i : NULL;
        jobs[i].psum = psum ? psum + i : NULL;
    }
    run_jobs(jobs, njobs, nthreads);
    free(jobs);
}

/* ------------------------------------------------------------------------ */
/* K8V4 cache: 8-bit K, NVFP4 V                                              */
/* ------------------------------------------------------------------------ */
/* "knoopx/ninfer" README, "Capabilities and limits": the engine stores KV
 * as BF16, INT8, FP8, NVFP4 or K8V4; the same README's note on its published
 * measurements names an "FP8 E4M3 row-256" KV.  Reading: K8V4 keeps V in
 * NVFP4 (as above) and K in that 8-bit format, one float scale per K row of
 * one token and one kv-head (D elements):
 *   scale = float(amax / 448)  (float division, round to nearest even),
 *   code  = E4M3 nearest to float(x / scale)  (float division, then E4M3
 *           rounding with ties to the even mantissa, saturating at 448),
 *   scale 0 (an all-zero row) gives codes 0; a magnitude that rounds to 0 is
 *   code 0 (no negative zero).
 * Both quotients are taken in float, as a kernel computes them, so the
 * decisions are the kernel's; the value is E4M3(code) * scale.            */
void oracle_k8_quantize_row(const uint16_t *x, int D, uint8_t *codes, float *scale) {
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) {
        float a = fabsf((float)oracle_bf16_value(x[d]));
        if (a > amax) amax = a;
    }
    float sc = amax / 448.0f;
    *scale = sc;
    for (int d = 0; d < D; ++d) {
        if (sc == 0.0f) {
            codes[d] = 0;
            continue;
        }
        float q = (float)oracle_bf16_value(x[d]) / sc;
        uint8_t mag = oracle_e4m3_round(fabs((double)q));
        codes[d] = (mag == 0) ? 0 : (uint8_t)((signbit(q) ? 0x80 : 0) | mag);
    }
}

double oracle_k8_dequant(int code, float scale) {
    return oracle_e4m3_value(code) * (double)scale;
}

void oracle_k8_qdq_row(const uint16_t *x, int D, double *out) {
    uint8_t codes[512];
    float sc;
    oracle_k8_quantize_row(x, D, codes, &sc);
    for (int d = 0; d < D; ++d) out[d] = oracle_k8_dequant(codes[d], sc);
}

/* K8V4 page layout: page p, kv-head h block of 25*D + 64 bytes at
 * (p * Hkv + h) * (25*D + 64):
 *   [0, 16D)            K codes [16 slots][D], one E4M3 byte per element
 *   [16D, 16D+64)       K scales [16 slots], IEEE binary32, little-endian
 *   [16D+64, 24D+64)    V codes [D][8]: byte (d, i) holds slot 2i in its low
 *                       nibble and slot 2i+1 in its high nibble
 *   [24D+64, 25D+64)    V scales [D/16][16 slots]                          */
size_t oracle_k8v4_page_bytes(int Hkv, int D) { return (size_t)Hkv * (25 * (size_t)D + 64); }

static size_t k8v4_base(int page, int h, int Hkv, int D) {
    return ((size_t)page * Hkv + h) * (25 * (size_t)D + 64);
}

void oracle_append_k8v4(uint8_t *pool, int Hkv, int D, const int32_t *page_table,
                        int max_pages_per_seq, const int32_t *kv_lens, int batch,
                        const uint16_t *k_new, const uint16_t *v_new, const int32_t *cu_new) {
    uint8_t kc[512], codes[16], sb;
    float ks;
    for (int b = 0; b < batch; ++b) {
        int n = cu_new[b + 1] - cu_new[b];
        const int32_t *page_row = page_table + (size_t)b * max_pages_per_seq;
        for (int i = 0; i < n; ++i) {
            int row = cu_new[b] + i;
            int pos = kv_lens[b] - n + i;
            int page = page_row[pos / 16], s = pos % 16;
            for (int h = 0; h < Hkv; ++h) {
                size_t base = k8v4_base(page, h, Hkv, D);
                const uint16_t *kr = k_new + ((size_t)row * Hkv + h) * D;
                const uint16_t *vr = v_new + ((size_t)row * Hkv + h) * D;
                oracle_k8_quantize_row(kr, D, kc, &ks);
                memcpy(pool + base + (size_t)s * D, kc, (size_t)D);
                memcpy(pool + base + 16 * (size_t)D + 4 * (size_t)s, &ks, 4);
                for (int g = 0; g < D / 16; ++g) {
                    oracle_quantize_group(vr + 16 * g, codes, &sb);
                    for (int e = 0; e < 16; ++e) {
                        int d = 16 * g + e;
                        size_t off = base + 16 * (size_t)D + 64 + (size_t)d * 8 + (size_t)(s >> 1);
                        put_nibble(pool, off, s & 1, codes[e]);
                    }
                    pool[base + 24 * (size_t)D + 64 + (size_t)g * 16 + s] = sb;
                }
            }
        }
    }
}

void oracle_k8v4_read_row(const uint8_t *pool, int Hkv, int D, const int32_t *page_row, int pos,
                          int h, int is_v, double *out) {
    int page = page_row[pos / 16], s = pos % 16;
    size_t base = k8v4_base(page, h, Hkv, D);
    if (!is_v) {
        float ks;
        memcpy(&ks, pool + base + 16 * (size_t)D + 4 * (size_t)s, 4);
        for (int d = 0; d < D; ++d) out[d] = oracle_k8_dequant(pool[base + (size_t)s * D + d], ks);
        return;
    }
    for (int d = 0; d < D; ++d) {
        int code = get_nibble(pool, base + 16 * (size_t)D + 64 + (size_t)d * 8 + (size_t)(s >> 1),
                              s & 1);
        int sb = pool[base + 24 * (size_t)D + 64 + (size_t)(d / 16) * 16 + s];
        out[d] = oracle_dequant(code, sb);
    }
}

/* Attention over a K8V4 cache: as oracle_attention_rows / _pool with K in
 * the 8-bit row format. */
void oracle_attention_rows_k8v4(int njobs, const uint16_t *const *k_seq,
                                const uint16_t *const *v_seq, int Hkv, int D, const int32_t *h,
                                const int32_t *n_visible, const uint16_t *const *q,
                                double sm_scale, double *out, double *lse, double *psum,
                                int nthreads) {
    oracle_job *jobs = (oracle_job *)calloc((size_t)njobs, sizeof(oracle_job));
    for (int i = 0; i < njobs; ++i) {
        jobs[i].k_rows = k_seq[i];
        jobs[i].v_rows = v_seq[i];
        jobs[i].Hkv = Hkv;
        jobs[i].D = D;
        jobs[i].h = h[i];
        jobs[i].n_visible = n_visible[i];
        jobs[i].q = q[i];
        jobs[i].sm_scale = sm_scale;
        jobs[i].out = out + (size_t)i * D;
        jobs[i].lse = lse ? lse + i : NULL;
        jobs[i].psum = psum ? psum + i : NULL;
        jobs[i].k8 = 1;
    }
    run_jobs(jobs, njobs, nthreads);
    free(jobs);
}

void oracle_attention_pool_k8v4(int njobs, const uint8_t *pool, int Hkv, int D,
                                const int32_t *const *page_rows, const int32_t *h,
                                const int32_t *n_visible, const uint16_t *const *q,
                                double sm_scale, double *out, double *lse, double *psum,
                                int nthreads) {
    oracle_job *jobs = (oracle_job *)calloc((size_t)njobs, sizeof(oracle_job));
    for (int i = 0; i < njobs; ++i) {
        jobs[i].pool = pool;
        jobs[i].page_row = page_rows[i];
        jobs[i].Hkv = Hkv;
        jobs[i].D = D;
        jobs[i].h = h[i];
        jobs[i].n_visible = n_visible[i];
        jobs[i].q = q[i];
        jobs[i].sm_scale = sm_scale;
        jobs[i].out = out + (size_t)i * D;
        jobs[i].lse = lse ? lse + i : NULL;
        jobs[i].psum = psum ? psum + i : NULL;
        jobs[i].k8 = 1;
    }
    run_jobs(jobs, njobs, nthreads);
    free(jobs);
}
