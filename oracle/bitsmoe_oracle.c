/*
 * bitsmoe_oracle.c -- plain, slow CPU reference of the BitsMoE spectral MoE
 * gate/up decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with the
 * CUDA library; both sides implement the same written specification
 * independently (the packed format and the quantiser described below).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * -ffp-contract=off matters: the quantiser is specified as separate IEEE fp32
 * operations (divide, then add), and an FMA contraction would change results.
 *
 * Sources followed (the BitsMoE study-note page, "BitsMoE: Cost-Aware Bit
 * Allocation In spectral Space for MoE LLM Quantization"):
 *   - Methodology, first split: W_e x = P_e (Phi^T x); z = Phi^T x does not
 *     depend on the expert and is reused by every selected expert.
 *   - second split: column normalisation W_e = sum_k a_{e,k} p_{e,k} phi_k^T
 *     with unit p_{e,k}; a measures strength, p is quantised at a chosen width.
 *   - Usage: the width set {0,1,2,3,4,6,8,16}; 0 = dropped, 16 = FP16.
 *   - Execution: components of equal width are put together and packed by
 *     bit plane.
 * The pages give no quantiser formula.  This file uses the mid-rise quantiser
 * w = s*(q - (2^b-1)/2), s = 2*max|p|/(2^b-1), one fp16 scale per component,
 * rounding to the nearest level with ties upward: q = clamp(floor(p/s + 2^(b-1))).
 *
 * Arithmetic: everything that defines a stored bit (scales, q) is done in IEEE
 * fp32 exactly as specified; everything that defines an output value (Z, Y) is
 * done in fp64 from the stored (dequantised) values.
 *
 * Every function here has pins in tests/test_oracle.py (closed forms, library
 * routines, brute force and a hand-built golden blob).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- status bits (device-side data errors; same meanings as the library's,
 *      written out again here from the specification) ---- */
#define ORC_ST_NONFINITE 1   /* a non-finite component element */
#define ORC_ST_BADSCALE 2    /* a scale that is negative, NaN or Inf */
#define ORC_ST_BADEXPERT 4   /* a routed expert id outside [0, E) */

/* ---- error returns ---- */
#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_EWIDTH (-2)
#define ORC_ESIZE (-3)
#define ORC_EFORMAT (-5)

/* Width order of the groups inside an expert: 16, 8, 6, 4, 3, 2, 1. */
static const int ORC_GROUP_WIDTH[7] = {16, 8, 6, 4, 3, 2, 1};

/* ------------------------------------------------------------------------- */
/* IEEE binary16 conversions, written from the format definition.            */
/* ------------------------------------------------------------------------- */

/* fp32 -> fp16 bits, round to nearest, ties to even.  Overflow gives +-Inf,
 * NaN gives the quiet NaN 0x7E00 (sign kept).  Pinned exhaustively against
 * numpy.float16 in the tests. */
uint16_t orc_f32_to_f16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ex = (x >> 23) & 0xFFu;
    uint32_t man = x & 0x7FFFFFu;
    if (ex == 0xFFu) return (uint16_t)(sign | (man ? 0x7E00u : 0x7C00u));
    if (ex == 0u) return (uint16_t)sign; /* fp32 subnormal: far below fp16's least subnormal */
    uint32_t m = man | 0x800000u;        /* 24-bit significand */
    int e16 = (int)ex - 127 + 15;        /* rebiased exponent */
    if (e16 >= 31) return (uint16_t)(sign | 0x7C00u);
    if (e16 >= 1) {
        /* normal: keep 10 fraction bits, round the 13 dropped bits */
        uint32_t h = ((uint32_t)e16 << 10) | (man >> 13);
        uint32_t rem = man & 0x1FFFu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u; /* carry may reach Inf: correct */
        return (uint16_t)(sign | h);
    }
    /* fp16 subnormal: value in units of 2^-24 is m * 2^(ex-126) */
    int s = 126 - (int)ex; /* >= 14 */
    if (s >= 25) return (uint16_t)sign; /* below a quarter unit (or a non-tie below half) */
    uint32_t h = m >> s;
    uint32_t rem = m & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    if (rem > half || (rem == half && (h & 1u))) h += 1u;
    return (uint16_t)(sign | h);
}

/* fp16 bits -> double (exact). */
double orc_f16_to_f64(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);
    return s ? -v : v;
}

/* fp16 bits -> float (exact: every fp16 value is an fp32 value). */
static float orc_f16_to_f32(uint16_t h) { return (float)orc_f16_to_f64(h); }

/* ------------------------------------------------------------------------- */
/* Widths and the packed layout (format v2).                                 */
/* ------------------------------------------------------------------------- */

static int orc_width_ok(int b) {
    return b == 0 || b == 1 || b == 2 || b == 3 || b == 4 || b == 6 || b == 8 || b == 16;
}

static uint64_t orc_roundup(uint64_t v, uint64_t m) { return (v + m - 1) / m * m; }

/* Bytes of one group of width b holding n members, rows padded to d_pad
 * (a multiple of 32; the planes are stored rows fastest, [b][W][d_pad]). */
static uint64_t orc_group_bytes(int b, uint64_t n, uint64_t d_pad) {
    if (n == 0) return 0;
    if (b == 16) {
        uint64_t np = orc_roundup(n, 8);
        return 2 * np + 4 * np + 2 * np * d_pad; /* idx u16, amp f32, w16 u16 [np][d_pad] */
    }
    uint64_t np = orc_roundup(n, 32);
    return 2 * np + 2 * np + 4 * np + 4 * (uint64_t)b * (np / 32) * d_pad; /* idx, scale, amp, planes */
}

/* Byte offset of plane word [plane j][word w][row i] inside a group's planes
 * (rows fastest); W = words per plane, d_pad = padded rows. */
static uint64_t orc_plane_off(uint64_t j, uint64_t w, uint64_t W, uint64_t d_pad, uint64_t i) {
    return 4 * ((j * W + w) * d_pad + i);
}

/* Count of each width for expert e: cnt[g] for groups g = 0..6 (widths
 * 16,8,6,4,3,2,1) and cnt[7] = zero-width count. */
static int orc_counts(int r, const uint8_t *wrow, uint32_t cnt[8]) {
    memset(cnt, 0, 8 * sizeof(uint32_t));
    for (int k = 0; k < r; k++) {
        int b = wrow[k];
        if (!orc_width_ok(b)) return ORC_EWIDTH;
        if (b == 0) {
            cnt[7]++;
            continue;
        }
        for (int g = 0; g < 7; g++)
            if (ORC_GROUP_WIDTH[g] == b) cnt[g]++;
    }
    return ORC_OK;
}

static int orc_dims_ok(int E, int r, int d_out) {
    return E >= 1 && r >= 1 && r <= 65535 && d_out >= 1 && d_out <= (1 << 30);
}

/* Total blob bytes for the given widths [E][r]; 0 on invalid input. */
uint64_t orc_blob_bytes(int E, int r, int d_out, const uint8_t *widths) {
    if (!orc_dims_ok(E, r, d_out) || !widths) return 0;
    uint64_t d_pad = orc_roundup((uint64_t)d_out, 32);
    uint64_t total = 64 + 64 * (uint64_t)E;
    for (int e = 0; e < E; e++) {
        uint32_t cnt[8];
        if (orc_counts(r, widths + (size_t)e * r, cnt) != ORC_OK) return 0;
        for (int g = 0; g < 7; g++) total += orc_group_bytes(ORC_GROUP_WIDTH[g], cnt[g], d_pad);
    }
    return total;
}

static void put16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put32(uint8_t *p, uint32_t v) {
    for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put64(uint8_t *p, uint64_t v) {
    for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint16_t get16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get32(const uint8_t *p) {
    uint32_t v = 0;
    for (int i = 3; i >= 0; i--) v = (v << 8) | p[i];
    return v;
}
static uint64_t get64(const uint8_t *p) {
    uint64_t v = 0;
    for (int i = 7; i >= 0; i--) v = (v << 8) | p[i];
    return v;
}

/* ------------------------------------------------------------------------- */
/* Scales and the quantiser.                                                 */
/* ------------------------------------------------------------------------- */

/* One fp16 scale per component of width b in {1,2,3,4,6,8}:
 *   m   = max_i |p_i|                       (exact in fp32)
 *   s32 = (2*m) / (2^b - 1)                 (IEEE fp32 divide, round to nearest)
 *   s   = fp16(s32)                         (round to nearest even)
 * Widths 0 and 16 get scale 0.  A component with a non-finite element gets
 * scale 0 and sets ORC_ST_NONFINITE.  Returns 0 or a negative error. */
int orc_compute_scales(int E, int r, int d_out, const float *comps, const uint8_t *widths,
                       uint16_t *scales, int32_t *status) {
    if (!orc_dims_ok(E, r, d_out) || !comps || !widths || !scales) return ORC_EINVAL;
    int32_t st = 0;
    for (int e = 0; e < E; e++)
        for (int k = 0; k < r; k++) {
            int b = widths[(size_t)e * r + k];
            if (!orc_width_ok(b)) return ORC_EWIDTH;
            uint16_t out = 0;
            if (b != 0 && b != 16) {
                const float *p = comps + ((size_t)e * r + k) * (size_t)d_out;
                float m = 0.0f;
                int bad = 0;
                for (int i = 0; i < d_out; i++) {
                    if (!isfinite(p[i])) bad = 1;
                    float a = fabsf(p[i]);
                    if (a > m) m = a;
                }
                if (bad) {
                    st |= ORC_ST_NONFINITE;
                } else {
                    float two_m = 2.0f * m;
                    float s32 = two_m / (float)((1 << b) - 1);
                    out = orc_f32_to_f16(s32);
                }
            }
            scales[(size_t)e * r + k] = out;
        }
    if (status) *status |= st;
    return ORC_OK;
}

/* Quantise one element p at width b with fp16 scale bits sh.
 *   t = p / s (fp32), u = t + 2^(b-1) (fp32), q = clamp(floor(u), 0, 2^b - 1).
 * A scale of +-0 gives q = 0.  A negative or non-finite scale gives q = 0 and
 * ORC_ST_BADSCALE; a non-finite p gives q = 0 and ORC_ST_NONFINITE. */
uint32_t orc_quantise(float p, int b, uint16_t sh, int32_t *st) {
    float s = orc_f16_to_f32(sh);
    if (!isfinite(s) || s < 0.0f) {
        *st |= ORC_ST_BADSCALE;
        return 0;
    }
    if (s == 0.0f) return 0;
    if (!isfinite(p)) {
        *st |= ORC_ST_NONFINITE;
        return 0;
    }
    float t = p / s;
    float u = t + (float)(1 << (b - 1));
    float qmax = (float)((1 << b) - 1);
    float f = floorf(u);
    if (f < 0.0f) return 0;
    if (f > qmax) return (uint32_t)qmax;
    return (uint32_t)f;
}

/* ------------------------------------------------------------------------- */
/* Pack.                                                                     */
/* ------------------------------------------------------------------------- */

/* Pack comps [E][r][d_out] (unit directions p_{e,k}), amps [E][r] and fp16
 * scales [E][r] into the format-v2 blob.  Every byte of the blob is written
 * (padding included).  Returns 0 or a negative error; data errors go to
 * *status as bits. */
int orc_pack(int E, int r, int d_out, const uint8_t *widths, const float *comps,
             const uint16_t *scales, const float *amps, uint8_t *blob, uint64_t blob_bytes,
             int32_t *status) {
    if (!orc_dims_ok(E, r, d_out) || !widths || !comps || !scales || !amps || !blob)
        return ORC_EINVAL;
    uint64_t need = orc_blob_bytes(E, r, d_out, widths);
    if (need == 0) return ORC_EWIDTH;
    if (blob_bytes < need) return ORC_ESIZE;
    memset(blob, 0, need);
    uint64_t d_pad = orc_roundup((uint64_t)d_out, 32);
    int32_t st = 0;

    /* header */
    put32(blob + 0, 0x454F4D42u); /* "BMOE" */
    put32(blob + 4, 2u);
    put32(blob + 8, (uint32_t)d_out);
    put32(blob + 12, (uint32_t)d_pad);
    put32(blob + 16, (uint32_t)E);
    put32(blob + 20, (uint32_t)r);
    put64(blob + 24, need);
    put64(blob + 32, 64u);
    put64(blob + 40, 64u + 64u * (uint64_t)E);

    uint64_t base = 64u + 64u * (uint64_t)E;
    for (int e = 0; e < E; e++) {
        const uint8_t *wrow = widths + (size_t)e * r;
        uint32_t cnt[8];
        orc_counts(r, wrow, cnt);
        uint8_t *dir = blob + 64 + 64 * (size_t)e;
        uint64_t off = 0;
        for (int g = 0; g < 7; g++) {
            int b = ORC_GROUP_WIDTH[g];
            put32(dir + 16 + 4 * g, (uint32_t)off);
            put16(dir + 44 + 2 * g, (uint16_t)cnt[g]);
            uint8_t *G = blob + base + off;
            uint64_t n = cnt[g];
            if (n > 0) {
                if (b == 16) {
                    uint64_t np = orc_roundup(n, 8);
                    uint8_t *idx = G, *amp = G + 2 * np, *w16 = G + 6 * np;
                    uint64_t m = 0;
                    for (int k = 0; k < r; k++) {
                        if (wrow[k] != 16) continue;
                        put16(idx + 2 * m, (uint16_t)k);
                        float a = amps[(size_t)e * r + k];
                        uint32_t abits;
                        memcpy(&abits, &a, 4);
                        put32(amp + 4 * m, abits);
                        const float *p = comps + ((size_t)e * r + k) * (size_t)d_out;
                        for (int i = 0; i < d_out; i++) {
                            uint16_t hb = 0;
                            if (isfinite(p[i]))
                                hb = orc_f32_to_f16(p[i]);
                            else
                                st |= ORC_ST_NONFINITE;
                            put16(w16 + 2 * (m * d_pad + (uint64_t)i), hb);
                        }
                        m++;
                    }
                } else {
                    uint64_t np = orc_roundup(n, 32), W = np / 32;
                    uint8_t *idx = G, *scl = G + 2 * np, *amp = G + 4 * np, *planes = G + 8 * np;
                    uint64_t m = 0;
                    for (int k = 0; k < r; k++) {
                        if (wrow[k] != b) continue;
                        uint16_t sh = scales[(size_t)e * r + k];
                        put16(idx + 2 * m, (uint16_t)k);
                        put16(scl + 2 * m, sh);
                        float a = amps[(size_t)e * r + k];
                        uint32_t abits;
                        memcpy(&abits, &a, 4);
                        put32(amp + 4 * m, abits);
                        const float *p = comps + ((size_t)e * r + k) * (size_t)d_out;
                        uint64_t w = m / 32, bit = m % 32;
                        for (int i = 0; i < d_out; i++) {
                            uint32_t q = orc_quantise(p[i], b, sh, &st);
                            for (int j = 0; j < b; j++) {
                                if (!((q >> j) & 1u)) continue;
                                uint8_t *word = planes + orc_plane_off((uint64_t)j, w, W, d_pad, (uint64_t)i);
                                put32(word, get32(word) | (1u << bit));
                            }
                        }
                        m++;
                    }
                }
            }
            off += orc_group_bytes(b, n, d_pad);
        }
        put16(dir + 44 + 2 * 7, (uint16_t)cnt[7]);
        put64(dir + 0, base);
        put64(dir + 8, off);
        base += off;
    }
    if (status) *status |= st;
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Reading a blob back.                                                      */
/* ------------------------------------------------------------------------- */

/* Check the header and the directory of a blob against its own size.
 * Returns 0 and fills the dims, or ORC_EFORMAT. */
int orc_blob_parse(const uint8_t *blob, uint64_t bytes, int *E, int *r, int *d_out) {
    if (!blob || bytes < 64) return ORC_EFORMAT;
    if (get32(blob) != 0x454F4D42u || get32(blob + 4) != 2u) return ORC_EFORMAT;
    uint64_t dout = get32(blob + 8), dpad = get32(blob + 12), ne = get32(blob + 16), rk = get32(blob + 20);
    if (!orc_dims_ok((int)ne, (int)rk, (int)dout) || dpad != orc_roundup(dout, 32)) return ORC_EFORMAT;
    uint64_t total = get64(blob + 24);
    if (total != bytes || get64(blob + 32) != 64u || get64(blob + 40) != 64u + 64u * ne) return ORC_EFORMAT;
    for (int i = 48; i < 64; i++)
        if (blob[i]) return ORC_EFORMAT;
    uint64_t base = 64u + 64u * ne;
    if (base > bytes) return ORC_EFORMAT;
    for (uint64_t e = 0; e < ne; e++) {
        const uint8_t *dir = blob + 64 + 64 * e;
        if (get64(dir) != base) return ORC_EFORMAT;
        uint64_t off = 0, members = 0;
        for (int g = 0; g < 7; g++) {
            if (get32(dir + 16 + 4 * g) != off) return ORC_EFORMAT;
            uint64_t n = get16(dir + 44 + 2 * g);
            members += n;
            off += orc_group_bytes(ORC_GROUP_WIDTH[g], n, dpad);
        }
        members += get16(dir + 44 + 14);
        if (members != rk || get64(dir + 8) != off || get32(dir + 60) != 0) return ORC_EFORMAT;
        base += off;
        if (base > bytes) return ORC_EFORMAT;
    }
    if (base != bytes) return ORC_EFORMAT;
    *E = (int)ne;
    *r = (int)rk;
    *d_out = (int)dout;
    return ORC_OK;
}

/* Unpack every component of a blob:
 *   q      [E][r][d_out]  u16: the b-bit integer for b in 1..8, the raw fp16
 *                         bits for b = 16, 0 for b = 0
 *   widths [E][r], scales [E][r] (fp16 bits; 0 for b = 0, 16), amps [E][r]
 *   (0 for b = 0).  Any output pointer may be NULL. */
int orc_unpack(const uint8_t *blob, uint64_t bytes, uint16_t *q, uint8_t *widths, uint16_t *scales,
               float *amps) {
    int E, r, d_out;
    int rc = orc_blob_parse(blob, bytes, &E, &r, &d_out);
    if (rc) return rc;
    uint64_t d_pad = orc_roundup((uint64_t)d_out, 32);
    if (q) memset(q, 0, sizeof(uint16_t) * (size_t)E * r * d_out);
    if (widths) memset(widths, 0, (size_t)E * r);
    if (scales) memset(scales, 0, sizeof(uint16_t) * (size_t)E * r);
    if (amps) memset(amps, 0, sizeof(float) * (size_t)E * r);
    for (int e = 0; e < E; e++) {
        const uint8_t *dir = blob + 64 + 64 * (size_t)e;
        uint64_t base = get64(dir);
        for (int g = 0; g < 7; g++) {
            int b = ORC_GROUP_WIDTH[g];
            uint64_t n = get16(dir + 44 + 2 * g);
            if (n == 0) continue;
            const uint8_t *G = blob + base + get32(dir + 16 + 4 * g);
            if (b == 16) {
                uint64_t np = orc_roundup(n, 8);
                for (uint64_t m = 0; m < n; m++) {
                    int k = get16(G + 2 * m);
                    if (k >= r) return ORC_EFORMAT;
                    size_t ek = (size_t)e * r + k;
                    if (widths) widths[ek] = 16;
                    if (amps) {
                        uint32_t ab = get32(G + 2 * np + 4 * m);
                        memcpy(&amps[ek], &ab, 4);
                    }
                    if (q)
                        for (int i = 0; i < d_out; i++)
                            q[ek * d_out + i] = get16(G + 6 * np + 2 * (m * d_pad + (uint64_t)i));
                }
            } else {
                uint64_t np = orc_roundup(n, 32), W = np / 32;
                const uint8_t *planes = G + 8 * np;
                for (uint64_t m = 0; m < n; m++) {
                    int k = get16(G + 2 * m);
                    if (k >= r) return ORC_EFORMAT;
                    size_t ek = (size_t)e * r + k;
                    if (widths) widths[ek] = (uint8_t)b;
                    if (scales) scales[ek] = get16(G + 2 * np + 2 * m);
                    if (amps) {
                        uint32_t ab = get32(G + 4 * np + 4 * m);
                        memcpy(&amps[ek], &ab, 4);
                    }
                    if (q)
                        for (int i = 0; i < d_out; i++) {
                            uint32_t v = 0;
                            for (int j = 0; j < b; j++) {
                                uint32_t word = get32(planes + orc_plane_off((uint64_t)j, m / 32, W, d_pad, (uint64_t)i));
                                v |= ((word >> (m % 32)) & 1u) << j;
                            }
                            q[ek * d_out + i] = (uint16_t)v;
                        }
                }
            }
        }
    }
    return ORC_OK;
}

/* Dequantised direction of one component (fp64):
 *   b in 1..8:  w = s * (q - (2^b - 1)/2)
 *   b = 16:     w = the fp16 value
 *   b = 0:      w = 0 */
static double orc_dequant(int b, uint16_t qv, uint16_t sh) {
    if (b == 0) return 0.0;
    if (b == 16) return orc_f16_to_f64(qv);
    return orc_f16_to_f64(sh) * ((double)qv - ((double)((1 << b) - 1)) / 2.0);
}

/* Dense dequantised directions of expert e: Wd [r][d_out] (fp64) and a [r]. */
int orc_dequant_expert(const uint8_t *blob, uint64_t bytes, int e, double *Wd, double *a) {
    int E, r, d_out;
    int rc = orc_blob_parse(blob, bytes, &E, &r, &d_out);
    if (rc) return rc;
    if (e < 0 || e >= E || !Wd) return ORC_EINVAL;
    size_t n = (size_t)E * r;
    uint16_t *q = (uint16_t *)malloc(sizeof(uint16_t) * n * d_out);
    uint8_t *w = (uint8_t *)malloc(n);
    uint16_t *s = (uint16_t *)malloc(sizeof(uint16_t) * n);
    float *am = (float *)malloc(sizeof(float) * n);
    if (!q || !w || !s || !am) {
        free(q); free(w); free(s); free(am);
        return ORC_EINVAL;
    }
    rc = orc_unpack(blob, bytes, q, w, s, am);
    if (!rc)
        for (int k = 0; k < r; k++) {
            size_t ek = (size_t)e * r + k;
            if (a) a[k] = (double)am[ek];
            for (int i = 0; i < d_out; i++) Wd[(size_t)k * d_out + i] = orc_dequant(w[ek], q[ek * d_out + i], s[ek]);
        }
    free(q); free(w); free(s); free(am);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* The two-step forward.                                                     */
/* ------------------------------------------------------------------------- */

/* Shared projection z = Phi^T x for T tokens (fp64 from fp16 inputs):
 *   Z[t][k] = sum_i PhiT[k][i] * X[t][i]
 * PhiT is [r][d_in] fp16 bits (row k = phi_k), X is [T][d_in] fp16 bits. */
void orc_shared_proj(const uint16_t *phi_t, const uint16_t *X, int T, int d_in, int r, double *Z) {
    for (int t = 0; t < T; t++)
        for (int k = 0; k < r; k++) {
            double acc = 0.0;
            for (int i = 0; i < d_in; i++)
                acc += orc_f16_to_f64(phi_t[(size_t)k * d_in + i]) * orc_f16_to_f64(X[(size_t)t * d_in + i]);
            Z[(size_t)t * r + k] = acc;
        }
}

/* Routed expert forward from a packed blob (fp64):
 *   Y_e[t][s][i] = sum_k a_{e,k} * w_{e,k,i} * Z[t][k]      with e = ids[t][s]
 *   Y_sum[t][i]  = sum_s g[t][s] * Y_e[t][s][i]
 * The sum over k runs over the stored components (widths 1..16); width-0
 * components are not in the blob and contribute nothing.  An id outside
 * [0, E) gives a zero row, is left out of Y_sum and sets ORC_ST_BADEXPERT.
 * Y_e may be NULL. */
int orc_expert_forward(const uint8_t *blob, uint64_t bytes, const double *Z, const int32_t *ids,
                       const float *g, int T, int top_k, double *Y_e, double *Y_sum, int32_t *status) {
    int E, r, d_out;
    int rc = orc_blob_parse(blob, bytes, &E, &r, &d_out);
    if (rc) return rc;
    if (T < 0 || top_k < 1 || !Z || !ids || !g || !Y_sum) return ORC_EINVAL;
    uint64_t d_pad = orc_roundup((uint64_t)d_out, 32);
    int32_t st = 0;
    double *y = (double *)malloc(sizeof(double) * (size_t)d_out);
    if (!y) return ORC_EINVAL;
    for (int t = 0; t < T; t++) {
        double *ys = Y_sum + (size_t)t * d_out;
        for (int i = 0; i < d_out; i++) ys[i] = 0.0;
        for (int s = 0; s < top_k; s++) {
            int e = ids[(size_t)t * top_k + s];
            for (int i = 0; i < d_out; i++) y[i] = 0.0;
            if (e < 0 || e >= E) {
                st |= ORC_ST_BADEXPERT;
            } else {
                const uint8_t *dir = blob + 64 + 64 * (size_t)e;
                uint64_t base = get64(dir);
                for (int gi = 0; gi < 7; gi++) {
                    int b = ORC_GROUP_WIDTH[gi];
                    uint64_t n = get16(dir + 44 + 2 * gi);
                    if (n == 0) continue;
                    const uint8_t *G = blob + base + get32(dir + 16 + 4 * gi);
                    uint64_t np = b == 16 ? orc_roundup(n, 8) : orc_roundup(n, 32);
                    for (uint64_t m = 0; m < n; m++) {
                        int k = get16(G + 2 * m);
                        uint32_t ab = get32(G + (b == 16 ? 2 * np : 4 * np) + 4 * m);
                        float af;
                        memcpy(&af, &ab, 4);
                        double c = (double)af * Z[(size_t)t * r + k];
                        uint16_t sh = b == 16 ? 0 : get16(G + 2 * np + 2 * m);
                        for (int i = 0; i < d_out; i++) {
                            uint16_t qv;
                            if (b == 16) {
                                qv = get16(G + 6 * np + 2 * (m * d_pad + (uint64_t)i));
                            } else {
                                uint64_t W = np / 32;
                                uint32_t v = 0;
                                for (int j = 0; j < b; j++) {
                                    uint32_t word = get32(G + 8 * np + orc_plane_off((uint64_t)j, m / 32, W, d_pad, (uint64_t)i));
                                    v |= ((word >> (m % 32)) & 1u) << j;
                                }
                                qv = (uint16_t)v;
                            }
                            y[i] += c * orc_dequant(b, qv, sh);
                        }
                    }
                }
                double gw = (double)g[(size_t)t * top_k + s];
                for (int i = 0; i < d_out; i++) ys[i] += gw * y[i];
            }
            if (Y_e)
                for (int i = 0; i < d_out; i++) Y_e[((size_t)t * top_k + s) * d_out + i] = y[i];
        }
    }
    free(y);
    if (status) *status |= st;
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Expert FFN output after the gate and up projections.                      */
/* ------------------------------------------------------------------------- */

/* The pages decompose only an expert's gate and up projections (Methodology:
 * the stacked gate/up matrices) and say nothing of what follows them.  This
 * is the usual gated MoE expert, with a dense fp16 down projection per
 * expert, in fp64 from the gate and up outputs:
 *   h[t][s][m] = SiLU(Yg[t][s][m]) * Yu[t][s][m],   SiLU(v) = v / (1 + e^(-v))
 *   out[t][i]  = sum_s g[t][s] * sum_m Wd[e][i][m] * h[t][s][m],  e = ids[t][s]
 * Yg, Yu are [T][top_k][d_ff] (the per-slot expert outputs of the gate and up
 * projections), Wd is [E][d_model][d_ff] fp16 bits (row i of expert e holds
 * the weights of output i), out is [T][d_model].  An id outside [0, E)
 * contributes nothing and sets ORC_ST_BADEXPERT. */
static double orc_silu(double v) { return v / (1.0 + exp(-v)); }

int orc_ffn_down(const double *Yg, const double *Yu, const uint16_t *w_down, const int32_t *ids, const float *g,
                 int T, int top_k, int E, int d_model, int d_ff, double *out, int32_t *status) {
    if (T < 0 || top_k < 1 || E < 1 || d_model < 1 || d_ff < 1) return ORC_EINVAL;
    if (T > 0 && (!Yg || !Yu || !w_down || !ids || !g || !out)) return ORC_EINVAL;
    int32_t st = 0;
    double *h = (double *)malloc(sizeof(double) * (size_t)d_ff);
    if (!h) return ORC_EINVAL;
    for (int t = 0; t < T; t++) {
        double *o = out + (size_t)t * d_model;
        for (int i = 0; i < d_model; i++) o[i] = 0.0;
        for (int s = 0; s < top_k; s++) {
            const size_t q = (size_t)t * top_k + s;
            const int e = ids[q];
            if (e < 0 || e >= E) {
                st |= ORC_ST_BADEXPERT;
                continue;
            }
            for (int m = 0; m < d_ff; m++) h[m] = orc_silu(Yg[q * d_ff + m]) * Yu[q * d_ff + m];
            const double gw = (double)g[q];
            for (int i = 0; i < d_model; i++) {
                const uint16_t *row = w_down + ((size_t)e * d_model + i) * d_ff;
                double acc = 0.0;
                for (int m = 0; m < d_ff; m++) acc += orc_f16_to_f64(row[m]) * h[m];
                o[i] += gw * acc;
            }
        }
    }
    free(h);
    if (status) *status |= st;
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Width-dependent distortion of each component (the FQCM cost's third factor). */
/* ------------------------------------------------------------------------- */

/* The pages name a width-dependent distortion eps_{e,k,b} but do not define it.
 * Read here as the squared error of storing the unit direction at width b:
 *   eps_{e,k,b} = sum_i (p_i - w_i)^2  (fp64),
 * w the stored value: b in 1..8, the quantiser above with the component's fp16
 * scale for that width, w = s (q - (2^b - 1)/2); b = 16, the fp16 value; b = 0,
 * w = 0 (so eps = ||p||^2).  Widths in the order 0,1,2,3,4,6,8,16: eps is
 * [E][r][8].  A component with a non-finite element gets NaN at every width. */
static const int ORC_WIDTH_SET[8] = {0, 1, 2, 3, 4, 6, 8, 16};

int orc_fqcm_eps(int E, int r, int d_out, const float *comps, double *eps) {
    if (!orc_dims_ok(E, r, d_out) || !comps || !eps) return ORC_EINVAL;
    for (int e = 0; e < E; e++)
        for (int k = 0; k < r; k++) {
            const float *p = comps + ((size_t)e * r + k) * (size_t)d_out;
            double *out = eps + ((size_t)e * r + k) * 8;
            float m = 0.0f;
            int bad = 0;
            for (int i = 0; i < d_out; i++) {
                if (!isfinite(p[i])) bad = 1;
                float a = fabsf(p[i]);
                if (a > m) m = a;
            }
            for (int wi = 0; wi < 8; wi++) {
                const int b = ORC_WIDTH_SET[wi];
                if (bad) {
                    out[wi] = NAN;
                    continue;
                }
                uint16_t sh = 0;
                if (b != 0 && b != 16) sh = orc_f32_to_f16((2.0f * m) / (float)((1 << b) - 1));
                double acc = 0.0;
                for (int i = 0; i < d_out; i++) {
                    double w;
                    if (b == 0) {
                        w = 0.0;
                    } else if (b == 16) {
                        w = orc_f16_to_f64(orc_f32_to_f16(p[i]));
                    } else {
                        int32_t st = 0;
                        uint32_t q = orc_quantise(p[i], b, sh, &st);
                        w = orc_dequant(b, (uint16_t)q, sh);
                    }
                    const double d = (double)p[i] - w;
                    acc += d * d;
                }
                out[wi] = acc;
            }
        }
    return ORC_OK;
}
