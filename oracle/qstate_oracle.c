/*
 * qstate_oracle.c -- plain, slow, scalar CPU oracle of the quantized
 * recurrent-state decode step.  TEST INFRASTRUCTURE ONLY (see the header):
 * the product path never includes, links or runs this file.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC -lm
 * (no contraction of a*b+c, so every float operation below is one IEEE
 * binary32 operation with round-to-nearest-even, except where fmaf is
 * written out; double is used only where the text says "exact").
 *
 * The recurrence is "Preserving Updates in Low-Bit Recurrent State
 * Quantization", Table 1; the scale modes are "When Dynamic Scaling Fails",
 * Abstract; BDR and the lost / moved / reversed taxonomy are the Abstract
 * and the Figure 4 caption of the first of these pages.  Everything the pages
 * do not fix is a reading, marked "Reading:" below.
 */
#include "qstate_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------
 * Number formats.  Written from the IEEE 754 definitions: binary16 has an
 * 11-bit significand, exponent bias 15, smallest normal 2^-14 and smallest
 * subnormal 2^-24; bfloat16 is the top 16 bits of binary32.
 * ---------------------------------------------------------------------- */
uint16_t or_f32_to_f16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
    double ax = fabs((double)x);              /* exact widening */
    /* 65520 is the midpoint between 65504 (odd significand) and 2^16, so
     * round-to-nearest-even sends it and everything above to infinity. */
    if (ax >= 65520.0) return (uint16_t)(sign | 0x7C00u);
    if (ax < 0x1p-14) {
        /* subnormal range: units of 2^-24; nearbyint rounds half to even */
        double n = nearbyint(ax * 0x1p24);    /* scaling by 2^24 is exact */
        return (uint16_t)(sign | (uint16_t)n);  /* n == 1024 is the smallest normal */
    }
    int e;
    (void)frexp(ax, &e);                      /* ax = f * 2^e, f in [0.5, 1) */
    int E = e - 1;                            /* ax in [2^E, 2^(E+1)) */
    double n = nearbyint(ldexp(ax, 10 - E));  /* significand in units of 2^(E-10) */
    if (n == 2048.0) { n = 1024.0; E += 1; }
    if (E + 15 >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(n - 1024.0));
}

float or_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return (float)(s ? -v : v);
}

float or_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t or_f32_to_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x40u);
    /* keep the top 16 bits, rounding the dropped 16 to nearest, ties to even */
    uint32_t low = u & 0xFFFFu, top = u >> 16;
    if (low > 0x8000u || (low == 0x8000u && (top & 1u))) top += 1;
    return (uint16_t)top;
}

/* ------------------------------------------------------------------------
 * Packed code layout of one d_k x d_v tile, row-major, packed along d_v.
 * Reading (the pages give no layout): two's-complement codes;
 *   8 bits: one byte per code;
 *   4 bits: code 2m in the low nibble of byte m, code 2m+1 in the high one;
 *   2 bits: code 4m+s in bits 2s..2s+1 of byte m;
 *   6 bits: two planes, first the low 4 bits of every code in the 4-bit
 *           layout (d_k*d_v/2 bytes), then the high 2 bits in the 2-bit
 *           layout (d_k*d_v/4 bytes).
 * ---------------------------------------------------------------------- */
int64_t or_tile_bytes(int bits, int d_k, int d_v)
{
    return (int64_t)d_k * d_v * bits / 8;
}

static void put_field(uint8_t* row, int j, int w, unsigned v)
{
    int per = 8 / w;
    row[j / per] |= (uint8_t)((v & ((1u << w) - 1u)) << (w * (j % per)));
}

static int get_field(const uint8_t* row, int j, int w)
{
    int per = 8 / w;
    return (row[j / per] >> (w * (j % per))) & ((1 << w) - 1);
}

void or_pack(int bits, int d_k, int d_v, const int8_t* codes, uint8_t* out)
{
    memset(out, 0, (size_t)or_tile_bytes(bits, d_k, d_v));
    for (int i = 0; i < d_k; i++) {
        for (int j = 0; j < d_v; j++) {
            int c = codes[(size_t)i * d_v + j];
            if (bits == 8) {
                out[(size_t)i * d_v + j] = (uint8_t)c;
            } else if (bits == 4 || bits == 2) {
                put_field(out + (size_t)i * d_v * bits / 8, j, bits, (unsigned)c);
            } else if (bits == 6) {
                uint8_t* lo = out + (size_t)i * d_v / 2;
                uint8_t* hi = out + (size_t)d_k * d_v / 2 + (size_t)i * d_v / 4;
                put_field(lo, j, 4, (unsigned)c & 15u);
                put_field(hi, j, 2, ((unsigned)c >> 4) & 3u);
            }
        }
    }
}

void or_unpack(int bits, int d_k, int d_v, const uint8_t* in, int8_t* codes)
{
    for (int i = 0; i < d_k; i++) {
        for (int j = 0; j < d_v; j++) {
            int u;
            if (bits == 8) {
                u = in[(size_t)i * d_v + j];
            } else if (bits == 4 || bits == 2) {
                u = get_field(in + (size_t)i * d_v * bits / 8, j, bits);
            } else {
                int lo = get_field(in + (size_t)i * d_v / 2, j, 4);
                int hi = get_field(in + (size_t)d_k * d_v / 2 + (size_t)i * d_v / 4, j, 2);
                u = (hi << 4) | lo;
            }
            if (u >= (1 << (bits - 1))) u -= (1 << bits);   /* sign-extend */
            codes[(size_t)i * d_v + j] = (int8_t)u;
        }
    }
}

/* ------------------------------------------------------------------------
 * Canonical reduction order of the two sums over the key index,
 *   r_j = sum_i (A S)_ij k_i   (GDN, Table 1)   and   o_j = sum_i S_ij q_i.
 * Reading (the pages fix no order): the rows are cut into blocks of 8
 * consecutive rows; each block is summed in ascending row order with a fused
 * multiply-add starting from +0; the block sums are then added pairwise,
 * adjacent blocks first, as a balanced binary tree.  n must be 8 times a
 * power of two.
 * ---------------------------------------------------------------------- */
float or_canon_dot(int n, const float* a, int stride, const float* b)
{
    float part[64];
    int nb = n / 8;
    for (int blk = 0; blk < nb; blk++) {
        float p = 0.0f;
        for (int r = 0; r < 8; r++) {
            int i = 8 * blk + r;
            p = fmaf(a[(size_t)i * stride], b[i], p);
        }
        part[blk] = p;
    }
    while (nb > 1) {
        for (int t = 0; t < nb / 2; t++) part[t] = part[2 * t] + part[2 * t + 1];
        nb /= 2;
    }
    return part[0];
}

/* ------------------------------------------------------------------------
 * Hadamard rotation (INT4+Had of Table 2 of "Preserving Updates ...": the
 * state is rotated by a Hadamard matrix before it is quantized to INT4; the
 * page says no more).
 * Reading: the rotation acts on the value axis of the state (the axis the
 * scale groups run along), S_rot = S H with H the Sylvester Hadamard matrix of
 * order d_v (entries +-1, symmetric, H H = d_v I).  Every decay A_t acts on the
 * key axis and every update is k w^T, so the rotated state follows the same
 * recurrence with the update k (H w)^T:
 *   rank-1:  S_rot,t = A_t S_rot,t-1 + k (H v)^T
 *   GDN:     r_rot = (A_t S_rot,t-1)^T k = H r, e_rot = H v - r_rot = H e
 * and the output is o = S^T q = H (S_rot^T q) / d_v.  The state is quantized
 * in the rotated form; unrotated H (no 1/sqrt(d_v)) keeps every entry exact
 * and the final 1/d_v is a power of two.
 * H x is evaluated by the butterfly: for h = 1, 2, 4, ..., n/2 and every i
 * with (i & h) == 0, (x_i, x_{i+h}) <- (x_i + x_{i+h}, x_i - x_{i+h}), one
 * binary32 rounding per operation, in this order.
 * ---------------------------------------------------------------------- */
void or_fwht(int n, float* x)
{
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i++)
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
}

/* ------------------------------------------------------------------------
 * Rounding.
 * Reading: symmetric codes in [-Qmax, Qmax], Qmax = 2^(b-1) - 1; the scaled
 * value is the exact product x * inv (exact in double: two 24-bit
 * significands), rounded half to even, then clamped.  A NaN product clamps
 * to -Qmax (the maxNum rule of fmax).
 * ---------------------------------------------------------------------- */
int or_round_rtn(float x, float inv, int qmax)
{
    double w = (double)x * (double)inv;
    double r = nearbyint(w);
    if (!(r >= -(double)qmax)) r = -(double)qmax;
    if (r > (double)qmax) r = (double)qmax;
    return (int)r;
}

/* BDR.  Reading of its rule (a reversed element is rounded in the direction
 * of its update instead) with the threshold eps_B of Table 6: the update of the element is d = x - a (a is
 * the decayed state before the update), u = a * inv is where the element
 * sits on the new grid without the update.  The element is reversed when its
 * RTN code lies on the far side of u from the update by more than eps_B grid
 * steps, measured as s = fma(a, inv, -c_rtn); it is then moved one grid
 * step toward its update (which is the nearest grid point on the update's
 * side of x), and clamped. */
int or_round(const or_cfg* c, float a, float x, float inv, int qmax, or_counts* cnt)
{
    int code = or_round_rtn(x, inv, qmax);
    if (c->round_mode == OR_BDR) {
        float d = x - a;
        if (d != 0.0f) {
            float s = fmaf(a, inv, -(float)code);
            if (d > 0.0f && s > c->eps_b) {
                code = code + 1 > qmax ? qmax : code + 1;
                if (cnt) cnt->bdr_applied++;
            } else if (d < 0.0f && s < -c->eps_b) {
                code = code - 1 < -qmax ? -qmax : code - 1;
                if (cnt) cnt->bdr_applied++;
            }
        }
    }
    return code;
}

/* Taxonomy of Figure 4 (left) under RTN, in grid units of the new scale.
 * Reading: an element with update d = x - a != 0 is "reversed" when its RTN
 * code lies strictly on the other side of u = a*inv from the update, "lost"
 * otherwise when the code equals the RTN code of u (the update left no
 * trace), and "moved" otherwise.  All comparisons are exact. */
int or_classify(float a, float x, float inv, int qmax)
{
    float d = x - a;
    if (!(d != 0.0f)) return OR_NONE;
    int c = or_round_rtn(x, inv, qmax);
    double u = (double)a * (double)inv;         /* exact */
    double diff = (double)c - u;                /* sign exact */
    if ((diff < 0.0 && d > 0.0f) || (diff > 0.0 && d < 0.0f)) return OR_REVERSED;
    return c == or_round_rtn(a, inv, qmax) ? OR_LOST : OR_MOVED;
}

/* ------------------------------------------------------------------------
 * Scale conversion to the stored precision.
 * Reading: binary16 scales (4.50 bits per INT4 element at group 32, Table 2
 * of "Preserving Updates ...") are rounded to nearest even; an overflow
 * saturates to 65504 and is counted.  binary32 scales are kept as is.
 * ---------------------------------------------------------------------- */
static float to_stored_scale(const or_cfg* c, float v, or_counts* cnt)
{
    if (c->scale_f32) return v;
    uint16_t h = or_f32_to_f16(v);
    if ((h & 0x7FFFu) == 0x7C00u) {
        h = (uint16_t)((h & 0x8000u) | 0x7BFFu);
        if (cnt) cnt->saturated++;
    }
    return or_f16_to_f32(h);
}

int or_n_scales(const or_cfg* c)
{
    return c->group ? c->d_k * (c->d_v / c->group) : 1;
}

static int valid_cfg(const or_cfg* c)
{
    if (c->d_k < 8 || c->d_k > 512 || c->d_k % 8) return 0;
    int nb = c->d_k / 8;
    if (nb & (nb - 1)) return 0;
    if (c->d_v < 8 || c->d_v % 8) return 0;
    if (c->group < 0 || (c->group && c->d_v % c->group)) return 0;
    if (c->kind < OR_RETNET || c->kind > OR_GDN) return 0;
    if (c->scale_mode < OR_DYNAMIC || c->scale_mode > OR_YOKED) return 0;
    if (c->round_mode < OR_RTN || c->round_mode > OR_BDR) return 0;
    if (c->rotate < 0 || c->rotate > 1) return 0;
    if (c->rotate && (c->d_v > 512 || (c->d_v & (c->d_v - 1)))) return 0;
    return 1;
}

static int finite_all(const float* p, int n)
{
    for (int i = 0; i < n; i++)
        if (!isfinite(p[i])) return 0;
    return 1;
}

/* One step of one tile.  The order of operations is the specification the
 * CUDA kernels implement; each line is one rounded binary32 operation. */
static void tile_step(const or_cfg* c, int bits, int8_t* codes, float* S, float* scales,
                      float* ref, const float* q, const float* k, const float* v,
                      const float* alpha, float beta, float* out, or_counts* cnt,
                      float* a, float* x, float* aref, float* xref, int8_t* cls)
{
    const int dk = c->d_k, dv = c->d_v;
    const int yoked = (c->scale_mode == OR_YOKED) && bits != 32;
    float vrot[512];
    if (c->rotate) {                    /* the update's value vector, rotated */
        memcpy(vrot, v, sizeof(float) * (size_t)dv);
        or_fwht(dv, vrot);
        v = vrot;
    }
    const int qmax = bits == 32 ? 0 : (1 << (bits - 1)) - 1;
    const int gs = c->group ? c->group : dv;             /* group width in columns */
    const int ng = dv / gs;                                /* groups per row */

    /* 1. decay, A_t S_{t-1} (Table 1, decay column).
     * Reading: the dequantized state S_hat = code * scale is decayed as
     * code * (alpha_i * scale), i.e. one product alpha_i * scale per group,
     * then one product per element. */
    for (int i = 0; i < dk; i++) {
        float al = c->kind == OR_RETNET ? c->gamma
                 : c->kind == OR_GLA    ? alpha[i] : alpha[0];
        for (int j = 0; j < dv; j++) {
            size_t e = (size_t)i * dv + j;
            if (bits == 32) {
                a[e] = S[e] * al;
            } else {
                float delta = c->group ? scales[i * ng + j / gs] : scales[0];
                float eta = al * delta;
                a[e] = (float)codes[e] * eta;
            }
            if (yoked) aref[e] = ref[e] * al;
        }
    }

    /* 2. update B_t (Table 1, update column). */
    if (c->kind == OR_GDN) {
        for (int j = 0; j < dv; j++) {
            float r = or_canon_dot(dk, a + j, dv, k);       /* ((A S)^T k)_j */
            float e = v[j] - r;
            float rr = 0.0f, er = 0.0f;
            if (yoked) { rr = or_canon_dot(dk, aref + j, dv, k); er = v[j] - rr; }
            for (int i = 0; i < dk; i++) {
                size_t idx = (size_t)i * dv + j;
                float kap = beta * k[i];
                x[idx] = fmaf(kap, e, a[idx]);
                if (yoked) xref[idx] = fmaf(kap, er, aref[idx]);
            }
        }
    } else {
        for (int i = 0; i < dk; i++)
            for (int j = 0; j < dv; j++) {
                size_t idx = (size_t)i * dv + j;
                x[idx] = fmaf(k[i], v[j], a[idx]);
                if (yoked) xref[idx] = fmaf(k[i], v[j], aref[idx]);
            }
    }

    /* 3. output o_t = S_t^T q_t from the updated, not yet rounded state.
     * Reading: the output is taken before the scale and rounding steps. */
    for (int j = 0; j < dv; j++) out[j] = or_canon_dot(dk, x + j, dv, q);
    if (c->rotate) {                    /* o = H (S_rot^T q) / d_v */
        or_fwht(dv, out);
        for (int j = 0; j < dv; j++) out[j] = out[j] * (1.0f / (float)dv);
    }
    int bad_out = !finite_all(out, dv);

    if (bits == 32) {                     /* quantization disabled */
        memcpy(S, x, sizeof(float) * (size_t)dk * dv);
        return;
    }

    int bad = !finite_all(q, dk) || !finite_all(k, dk) || !finite_all(v, dv);
    if (c->kind == OR_GLA) bad |= !finite_all(alpha, dk);
    else if (c->kind != OR_RETNET) bad |= !isfinite(alpha[0]);
    if (c->kind == OR_GDN) bad |= !isfinite(beta);
    bad |= bad_out;

    /* 4-6. scale and rounding, group by group (a group is gs consecutive
     * columns of one row, or the whole tile for a per-token scale). */
    const int ngroups = or_n_scales(c);
    const float fq = (float)qmax;
    for (int g = 0; g < ngroups; g++) {
        int i0 = c->group ? g / ng : 0, i1 = c->group ? i0 + 1 : dk;
        int j0 = c->group ? (g % ng) * gs : 0, j1 = c->group ? j0 + gs : dv;
        float m = 0.0f, mref = 0.0f;
        for (int i = i0; i < i1; i++)
            for (int j = j0; j < j1; j++) {
                m = fmaxf(m, fabsf(x[(size_t)i * dv + j]));
                if (yoked) mref = fmaxf(mref, fabsf(xref[(size_t)i * dv + j]));
            }
        if (!isfinite(m) || (yoked && !isfinite(mref))) bad = 1;
        float delta;
        if (c->scale_mode == OR_DYNAMIC) {
            /* re-derived from this step's state */
            delta = to_stored_scale(c, m / fq, cnt);
        } else if (c->scale_mode == OR_PERSISTENT) {
            /* Reading: carried across steps and regrown only when the group
             * maximum overflows the code range of the carried scale. */
            float dp = scales[g];
            delta = (m > fq * dp) ? to_stored_scale(c, m / fq, cnt) : dp;
        } else {
            /* yoked to the full-precision reference state of this step */
            delta = to_stored_scale(c, mref / fq, cnt);
        }
        scales[g] = delta;
        float inv = delta == 0.0f ? 0.0f : 1.0f / delta;
        for (int i = i0; i < i1; i++)
            for (int j = j0; j < j1; j++) {
                size_t e = (size_t)i * dv + j;
                if ((cnt && c->taxonomy) || cls) {
                    int k3 = or_classify(a[e], x[e], inv, qmax);
                    if (cls) cls[e] = (int8_t)k3;
                    if (cnt && c->taxonomy) {
                        if (k3 == OR_LOST) cnt->lost++;
                        else if (k3 == OR_MOVED) cnt->moved++;
                        else if (k3 == OR_REVERSED) cnt->reversed++;
                    }
                }
                codes[e] = (int8_t)or_round(c, a[e], x[e], inv, qmax, cnt);
            }
    }
    if (yoked) memcpy(ref, xref, sizeof(float) * (size_t)dk * dv);
    if (bad && cnt) cnt->nonfinite++;
}

int or_step(const or_cfg* c, int64_t ntiles, const int* tile_bits,
            int8_t* codes, float* S, float* scales, float* ref,
            const float* q, const float* k, const float* v,
            const float* alpha, const float* beta, float* out, or_counts* cnt)
{
    return or_step_trace(c, ntiles, tile_bits, codes, S, scales, ref, q, k, v, alpha, beta,
                         out, cnt, NULL, NULL, NULL);
}

int or_step_trace(const or_cfg* c, int64_t ntiles, const int* tile_bits,
                  int8_t* codes, float* S, float* scales, float* ref,
                  const float* q, const float* k, const float* v,
                  const float* alpha, const float* beta, float* out, or_counts* cnt,
                  float* a_out, float* x_out, int8_t* cls_out)
{
    if (!valid_cfg(c)) return -1;
    const int dk = c->d_k, dv = c->d_v;
    const size_t n = (size_t)dk * dv;
    const int nsc = or_n_scales(c);
    const int na = c->kind == OR_GLA ? dk : 1;
    for (int64_t t = 0; t < ntiles; t++) {
        int b = tile_bits[t];
        if (!(b == 2 || b == 4 || b == 6 || b == 8 || b == 32)) return -1;
        if (c->scale_mode == OR_YOKED && b != 32 && !ref) return -1;
    }
    float* buf = (float*)malloc(sizeof(float) * n * 4);
    if (!buf) return -1;
    for (int64_t t = 0; t < ntiles; t++) {
        tile_step(c, tile_bits[t],
                  codes ? codes + t * n : NULL, S ? S + t * n : NULL,
                  scales ? scales + t * nsc : NULL, ref ? ref + t * n : NULL,
                  q + t * dk, k + t * dk, v + t * dv,
                  alpha ? alpha + t * na : NULL, beta ? beta[t] : 0.0f,
                  out + t * dv, cnt,
                  a_out ? a_out + t * n : buf, x_out ? x_out + t * n : buf + n,
                  buf + 2 * n, buf + 3 * n, cls_out ? cls_out + t * n : NULL);
    }
    free(buf);
    return 0;
}

void or_dequant(const or_cfg* c, int bits, const int8_t* codes, const float* scales,
                float* S_out)
{
    (void)bits;
    const int dk = c->d_k, dv = c->d_v;
    const int gs = c->group ? c->group : dv, ng = dv / gs;
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            float delta = c->group ? scales[i * ng + j / gs] : scales[0];
            S_out[(size_t)i * dv + j] = (float)codes[(size_t)i * dv + j] * delta;
        }
}

/* ========================================================================
 * Low-Rank Bypass (LRB), "Preserving Updates in Low-Bit Recurrent State
 * Quantization": the Abstract (small updates collect in a low-rank buffer,
 * and the buffer's large elements go into the state from time to time),
 * Figure 3 (updates go to the bypass and are written into
 * the quantized state every m steps), Table 6 (k, m, eps_L per model, and
 * the average / peak storage per state element) and Tables 8-9 (the rank k
 * and the number k + m of bypass columns).
 *
 * Readings (the pages give the structure and the storage, not the rule):
 *  L1 The bypass of a tile holds up to k + m column pairs (u_l in R^{d_k},
 *     w_l in R^{d_v}) in binary16 with one binary32 coefficient g_l each; it
 *     stands for P = sum_l g_l u_l w_l^T, and the tile's state is the
 *     dequantized codes plus P.  Storage per column: (d_k + d_v) 16-bit
 *     values plus the 32-bit coefficient (this reproduces the bits of
 *     Tables 6, 8 and 9; see or_lrb_bits).
 *  L2 Slots 0 .. n_res-1 hold the rank-k residual, slots n_res .. n-1 the
 *     fresh updates in arrival order.
 *  L3 Between merges the codes and scales are not touched: the decay since
 *     the last merge accumulates in one binary32 factor D per tile,
 *     D <- alpha * D (scalar decays: RetNet gamma, Mamba2 and GDN alpha_t),
 *     so the decayed quantized part is a_ij = code_ij * (D * scale_ij), the
 *     plain step's decay with D for alpha; rounding happens only at a merge
 *     (a re-rounding every step would lose the decay of every code below
 *     1 / (2 (1 - alpha)) under a persistent scale).  The per-row decay of
 *     GLA would need a factor per row (one binary32 per row: the extra 1/16
 *     bit of GLA in Table 6 at d_v = 512) and is not read here.  Every
 *     column's coefficient decays with its own product since insertion,
 *     g_l <- alpha * g_l, a new column starting at g = 1.
 *  L4 The step's update enters the bypass as a new column: rank-1 kinds
 *     (binary16(k), binary16(v), 1); GDN (binary16(beta k), binary16(e), 1)
 *     with e = v - r and r = (A_t S_{t-1})^T k over the whole state:
 *     r_j = csum_i(a_ij k_i), then for each column l in slot order
 *     r_j <- fma(g_l * csum_i(u_li k_i), w_lj, r_j).
 *  L5 The output is o_t = (a + P_t)^T q_t in the same form: the canonical
 *     sum over the decayed quantized part, then the columns in slot order.
 *  L7 GLA (decay Diag(alpha_t)): D is one binary32 factor per key row
 *     (D_i <- alpha_t,i * D_i; the 32 bits per row are the extra 1/16 bit of
 *     GLA in Table 6 at d_v = 512); no coefficient decays (g stays 1); a
 *     column's key side is stored divided by the row factors of its step,
 *     binary16(k_i / D_i), and read as D_i * u_i, which carries every later
 *     step's decay of row i; the merge threshold uses D_i of the element's
 *     row.
 *  L6 When the m-th fresh column arrives the bypass is merged: the dense
 *     P_ij = sum_l fma(g_l * u_li, w_lj, .) (slots in order, from +0) is
 *     formed; an element is merged when |P_ij| >= eps_L * (D * scale_ij), eps_L
 *     grid steps of the decayed grid it lives on; the state is requantized
 *     from x = a + P on merged elements and x = a elsewhere (the scale rule
 *     and the rounding rule of the plain step, BDR with d = x - a) and D is
 *     reset to 1; the unmerged part R (P with the merged elements zeroed) is
 *     replaced by its best rank-k approximation (truncated SVD, Eckart-Young)
 *     stored as u_l = binary16(sqrt(s_l) U_l), w_l = binary16(sqrt(s_l) V_l),
 *     g_l = 1; the fresh slots are emptied.  With k = 0, m = 1 and eps_L = 0
 *     this is the plain quantized step (a + u w rounds once, as fma(k, v, a),
 *     when k and v are exact in binary16).
 * ====================================================================== */

/* binary16 round trip of a binary32 value (the stored bypass precision) */
static float f16r(float x) { return or_f16_to_f32(or_f32_to_f16(x)); }

/* Top-k singular triplets of R (rows x cols, row-major, fp64) by cyclic
 * Jacobi on the Gram matrix R^T R (cols x cols): eigenvalues s^2 and
 * eigenvectors V; U_l = R V_l / s_l.  Writes s[k], U[k][rows], V[k][cols]
 * (zeros past the rank). */
void or_rank_k(int rows, int cols, const double* R, int k, double* s, double* U, double* V)
{
    double* A = (double*)calloc((size_t)cols * cols, sizeof(double));
    double* E = (double*)calloc((size_t)cols * cols, sizeof(double));
    for (int a = 0; a < cols; a++) {
        E[(size_t)a * cols + a] = 1.0;
        for (int b = 0; b < cols; b++) {
            double t = 0.0;
            for (int i = 0; i < rows; i++) t += R[(size_t)i * cols + a] * R[(size_t)i * cols + b];
            A[(size_t)a * cols + b] = t;
        }
    }
    for (int sweep = 0; sweep < 60; sweep++) {
        double off = 0.0, diag = 0.0;
        for (int a = 0; a < cols; a++) {
            diag += A[(size_t)a * cols + a] * A[(size_t)a * cols + a];
            for (int b = a + 1; b < cols; b++) off += A[(size_t)a * cols + b] * A[(size_t)a * cols + b];
        }
        if (off <= 1e-30 * (diag + 1e-300)) break;
        for (int p = 0; p < cols; p++)
            for (int q = p + 1; q < cols; q++) {
                double apq = A[(size_t)p * cols + q];
                if (apq == 0.0) continue;
                double app = A[(size_t)p * cols + p], aqq = A[(size_t)q * cols + q];
                double theta = (aqq - app) / (2.0 * apq);
                double t = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                double cs = 1.0 / sqrt(t * t + 1.0), sn = t * cs;
                for (int r = 0; r < cols; r++) {          /* A <- J^T A J */
                    double arp = A[(size_t)r * cols + p], arq = A[(size_t)r * cols + q];
                    A[(size_t)r * cols + p] = cs * arp - sn * arq;
                    A[(size_t)r * cols + q] = sn * arp + cs * arq;
                }
                for (int r = 0; r < cols; r++) {
                    double apr = A[(size_t)p * cols + r], aqr = A[(size_t)q * cols + r];
                    A[(size_t)p * cols + r] = cs * apr - sn * aqr;
                    A[(size_t)q * cols + r] = sn * apr + cs * aqr;
                }
                for (int r = 0; r < cols; r++) {          /* E <- E J */
                    double erp = E[(size_t)r * cols + p], erq = E[(size_t)r * cols + q];
                    E[(size_t)r * cols + p] = cs * erp - sn * erq;
                    E[(size_t)r * cols + q] = sn * erp + cs * erq;
                }
            }
    }
    /* pick the k largest eigenvalues */
    char* used = (char*)calloc((size_t)cols, 1);
    for (int l = 0; l < k; l++) {
        int best = -1;
        for (int a = 0; a < cols; a++)
            if (!used[a] && (best < 0 || A[(size_t)a * cols + a] > A[(size_t)best * cols + best])) best = a;
        double lam = best >= 0 ? A[(size_t)best * cols + best] : 0.0;
        double sig = lam > 0.0 ? sqrt(lam) : 0.0;
        s[l] = sig;
        for (int b = 0; b < cols; b++) V[(size_t)l * cols + b] = (best >= 0 && sig > 0.0) ? E[(size_t)b * cols + best] : 0.0;
        for (int i = 0; i < rows; i++) {
            double t = 0.0;
            if (sig > 0.0)
                for (int b = 0; b < cols; b++) t += R[(size_t)i * cols + b] * V[(size_t)l * cols + b];
            U[(size_t)l * rows + i] = sig > 0.0 ? t / sig : 0.0;
        }
        if (best >= 0) used[best] = 1;
    }
    free(used);
    free(A);
    free(E);
}

/* Storage per state element of a tile with `cols_used` bypass columns. */
double or_lrb_bits(int bits, int group, int scale_bits, int d_k, int d_v, double cols_used)
{
    double base = (double)bits + (group ? (double)scale_bits / group : (double)scale_bits / ((double)d_k * d_v));
    return base + cols_used * 16.0 * (d_k + d_v + 2) / ((double)d_k * d_v);
}

static int valid_lrb(const or_cfg* c, const or_lrb_cfg* L)
{
    if (!valid_cfg(c) || !L) return 0;
    if (c->scale_mode == OR_YOKED || c->rotate) return 0;
    if (L->k < 0 || L->m < 1 || L->k + L->m > OR_LRB_MAX_COLS) return 0;
    if (!(L->eps_l >= 0.0f)) return 0;
    return 1;
}

/* One LRB step of one tile (bits 2..8).  u, w: [k+m][d_k], [k+m][d_v]
 * binary16 bit patterns; g: [k+m]; nres, nnew: slot counts. */
static void lrb_tile_step(const or_cfg* c, const or_lrb_cfg* L, int bits, int8_t* codes,
                          float* scales, uint16_t* u, uint16_t* w, float* g, int* nres, int* nnew,
                          float* D,
                          const float* q, const float* k, const float* v, const float* alpha,
                          float beta, float* out, or_counts* cnt, int* merged_out,
                          float* resid_out)
{
    const int dk = c->d_k, dv = c->d_v;
    const int qmax = (1 << (bits - 1)) - 1;
    const int gs = c->group ? c->group : dv, ng = dv / gs;
    const size_t n_el = (size_t)dk * dv;
    float* a = (float*)malloc(sizeof(float) * n_el);
    float* x = (float*)malloc(sizeof(float) * n_el);
    float* P = (float*)malloc(sizeof(float) * n_el);
    float uf[OR_LRB_MAX_COLS][512], wf[OR_LRB_MAX_COLS][512];
    const int gla = c->kind == OR_GLA;
    const float al = c->kind == OR_RETNET ? c->gamma : alpha[0];

    /* L3: the decay accumulates in D (GLA: one factor per key row, L7); the
     * decayed quantized part as the plain step's decay with D for alpha; the
     * columns' own decays (scalar decays: their coefficients) */
    if (gla) {
        for (int i = 0; i < dk; i++) D[i] = alpha[i] * D[i];
    } else {
        *D = al * *D;
    }
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            size_t e = (size_t)i * dv + j;
            float delta = c->group ? scales[i * ng + j / gs] : scales[0];
            a[e] = (float)codes[e] * ((gla ? D[i] : *D) * delta);
        }
    int n = *nres + *nnew;
    if (!gla)
        for (int l = 0; l < n; l++) g[l] = al * g[l];

    /* L4: the update as a new column (GLA, L7: the key side held divided by
     * D, each column's effective key side D * u formed when it is read) */
    for (int l = 0; l < n; l++) {
        for (int i = 0; i < dk; i++) {
            uf[l][i] = or_f16_to_f32(u[(size_t)l * dk + i]);
            if (gla) uf[l][i] = D[i] * uf[l][i];
        }
        for (int j = 0; j < dv; j++) wf[l][j] = or_f16_to_f32(w[(size_t)l * dv + j]);
    }
    float wnew[512], unew[512];
    if (c->kind == OR_GDN) {
        float r[512];
        for (int j = 0; j < dv; j++) r[j] = or_canon_dot(dk, a + j, dv, k);
        for (int l = 0; l < n; l++) {
            float cl = g[l] * or_canon_dot(dk, uf[l], 1, k);
            for (int j = 0; j < dv; j++) r[j] = fmaf(cl, wf[l][j], r[j]);
        }
        for (int j = 0; j < dv; j++) wnew[j] = f16r(v[j] - r[j]);
        for (int i = 0; i < dk; i++) unew[i] = f16r(beta * k[i]);
    } else {
        for (int j = 0; j < dv; j++) wnew[j] = f16r(v[j]);
        for (int i = 0; i < dk; i++) unew[i] = f16r(gla ? k[i] / D[i] : k[i]);
    }
    for (int i = 0; i < dk; i++) {
        u[(size_t)n * dk + i] = or_f32_to_f16(unew[i]);
        uf[n][i] = gla ? D[i] * unew[i] : unew[i];
    }
    for (int j = 0; j < dv; j++) { w[(size_t)n * dv + j] = or_f32_to_f16(wnew[j]); wf[n][j] = wnew[j]; }
    g[n] = 1.0f;
    n++;
    (*nnew)++;

    /* L5: output */
    for (int j = 0; j < dv; j++) out[j] = or_canon_dot(dk, a + j, dv, q);
    for (int l = 0; l < n; l++) {
        float cl = g[l] * or_canon_dot(dk, uf[l], 1, q);
        for (int j = 0; j < dv; j++) out[j] = fmaf(cl, wf[l][j], out[j]);
    }

    /* L6: merge every m fresh columns; otherwise requantize the decayed state */
    const int merge = *nnew == L->m;
    int n_merged = 0;
    memcpy(x, a, sizeof(float) * n_el);
    if (merge) {
        for (size_t e = 0; e < n_el; e++) P[e] = 0.0f;
        for (int l = 0; l < n; l++)
            for (int i = 0; i < dk; i++) {
                float gu = g[l] * uf[l][i];
                for (int j = 0; j < dv; j++)
                    P[(size_t)i * dv + j] = fmaf(gu, wf[l][j], P[(size_t)i * dv + j]);
            }
        for (int i = 0; i < dk; i++)
            for (int j = 0; j < dv; j++) {
                size_t e = (size_t)i * dv + j;
                float dprev = c->group ? scales[i * ng + j / gs] : scales[0];
                if (fabsf(P[e]) >= L->eps_l * ((gla ? D[i] : *D) * dprev)) {
                    x[e] = a[e] + P[e];
                    P[e] = 0.0f;                     /* merged: leaves the residual */
                    n_merged++;
                }
            }
    }
    if (!merge) {                  /* L3: nothing is rounded between merges */
        if (merged_out) *merged_out = 0;
        free(a);
        free(x);
        free(P);
        return;
    }
    /* scale and rounding (the plain step's rules, on x, with a for BDR) */
    const int ngroups = or_n_scales(c);
    const float fq = (float)qmax;
    for (int gi = 0; gi < ngroups; gi++) {
        int i0 = c->group ? gi / ng : 0, i1 = c->group ? i0 + 1 : dk;
        int j0 = c->group ? (gi % ng) * gs : 0, j1 = c->group ? j0 + gs : dv;
        float m = 0.0f;
        for (int i = i0; i < i1; i++)
            for (int j = j0; j < j1; j++) m = fmaxf(m, fabsf(x[(size_t)i * dv + j]));
        float delta;
        if (c->scale_mode == OR_DYNAMIC) {
            delta = to_stored_scale(c, m / fq, cnt);
        } else {
            float dp = scales[gi];
            delta = (m > fq * dp) ? to_stored_scale(c, m / fq, cnt) : dp;
        }
        scales[gi] = delta;
        float inv = delta == 0.0f ? 0.0f : 1.0f / delta;
        for (int i = i0; i < i1; i++)
            for (int j = j0; j < j1; j++) {
                size_t e = (size_t)i * dv + j;
                codes[e] = (int8_t)or_round(c, a[e], x[e], inv, qmax, cnt);
            }
    }
    if (merge) {
        if (resid_out) memcpy(resid_out, P, sizeof(float) * n_el);
        /* the unmerged residual as its best rank-k approximation */
        const int kk = L->k;
        if (kk > 0) {
            double* R = (double*)malloc(sizeof(double) * n_el);
            double* U = (double*)malloc(sizeof(double) * (size_t)kk * dk);
            double* V = (double*)malloc(sizeof(double) * (size_t)kk * dv);
            double s[OR_LRB_MAX_COLS];
            for (size_t e = 0; e < n_el; e++) R[e] = P[e];
            or_rank_k(dk, dv, R, kk, s, U, V);
            for (int l = 0; l < kk; l++) {
                double rs = sqrt(s[l]);
                for (int i = 0; i < dk; i++)
                    u[(size_t)l * dk + i] = or_f32_to_f16((float)(rs * U[(size_t)l * dk + i]));
                for (int j = 0; j < dv; j++)
                    w[(size_t)l * dv + j] = or_f32_to_f16((float)(rs * V[(size_t)l * dv + j]));
                g[l] = 1.0f;
            }
            free(R);
            free(U);
            free(V);
        }
        *nres = kk;
        *nnew = 0;
        if (gla)
            for (int i = 0; i < dk; i++) D[i] = 1.0f;
        else
            *D = 1.0f;
    }
    if (merged_out) *merged_out = n_merged;
    free(a);
    free(x);
    free(P);
}

int or_lrb_step(const or_cfg* c, const or_lrb_cfg* L, int64_t ntiles, const int* tile_bits,
                int8_t* codes, float* scales, uint16_t* u, uint16_t* w, float* g, int* nres,
                int* nnew, float* D, const float* q, const float* k, const float* v,
                const float* alpha, const float* beta, float* out, or_counts* cnt, int* merged,
                float* resid)
{
    if (!valid_lrb(c, L)) return -1;
    const int dk = c->d_k, dv = c->d_v, K = L->k + L->m, nsc = or_n_scales(c);
    for (int64_t t = 0; t < ntiles; t++)
        if (tile_bits[t] < 2 || tile_bits[t] > 8 || tile_bits[t] % 2) return -1;
    for (int64_t t = 0; t < ntiles; t++)
        lrb_tile_step(c, L, tile_bits[t], codes + t * dk * dv, scales + t * nsc,
                      u + t * K * dk, w + t * K * dv, g + t * K, nres + t, nnew + t,
                      D + (c->kind == OR_GLA ? t * dk : t), q + t * dk, k + t * dk, v + t * dv,
                      alpha ? alpha + (c->kind == OR_GLA ? t * dk : t) : NULL,
                      beta ? beta[t] : 0.0f, out + t * dv, cnt, merged ? merged + t : NULL,
                      resid ? resid + t * (int64_t)dk * dv : NULL);
    return 0;
}


/* ------------------------------------------------------------------------
 * Pure-write sliding window (PW) of "Low-Bit GDN Recurrent-State
 * Quantization: Global Gradient-aware Allocation and Pure-Write Sliding
 * Windows" (Abstract).  The page gives the method in one sentence: the
 * recent pure writes are kept as FP8 vector pairs, carried through the full
 * Gated DeltaNet transition, and merged into the low-bit history only once
 * they leave the window.  Readings:
 *  W1 the pure write of step t is beta_t k_t v_t^T (the update without its
 *     erase term); its pair is (fp8(beta_t k_t), fp8(v_t)), beta_t k_t the
 *     binary32 product;
 *  W2 FP8 is OCP E4M3 without per-vector scales, encoded to nearest with
 *     ties to even and saturating at 448;
 *  W3 the transition A_t = alpha_t (I - beta_t k_t k_t^T) acts on every
 *     part of the state: the history as the plain Gated DeltaNet step with
 *     v = 0 (a = alpha (x) S_hat, r = a^T k, x = fma(beta k_i, -r_j, a_ij)),
 *     and each stored pair on its key side:
 *     s = canon(a_l . k), t_i = fma(-(beta (x) s), k_i, a_l,i),
 *     a_l,i <- fp8(alpha (x) t_i), the value side unchanged;
 *  W4 a window of W pairs: after the transition, when W pairs are held, the
 *     oldest leaves and is merged into the history, x_ij = fma(a_i, b_j, x_ij);
 *     then the step's own pair enters (in the slot the leaver freed);
 *  W5 the output is the whole state's: o = canon(x^T q), then for every pair
 *     held after the step, oldest first, o_j = fma(canon(a_l . q), b_l,j, o_j);
 *  W6 the history is requantized every step with the object's scale and
 *     rounding rules (BDR with d = x - a, a the decayed history).
 * ---------------------------------------------------------------------- */
float or_e4m3_to_f32(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    float v = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    return (b & 0x80) ? -v : v;
}

uint8_t or_f32_to_e4m3(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t s = signbit(x) ? 0x80 : 0;
    double ax = fabs((double)x);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 127; c++) {      /* the finite non-negative codes, ascending */
        double d = fabs((double)or_e4m3_to_f32((uint8_t)c) - ax);
        if (d < bd || (d == bd && !(c & 1))) {
            bd = d;
            best = c;
        }
    }
    return (uint8_t)(s | best);
}

static void pw_tile_step(const or_cfg* c, int W, int bits, int8_t* codes, float* S,
                         float* scales, uint8_t* A, uint8_t* B, int* head, int* count,
                         const float* q, const float* k, const float* v, float al, float be,
                         float* out, or_counts* cnt)
{
    const int dk = c->d_k, dv = c->d_v;
    const size_t n_el = (size_t)dk * dv;
    const int gs = c->group ? c->group : dv, ng = dv / gs;
    float* a = (float*)malloc(sizeof(float) * n_el);
    float* x = (float*)malloc(sizeof(float) * n_el);
    float al_[512], bl_[512];

    /* W3: the history's transition */
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            size_t e = (size_t)i * dv + j;
            if (bits == 32) {
                a[e] = S[e] * al;
            } else {
                float delta = c->group ? scales[i * ng + j / gs] : scales[0];
                a[e] = (float)codes[e] * (al * delta);
            }
        }
    for (int j = 0; j < dv; j++) {
        float r = or_canon_dot(dk, a + j, dv, k);
        float e = -r;
        for (int i = 0; i < dk; i++) {
            size_t idx = (size_t)i * dv + j;
            x[idx] = fmaf(be * k[i], e, a[idx]);
        }
    }
    /* W3: the pairs' key sides */
    int h = *head, n = *count;
    for (int l = 0; l < n; l++) {
        uint8_t* Ak = A + (size_t)((h + l) % W) * dk;
        for (int i = 0; i < dk; i++) al_[i] = or_e4m3_to_f32(Ak[i]);
        float s = or_canon_dot(dk, al_, 1, k);
        float cs = be * s;
        for (int i = 0; i < dk; i++) Ak[i] = or_f32_to_e4m3(al * fmaf(-cs, k[i], al_[i]));
    }
    /* W4: the oldest leaves a full window into the history; the new pair */
    int slot;
    if (n == W) {
        uint8_t* Ak = A + (size_t)h * dk;
        uint8_t* Bv = B + (size_t)h * dv;
        for (int i = 0; i < dk; i++) al_[i] = or_e4m3_to_f32(Ak[i]);
        for (int j = 0; j < dv; j++) bl_[j] = or_e4m3_to_f32(Bv[j]);
        for (int i = 0; i < dk; i++)
            for (int j = 0; j < dv; j++) {
                size_t idx = (size_t)i * dv + j;
                x[idx] = fmaf(al_[i], bl_[j], x[idx]);
            }
        slot = h;
        h = (h + 1) % W;
    } else {
        slot = (h + n) % W;
        n++;
    }
    for (int i = 0; i < dk; i++) A[(size_t)slot * dk + i] = or_f32_to_e4m3(be * k[i]);
    for (int j = 0; j < dv; j++) B[(size_t)slot * dv + j] = or_f32_to_e4m3(v[j]);
    *head = h;
    *count = n;

    /* W5: the output of the whole state */
    for (int j = 0; j < dv; j++) out[j] = or_canon_dot(dk, x + j, dv, q);
    for (int l = 0; l < n; l++) {
        int sl = (h + l) % W;
        for (int i = 0; i < dk; i++) al_[i] = or_e4m3_to_f32(A[(size_t)sl * dk + i]);
        float cq = or_canon_dot(dk, al_, 1, q);
        for (int j = 0; j < dv; j++) out[j] = fmaf(cq, or_e4m3_to_f32(B[(size_t)sl * dv + j]), out[j]);
    }

    /* W6: requantize the history */
    if (bits == 32) {
        memcpy(S, x, sizeof(float) * n_el);
    } else {
        const int qmax = (1 << (bits - 1)) - 1;
        const float fq = (float)qmax;
        for (int g = 0; g < or_n_scales(c); g++) {
            int i0 = c->group ? g / ng : 0, i1 = c->group ? i0 + 1 : dk;
            int j0 = c->group ? (g % ng) * gs : 0, j1 = c->group ? j0 + gs : dv;
            float m = 0.0f;
            for (int i = i0; i < i1; i++)
                for (int j = j0; j < j1; j++) m = fmaxf(m, fabsf(x[(size_t)i * dv + j]));
            float delta;
            if (c->scale_mode == OR_DYNAMIC) {
                delta = to_stored_scale(c, m / fq, cnt);
            } else {
                float dp = scales[g];
                delta = (m > fq * dp) ? to_stored_scale(c, m / fq, cnt) : dp;
            }
            scales[g] = delta;
            float inv = delta == 0.0f ? 0.0f : 1.0f / delta;
            for (int i = i0; i < i1; i++)
                for (int j = j0; j < j1; j++) {
                    size_t e = (size_t)i * dv + j;
                    codes[e] = (int8_t)or_round(c, a[e], x[e], inv, qmax, cnt);
                }
        }
    }
    free(a);
    free(x);
}

int or_pw_step(const or_cfg* c, int W, int64_t ntiles, const int* tile_bits,
               int8_t* codes, float* S, float* scales, uint8_t* A, uint8_t* B, int* head,
               int* count, const float* q, const float* k, const float* v,
               const float* alpha, const float* beta, float* out, or_counts* cnt)
{
    if (!valid_cfg(c) || c->kind != OR_GDN || c->scale_mode == OR_YOKED || c->rotate) return -1;
    if (W < 1 || W > OR_PW_MAX_W || c->d_k > 512 || c->d_v > 512) return -1;
    const int dk = c->d_k, dv = c->d_v, nsc = or_n_scales(c);
    for (int64_t t = 0; t < ntiles; t++) {
        int b = tile_bits[t];
        if (!(b == 32 || (b >= 2 && b <= 8 && b % 2 == 0))) return -1;
    }
    for (int64_t t = 0; t < ntiles; t++)
        pw_tile_step(c, W, tile_bits[t], codes + t * dk * dv, S + t * dk * dv, scales + t * nsc,
                     A + t * (int64_t)W * dk, B + t * (int64_t)W * dv, head + t, count + t,
                     q + t * dk, k + t * dk, v + t * dv, alpha[t], beta[t], out + t * dv, cnt);
    return 0;
}


/* ------------------------------------------------------------------------
 * Key-row x value-column scales ("STEPQuant: When and Where Errors Matter
 * in Delta-Rule Recurrent State Quantization", Abstract: key-row and
 * value-column scales fitted jointly from the state's distribution, the
 * state's magnitudes varying along both rows and columns).  The page fits
 * them offline against trained models' output error (out of scope here);
 * this is the plainest joint fit from the state alone.  Readings:
 *  R1 a tile holds row scales rho_i (i < d_k) and column scales kappa_j
 *     (j < d_v) in the object's scale format; the grid step of element
 *     (i, j) is Delta_ij = rho_i * kappa_j (a binary32 product, exact for
 *     binary16 scales);
 *  R2 fitted every step from the updated state x before rounding: kappa_j =
 *     cvt(max_i |x_ij|) (the column maxima), ikappa_j = 1/kappa_j (0 for
 *     0); rho_i = cvt(max_j(|x_ij| * ikappa_j) / Qmax) (each row's largest
 *     column-normalised magnitude spread over the code range), irho_i =
 *     1/rho_i (0 for 0);
 *  R3 c_ij = clamp(rne(x_ij * inv_ij)), inv_ij = irho_i * ikappa_j (the
 *     exact product x * inv rounded to nearest even, as the plain step);
 *     BDR with a = the decayed state and the same inv;
 *  R4 the decay of a quantized tile: a_ij = code_ij * ((alpha_i * rho_i) *
 *     kappa_j), alpha_i the row's decay (GLA) or the scalar one;
 *  R5 dynamic scales only (a carried or yoked rule is not defined for a
 *     two-factor scale).
 * ---------------------------------------------------------------------- */
static void rc_tile_step(const or_cfg* c, int bits, int8_t* codes, float* scales,
                         const float* q, const float* k, const float* v, const float* alpha,
                         float beta, float* out, or_counts* cnt)
{
    const int dk = c->d_k, dv = c->d_v;
    const size_t n_el = (size_t)dk * dv;
    const int qmax = (1 << (bits - 1)) - 1;
    const float fq = (float)qmax;
    float* rho = scales;
    float* kap = scales + dk;
    float* a = (float*)malloc(sizeof(float) * n_el);
    float* x = (float*)malloc(sizeof(float) * n_el);

    /* R4: decay */
    for (int i = 0; i < dk; i++) {
        float al = c->kind == OR_RETNET ? c->gamma : c->kind == OR_GLA ? alpha[i] : alpha[0];
        float ar = al * rho[i];
        for (int j = 0; j < dv; j++) {
            size_t e = (size_t)i * dv + j;
            a[e] = (float)codes[e] * (ar * kap[j]);
        }
    }
    /* update and output: the plain step's */
    if (c->kind == OR_GDN) {
        for (int j = 0; j < dv; j++) {
            float r = or_canon_dot(dk, a + j, dv, k);
            float e = v[j] - r;
            for (int i = 0; i < dk; i++) {
                size_t idx = (size_t)i * dv + j;
                x[idx] = fmaf(beta * k[i], e, a[idx]);
            }
        }
    } else {
        for (int i = 0; i < dk; i++)
            for (int j = 0; j < dv; j++) {
                size_t idx = (size_t)i * dv + j;
                x[idx] = fmaf(k[i], v[j], a[idx]);
            }
    }
    for (int j = 0; j < dv; j++) out[j] = or_canon_dot(dk, x + j, dv, q);

    /* R2: the scales */
    float ikap[512], irho[512];
    for (int j = 0; j < dv; j++) {
        float m = 0.0f;
        for (int i = 0; i < dk; i++) m = fmaxf(m, fabsf(x[(size_t)i * dv + j]));
        kap[j] = to_stored_scale(c, m, cnt);
        ikap[j] = kap[j] == 0.0f ? 0.0f : 1.0f / kap[j];
    }
    for (int i = 0; i < dk; i++) {
        float m = 0.0f;
        for (int j = 0; j < dv; j++) m = fmaxf(m, fabsf(x[(size_t)i * dv + j]) * ikap[j]);
        rho[i] = to_stored_scale(c, m / fq, cnt);
        irho[i] = rho[i] == 0.0f ? 0.0f : 1.0f / rho[i];
    }
    /* R3: rounding */
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            size_t e = (size_t)i * dv + j;
            codes[e] = (int8_t)or_round(c, a[e], x[e], irho[i] * ikap[j], qmax, cnt);
        }
    int bad = !finite_all(out, dv) || !finite_all(x, (int)n_el);
    if (bad && cnt) cnt->nonfinite++;
    free(a);
    free(x);
}

int or_rc_step(const or_cfg* c, int64_t ntiles, const int* tile_bits, int8_t* codes,
               float* scales, const float* q, const float* k, const float* v,
               const float* alpha, const float* beta, float* out, or_counts* cnt)
{
    if (!valid_cfg(c) || c->scale_mode != OR_DYNAMIC || c->rotate) return -1;
    if (c->d_k > 512 || c->d_v > 512) return -1;
    const int dk = c->d_k, dv = c->d_v;
    for (int64_t t = 0; t < ntiles; t++)
        if (tile_bits[t] < 2 || tile_bits[t] > 8 || tile_bits[t] % 2) return -1;
    const int na = c->kind == OR_GLA ? dk : 1;
    for (int64_t t = 0; t < ntiles; t++)
        rc_tile_step(c, tile_bits[t], codes + t * dk * dv, scales + t * (dk + dv), q + t * dk,
                     k + t * dk, v + t * dv, alpha ? alpha + t * na : NULL,
                     beta ? beta[t] : 0.0f, out + t * dv, cnt);
    return 0;
}

void or_rc_dequant(const or_cfg* c, const int8_t* codes, const float* scales, float* S_out)
{
    const int dk = c->d_k, dv = c->d_v;
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++)
            S_out[(size_t)i * dv + j] = (float)codes[(size_t)i * dv + j] * (scales[i] * scales[dk + j]);
}
