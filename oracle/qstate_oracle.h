/*
 * qstate_oracle.h -- plain, slow, scalar CPU oracle of the quantized
 * recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this code; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant table with the
 * CUDA library.
 *
 * What it follows (all citations are to the source pages):
 *  - "Preserving Updates in Low-Bit Recurrent State Quantization", Table 1:
 *    the recurrence S_t = A_t S_{t-1} + B_t with
 *      RetNet  A = gamma I,        B = k v^T
 *      Mamba2  A = alpha_t I,      B = k v^T
 *      GLA     A = Diag(alpha_t),  B = k v^T
 *      GDN     A = alpha_t I,      B = beta_t k (v - (A S_{t-1})^T k)^T
 *    and the output o_t = S_t^T q_t.
 *  - same page, Abstract: the state is requantized after every update; a
 *    reversed element is rounded toward its update (Bounded Directional
 *    Rounding), Figure 4 caption: lost / moved / reversed updates; Table 6:
 *    the BDR threshold eps_B.
 *  - "When Dynamic Scaling Fails", Abstract: dynamic scale re-derived from the
 *    state each step, persistent scale, and a scale yoked to a full-precision
 *    reference state.
 *  - same page and Table 2 of the second page: group-wise INT4 at 4.50 bits
 *    per element (4-bit codes plus one 16-bit scale per 32 elements).
 *  - "Low-Bit Recurrent States in Hybrid Language Models", Abstract: per-token
 *    (one scale per head per step) state quantization and mixed bit widths.
 *
 * Readings of points the pages leave open are stated next to the code that
 * implements them in qstate_oracle.c.
 */
#ifndef QSTATE_ORACLE_H
#define QSTATE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_RETNET = 0, OR_MAMBA2 = 1, OR_GLA = 2, OR_GDN = 3 };
enum { OR_DYNAMIC = 0, OR_PERSISTENT = 1, OR_YOKED = 2 };
enum { OR_RTN = 0, OR_BDR = 1 };
enum { OR_NONE = 0, OR_LOST = 1, OR_MOVED = 2, OR_REVERSED = 3 };

typedef struct {
    int d_k, d_v;     /* state is d_k rows (key index) x d_v columns (value index) */
    int kind;         /* OR_RETNET .. OR_GDN */
    int group;        /* columns per scale group along d_v; 0 = one scale per tile */
    int scale_mode;   /* OR_DYNAMIC, OR_PERSISTENT, OR_YOKED */
    int round_mode;   /* OR_RTN, OR_BDR */
    int scale_f32;    /* 0: scales stored as IEEE binary16, 1: binary32 */
    float gamma;      /* RetNet decay */
    float eps_b;      /* BDR threshold, in grid steps of the new scale */
    int taxonomy;     /* nonzero: count lost / moved / reversed elements */
    int rotate;       /* 1: the state is kept rotated by a Hadamard matrix along d_v
                         (INT4+Had of Table 2 of "Preserving Updates ..."); 0: none */
} or_cfg;

typedef struct {
    int64_t nonfinite;   /* tile-steps with a non-finite input, output or group maximum */
    int64_t saturated;   /* binary16 scale conversions that overflowed */
    int64_t lost, moved, reversed, bdr_applied;  /* rounding taxonomy counts */
} or_counts;

/* ---- number formats ---------------------------------------------------- */
uint16_t or_f32_to_f16(float x);      /* IEEE round-to-nearest-even; inf on overflow */
float    or_f16_to_f32(uint16_t h);
float    or_bf16_to_f32(uint16_t h);
uint16_t or_f32_to_bf16(float x);     /* round-to-nearest-even */

/* ---- packed code layout ---------------------------------------------- */
int64_t or_tile_bytes(int bits, int d_k, int d_v);
void or_pack(int bits, int d_k, int d_v, const int8_t* codes, uint8_t* out);
void or_unpack(int bits, int d_k, int d_v, const uint8_t* in, int8_t* codes);

/* ---- Walsh-Hadamard transform, in place: x <- H x, H the n x n Sylvester
 * Hadamard matrix (entries +-1, H H = n I), n a power of two ------------- */
void or_fwht(int n, float* x);

/* ---- canonical reduction: sum_i a[i*stride] * b[i], i < n ------------- */
float or_canon_dot(int n, const float* a, int stride, const float* b);

/* ---- rounding ---------------------------------------------------------- */
int or_round_rtn(float x, float inv, int qmax);
int or_round(const or_cfg* c, float a, float x, float inv, int qmax, or_counts* cnt);
int or_classify(float a, float x, float inv, int qmax);

/* ---- one step over ntiles independent tiles --------------------------- *
 * tile_bits[t]: 2, 4, 6, 8 or 32 (32 = unquantized fp32 state).
 * codes  [ntiles][d_k][d_v] int8 (ignored for 32-bit tiles)
 * S      [ntiles][d_k][d_v] f32  (the fp32 state of 32-bit tiles)
 * scales [ntiles][n_scales]  f32 holding the stored value exactly
 * ref    [ntiles][d_k][d_v] f32  (yoked mode only, else NULL)
 * q,k    [ntiles][d_k], v [ntiles][d_v]
 * alpha  [ntiles][n_alpha] (n_alpha = d_k for GLA, 1 for Mamba2/GDN, unused
 *        for RetNet), beta [ntiles] (GDN only)
 * out    [ntiles][d_v]
 * Returns 0, or -1 on an invalid configuration. */
int or_step(const or_cfg* c, int64_t ntiles, const int* tile_bits,
            int8_t* codes, float* S, float* scales, float* ref,
            const float* q, const float* k, const float* v,
            const float* alpha, const float* beta, float* out, or_counts* cnt);

/* or_step, also returning per tile the decayed state a [ntiles][d_k][d_v],
 * the updated state before rounding x (same layout) and, for quantized
 * tiles, each element's rounding class (OR_NONE / OR_LOST / OR_MOVED /
 * OR_REVERSED, or_classify); any of the three may be NULL. */
int or_step_trace(const or_cfg* c, int64_t ntiles, const int* tile_bits,
                  int8_t* codes, float* S, float* scales, float* ref,
                  const float* q, const float* k, const float* v,
                  const float* alpha, const float* beta, float* out, or_counts* cnt,
                  float* a_out, float* x_out, int8_t* cls_out);

int or_n_scales(const or_cfg* c);

/* Dequantized state of one tile: S_hat = code * scale. */
void or_dequant(const or_cfg* c, int bits, const int8_t* codes, const float* scales,
                float* S_out);

/* ---- Low-Rank Bypass (LRB): readings L1-L6 in qstate_oracle.c ---------- */
#define OR_LRB_MAX_COLS 32

typedef struct {
    int k;            /* rank of the residual kept across merges */
    int m;            /* fresh columns (steps) between merges */
    float eps_l;      /* merge threshold, in grid steps of the element's scale */
} or_lrb_cfg;

/* One LRB step over ntiles tiles (quantized widths 2..8 only; all four
 * kinds; dynamic or persistent scales).  Bypass per tile: u
 * [k+m][d_k] and w [k+m][d_v] binary16 bit patterns, g [k+m] binary32,
 * nres / nnew the residual and fresh slot counts, D [ntiles] the decay since
 * the last merge (GLA: [ntiles][d_k], one per key row; 1 at the start).  merged (may be NULL):
 * per tile, the number of elements merged by this step.  resid (may be
 * NULL): [ntiles][d_k][d_v], at a merge the unmerged rest of the bypass
 * (before its rank-k approximation), untouched otherwise.  -1 if invalid. */
int or_lrb_step(const or_cfg* c, const or_lrb_cfg* L, int64_t ntiles, const int* tile_bits,
                int8_t* codes, float* scales, uint16_t* u, uint16_t* w, float* g, int* nres,
                int* nnew, float* D, const float* q, const float* k, const float* v,
                const float* alpha, const float* beta, float* out, or_counts* cnt, int* merged,
                float* resid);

/* Top-k singular triplets of a rows x cols fp64 matrix (Jacobi on R^T R). */
void or_rank_k(int rows, int cols, const double* R, int k, double* s, double* U, double* V);

/* Storage per state element: bits + scale bits per element + cols_used
 * bypass columns of (d_k + d_v) 16-bit values and a 32-bit coefficient. */
double or_lrb_bits(int bits, int group, int scale_bits, int d_k, int d_v, double cols_used);

/* ---- Pure-write sliding window (PW): readings W1-W6 in qstate_oracle.c -- */
#define OR_PW_MAX_W 16

/* OCP FP8 E4M3 ("E4M3FN"): 1 sign, 4 exponent bits (bias 7), 3 fraction bits,
 * no infinities, 0x7F / 0xFF NaN, largest finite 448.  Encoding: nearest,
 * ties to the even code; magnitudes beyond 448 give 448 (saturating). */
float or_e4m3_to_f32(uint8_t b);
uint8_t or_f32_to_e4m3(float x);

/* One PW step of ntiles Gated DeltaNet tiles (history widths 2..8 quantized,
 * or 32 = an fp32 history; dynamic or persistent scales).  Window per tile:
 * A [W][d_k] and B [W][d_v] FP8 E4M3 bytes (key and value sides of the
 * pairs), head the slot of the oldest pair, count the pairs held.  W in
 * 1 .. OR_PW_MAX_W.  -1 if invalid. */
int or_pw_step(const or_cfg* c, int W, int64_t ntiles, const int* tile_bits,
               int8_t* codes, float* S, float* scales, uint8_t* A, uint8_t* B, int* head,
               int* count, const float* q, const float* k, const float* v,
               const float* alpha, const float* beta, float* out, or_counts* cnt);

/* ---- Key-row x value-column scales: readings R1-R5 in qstate_oracle.c --- */

/* One step of ntiles tiles whose scales are a row vector rho [d_k] and a
 * column vector kappa [d_v] per tile (scales [ntiles][d_k + d_v], rho
 * first, in the configuration's scale format); widths 2..8, dynamic scales,
 * all four kinds, RTN or BDR.  -1 if invalid. */
int or_rc_step(const or_cfg* c, int64_t ntiles, const int* tile_bits, int8_t* codes,
               float* scales, const float* q, const float* k, const float* v,
               const float* alpha, const float* beta, float* out, or_counts* cnt);

/* Dequantized tile of a row x column-scaled state: code * (rho_i * kappa_j). */
void or_rc_dequant(const or_cfg* c, const int8_t* codes, const float* scales, float* S_out);

#ifdef __cplusplus
}
#endif
#endif
