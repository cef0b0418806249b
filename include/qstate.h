/*
 * qstate.h -- C ABI of the fused quantized recurrent-state decode step
 * (sm_100a).  Library: bit_recurrent_state_decode_b200/libqstate.so.
 *
 * WHAT ONE STEP COMPUTES
 * The state of one (layer, batch, head) tile is a d_k x d_v matrix S stored in
 * low-bit codes with per-group scales.  One step, per tile:
 *   1. unpack the codes and decay the state: a = A_t S_hat_{t-1}
 *   2. add the update:                       x = a + B_t
 *   3. emit the output:                      o_t = x^T q_t
 *   4. re-derive or carry the scale, 5. round, 6. repack.
 * The recurrence (decay A_t, update B_t) is Table 1 of "Preserving Updates in
 * Low-Bit Recurrent State Quantization":
 *   RetNet  A = gamma I,        B = k v^T
 *   Mamba2  A = alpha_t I,      B = k v^T
 *   GLA     A = Diag(alpha_t),  B = k v^T          (alpha over the d_k rows)
 *   GDN     A = alpha_t I,      B = beta_t k (v - (A S_{t-1})^T k)^T
 * The scale modes (dynamic: re-derived from the state every step;
 * persistent: carried and regrown only on overflow; yoked: derived from a
 * full-precision reference state stepped in lockstep) are the Abstract of
 * "When Dynamic Scaling Fails".  Round-to-nearest and Bounded Directional
 * Rounding (a reversed element is rounded toward its update) are the Abstract
 * and Figure 4 of the first page; eps_B is its Table 6.  Per-token scales and
 * mixed per-head bit widths are the Abstract of "Low-Bit Recurrent States in
 * Hybrid Language Models".
 *
 * EXACT ARITHMETIC (binary32, round-to-nearest-even, in this order)
 *   eta_i   = alpha_i * scale_prev(i, g)            one per (row, group)
 *   a_ij    = code_ij * eta_i                        (32-bit state: S_ij * alpha_i)
 *   rank-1:  x_ij = fma(k_i, v_j, a_ij)
 *   GDN:     r_j = csum_i(a_ij k_i);  e_j = v_j - r_j;  kap_i = beta * k_i;
 *            x_ij = fma(kap_i, e_j, a_ij)
 *   o_j     = csum_i(x_ij q_i)                       (before rounding)
 *   m       = max |x| over the group (a group is `group` consecutive columns
 *             of one row, or the whole tile when group == 0)
 *   dynamic:    scale = cvt(m / Qmax)
 *   persistent: scale = (m > Qmax * scale_prev) ? cvt(m / Qmax) : scale_prev
 *   yoked:      scale = cvt(m_ref / Qmax), m_ref from the reference state
 *               stepped with the same arithmetic on 32-bit values
 *   inv     = scale == 0 ? 0 : 1 / scale
 *   RTN:     code = clamp(round_half_even(x * inv exact), -Qmax, Qmax)
 *   BDR:     d = x - a; s = fma(a, inv, -code);  if d > 0 and s > eps_B:
 *            code = min(code + 1, Qmax); if d < 0 and s < -eps_B:
 *            code = max(code - 1, -Qmax)
 * csum is the canonical order: rows in blocks of 8 consecutive rows, each
 * block an ascending fma chain from +0, block sums added as a balanced
 * pairwise tree (adjacent blocks first).  cvt is binary16 round-to-nearest-
 * even (overflow saturates to 65504 and is counted) or the identity for
 * binary32 scales.  Qmax = 2^(bits-1) - 1 (codes are symmetric; the code
 * -2^(bits-1) is accepted on input).
 *
 * MEMORY LAYOUT (all device memory, row-major, tile = (layer, b, h),
 * tile index t = (layer * batch + b) * heads + h)
 *   q, k   [layers][batch][heads][d_k]   qkv_dtype (f32 or bf16)
 *   v      [layers][batch][heads][d_v]   qkv_dtype
 *   gates  [layers][batch][heads][n_gate] gate_dtype, n_gate = 0 (RetNet),
 *          1 (Mamba2: alpha), d_k (GLA: alpha_i), 2 (GDN: alpha, beta)
 *   out    [layers][batch][heads][d_v]   float32
 *   codes (library-owned): per tile d_k*d_v*bits/8 bytes, two's complement,
 *          packed along d_v: 8-bit one byte per code; 4-bit code 2m in the
 *          low nibble of byte m; 2-bit code 4m+s in bits 2s..2s+1 of byte m;
 *          6-bit a low-nibble plane (4-bit layout of code & 15) for the whole
 *          tile followed by a high plane (2-bit layout of (code >> 4) & 3);
 *          32-bit: the fp32 state itself.  Tiles are contiguous in tile order;
 *          with per-head bit widths the tile (layer, b, h) starts at
 *          (layer*batch + b) * sum_h(tile_bytes_h) + sum_{h'<h} tile_bytes_h'.
 *   scales (library-owned): [tiles][d_k][d_v/group] (group > 0) or [tiles],
 *          binary16 or binary32.
 *   ref   (library-owned, yoked only): [tiles][d_k][d_v] float32.
 * q, k, v, gates and out must be 16-byte aligned.
 *
 * ERRORS AND OWNERSHIP
 * Every call returns QSTATE_OK (0) or a negative code; nothing throws across
 * the ABI.  Invalid arguments are rejected before any CUDA call.  Kernels
 * never trap: non-finite inputs and binary16 scale overflow are counted in
 * sticky device counters read by qstate_status().  A qstate object owns its
 * device memory; its calls are asynchronous on the stream passed and an
 * object must not be stepped from two streams at once.  All pointers other
 * than the object are borrowed for the duration of the call's device work.
 */
#ifndef QSTATE_H
#define QSTATE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Compatible with cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* qstate_stream;

enum {
    QSTATE_OK = 0,
    QSTATE_EINVAL = -1,       /* invalid argument or layout */
    QSTATE_ENOMEM = -2,       /* device or host allocation failed */
    QSTATE_ECUDA = -3,        /* a CUDA runtime call failed */
    QSTATE_EUNSUPPORTED = -4  /* valid but not built (e.g. d_k outside {64,128}) */
};

typedef enum { QSTATE_RETNET = 0, QSTATE_MAMBA2 = 1, QSTATE_GLA = 2, QSTATE_GDN = 3 } qstate_kind;
typedef enum { QSTATE_DYNAMIC = 0, QSTATE_PERSISTENT = 1, QSTATE_YOKED = 2 } qstate_scale_mode;
typedef enum { QSTATE_RTN = 0, QSTATE_BDR = 1 } qstate_round_mode;
typedef enum { QSTATE_F32 = 0, QSTATE_BF16 = 1, QSTATE_F16 = 2 } qstate_dtype;

typedef struct qstate_layout {
    int32_t batch;            /* >= 0 (0: an empty object, steps are no-ops) */
    int32_t heads;            /* >= 1 */
    int32_t d_k, d_v;         /* each 64 or 128 */
    int32_t layers;           /* independent layers held by the object, >= 1;
                                 layers * batch * heads < 2^31 */
    int32_t kind;             /* qstate_kind */
    float gamma;              /* RetNet decay (ignored for the other kinds) */
    int32_t qkv_dtype;        /* QSTATE_F32 or QSTATE_BF16 */
    int32_t gate_dtype;       /* QSTATE_F32 or QSTATE_BF16 */
    int32_t scale_dtype;      /* QSTATE_F16 or QSTATE_F32 */
    const uint8_t* head_bits; /* NULL, or host array [heads] of 2/4/6/8 (copied);
                                 overrides `bits` of qstate_create */
    int32_t rotation;         /* 0: none; 1: the state is kept rotated by the
                                 Hadamard matrix H along d_v (INT4+Had of Table 2
                                 of "Preserving Updates in Low-Bit Recurrent State
                                 Quantization"): the stored state is S H, each
                                 step takes H v for v and emits o = H (S H)^T q
                                 / d_v, H the Sylvester matrix (entries +-1)
                                 applied by the butterfly of its order; the
                                 outputs are those of S, qstate_dequant returns
                                 the stored S H */
} qstate_layout;

typedef struct qstate qstate;

typedef struct qstate_counters {
    uint64_t nonfinite;       /* tile-steps with a non-finite output or group
                                 maximum (any non-finite input produces one) */
    uint64_t saturated;       /* binary16 scale conversions that overflowed */
    uint64_t pipeline_timeouts; /* CTAs that gave up a bounded wait for their input
                                   copies (the step's results are then undefined) */
    uint64_t exact_path_warps; /* warp-tiles that rounded element by element (the
                                  general form, taken when the fast form's
                                  conditions do not hold for every row of the
                                  warp); counted while qstate_set_taxonomy is on */
    /* Rounding taxonomy (only while qstate_set_taxonomy is on): elements with a
     * nonzero update d = x - a, classified on the grid of the new scale with
     * u = a * inv, w = x * inv and c = clamp(RTN(w)): reversed when c lies
     * strictly beyond u on the side away from the update, else lost when
     * c = clamp(RTN(u)), else moved (Figure 4 of "Preserving Updates in
     * Low-Bit Recurrent State Quantization"); and the BDR steps applied. */
    uint64_t lost, moved, reversed, bdr_applied;
} qstate_counters;

typedef struct qstate_sizes {
    int64_t tiles;            /* layers * batch * heads */
    int64_t code_bytes;       /* packed codes (or fp32 state) of all tiles */
    int64_t scale_bytes;      /* all scales */
    int64_t ref_bytes;        /* yoked reference state (0 otherwise) */
    int64_t n_scales;         /* scales per tile */
    int64_t n_gate;           /* gate values per tile */
    int64_t q_bytes, v_bytes, gate_bytes, out_bytes;  /* step operand sizes */
} qstate_sizes;

/* Create a zero state (codes, scales and reference all zero).
 * The layer kinds are the rows of Table 1 of "Preserving Updates in Low-Bit
 * Recurrent State Quantization"; the scale modes `sm` are the three of the
 * Abstract of "When Dynamic Scaling Fails"; group-wise INT4 at 4.50 bits
 * (group 32, binary16 scales) is Table 2 of the first page; per-token scales
 * (group 0) and per-head widths (L->head_bits) are the Abstract of "Low-Bit
 * Recurrent States in Hybrid Language Models"; `rm` and `eps_b` are BDR and
 * its threshold eps_B (Abstract, Figure 4 and Table 6 of the first page).
 * bits: 2, 4, 6, 8, or 32 (quantization disabled, fp32 state); ignored when
 *   L->head_bits is given.
 * group: columns per scale group along d_v, a multiple of 8 dividing d_v, or
 *   0 for one scale per tile per step (per-token).
 * sm / rm / eps_b: scale mode, rounding mode, BDR threshold (>= 0, in grid
 *   steps of the new scale).  YOKED needs bits < 32.
 * On success *out owns the device memory; free it with qstate_destroy. */
int qstate_create(const qstate_layout* L, int bits, int group, qstate_scale_mode sm,
                  qstate_round_mode rm, float eps_b, qstate** out);
int qstate_destroy(qstate* s);

/* Zero the state again (asynchronous on stream). */
int qstate_reset(qstate* s, qstate_stream stream);

/* One decode step of every tile (one kernel launch), asynchronous on stream:
 * S_t = A_t S_{t-1} + B_t with the decay and update of the object's layer
 * kind (Table 1 of "Preserving Updates in Low-Bit Recurrent State
 * Quantization"), o_t = S_t^T q_t, then the scale, rounding and repacking of
 * the state in the order given at the top of this file.
 * q, k, v, gates, out: caller-owned DEVICE buffers in the layouts above
 * (gates may be NULL for RetNet), each starting on a 16-byte boundary;
 * QSTATE_EINVAL for a NULL or misaligned one, also for an object of no
 * tiles, whose step then does nothing.  Returns after the launch. */
int qstate_step(qstate* s, const void* q, const void* k, const void* v, const void* gates,
                float* out, qstate_stream stream);

/* The same step from HOST buffers: copies q, k, v, gates host->device into
 * library-owned staging buffers, launches the step on stream and copies out
 * device->host on stream, all asynchronous (synchronise the stream before
 * reading out: its completion covers this call's copies and step).  The
 * input copies run on a stream of the object's own, into one of two staging
 * sets used by alternate calls, so that a call's input copies overlap the
 * previous call's step; the step waits for them.  Pinned host memory makes
 * the copies asynchronous; the caller keeps its input buffers unchanged
 * until the stream has completed the call.  The staging buffers, the copy
 * stream and its events are allocated by the first call and shared by every
 * later call on the object: issue all qstate_step_host calls of one object
 * on one stream (calls on different streams would overwrite each other's
 * operands).  The output copy runs on a second stream of the object's own,
 * which `stream` waits for before the call returns control to later work. */
int qstate_step_host(qstate* s, const void* q, const void* k, const void* v,
                     const void* gates, float* out, qstate_stream stream);

/* qstate_step_host for a stream of calls (no counterpart on the pages): the
 * same copies and step, but the output copy runs on a stream of the
 * object's own, into the caller's `out` of this call, so that it overlaps
 * the next call's step; completion of `stream` covers this call's input
 * copies and step and the output copies of the calls before it.  The output
 * of the last call is in host memory once `stream` has completed a
 * following qstate_step_host_sync (or a following host-buffer call).  The
 * same single-stream rule and staging buffers as qstate_step_host, with
 * which it may be mixed. */
int qstate_step_host_pipelined(qstate* s, const void* q, const void* k, const void* v,
                               const void* gates, float* out, qstate_stream stream);

/* Make `stream` wait for the output copy of the object's last host-buffer
 * call (a no-op before the first). */
int qstate_step_host_sync(qstate* s, qstate_stream stream);

/* Size of the device array that qstate_step_host_static stages operands in. */
#define QSTATE_STATIC_STAGING_BYTES (16u << 20)

/* qstate_step_host for callers that must not allocate device memory.  No
 * counterpart on the pages: it exists for the callers of this library that
 * cannot call cudaMalloc, such as a serving process whose device memory is
 * all handed out by its own pool allocator, or a decode loop that must not
 * stall (cudaMalloc may synchronise the device).  qstate_step_host allocates
 * its staging buffers on its first call; this call allocates nothing: it
 * copies q, k, v and gates into one fixed device array of
 * QSTATE_STATIC_STAGING_BYTES bytes that the library image holds on every GPU
 * that loads it until the process exits, launches the step on that copy and
 * copies out back, all asynchronous on stream.  The object itself is still
 * created (and its state allocated) by qstate_create.
 *  - Size limit: q, k, v, gates and out of the object (qstate_get_sizes),
 *    each rounded up to 256 bytes, must fit in QSTATE_STATIC_STAGING_BYTES;
 *    larger objects get QSTATE_EINVAL and nothing is copied.
 *  - The first call on a device looks up the array's device address (once
 *    per device, under a lock); make that first call before capturing any
 *    stream on that device.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents; nothing in it needs clearing, since each call copies in every
 *    operand the step reads and the step writes every element of out.  Calls
 *    that overlap on the GPU (other streams, other objects) race on the
 *    array: issue them on one stream, or order them with events.
 *  - Pinned host memory makes the copies asynchronous. */
int qstate_step_host_static(qstate* s, const void* q, const void* k, const void* v,
                            const void* gates, float* out, qstate_stream stream);

/* Dequantized state S_hat = code * scale, float32 [tiles][d_k][d_v] (device):
 * the state a quantized recurrence carries ("Preserving Updates in Low-Bit
 * Recurrent State Quantization", Abstract). */
int qstate_dequant(const qstate* s, float* S_out, qstate_stream stream);

/* Copy the raw state out to / in from caller device buffers of
 * qstate_sizes() bytes (codes, scales, ref; ref may be NULL if not yoked).
 * Used for checkpoints and teacher-forced parity (no counterpart on the
 * pages; the layouts are the ones above).  With a Low-Rank Bypass these are
 * the quantized part only (qstate_dequant likewise); import also empties the
 * bypass and sets D = 1.  With a pure-write window they are the history
 * only; import also empties the window. */
int qstate_export(const qstate* s, void* codes, void* scales, float* ref,
                  qstate_stream stream);
int qstate_import(qstate* s, const void* codes, const void* scales, const float* ref,
                  qstate_stream stream);

int qstate_get_sizes(const qstate* s, qstate_sizes* out);

/* Algorithmic bytes one step must move: packed state read + write, scales
 * read + write, q, k, v and gates read, out written, and in yoked mode the
 * float32 reference state read + write (the memory traffic that makes FP32
 * states costly at large batch, Abstract of "Preserving Updates in Low-Bit
 * Recurrent State Quantization").  Returns -1 on a NULL object. */
int64_t qstate_bytes_per_step(const qstate* s);

/* Read the sticky counters: copies them device->host on stream and
 * synchronises that stream (no counterpart on the pages). */
int qstate_status(qstate* s, qstate_counters* out, qstate_stream stream);

/* Count the rounding taxonomy of every element of every following step
 * (on = 1) or stop (on = 0, the default) into the lost / moved / reversed /
 * bdr_applied counters of qstate_status.  The counts are diagnostics of the
 * error accounting of "Preserving Updates in Low-Bit Recurrent State
 * Quantization" (Figure 4, Table 5: the lost fraction); while on, steps run
 * the general kernel and classify each element again, so they are slower;
 * the state and outputs are unchanged.  QSTATE_EINVAL for other values. */
int qstate_set_taxonomy(qstate* s, int on);

/* With the taxonomy on, each step also keeps, per tile and key row, the
 * squared rounding error it added, sum_j (S_hat_t - x_t)_ij^2 (S_hat_t the
 * dequantized new state, x_t the updated state before rounding; binary32):
 * the per-step R_t of the error accounting of "Preserving Updates in Low-Bit
 * Recurrent State Quantization" (Figures 1 and 2, Table 5), from which a
 * caller forms D_T = sum_t ||a_{t:T} R_t||^2 and the coherent gain.  Copies
 * the last such step's values, [tiles][d_k] binary32, to `out` (device or
 * host) on stream.  QSTATE_EINVAL if the taxonomy was never switched on
 * (the buffer is allocated by the first qstate_set_taxonomy(s, 1), which may
 * return QSTATE_ENOMEM).  Objects with a bypass, a window or row x column
 * scales do not keep it. */
int qstate_error_rows(const qstate* s, float* out, qstate_stream stream);

/* Switch the object to steps with a Low-Rank Bypass (LRB) of "Preserving
 * Updates in Low-Bit Recurrent State Quantization" (Abstract, Figure 3,
 * Tables 6, 8, 9), before its first step.  Each tile keeps, next to its
 * codes and scales, up to k + m bypass columns (u in binary16 [d_k], w in
 * binary16 [d_v], a binary32 coefficient) and a binary32 decay D: every step
 * decays D and the coefficients, adds the step's update as a new column
 * (Gated DeltaNet: e = v - r with r over the whole state, codes plus bypass)
 * and emits o from the whole state; codes and scales change only every m
 * steps, when the bypass elements at least eps_l grid steps (of the decayed
 * grid) large are merged into the state and it is requantized with the
 * object's scale and rounding modes (BDR with the merged update as d), D
 * reset to 1 and the rest kept as its leading singular pair (k = 1, found by
 * power iteration) or dropped (k = 0).  The state a tile stands for is
 * D * dequant(codes) + sum_l g_l u_l w_l^T.  GLA (decay Diag(alpha)) keeps
 * one D per key row instead: the coefficients do not decay, a column's key
 * side is stored as fp16(k / D) of its step and read as D_i u_i, and the
 * tile stands for Diag(D) (dequant(codes) + sum_l g_l u_l w_l^T).
 * k in {0, 1}, m >= 1, k + m <= 32, eps_l >= 0.  Supported for all four
 * kinds with one code width of 4 or 8 bits, d_k = d_v in {64, 128},
 * dynamic or persistent scales, no rotation (QSTATE_EUNSUPPORTED
 * otherwise); allocates the bypass (QSTATE_ENOMEM).
 * QSTATE_EINVAL if a bypass, a window or row x column scales are already set
 * or for invalid k, m, eps_l. */
int qstate_set_lrb(qstate* s, int k, int m, float eps_l);

/* Switch a Gated DeltaNet object to steps with a pure-write sliding window
 * (PW) of "Low-Bit GDN Recurrent-State Quantization: Global Gradient-aware
 * Allocation and Pure-Write Sliding Windows" (Abstract), before its first
 * step.  Each tile keeps, next to its quantized history (codes, scales), the
 * W most recent pure writes beta k v^T as pairs of FP8 E4M3 vectors
 * (a = beta k, b = v; OCP E4M3, nearest-even, saturating at 448).  Every
 * step applies the transition alpha (I - beta k k^T) to the history (a
 * Gated DeltaNet step without a write, requantized with the object's scale
 * and rounding rules) and to every pair's key side (re-encoded in E4M3);
 * when W pairs are held the oldest then leaves into the history before the
 * step's own pair takes its slot; o is the whole state's output.  The state
 * a tile stands for is dequant(codes) + sum over the pairs of a b^T.
 * 1 <= W <= 16.  Supported for Gated DeltaNet objects with one code width
 * of 4 or 8 bits, d_k = d_v in {64, 128}, dynamic or persistent scales, no
 * rotation (QSTATE_EUNSUPPORTED otherwise); allocates the window
 * (QSTATE_ENOMEM).  QSTATE_EINVAL if a window, a bypass or row x column
 * scales are already set, or for an invalid W.  qstate_reset and
 * qstate_import empty the window. */
int qstate_set_pw(qstate* s, int W);

/* Copy a PW object's window to caller buffers (device or host): A
 * [tiles][W][d_k] and B [tiles][W][d_v] E4M3 bytes by slot, head [tiles]
 * the slot of the oldest pair, count [tiles] the pairs held. */
int qstate_pw_export(const qstate* s, uint8_t* A, uint8_t* B, int32_t* head, int32_t* count,
                     qstate_stream stream);

/* Switch the object to key-row x value-column scales ("STEPQuant: When and
 * Where Errors Matter in Delta-Rule Recurrent State Quantization",
 * Abstract), before its first step: the scales become, per tile, row scales
 * rho [d_k] then column scales kappa [d_v] (scales [tiles][d_k + d_v] in the
 * layout's scale format; qstate_get_sizes reports the new size), the grid
 * step of element (i, j) is rho_i * kappa_j, and every step fits them from
 * the updated state x before rounding: kappa_j = cvt(max_i |x_ij|),
 * rho_i = cvt(max_j(|x_ij| * (1/kappa_j)) / Qmax), codes
 * c = clamp(rne(x * ((1/rho_i) * (1/kappa_j)))) (BDR with d = x - a), the
 * decay a = code * ((alpha_i * rho_i) * kappa_j).  The update and output
 * are the plain step's.  The page fits these scales offline against trained
 * models; this joint fit from the state alone is this library's reading.
 * Supported for all four kinds, one code width of 4 or 8 bits, dynamic
 * scales, no rotation (QSTATE_EUNSUPPORTED otherwise); the state is reset.
 * QSTATE_EINVAL if already set or with a bypass or window.  The taxonomy
 * counts are not kept for such objects. */
int qstate_set_rowcol(qstate* s);

/* Name of the kernel the object's next step launches ("step_kernel",
 * "rows_kernel", "lrb_kernel", "pw_kernel" or "rc_kernel"; "" for NULL): for reports and profiles, no
 * counterpart on the pages.  The string is static. */
const char* qstate_kernel(const qstate* s);

/* Copy an LRB object's bypass to caller buffers (device or host):
 * u [tiles][k+m][d_k] and w [tiles][k+m][d_v] binary16 bit patterns,
 * g [tiles][k+m], n [tiles][2] (residual and fresh columns held), D [tiles]
 * (GLA: [tiles][d_k]). */
int qstate_lrb_export(const qstate* s, uint16_t* u, uint16_t* w, float* g, int32_t* n, float* D,
                      qstate_stream stream);

/* Fault injection for tests of the bounded waits (no counterpart on the
 * pages).  The step kernel stages each tile's inputs with asynchronous bulk
 * copies and waits for them with at most `wait_polls` polls (default 2^24,
 * several seconds).  With drop_from_tile >= 0 the copies of every tile with
 * index >= drop_from_tile are never issued, so those waits run out: the
 * affected CTAs count a pipeline timeout and return, the step's results are
 * undefined, and the CUDA context stays usable.  drop_from_tile = -1 restores
 * normal operation.  Returns QSTATE_EINVAL for wait_polls == 0. */
int qstate_debug_set(qstate* s, int64_t drop_from_tile, uint32_t wait_polls);

/* Static, human-readable name of a return code. */
const char* qstate_error_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* QSTATE_H */
