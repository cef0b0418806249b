// qstate_kernel.cuh -- sm_100a kernels of the fused quantized recurrent-state
// decode step.  The arithmetic and its order are specified in include/qstate.h
// (recurrence: "Preserving Updates in Low-Bit Recurrent State Quantization",
// Table 1; scale modes: "When Dynamic Scaling Fails", Abstract; BDR: the
// Abstract and Figure 4 of the first page).
//
// Work decomposition.  One CTA steps one (layer, batch, head) tile at a time
// and walks tiles with a grid stride (the grid is sized to the SM count times
// the resident CTAs per SM).  Each thread owns an 8 x 8 block of the tile:
// 8 consecutive rows (one "row block" of the canonical reduction) and 8
// consecutive columns.  A warp covers all d_v columns of 32/(d_v/8) row
// blocks, so
//   - the column sums r_j, o_j are an in-thread fma chain over the block
//     (exactly the canonical block sum), an xor butterfly across the row
//     blocks of the warp (adjacent blocks first), and a pairwise tree across
//     warps through shared memory;
//   - the group maximum along d_v is an in-thread max plus an xor butterfly
//     across the lanes that share the group;
// and every load of a warp is a set of fully used 32-byte sectors.  The
// state is read once and written once per step; nothing spills to global
// scratch.  No tensor cores: the step is a rank-1 update plus two
// matrix-vector products per tile.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qs {

enum { K_RETNET = 0, K_MAMBA2 = 1, K_GLA = 2, K_GDN = 3 };
enum { M_DYNAMIC = 0, M_PERSISTENT = 1, M_YOKED = 2 };

struct StepParams {
    uint8_t* codes;                 // packed codes, or the fp32 state (32-bit tiles)
    void* scales;                   // [tiles][n_scales] binary16 or binary32
    float* ref;                     // yoked reference state [tiles][d_k][d_v]
    const void* q;
    const void* k;
    const void* v;
    const void* gates;
    float* out;
    unsigned long long* counters;   // [0] non-finite tile-steps, [1] saturated scales
    const long long* head_off;      // per-head byte offset in a (layer, batch) row, or null
    const unsigned char* head_bits; // per-head bit width, or null (uniform)
    long long row_bytes;            // code bytes of one (layer, batch) row (mixed bits)
    long long tile_bytes;           // code bytes of one tile (uniform bits)
    long long ntiles;
    int heads;
    int bits;                       // uniform bit width (2/4/6/8/32)
    int group;                      // columns per scale group, 0 = whole tile
    int n_scales;                   // scales per tile
    int kind;
    int scale_mode;
    int n_gate;
    int qkv_bf16, gate_bf16, scale_f32;
    float gamma, eps_b;
};

template <int DK, int DV>
struct Geo {
    static constexpr int CBW = DV / 8;          // column blocks per row (lanes per row)
    static constexpr int RBW = 32 / CBW;        // row blocks per warp
    static constexpr int NWARPS = DK / (8 * RBW);
    static constexpr int NT = 32 * NWARPS;
    static_assert(CBW * RBW == 32, "d_v must be 64 or 128");
    static_assert(NWARPS >= 1 && (NWARPS & (NWARPS - 1)) == 0, "warps must be a power of two");
};

constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23: rounds to integers in [2^23, 2^24)
constexpr int kMagicBits = 0x4B400000;

// ------------------------------------------------------------------ loads
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

// 8 consecutive values (element index idx, a multiple of 8) as float.
__device__ __forceinline__ void load8(const void* base, long long idx, bool bf16, float (&o)[8]) {
    if (bf16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + idx));
        bf16x2_to_f32(u.x, o[0], o[1]);
        bf16x2_to_f32(u.y, o[2], o[3]);
        bf16x2_to_f32(u.z, o[4], o[5]);
        bf16x2_to_f32(u.w, o[6], o[7]);
    } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
}

__device__ __forceinline__ float load1(const void* base, long long idx, bool bf16) {
    if (bf16) return __uint_as_float(uint32_t(__ldg(static_cast<const uint16_t*>(base) + idx)) << 16);
    return __ldg(static_cast<const float*>(base) + idx);
}

__device__ __forceinline__ float load_scale(const void* base, long long idx, bool f32) {
    if (f32) return static_cast<const float*>(base)[idx];
    return __half2float(static_cast<const __half*>(base)[idx]);
}

// Convert a scale to its stored precision; returns the stored value widened.
__device__ __forceinline__ float to_stored(float v, bool f32, bool& saturated) {
    if (f32) return v;
    __half h = __float2half_rn(v);
    if (__hisinf(h)) {
        saturated = true;
        return 65504.0f;
    }
    return __half2float(h);
}

__device__ __forceinline__ void store_scale(void* base, long long idx, bool f32, float v) {
    if (f32) static_cast<float*>(base)[idx] = v;
    else static_cast<__half*>(base)[idx] = __float2half_rn(v);   // exact: v is a binary16 value
}

// ------------------------------------------------------------------ codes
// One thread's 8 codes of one row, for each bit width.  `t` is the tile base.
template <int BITS, int DK, int DV>
struct Codec;

template <int DK, int DV>
struct Codec<4, DK, DV> {
    struct W { uint32_t w; };
    static __device__ __forceinline__ W load(const uint8_t* t, int i, int cb) {
        return W{*reinterpret_cast<const uint32_t*>(t + i * (DV / 2) + cb * 4)};
    }
    static __device__ __forceinline__ int get(const W& w, int c) {
        return int(w.w << (28 - 4 * c)) >> 28;
    }
    static __device__ __forceinline__ void store(uint8_t* t, int i, int cb, const int (&c)[8]) {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; e++) w |= (uint32_t(c[e]) & 15u) << (4 * e);
        *reinterpret_cast<uint32_t*>(t + i * (DV / 2) + cb * 4) = w;
    }
};

template <int DK, int DV>
struct Codec<8, DK, DV> {
    struct W { uint2 w; };
    static __device__ __forceinline__ W load(const uint8_t* t, int i, int cb) {
        return W{*reinterpret_cast<const uint2*>(t + i * DV + cb * 8)};
    }
    static __device__ __forceinline__ int get(const W& w, int c) {
        const uint32_t v = c < 4 ? w.w.x : w.w.y;
        return int(v << (24 - 8 * (c & 3))) >> 24;
    }
    static __device__ __forceinline__ void store(uint8_t* t, int i, int cb, const int (&c)[8]) {
        uint2 w = make_uint2(0u, 0u);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            w.x |= (uint32_t(c[e]) & 255u) << (8 * e);
            w.y |= (uint32_t(c[e + 4]) & 255u) << (8 * e);
        }
        *reinterpret_cast<uint2*>(t + i * DV + cb * 8) = w;
    }
};

template <int DK, int DV>
struct Codec<2, DK, DV> {
    struct W { uint32_t w; };
    static __device__ __forceinline__ W load(const uint8_t* t, int i, int cb) {
        return W{*reinterpret_cast<const uint16_t*>(t + i * (DV / 4) + cb * 2)};
    }
    static __device__ __forceinline__ int get(const W& w, int c) {
        return int(w.w << (30 - 2 * c)) >> 30;
    }
    static __device__ __forceinline__ void store(uint8_t* t, int i, int cb, const int (&c)[8]) {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; e++) w |= (uint32_t(c[e]) & 3u) << (2 * e);
        *reinterpret_cast<uint16_t*>(t + i * (DV / 4) + cb * 2) = uint16_t(w);
    }
};

template <int DK, int DV>
struct Codec<6, DK, DV> {
    // low-nibble plane (4-bit layout) then high 2-bit plane (2-bit layout)
    struct W { uint32_t lo, hi; };
    static __device__ __forceinline__ W load(const uint8_t* t, int i, int cb) {
        return W{*reinterpret_cast<const uint32_t*>(t + i * (DV / 2) + cb * 4),
                 *reinterpret_cast<const uint16_t*>(t + DK * DV / 2 + i * (DV / 4) + cb * 2)};
    }
    static __device__ __forceinline__ int get(const W& w, int c) {
        const uint32_t u = ((w.lo >> (4 * c)) & 15u) | (((w.hi >> (2 * c)) & 3u) << 4);
        return int(u << 26) >> 26;
    }
    static __device__ __forceinline__ void store(uint8_t* t, int i, int cb, const int (&c)[8]) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            lo |= (uint32_t(c[e]) & 15u) << (4 * e);
            hi |= ((uint32_t(c[e]) >> 4) & 3u) << (2 * e);
        }
        *reinterpret_cast<uint32_t*>(t + i * (DV / 2) + cb * 4) = lo;
        *reinterpret_cast<uint16_t*>(t + DK * DV / 2 + i * (DV / 4) + cb * 2) = uint16_t(hi);
    }
};

// ------------------------------------------------------------------ reductions
// Canonical column sums of a thread-owned 8x8 block: sum_i val[r][c] * w[r].
// The in-thread chain is the block sum, the xor butterfly over offsets
// CBW, 2*CBW, ... joins adjacent row blocks of the warp, and the pairwise tree
// over warps finishes the balanced tree.  Every thread receives its 8 column
// totals.  red: shared [NWARPS][DV]; tot: shared [DV].
template <int DK, int DV>
__device__ __forceinline__ void colsum(const float (&val)[8][8], const float (&w)[8],
                                       float (&res)[8], float* red, float* tot,
                                       int warp, int rbl, int j0) {
    using G = Geo<DK, DV>;
    float p[8];
#pragma unroll
    for (int c = 0; c < 8; c++) {
        float s = 0.0f;
#pragma unroll
        for (int r = 0; r < 8; r++) s = __fmaf_rn(val[r][c], w[r], s);
        p[c] = s;
    }
#pragma unroll
    for (int off = G::CBW; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 8; c++) p[c] = __fadd_rn(p[c], __shfl_xor_sync(0xFFFFFFFFu, p[c], off));
    }
    if (G::NWARPS == 1) {
#pragma unroll
        for (int c = 0; c < 8; c++) res[c] = p[c];
        return;
    }
    if (rbl == 0) {
#pragma unroll
        for (int c = 0; c < 8; c++) red[warp * DV + j0 + c] = p[c];
    }
    __syncthreads();
    if (threadIdx.x < DV) {
        float t[G::NWARPS];
#pragma unroll
        for (int w2 = 0; w2 < G::NWARPS; w2++) t[w2] = red[w2 * DV + threadIdx.x];
#pragma unroll
        for (int n = G::NWARPS; n > 1; n >>= 1) {
#pragma unroll
            for (int u = 0; u < n / 2; u++) t[u] = __fadd_rn(t[2 * u], t[2 * u + 1]);
        }
        tot[threadIdx.x] = t[0];
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 8; c++) res[c] = tot[j0 + c];
    __syncthreads();   // red/tot are reused by the next reduction
}

// Row-group maxima: in-thread over 8 columns then across the lanes of a group
// (group > 0), or over the whole tile (group == 0, result in every m[r]).
template <int DK, int DV>
__device__ __forceinline__ void groupmax(float (&m)[8], int group, float* wred, int warp) {
    using G = Geo<DK, DV>;
    if (group > 0) {
        const int lanes = group / 8;
        for (int off = 1; off < lanes; off <<= 1) {
#pragma unroll
            for (int r = 0; r < 8; r++) m[r] = fmaxf(m[r], __shfl_xor_sync(0xFFFFFFFFu, m[r], off));
        }
        return;
    }
    float t = m[0];
#pragma unroll
    for (int r = 1; r < 8; r++) t = fmaxf(t, m[r]);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) t = fmaxf(t, __shfl_xor_sync(0xFFFFFFFFu, t, off));
    if ((threadIdx.x & 31) == 0) wred[warp] = t;
    __syncthreads();
    t = wred[0];
#pragma unroll
    for (int w2 = 1; w2 < G::NWARPS; w2++) t = fmaxf(t, wred[w2]);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; r++) m[r] = t;
}

// Round one element (RTN, then BDR when enabled).  Returns the code.
template <bool BDR>
__device__ __forceinline__ int round_code(float a, float x, float inv, int qmax, float eps_b) {
    float t = __fmaf_rn(x, inv, kMagic);                  // one rounding of the exact product
    t = fminf(fmaxf(t, kMagic - float(qmax)), kMagic + float(qmax));
    int c = __float_as_int(t) - kMagicBits;
    if (BDR) {
        const float d = __fsub_rn(x, a);
        if (d != 0.0f) {
            const float s = __fmaf_rn(a, inv, -float(c));
            if (d > 0.0f && s > eps_b) c = min(c + 1, qmax);
            else if (d < 0.0f && s < -eps_b) c = max(c - 1, -qmax);
        }
    }
    return c;
}

__device__ __forceinline__ bool all_finite8(const float (&v)[8]) {
    bool ok = true;
#pragma unroll
    for (int e = 0; e < 8; e++) ok &= isfinite(v[e]);
    return ok;
}

// ------------------------------------------------------------------ one tile
template <int DK, int DV, int BITS, bool GDN, bool YOKED, bool BDR>
__device__ __forceinline__ void step_tile(const StepParams& p, long long tile, uint8_t* ct,
                                          float* red, float* tot, float* wred) {
    using G = Geo<DK, DV>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane % G::CBW, rbl = lane / G::CBW;
    const int i0 = (warp * G::RBW + rbl) * 8, j0 = cb * 8;
    constexpr int QMAX = BITS == 32 ? 0 : (1 << (BITS - 1)) - 1;
    const bool bf = p.qkv_bf16 != 0, gbf = p.gate_bf16 != 0, sf32 = p.scale_f32 != 0;

    // step inputs
    float kk[8], qq[8], vv[8], al[8];
    load8(p.k, tile * DK + i0, bf, kk);
    load8(p.q, tile * DK + i0, bf, qq);
    load8(p.v, tile * DV + j0, bf, vv);
    bool bad = !(all_finite8(kk) && all_finite8(qq) && all_finite8(vv));
    if (p.kind == K_GLA) {
        load8(p.gates, tile * p.n_gate + i0, gbf, al);
        bad |= !all_finite8(al);
    } else {
        const float s = p.kind == K_RETNET ? p.gamma : load1(p.gates, tile * p.n_gate, gbf);
        bad |= !isfinite(s);
#pragma unroll
        for (int r = 0; r < 8; r++) al[r] = s;
    }
    float beta = 0.0f;
    if (GDN) {
        beta = load1(p.gates, tile * p.n_gate + 1, gbf);
        bad |= !isfinite(beta);
    }

    const int group = p.group;
    const int ng = group ? DV / group : 1;                 // groups per row
    const long long sbase = tile * (long long)p.n_scales;
    auto sidx = [&](int r) -> long long {
        return group ? sbase + (long long)(i0 + r) * ng + j0 / group : sbase;
    };

    // 1. decay
    float a[8][8];
    float dprev[8];
    if (BITS == 32) {
#pragma unroll
        for (int r = 0; r < 8; r++) {
            const float4* sp = reinterpret_cast<const float4*>(
                reinterpret_cast<const float*>(ct) + (i0 + r) * DV + j0);
            const float4 u0 = sp[0], u1 = sp[1];
            const float s8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int c = 0; c < 8; c++) a[r][c] = __fmul_rn(s8[c], al[r]);
            dprev[r] = 0.0f;
        }
    } else {
        using CD = Codec<(BITS == 32 ? 8 : BITS), DK, DV>;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            dprev[r] = load_scale(p.scales, sidx(r), sf32);
            const float eta = __fmul_rn(al[r], dprev[r]);
            const auto w = CD::load(ct, i0 + r, cb);
#pragma unroll
            for (int c = 0; c < 8; c++) a[r][c] = __fmul_rn(float(CD::get(w, c)), eta);
        }
    }

    // yoked reference state: stepped first, only its group maxima are kept
    float mref[8];
    if (YOKED) {
        float ar[8][8];
#pragma unroll
        for (int r = 0; r < 8; r++) {
            const float4* sp = reinterpret_cast<const float4*>(
                p.ref + (tile * DK + i0 + r) * (long long)DV + j0);
            const float4 u0 = sp[0], u1 = sp[1];
            const float s8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int c = 0; c < 8; c++) ar[r][c] = __fmul_rn(s8[c], al[r]);
        }
        if (GDN) {
            float rr[8];
            colsum<DK, DV>(ar, kk, rr, red, tot, warp, rbl, j0);
#pragma unroll
            for (int c = 0; c < 8; c++) rr[c] = __fsub_rn(vv[c], rr[c]);
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const float kap = __fmul_rn(beta, kk[r]);
#pragma unroll
                for (int c = 0; c < 8; c++) ar[r][c] = __fmaf_rn(kap, rr[c], ar[r][c]);
            }
        } else {
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int c = 0; c < 8; c++) ar[r][c] = __fmaf_rn(kk[r], vv[c], ar[r][c]);
        }
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float4* sp = reinterpret_cast<float4*>(p.ref + (tile * DK + i0 + r) * (long long)DV + j0);
            sp[0] = make_float4(ar[r][0], ar[r][1], ar[r][2], ar[r][3]);
            sp[1] = make_float4(ar[r][4], ar[r][5], ar[r][6], ar[r][7]);
            float mm = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; c++) mm = fmaxf(mm, fabsf(ar[r][c]));
            mref[r] = mm;
        }
        groupmax<DK, DV>(mref, group, wred, warp);
    }

    // 2. update
    float x[8][8];
    if (GDN) {
        float e[8];
        colsum<DK, DV>(a, kk, e, red, tot, warp, rbl, j0);
#pragma unroll
        for (int c = 0; c < 8; c++) e[c] = __fsub_rn(vv[c], e[c]);
#pragma unroll
        for (int r = 0; r < 8; r++) {
            const float kap = __fmul_rn(beta, kk[r]);
#pragma unroll
            for (int c = 0; c < 8; c++) x[r][c] = __fmaf_rn(kap, e[c], a[r][c]);
        }
    } else {
#pragma unroll
        for (int r = 0; r < 8; r++)
#pragma unroll
            for (int c = 0; c < 8; c++) x[r][c] = __fmaf_rn(kk[r], vv[c], a[r][c]);
    }

    // 3. output from the updated, not yet rounded state
    {
        float o[8];
        colsum<DK, DV>(x, qq, o, red, tot, warp, rbl, j0);
        if (rbl == 0 && warp == 0) {
            float4* op = reinterpret_cast<float4*>(p.out + tile * DV + j0);
            op[0] = make_float4(o[0], o[1], o[2], o[3]);
            op[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
    }

    if (BITS == 32) {
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float4* sp = reinterpret_cast<float4*>(reinterpret_cast<float*>(ct) + (i0 + r) * DV + j0);
            sp[0] = make_float4(x[r][0], x[r][1], x[r][2], x[r][3]);
            sp[1] = make_float4(x[r][4], x[r][5], x[r][6], x[r][7]);
        }
        return;
    }

    // 4. scale
    float m[8];
#pragma unroll
    for (int r = 0; r < 8; r++) {
        float mm = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; c++) mm = fmaxf(mm, fabsf(x[r][c]));
        m[r] = mm;
    }
    groupmax<DK, DV>(m, group, wred, warp);
    const float fq = float(QMAX);
    float inv[8];
    // one lane per (row, group) stores the scale and counts its overflow
    const bool writer = group ? (cb % (group / 8)) == 0 : threadIdx.x == 0;
    unsigned nsat = 0;
#pragma unroll
    for (int r = 0; r < 8; r++) {
        bad |= !isfinite(m[r]);
        bool sat = false;
        float d;
        if (YOKED) {
            bad |= !isfinite(mref[r]);
            d = to_stored(__fdiv_rn(mref[r], fq), sf32, sat);
        } else if (p.scale_mode == M_PERSISTENT) {
            d = (m[r] > __fmul_rn(fq, dprev[r])) ? to_stored(__fdiv_rn(m[r], fq), sf32, sat)
                                                  : dprev[r];
        } else {
            d = to_stored(__fdiv_rn(m[r], fq), sf32, sat);
        }
        inv[r] = d == 0.0f ? 0.0f : __frcp_rn(d);
        if (writer && (group || r == 0)) {
            store_scale(p.scales, sidx(r), sf32, d);
            nsat += sat ? 1u : 0u;
        }
    }
    if (nsat) atomicAdd(p.counters + 1, (unsigned long long)nsat);

    // 5-6. round and repack
    using CD = Codec<(BITS == 32 ? 8 : BITS), DK, DV>;
#pragma unroll
    for (int r = 0; r < 8; r++) {
        int c8[8];
#pragma unroll
        for (int c = 0; c < 8; c++) c8[c] = round_code<BDR>(a[r][c], x[r][c], inv[r], QMAX, p.eps_b);
        CD::store(ct, i0 + r, cb, c8);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicAdd(p.counters, 1ull);
}

template <int DK, int DV, bool GDN, bool YOKED, bool BDR>
__global__ void __launch_bounds__(Geo<DK, DV>::NT)
step_kernel(const StepParams p) {
    using G = Geo<DK, DV>;
    __shared__ __align__(16) float red[G::NWARPS * DV];
    __shared__ __align__(16) float tot[DV];
    __shared__ float wred[G::NWARPS];
    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        int bits = p.bits;
        uint8_t* ct;
        if (p.head_bits) {
            const int h = int(tile % p.heads);
            bits = p.head_bits[h];
            ct = p.codes + (tile / p.heads) * p.row_bytes + p.head_off[h];
        } else {
            ct = p.codes + tile * p.tile_bytes;
        }
        // warm L2 with the next tile of this CTA (bulk prefetch, no completion)
        if (threadIdx.x == 0 && !p.head_bits && tile + gridDim.x < p.ntiles) {
            const uint8_t* nxt = p.codes + (tile + gridDim.x) * p.tile_bytes;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                         :: "l"(nxt), "r"(uint32_t(p.tile_bytes)) : "memory");
        }
        switch (bits) {
            case 2: step_tile<DK, DV, 2, GDN, YOKED, BDR>(p, tile, ct, red, tot, wred); break;
            case 4: step_tile<DK, DV, 4, GDN, YOKED, BDR>(p, tile, ct, red, tot, wred); break;
            case 6: step_tile<DK, DV, 6, GDN, YOKED, BDR>(p, tile, ct, red, tot, wred); break;
            case 8: step_tile<DK, DV, 8, GDN, YOKED, BDR>(p, tile, ct, red, tot, wred); break;
            default:
                if (!YOKED) step_tile<DK, DV, 32, GDN, false, BDR>(p, tile, ct, red, tot, wred);
                break;
        }
    }
}

// Dequantized state S_hat = code * scale, one thread per 8-column block.
template <int DK, int DV>
__global__ void dequant_kernel(const StepParams p, float* S) {
    const long long nblk = p.ntiles * DK * (DV / 8);
    for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < nblk;
         b += (long long)gridDim.x * blockDim.x) {
        const long long tile = b / (DK * (DV / 8));
        const int rem = int(b % (DK * (DV / 8)));
        const int i = rem / (DV / 8), cb = rem % (DV / 8);
        int bits = p.bits;
        const uint8_t* ct;
        if (p.head_bits) {
            const int h = int(tile % p.heads);
            bits = p.head_bits[h];
            ct = p.codes + (tile / p.heads) * p.row_bytes + p.head_off[h];
        } else {
            ct = p.codes + tile * p.tile_bytes;
        }
        float* dst = S + (tile * DK + i) * (long long)DV + cb * 8;
        if (bits == 32) {
            const float* src = reinterpret_cast<const float*>(ct) + i * DV + cb * 8;
#pragma unroll
            for (int c = 0; c < 8; c++) dst[c] = src[c];
            continue;
        }
        const int group = p.group, ng = group ? DV / group : 1;
        const long long si = tile * (long long)p.n_scales + (group ? (long long)i * ng + cb * 8 / group : 0);
        const float d = load_scale(p.scales, si, p.scale_f32 != 0);
        int c8[8];
        switch (bits) {
            case 2: { auto w = Codec<2, DK, DV>::load(ct, i, cb);
                      for (int c = 0; c < 8; c++) c8[c] = Codec<2, DK, DV>::get(w, c); } break;
            case 4: { auto w = Codec<4, DK, DV>::load(ct, i, cb);
                      for (int c = 0; c < 8; c++) c8[c] = Codec<4, DK, DV>::get(w, c); } break;
            case 6: { auto w = Codec<6, DK, DV>::load(ct, i, cb);
                      for (int c = 0; c < 8; c++) c8[c] = Codec<6, DK, DV>::get(w, c); } break;
            default: { auto w = Codec<8, DK, DV>::load(ct, i, cb);
                       for (int c = 0; c < 8; c++) c8[c] = Codec<8, DK, DV>::get(w, c); } break;
        }
#pragma unroll
        for (int c = 0; c < 8; c++) dst[c] = __fmul_rn(float(c8[c]), d);
    }
}

}  // namespace qs
