// qstate_lrb.cuh -- the decode step with a Low-Rank Bypass (LRB) of
// "Preserving Updates in Low-Bit Recurrent State Quantization" (Abstract,
// Figure 3, Tables 6, 8, 9), for uniform 4- or 8-bit states of RetNet,
// Mamba2, GLA and Gated DeltaNet tiles with d_k = d_v.
//
// A tile's state is D * S_hat + P: the quantized part S_hat (codes, scales)
// times the decay D accumulated since the last merge, plus the bypass
// P = sum_l g_l u_l w_l^T of up to k + m columns (u, w in binary16, g in
// binary32; slots 0 .. n_res - 1 the rank-k residual, then the fresh updates
// in arrival order).  Every step decays D and every g_l by alpha, forms the
// update (GDN: e = v - r with r = (A S)^T k over the whole state) as a new
// column, and emits o = (A S + B)^T q; codes and scales are not touched.
// When the m-th fresh column arrives, the bypass elements at least eps_L
// grid steps of the decayed grid large are merged: x = a + P there, x = a
// elsewhere, requantized with the object's scale and rounding rules (BDR with
// d = x - a), D reset to 1, and the unmerged rest kept as its leading
// singular pair (k = 1, by power iteration) or dropped (k = 0).  GLA's decay
// Diag(alpha) keeps one D per key row instead: the coefficients do not
// decay, a column's key side is stored divided by the D of its step and read
// as D_i u_i, and the tile stands for Diag(D) (S_hat + P).
//
// Arithmetic and order follow the specification of the bypass (canonical
// sums; each column in slot order as one fma per element); every result is
// the same as the element-wise definition except the rank-1 residual, which
// approximates the truncated SVD.  One tile per CTA at a time, plain loads:
// this is the reference decomposition of the method, not the streaming
// pipeline of step_kernel.
#pragma once

#include "qstate_kernel.cuh"

namespace qs {

constexpr int kLrbMaxCols = 32;
constexpr int kLrbPowerIters = 16;

struct LrbParams {
    uint16_t* u;      // [tiles][k + m][d_k] binary16
    uint16_t* w;      // [tiles][k + m][d_v] binary16
    float* g;         // [tiles][k + m]
    int* n;           // [tiles][2]: residual slots in use, fresh slots in use
    float* D;         // [tiles] (GLA: [tiles][d_k]): decay since the last merge
    int k, m;
    float eps_l;
};

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t f2h(float x) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ float f16r(float x) { return __half2float(__float2half_rn(x)); }

// Eight consecutive binary16 values (16-byte aligned) as binary32
__device__ __forceinline__ void h8(const uint16_t* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Canonical sum over i < DK of x_i y_i (blocks of 8 rows, ascending fma from
// +0, then the adjacent-pairs tree), by one warp: lane b < DK/8 sums block b,
// the xor butterfly over those lanes is the tree, and lane 0's total goes to
// every lane (the lanes above DK/8 hold only their own zeros).
template <int DK, class X, class Y>
__device__ __forceinline__ float warp_canon_dot(X x, Y y, int lane) {
    constexpr int NB = DK / 8;
    float p = 0.0f;
    if (lane < NB) {
#pragma unroll
        for (int r = 0; r < 8; r++) p = __fmaf_rn(x(8 * lane + r), y(8 * lane + r), p);
    }
#pragma unroll
    for (int off = 1; off < NB; off <<= 1) p = __fadd_rn(p, __shfl_xor_sync(0xFFFFFFFFu, p, off));
    return __shfl_sync(0xFFFFFFFFu, p, 0);
}

template <int DK, int DV>
struct __align__(16) LrbShared {
    using G = Geo<DK, DV>;
    Xchg<DK, DV, false> xs;
    float red[G::NWARPS * DV];       // column-sum partials (r, power iteration)
    float tot[DV];
    float vec[DK > DV ? DK : DV];    // power iteration vector
    float nrm[G::NWARPS];
    float gco[kLrbMaxCols];          // decayed coefficients, the new column's = 1
    float ck[kLrbMaxCols], cq[kLrbMaxCols];   // g_l (u_l . k), g_l (u_l . q)
    float unew[DK], wnew[DV];        // the new column (binary16 values)
    float drow[DK];                  // GLA: the per-row decay since the last merge, this step's
    // the tile's scales before the step, in their stored format
    __align__(16) uint8_t sprev[DK * (DV / 8) * 4];
    // the columns held at the start of the step (binary16 patterns)
    __align__(16) uint16_t ucol[kLrbMaxCols * DK];
    __align__(16) uint16_t wcol[kLrbMaxCols * DV];
};

// Ask L2 for [p, p + bytes) (128-byte lines, spread over the CTA's threads)
template <int NT>
__device__ __forceinline__ void prefetch_l2(const void* p, long long bytes) {
    const char* c = static_cast<const char*>(p);
    for (long long o = (long long)threadIdx.x * 128; o < bytes; o += (long long)NT * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(c + o));
}

// Round x with the scale's reciprocal: code = clamp(RTN(x * inv)); with BDR
// a reversed element (d = x - a, s = fma(a, inv, -code), d > 0 and s > eps_B,
// or d < 0 and s < -eps_B) moves one code toward its update, clamped.
// arow(r, a8) gives row r of this thread's decayed state a (read only with
// BDR, before row r's codes are written).
template <int DK, int DV, int BITS, bool BDR, class ARow>
__device__ __forceinline__ void round_pack_ax(ARow arow, const float (&x)[8][8],
                                              const float (&inv)[8], float eps_b, uint8_t* ct,
                                              int i0, int cb) {
    constexpr float fq = float((1 << (BITS - 1)) - 1);
#pragma unroll
    for (int r = 0; r < 8; r++) {
        float t8[8];
        float ar[8];
        if (BDR) arow(r, ar);
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float2 x2 = f2(x[r][c], x[r][c + 1]);
            float2 t2 = rtn2(x2, inv[r]);
            t2.x = fminf(fmaxf(t2.x, kMagic - fq), kMagic + fq);
            t2.y = fminf(fmaxf(t2.y, kMagic - fq), kMagic + fq);
            if (BDR) {
                const float2 a2 = f2(ar[c], ar[c + 1]);
                const float2 d2 = ffma2(a2, f2(-1.0f, -1.0f), x2);                  // x - a
                const float2 cn = ffma2(t2, f2(-1.0f, -1.0f), f2(kMagic, kMagic));  // -code
                const float2 s2 = ffma2(a2, f2(inv[r], inv[r]), cn);
                t2.x = fminf(fmaxf(bdr1(t2.x, s2.x, d2.x, eps_b), kMagic - fq), kMagic + fq);
                t2.y = fminf(fmaxf(bdr1(t2.y, s2.y, d2.y, eps_b), kMagic - fq), kMagic + fq);
            }
            t8[c] = t2.x;
            t8[c + 1] = t2.y;
        }
        pack_row<DK, DV, BITS>(ct, i0 + r, cb, t8);
    }
}

// Sum over the row blocks of a warp and then over the warps (any order: the
// power iteration only) of a per-thread 8-column partial; every thread gets
// its 8 column totals.
template <int DK, int DV>
__device__ __forceinline__ void colsum_any(float (&p)[8], float* red, float* tot, int warp, int rbl,
                                           int j0, float (&res)[8]) {
    colsum_finish<DK, DV>(p, red, tot, warp, rbl, j0, res);
}

// Requantize a tile's updated state x (arow: rows of the decayed state a
// before the update, for BDR) with the object's scale rule (dynamic or
// persistent, per-group or per-token; previous scales in `sprev`, in their
// stored format): new scales and codes written to HBM, saturated scales and
// non-finite group maxima counted.  Every thread of the CTA calls it.
template <int DK, int DV, int BITS, bool BDR, class XS, class ARow>
__device__ __forceinline__ void requantize(const StepParams& p, XS& xs, const uint8_t* sprev,
                                           long long sbase, uint8_t* ct, ARow arow,
                                           const float (&x)[8][8], int lane, int warp, int cb,
                                           int i0, int ng, int gcol) {
    using G = Geo<DK, DV>;
    constexpr int QMAX = (1 << (BITS - 1)) - 1;
    constexpr float fq = float(QMAX);
    constexpr float rq = QMAX == 7 ? 0x1.24924ap-3f : 0x1.020408p-7f;
    const bool sf32 = p.scale_f32 != 0;
    const int group = p.group;
    auto prev_scale = [&](int idx) -> float {
        if (sf32) return reinterpret_cast<const float*>(sprev)[idx];
        return __half2float(reinterpret_cast<const __half*>(sprev)[idx]);
    };
    // group maxima of |x| and the new scales
    float m[8];
#pragma unroll
    for (int r = 0; r < 8; r++) {
        float mx = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; c++) mx = fmaxf(mx, fabsf(x[r][c]));
        m[r] = mx;
    }
    if (group) {
        float4* r4 = reinterpret_cast<float4*>(&xs.rmax[cb][i0]);
        r4[0] = make_float4(m[0], m[1], m[2], m[3]);
        r4[1] = make_float4(m[4], m[5], m[6], m[7]);
    } else {
        float t = m[0];
#pragma unroll
        for (int r = 1; r < 8; r++) t = fmaxf(t, m[r]);
        t = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(t)));
        if (lane == 0) xs.wred[0][warp] = t;
    }
    __syncthreads();
    float inv[8];
    unsigned nsat = 0;
    bool bad = false;
    auto new_scale = [&](float mm, float, float dp, bool& sat, auto sfc) -> float {
        const bool F = as_bool(sfc);
        sat = false;
        if (p.scale_mode == M_PERSISTENT)
            return (mm > __fmul_rn(fq, dp)) ? to_stored(div_by_qmax(mm, fq, rq), F, sat) : dp;
        return to_stored(div_by_qmax(mm, fq, rq), F, sat);
    };
    if (group) {
        auto gs = [&](auto lc, auto sfc) {
            group_scales<DK, DV, decltype(lc)::value, decltype(sfc)::value>(
                cb, lane, i0, xs, false, inv, nsat, bad, new_scale, sprev, p, sbase, ng, gcol);
        };
        auto gs_l = [&](auto lc) {
            if (sf32) gs(lc, std::true_type{});
            else gs(lc, std::false_type{});
        };
        switch (group / 8) {
            case 1: gs_l(std::integral_constant<int, 1>{}); break;
            case 2: gs_l(std::integral_constant<int, 2>{}); break;
            case 4: gs_l(std::integral_constant<int, 4>{}); break;
            case 8: gs_l(std::integral_constant<int, 8>{}); break;
            default: gs_l(std::integral_constant<int, 16>{}); break;
        }
    } else {
        float tmax = xs.wred[0][0];
#pragma unroll
        for (int w2 = 1; w2 < G::NWARPS; w2++) tmax = fmaxf(tmax, xs.wred[0][w2]);
        bool sat;
        const float d = new_scale(tmax, 0.0f, prev_scale(0), sat, sf32);
        const float iv = d == 0.0f ? 0.0f : __frcp_rn(d);
#pragma unroll
        for (int r = 0; r < 8; r++) inv[r] = iv;
        bad |= !isfinite(tmax);
        if (threadIdx.x == G::NT - 1) {
            store_scale(p.scales, sbase, sf32, d);
            nsat += sat ? 1u : 0u;
        }
    }
    if (nsat) atomicAdd(p.counters + 1, (unsigned long long)nsat);
    if (bad && threadIdx.x == 0) atomicAdd(p.counters, 1ull);
    round_pack_ax<DK, DV, BITS, BDR>(arow, x, inv, p.eps_b, ct, i0, cb);
}

// Two CTAs per SM: the decayed quantized part a is re-derived from the codes
// (an L1 hit after the first read) wherever the step needs it, so only the
// merge's 8 x 8 block stays in registers.
// VEC: GLA's per-row decay: D holds one factor per key row, the coefficients
// do not decay, and a column's key side is held divided by the row factors of
// its step and read as D_i * u_i.
template <int DK, int DV, int BITS, bool GDN, bool VEC, bool BDR, bool BF>
__global__ void __launch_bounds__(Geo<DK, DV>::NT, 2) lrb_kernel(const StepParams p, const LrbParams L) {
    using G = Geo<DK, DV>;
    static_assert(DK == DV, "square tiles");
    static_assert(!(GDN && VEC), "the delta rule has a scalar decay");
    static_assert(BITS == 4 || BITS == 8, "4- or 8-bit codes");
    constexpr int QMAX = (1 << (BITS - 1)) - 1;
    constexpr float fq = float(QMAX);
    constexpr float rq = QMAX == 7 ? 0x1.24924ap-3f : 0x1.020408p-7f;
    __shared__ LrbShared<DK, DV> sh;
    extern __shared__ __align__(16) float resid[];     // [64][NT]: the unmerged residual (k = 1)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane % G::CBW, rbl = lane / G::CBW;
    const int i0 = (warp * G::RBW + rbl) * 8, j0 = cb * 8;
    const int K = L.k + L.m;
    const bool sf32 = p.scale_f32 != 0;
    const int group = p.group;
    const int gsh = group ? __ffs(group) - 1 : 0;
    const int ng = group ? DV >> gsh : 1;
    const int gcol = group ? j0 >> gsh : 0;

    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        const int nres = L.n[2 * tile], nnew = L.n[2 * tile + 1];
        const int n = nres + nnew;                         // columns before this step
        const uint16_t* U = L.u + tile * K * DK;
        const uint16_t* Wc = L.w + tile * K * DV;
        uint8_t* ct = p.codes + tile * p.tile_bytes;
        const long long sbase = tile * (long long)p.n_scales;
        const float alpha = VEC ? 1.0f
                          : p.kind == K_RETNET ? p.gamma : ldg1(p.gates, tile * p.n_gate, p.gate_bf16 != 0);
        const float beta = GDN ? ldg1(p.gates, tile * p.n_gate + 1, p.gate_bf16 != 0) : 0.0f;
        const float Dn = VEC ? 0.0f : __fmul_rn(alpha, L.D[tile]);
        if constexpr (VEC) {
            for (int i = threadIdx.x; i < DK; i += G::NT)
                sh.drow[i] = __fmul_rn(ldg1(p.gates, tile * p.n_gate + i, p.gate_bf16 != 0),
                                       L.D[tile * DK + i]);
        }

        // the next tile's bytes on their way to L2 while this one is stepped
        {
            const long long nt = tile + gridDim.x;
            if (nt < p.ntiles) {
                const int ssz = sf32 ? 4 : 2;
                const int isz = BF ? 2 : 4;
                prefetch_l2<G::NT>(p.codes + nt * p.tile_bytes, p.tile_bytes);
                prefetch_l2<G::NT>(static_cast<const uint8_t*>(p.scales) + nt * p.n_scales * ssz,
                                   (long long)p.n_scales * ssz);
                // only the columns that tile holds (its counts: one cached line)
                const int nn = L.n[2 * nt] + L.n[2 * nt + 1];
                prefetch_l2<G::NT>(L.u + nt * K * DK, (long long)nn * DK * 2);
                prefetch_l2<G::NT>(L.w + nt * K * DV, (long long)nn * DV * 2);
                if (threadIdx.x == 0) {
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.q) + nt * DK * isz));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.k) + nt * DK * isz));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.v) + nt * DV * isz));
                }
            }
        }
        // the tile's scales before the step, its columns, and the decayed
        // coefficients (16-byte loads: every region starts on a 16-byte
        // boundary and holds a multiple of 16 bytes, or is copied bytewise)
        {
            const int ssz = sf32 ? 4 : 2;
            const uint8_t* src = static_cast<const uint8_t*>(p.scales) + sbase * ssz;
            const int sb = p.n_scales * ssz;
            if ((sb & 15) == 0 && ((sbase * ssz) & 15) == 0) {
                for (int i = threadIdx.x; i < sb / 16; i += G::NT)
                    reinterpret_cast<uint4*>(sh.sprev)[i] = reinterpret_cast<const uint4*>(src)[i];
            } else {
                for (int i = threadIdx.x; i < sb; i += G::NT) sh.sprev[i] = src[i];
            }
            for (int i = threadIdx.x; i < n * DK / 8; i += G::NT)
                reinterpret_cast<uint4*>(sh.ucol)[i] = reinterpret_cast<const uint4*>(U)[i];
            for (int i = threadIdx.x; i < n * DV / 8; i += G::NT)
                reinterpret_cast<uint4*>(sh.wcol)[i] = reinterpret_cast<const uint4*>(Wc)[i];
        }
        auto prev_scale = [&](int idx) -> float {
            if (sf32) return reinterpret_cast<const float*>(sh.sprev)[idx];
            return __half2float(reinterpret_cast<const __half*>(sh.sprev)[idx]);
        };
        for (int l = threadIdx.x; l < n; l += G::NT)
            sh.gco[l] = VEC ? L.g[tile * K + l] : __fmul_rn(alpha, L.g[tile * K + l]);
        __syncthreads();
        // a column's key side as the step reads it (GLA: D_i * u_i)
        auto ueff = [&](int l, int i) -> float {
            const float u = h2f(sh.ucol[l * DK + i]);
            return VEC ? __fmul_rn(sh.drow[i], u) : u;
        };
        // g_l (u_l . k) and g_l (u_l . q) for the columns held
        const uint8_t* kin = static_cast<const uint8_t*>(p.k) + tile * DK * (BF ? 2 : 4);
        const uint8_t* qin = static_cast<const uint8_t*>(p.q) + tile * DK * (BF ? 2 : 4);
        auto kval = [&](int i) { return ldg1(kin, i, BF); };
        auto qval = [&](int i) { return ldg1(qin, i, BF); };
        for (int l = warp; l < n; l += G::NWARPS) {
            auto uval = [&](int i) { return ueff(l, i); };
            const float dk_ = GDN ? warp_canon_dot<DK>(uval, kval, lane) : 0.0f;
            const float dq_ = warp_canon_dot<DK>(uval, qval, lane);
            if (lane == 0) {
                sh.ck[l] = __fmul_rn(sh.gco[l], dk_);
                sh.cq[l] = __fmul_rn(sh.gco[l], dq_);
            }
        }

        // the decayed quantized part a = code * (D * scale)
        float kk[8], qq[8], vv[8], eta[8];
#pragma unroll
        for (int r = 0; r < 8; r++) {
            kk[r] = kval(i0 + r);
            qq[r] = qval(i0 + r);
            const float dp = prev_scale(group ? (i0 + r) * ng + gcol : 0);
            eta[r] = __fmul_rn(VEC ? sh.drow[i0 + r] : Dn, dp);
        }
        {
            const uint8_t* vin = static_cast<const uint8_t*>(p.v) + tile * DV * (BF ? 2 : 4);
#pragma unroll
            for (int c = 0; c < 8; c++) vv[c] = ldg1(vin, j0 + c, BF);
        }
        // row r of this thread's a = code * (D * scale)
        auto arow = [&](int r, float (&ar)[8]) {
            float c8[8];
            if constexpr (BITS == 4) Decode<4>::run(ct + (i0 + r) * (DV / 2), cb, c8);
            else Decode<8>::run(ct + (i0 + r) * DV, cb, c8);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 a2 = fmul2(f2(c8[c], c8[c + 1]), f2(eta[r], eta[r]));
                ar[c] = a2.x;
                ar[c + 1] = a2.y;
            }
        };
        __syncthreads();                                   // ck, cq complete

        // the update: GDN e = v - r over the whole state; the new column
        float wn[8];
        if constexpr (GDN) {
            float pr[8];
#pragma unroll
            for (int c = 0; c < 8; c++) pr[c] = 0.0f;
#pragma unroll
            for (int r = 0; r < 8; r++) {
                float ar[8];
                arow(r, ar);
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 p2 = ffma2(f2(ar[c], ar[c + 1]), f2(kk[r], kk[r]), f2(pr[c], pr[c + 1]));
                    pr[c] = p2.x;
                    pr[c + 1] = p2.y;
                }
            }
            float rr[8];
            colsum_finish<DK, DV>(pr, sh.red, sh.tot, warp, rbl, j0, rr);
            for (int l = 0; l < n; l++) {
                float w8[8];
                h8(sh.wcol + l * DV + j0, w8);
                const float cl = sh.ck[l];
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 r2 = ffma2(f2(cl, cl), f2(w8[c], w8[c + 1]), f2(rr[c], rr[c + 1]));
                    rr[c] = r2.x;
                    rr[c + 1] = r2.y;
                }
            }
#pragma unroll
            for (int c = 0; c < 8; c++) wn[c] = f16r(__fsub_rn(vv[c], rr[c]));
        } else {
#pragma unroll
            for (int c = 0; c < 8; c++) wn[c] = f16r(vv[c]);
        }
        if (rbl == 0 && warp == 0) {
#pragma unroll
            for (int c = 0; c < 8; c++) sh.wnew[j0 + c] = wn[c];
        }
        if (cb == 0) {
#pragma unroll
            for (int r = 0; r < 8; r++)
                sh.unew[i0 + r] = f16r(GDN ? __fmul_rn(beta, kk[r])
                                           : VEC ? __fdiv_rn(kk[r], sh.drow[i0 + r]) : kk[r]);
        }
        __syncthreads();
        if (warp == 0) {
            auto uval = [&](int i) { return VEC ? __fmul_rn(sh.drow[i], sh.unew[i]) : sh.unew[i]; };
            const float dq_ = warp_canon_dot<DK>(uval, qval, lane);
            if (lane == 0) {
                sh.cq[n] = __fmul_rn(1.0f, dq_);
                sh.gco[n] = 1.0f;
            }
        }

        // output o = a^T q, then the columns in slot order (the new one last)
        {
            float po[8];
#pragma unroll
            for (int c = 0; c < 8; c++) po[c] = 0.0f;
#pragma unroll
            for (int r = 0; r < 8; r++) {
                float ar[8];
                arow(r, ar);
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 p2 = ffma2(f2(ar[c], ar[c + 1]), f2(qq[r], qq[r]), f2(po[c], po[c + 1]));
                    po[c] = p2.x;
                    po[c + 1] = p2.y;
                }
            }
            float oo[8];
            colsum_finish<DK, DV>(po, sh.red, sh.tot, warp, rbl, j0, oo);    // syncs: cq[n] visible
            for (int l = 0; l < n; l++) {
                float w8[8];
                h8(sh.wcol + l * DV + j0, w8);
                const float cl = sh.cq[l];
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 o2 = ffma2(f2(cl, cl), f2(w8[c], w8[c + 1]), f2(oo[c], oo[c + 1]));
                    oo[c] = o2.x;
                    oo[c + 1] = o2.y;
                }
            }
#pragma unroll
            for (int c = 0; c < 8; c++) oo[c] = __fmaf_rn(sh.cq[n], sh.wnew[j0 + c], oo[c]);
            if (rbl == 0 && warp == 0) {
#pragma unroll
                for (int c = 0; c < 8; c++) p.out[tile * DV + j0 + c] = oo[c];
            }
        }

        // append the new column; the decayed coefficients
        for (int i = threadIdx.x; i < DK; i += G::NT) L.u[(tile * K + n) * DK + i] = f2h(sh.unew[i]);
        for (int j = threadIdx.x; j < DV; j += G::NT) L.w[(tile * K + n) * DV + j] = f2h(sh.wnew[j]);
        for (int l = threadIdx.x; l <= n; l += G::NT) L.g[tile * K + l] = sh.gco[l];

        if (nnew + 1 < L.m) {                              // no merge: codes untouched
            if constexpr (VEC) {
                for (int i = threadIdx.x; i < DK; i += G::NT) L.D[tile * DK + i] = sh.drow[i];
            }
            if (threadIdx.x == 0) {
                if (!VEC) L.D[tile] = Dn;
                L.n[2 * tile + 1] = nnew + 1;
            }
            __syncthreads();
            continue;
        }

        // ---- merge: the dense bypass, the threshold, requantization (x is
        // formed in place of the bypass block P)
        float x[8][8];
        {
            auto& P = x;
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int c = 0; c < 8; c++) P[r][c] = 0.0f;
            for (int l = 0; l <= n; l++) {
                const float gl = sh.gco[l];
                float u8[8], w8[8];
                if (l < n) {
                    h8(sh.ucol + l * DK + i0, u8);
                    h8(sh.wcol + l * DV + j0, w8);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        u8[i] = sh.unew[i0 + i];
                        w8[i] = sh.wnew[j0 + i];
                    }
                }
                if constexpr (VEC) {
#pragma unroll
                    for (int i = 0; i < 8; i++) u8[i] = __fmul_rn(sh.drow[i0 + i], u8[i]);
                }
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    const float gu = __fmul_rn(gl, u8[r]);
#pragma unroll
                    for (int c = 0; c < 8; c += 2) {
                        const float2 p2 = ffma2(f2(gu, gu), f2(w8[c], w8[c + 1]), f2(P[r][c], P[r][c + 1]));
                        P[r][c] = p2.x;
                        P[r][c + 1] = p2.y;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const float thr = __fmul_rn(L.eps_l, eta[r]);
                float ar[8];
                arow(r, ar);
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    const float pc = P[r][c];
                    const bool mg = fabsf(pc) >= thr;
                    if (L.k == 1) resid[(r * 8 + c) * G::NT + threadIdx.x] = mg ? 0.0f : pc;
                    x[r][c] = mg ? __fadd_rn(ar[c], pc) : ar[c];
                }
            }
        }
        requantize<DK, DV, BITS, BDR>(p, sh.xs, sh.sprev, sbase, ct, arow, x, lane, warp, cb, i0, ng,
                                      gcol);

        // the unmerged rest: its leading singular pair (k = 1) or nothing
        if (L.k == 1) {
            auto R = [&](int r, int c) { return resid[(r * 8 + c) * G::NT + threadIdx.x]; };
            // start from the previous residual's value vector when it is not
            // zero, else from a fixed vector of unequal positive entries (not
            // orthogonal to the leading singular vector of a residual whose
            // rows sum to zero, as all ones would be)
            bool nz = false;
            for (int j = threadIdx.x; j < DV; j += G::NT) {
                const float v0 = nres > 0 ? h2f(sh.wcol[j]) : 0.0f;
                sh.vec[j] = v0;
                nz |= v0 != 0.0f;
            }
            if (!__syncthreads_or(nz)) {
                for (int j = threadIdx.x; j < DV; j += G::NT) sh.vec[j] = 1.0f + float((5 * j) % 7) * 0.125f;
            }
            __syncthreads();
            float y[8], vj[8];
#pragma unroll
            for (int c = 0; c < 8; c++) vj[c] = sh.vec[j0 + c];
            for (int itp = 0; itp <= kLrbPowerIters; itp++) {
                // y = R v over this thread's rows, joined across its row's lanes
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    float t = 0.0f;
#pragma unroll
                    for (int c = 0; c < 8; c++) t = __fmaf_rn(R(r, c), vj[c], t);
                    for (int off = 1; off < G::CBW; off <<= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, off);
                    y[r] = t;
                }
                if (itp == kLrbPowerIters) break;
                // v = R^T y / |R^T y|: every warp forms the norm from the column
                // totals itself (same values, same order), so v stays in registers
                float z[8], zt[8];
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    float t = 0.0f;
#pragma unroll
                    for (int r = 0; r < 8; r++) t = __fmaf_rn(R(r, c), y[r], t);
                    z[c] = t;
                }
                colsum_any<DK, DV>(z, sh.red, sh.tot, warp, rbl, j0, zt);
                float s2 = 0.0f;
                for (int j = lane; j < DV; j += 32) s2 = __fmaf_rn(sh.tot[j], sh.tot[j], s2);
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, off);
                const float iz = s2 > 0.0f ? rsqrtf(s2) : 0.0f;
#pragma unroll
                for (int c = 0; c < 8; c++) vj[c] = zt[c] * iz;
            }
            if (rbl == 0 && warp == 0) {
#pragma unroll
                for (int c = 0; c < 8; c++) sh.vec[j0 + c] = vj[c];
            }
            // sigma = |R v|, u = R v / sigma: columns of the new residual slot 0
            float s2 = 0.0f;
            if (cb == 0) {
#pragma unroll
                for (int r = 0; r < 8; r++) s2 = __fmaf_rn(y[r], y[r], s2);
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, off);
            if (lane == 0) sh.nrm[warp] = s2;
            __syncthreads();
            float tot2 = 0.0f;
#pragma unroll
            for (int w2 = 0; w2 < G::NWARPS; w2++) tot2 += sh.nrm[w2];
            const float sig = sqrtf(tot2);
            const float rs = sqrtf(sig);
            if (cb == 0) {
#pragma unroll
                for (int r = 0; r < 8; r++)
                    L.u[(tile * K) * DK + i0 + r] = f2h(sig > 0.0f ? rs * (y[r] / sig) : 0.0f);
            }
            for (int j = threadIdx.x; j < DV; j += G::NT)
                L.w[(tile * K) * DV + j] = f2h(sig > 0.0f ? rs * sh.vec[j] : 0.0f);
            if (threadIdx.x == 0) L.g[tile * K] = 1.0f;
        }
        if constexpr (VEC) {
            for (int i = threadIdx.x; i < DK; i += G::NT) L.D[tile * DK + i] = 1.0f;
        }
        if (threadIdx.x == 0) {
            if (!VEC) L.D[tile] = 1.0f;
            L.n[2 * tile] = L.k;
            L.n[2 * tile + 1] = 0;
        }
        __syncthreads();
    }
}

}  // namespace qs
