// qstate_rc.cuh -- the decode step of a state quantized with key-row x
// value-column scales ("STEPQuant: When and Where Errors Matter in
// Delta-Rule Recurrent State Quantization", Abstract), fitted every step
// from the state itself: kappa_j = cvt(max_i |x_ij|), rho_i =
// cvt(max_j(|x_ij| / kappa_j) / Qmax), grid step rho_i * kappa_j.
//
// Per tile: a_ij = code * ((alpha_i * rho_i) * kappa_j); the update and the
// output are the plain step's (rank-1, or the delta rule with r = a^T k);
// then the column maxima, the column scales and their reciprocals, the row
// maxima of the column-normalised magnitudes, the row scales, and
// c = clamp(rne(x * (1/rho_i * 1/kappa_j))) (BDR with d = x - a).  Every
// result is defined element by element and matches the definition bit for
// bit.  One tile per CTA at a time, plain loads with the next tile's bytes
// prefetched to L2 (like the bypass and window steps).
#pragma once

#include "qstate_lrb.cuh"

namespace qs {

template <int DK, int DV>
struct __align__(16) RcShared {
    using G = Geo<DK, DV>;
    float red[G::NWARPS * DV];
    float tot[DV];
    float rho[DK];                   // alpha_i * the previous row scale
    float kap[DV];                   // the previous column scales
    int bad;
};

// Maximum over the row blocks of a warp and then over the warps of a
// per-thread 8-column partial (max is exact: any order); every thread gets
// its 8 column maxima.
template <int DK, int DV>
__device__ __forceinline__ void colmax_finish(float (&p)[8], float* red, float* tot, int warp,
                                              int rbl, int j0, float (&res)[8]) {
    using G = Geo<DK, DV>;
#pragma unroll
    for (int off = G::CBW; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 8; c++) p[c] = fmaxf(p[c], __shfl_xor_sync(0xFFFFFFFFu, p[c], off));
    }
    if (rbl == 0) {
#pragma unroll
        for (int c = 0; c < 8; c++) red[warp * DV + j0 + c] = p[c];
    }
    __syncthreads();
    for (int j = threadIdx.x; j < DV; j += G::NT) {
        float t = red[j];
#pragma unroll
        for (int w2 = 1; w2 < G::NWARPS; w2++) t = fmaxf(t, red[w2 * DV + j]);
        tot[j] = t;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 8; c++) res[c] = tot[j0 + c];
}

// Two CTAs per SM: only the updated state x stays in registers; the decayed
// state a is re-derived from the codes (an L1 hit after the first read)
// wherever a step needs it.
template <int DK, int DV, int BITS, bool GDN, bool BDR, bool BF>
__global__ void __launch_bounds__(Geo<DK, DV>::NT, 2) rc_kernel(const StepParams p) {
    using G = Geo<DK, DV>;
    static_assert(BITS == 4 || BITS == 8, "4- or 8-bit codes");
    constexpr int QMAX = (1 << (BITS - 1)) - 1;
    constexpr float fq = float(QMAX);
    constexpr float rq = QMAX == 7 ? 0x1.24924ap-3f : 0x1.020408p-7f;
    __shared__ RcShared<DK, DV> sh;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane % G::CBW, rbl = lane / G::CBW;
    const int i0 = (warp * G::RBW + rbl) * 8, j0 = cb * 8;
    const bool sf32 = p.scale_f32 != 0;
    const int isz = BF ? 2 : 4;

    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        uint8_t* ct = p.codes + tile * p.tile_bytes;
        const long long sbase = tile * (long long)(DK + DV);
        {
            const long long nt = tile + gridDim.x;
            if (nt < p.ntiles) {
                const int ssz = sf32 ? 4 : 2;
                prefetch_l2<G::NT>(p.codes + nt * p.tile_bytes, p.tile_bytes);
                prefetch_l2<G::NT>(static_cast<const uint8_t*>(p.scales) + nt * (DK + DV) * ssz,
                                   (long long)(DK + DV) * ssz);
                if (threadIdx.x < 3) {
                    const void* src = threadIdx.x == 0 ? p.q : threadIdx.x == 1 ? p.k : p.v;
                    const int n = threadIdx.x == 2 ? DV : DK;
                    const char* b = static_cast<const char*>(src) + nt * n * isz;
                    for (int o = 0; o < n * isz; o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(b + o));
                }
            }
        }
        for (int i = threadIdx.x; i < DK + DV; i += G::NT) {
            const float s = scale_at(p.scales, sbase + i, sf32);
            if (i < DK) {
                const float al = p.kind == K_RETNET ? p.gamma
                               : p.kind == K_GLA    ? ldg1(p.gates, tile * p.n_gate + i, p.gate_bf16 != 0)
                                                    : ldg1(p.gates, tile * p.n_gate, p.gate_bf16 != 0);
                sh.rho[i] = __fmul_rn(al, s);            // alpha_i * rho_i
            } else {
                sh.kap[i - DK] = s;
            }
        }
        if (threadIdx.x == 0) sh.bad = 0;
        const uint8_t* kin = static_cast<const uint8_t*>(p.k) + tile * DK * isz;
        const uint8_t* qin = static_cast<const uint8_t*>(p.q) + tile * DK * isz;
        const uint8_t* vin = static_cast<const uint8_t*>(p.v) + tile * DV * isz;
        float kk[8];
#pragma unroll
        for (int r = 0; r < 8; r++) kk[r] = ldg1(kin, i0 + r, BF);
        const float beta = GDN ? ldg1(p.gates, tile * p.n_gate + 1, p.gate_bf16 != 0) : 0.0f;
        __syncthreads();

        float kp[8];
#pragma unroll
        for (int c = 0; c < 8; c++) kp[c] = sh.kap[j0 + c];
        // a_ij = code * ((alpha_i * rho_i) * kappa_j) of row r of this thread
        auto decayed_row = [&](int r, float (&ar)[8]) {
            float c8[8];
            if constexpr (BITS == 4) Decode<4>::run(ct + (i0 + r) * (DV / 2), cb, c8);
            else Decode<8>::run(ct + (i0 + r) * DV, cb, c8);
            const float arho = sh.rho[i0 + r];
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 a2 = fmul2(f2(c8[c], c8[c + 1]), fmul2(f2(arho, arho), f2(kp[c], kp[c + 1])));
                ar[c] = a2.x;
                ar[c + 1] = a2.y;
            }
        };
        // the update
        float x[8][8];
        float e[8];
        if constexpr (GDN) {
            float2 pr[4];
#pragma unroll
            for (int c = 0; c < 4; c++) pr[c] = f2(0.0f, 0.0f);
#pragma unroll
            for (int r = 0; r < 8; r++) {
                float ar[8];
                decayed_row(r, ar);
#pragma unroll
                for (int c = 0; c < 4; c++) pr[c] = ffma2(f2(ar[2 * c], ar[2 * c + 1]), f2(kk[r], kk[r]), pr[c]);
            }
            float p8[8], rr[8];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                p8[2 * c] = pr[c].x;
                p8[2 * c + 1] = pr[c].y;
            }
            colsum_finish<DK, DV>(p8, sh.red, sh.tot, warp, rbl, j0, rr);
#pragma unroll
            for (int c = 0; c < 8; c++) e[c] = __fsub_rn(ldg1(vin, j0 + c, BF), rr[c]);
        } else {
#pragma unroll
            for (int c = 0; c < 8; c++) e[c] = ldg1(vin, j0 + c, BF);
        }
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float ar[8];
            decayed_row(r, ar);
            const float kr = GDN ? __fmul_rn(beta, kk[r]) : kk[r];
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 x2 = ffma2(f2(kr, kr), f2(e[c], e[c + 1]), f2(ar[c], ar[c + 1]));
                x[r][c] = x2.x;
                x[r][c + 1] = x2.y;
            }
        }
        // the output from the state before rounding
        bool bad = false;
        {
            float2 po[4];
#pragma unroll
            for (int c = 0; c < 4; c++) po[c] = f2(0.0f, 0.0f);
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const float qr = ldg1(qin, i0 + r, BF);
#pragma unroll
                for (int c = 0; c < 4; c++) po[c] = ffma2(f2(x[r][2 * c], x[r][2 * c + 1]), f2(qr, qr), po[c]);
            }
            float p8[8], oo[8];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                p8[2 * c] = po[c].x;
                p8[2 * c + 1] = po[c].y;
            }
            colsum_finish<DK, DV>(p8, sh.red, sh.tot, warp, rbl, j0, oo);
            if (rbl == 0 && warp == 0) {
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    p.out[tile * DV + j0 + c] = oo[c];
                    bad |= !isfinite(oo[c]);
                }
            }
        }
        // the column scales and their reciprocals
        float ik[8];
        unsigned nsat = 0;
        {
            float m[8];
#pragma unroll
            for (int c = 0; c < 8; c++) {
                float t = fmaxf(fabsf(x[0][c]), fabsf(x[1][c]));
#pragma unroll
                for (int r = 2; r < 8; r += 2) t = fmaxf(t, fmaxf(fabsf(x[r][c]), fabsf(x[r + 1][c])));
                m[c] = t;
            }
            // x * 0 is NaN exactly for a NaN or infinite x: one packed fma per
            // pair finds any non-finite element of the block
            float2 nf = f2(0.0f, 0.0f);
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int c = 0; c < 8; c += 2) nf = ffma2(f2(x[r][c], x[r][c + 1]), f2(0.0f, 0.0f), nf);
            bad |= (nf.x != nf.x) || (nf.y != nf.y);
            float cm[8];
            colmax_finish<DK, DV>(m, sh.red, sh.tot, warp, rbl, j0, cm);
#pragma unroll
            for (int c = 0; c < 8; c++) {
                bool sat = false;
                const float kap = to_stored(cm[c], sf32, sat);
                ik[c] = kap == 0.0f ? 0.0f : __frcp_rn(kap);
                if (rbl == 0 && warp == 0) {
                    store_scale(p.scales, sbase + DK + j0 + c, sf32, kap);
                    nsat += sat ? 1u : 0u;
                }
            }
        }
        // row by row: the row scale from the column-normalised magnitudes, then
        // round (BDR: a reversed element moves one code toward its update) and pack
        constexpr float lo = kMagic - fq, hi = kMagic + fq;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float t = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 y2 = fmul2(f2(fabsf(x[r][c]), fabsf(x[r][c + 1])), f2(ik[c], ik[c + 1]));
                t = fmaxf(t, fmaxf(y2.x, y2.y));
            }
#pragma unroll
            for (int off = 1; off < G::CBW; off <<= 1) t = fmaxf(t, __shfl_xor_sync(0xFFFFFFFFu, t, off));
            bool sat = false;
            const float rho = to_stored(div_by_qmax(t, fq, rq), sf32, sat);
            const float ir = rho == 0.0f ? 0.0f : __frcp_rn(rho);
            if (cb == 0) {
                store_scale(p.scales, sbase + i0 + r, sf32, rho);
                nsat += sat ? 1u : 0u;
            }
            float ar[8];
            if (BDR) decayed_row(r, ar);
            float t8[8];
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 inv2 = fmul2(f2(ir, ir), f2(ik[c], ik[c + 1]));
                const float2 x2 = f2(x[r][c], x[r][c + 1]);
                float2 t2 = ffma2(x2, inv2, f2(kMagic, kMagic));
                t2.x = fminf(fmaxf(t2.x, lo), hi);
                t2.y = fminf(fmaxf(t2.y, lo), hi);
                if (BDR) {
                    const float2 a2 = f2(ar[c], ar[c + 1]);
                    const float2 d2 = ffma2(a2, f2(-1.0f, -1.0f), x2);                  // x - a
                    const float2 cn = ffma2(t2, f2(-1.0f, -1.0f), f2(kMagic, kMagic));  // -code
                    const float2 s2 = ffma2(a2, inv2, cn);
                    t2.x = fminf(fmaxf(bdr1(t2.x, s2.x, d2.x, p.eps_b), lo), hi);
                    t2.y = fminf(fmaxf(bdr1(t2.y, s2.y, d2.y, p.eps_b), lo), hi);
                }
                t8[c] = t2.x;
                t8[c + 1] = t2.y;
            }
            pack_row<DK, DV, BITS>(ct, i0 + r, cb, t8);
        }
        if (nsat) atomicAdd(p.counters + 1, (unsigned long long)nsat);
        if (bad) sh.bad = 1;
        __syncthreads();
        if (threadIdx.x == 0 && sh.bad) atomicAdd(p.counters, 1ull);
    }
}

// Dequantized state of a row x column-scaled object: code * (rho_i * kappa_j).
template <int DK, int DV, int BITS>
__global__ void __launch_bounds__(Geo<DK, DV>::NT) rc_dequant_kernel(const StepParams p, float* S) {
    using G = Geo<DK, DV>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane % G::CBW, rbl = lane / G::CBW;
    const int i0 = (warp * G::RBW + rbl) * 8, j0 = cb * 8;
    const bool sf32 = p.scale_f32 != 0;
    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        const uint8_t* ct = p.codes + tile * p.tile_bytes;
        const long long sbase = tile * (long long)(DK + DV);
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float c8[8];
            if constexpr (BITS == 4) Decode<4>::run(ct + (i0 + r) * (DV / 2), cb, c8);
            else Decode<8>::run(ct + (i0 + r) * DV, cb, c8);
            const float rho = scale_at(p.scales, sbase + i0 + r, sf32);
#pragma unroll
            for (int c = 0; c < 8; c++) {
                const float kap = scale_at(p.scales, sbase + DK + j0 + c, sf32);
                S[(tile * DK + i0 + r) * DV + j0 + c] = __fmul_rn(c8[c], __fmul_rn(rho, kap));
            }
        }
    }
}

}  // namespace qs
