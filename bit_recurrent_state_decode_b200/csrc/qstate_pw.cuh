// qstate_pw.cuh -- the Gated DeltaNet decode step with a pure-write sliding
// window (PW) of "Low-Bit GDN Recurrent-State Quantization: Global
// Gradient-aware Allocation and Pure-Write Sliding Windows" (Abstract), for
// uniform 4- or 8-bit histories of tiles with d_k = d_v.
//
// A tile's state is its quantized history plus the W most recent pure writes
// beta k v^T, each held as a pair of FP8 E4M3 vectors (a = beta k on the key
// side, b = v).  Every step applies the transition alpha (I - beta k k^T) to
// each part: to the history as a Gated DeltaNet step without a write
// (x = a + (beta k)(-r)^T, r = a^T k), and to every pair's key side
// (a <- fp8(alpha (a - beta (a . k) k))).  When the window is full the
// oldest pair, after its transition, leaves into the history
// (x += a_old b_old^T); then the step's own pair takes its slot.  The output
// is the whole state's, o = x^T q + sum over the pairs held (oldest first)
// of (a_l . q) b_l, and the history is requantized every step with the
// object's scale and rounding rules.
//
// Arithmetic and order follow the specification element by element (the
// canonical sums, one fma per pair and element), so every result is the same
// bits as the definition.  One tile per CTA at a time, plain loads with the
// next tile's bytes prefetched to L2, like the LRB step.
#pragma once

#include <cuda_fp8.h>

#include "qstate_lrb.cuh"

namespace qs {

constexpr int kPwMaxW = 16;

struct PwParams {
    uint8_t* A;       // [tiles][W][d_k] E4M3: the pairs' key sides, by slot
    uint8_t* B;       // [tiles][W][d_v] E4M3: the pairs' value sides
    int* head;        // [tiles]: slot of the oldest pair
    int* count;       // [tiles]: pairs held
    int W;
};

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
    return __half2float(__half(__nv_cvt_fp8_to_halfraw(b, __NV_E4M3)));
}
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
    return __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

template <int DK, int DV>
struct __align__(16) PwShared {
    using G = Geo<DK, DV>;
    Xchg<DK, DV, false> xs;
    float red[G::NWARPS * DV];
    float tot[DV];
    float cq[kPwMaxW];               // (a_l . q) of the pairs held after the step, by age
    __align__(16) uint8_t sprev[DK * (DV / 8) * 4];
    __align__(16) uint8_t sa[kPwMaxW * DK];    // key sides by slot (propagated in place)
    __align__(16) uint8_t sb[kPwMaxW * DV];    // value sides by slot
};

// Two CTAs per SM: the decayed history a is re-derived from the codes (an L1
// hit after the first read) wherever the step needs it.
template <int DK, int DV, int BITS, bool BDR, bool BF>
__global__ void __launch_bounds__(Geo<DK, DV>::NT, 2) pw_kernel(const StepParams p, const PwParams P) {
    using G = Geo<DK, DV>;
    static_assert(DK == DV, "square tiles");
    static_assert(BITS == 4 || BITS == 8, "4- or 8-bit codes");
    __shared__ PwShared<DK, DV> sh;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane % G::CBW, rbl = lane / G::CBW;
    const int i0 = (warp * G::RBW + rbl) * 8, j0 = cb * 8;
    const int W = P.W;
    const bool sf32 = p.scale_f32 != 0;
    const int group = p.group;
    const int gsh = group ? __ffs(group) - 1 : 0;
    const int ng = group ? DV >> gsh : 1;
    const int gcol = group ? j0 >> gsh : 0;

    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        const int h = P.head[tile], n = P.count[tile];
        uint8_t* ct = p.codes + tile * p.tile_bytes;
        uint8_t* At = P.A + tile * (long long)W * DK;
        uint8_t* Bt = P.B + tile * (long long)W * DV;
        const long long sbase = tile * (long long)p.n_scales;
        const float alpha = ldg1(p.gates, tile * p.n_gate, p.gate_bf16 != 0);
        const float beta = ldg1(p.gates, tile * p.n_gate + 1, p.gate_bf16 != 0);

        // the next tile's bytes on their way to L2 while this one is stepped
        {
            const long long nt = tile + gridDim.x;
            if (nt < p.ntiles) {
                const int ssz = sf32 ? 4 : 2;
                const int isz = BF ? 2 : 4;
                prefetch_l2<G::NT>(p.codes + nt * p.tile_bytes, p.tile_bytes);
                prefetch_l2<G::NT>(static_cast<const uint8_t*>(p.scales) + nt * p.n_scales * ssz,
                                   (long long)p.n_scales * ssz);
                prefetch_l2<G::NT>(P.A + nt * (long long)W * DK, (long long)W * DK);
                prefetch_l2<G::NT>(P.B + nt * (long long)W * DV, (long long)W * DV);
                if (threadIdx.x == 0) {
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.q) + nt * DK * isz));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.k) + nt * DK * isz));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.v) + nt * DV * isz));
                }
            }
        }
        // the tile's previous scales and its pairs (16-byte loads where every
        // region starts on a 16-byte boundary and holds a multiple of 16 bytes)
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
            for (int i = threadIdx.x; i < W * DK / 16; i += G::NT)
                reinterpret_cast<uint4*>(sh.sa)[i] = reinterpret_cast<const uint4*>(At)[i];
            for (int i = threadIdx.x; i < W * DV / 16; i += G::NT)
                reinterpret_cast<uint4*>(sh.sb)[i] = reinterpret_cast<const uint4*>(Bt)[i];
        }
        auto prev_scale = [&](int idx) -> float {
            if (sf32) return reinterpret_cast<const float*>(sh.sprev)[idx];
            return __half2float(reinterpret_cast<const __half*>(sh.sprev)[idx]);
        };
        const uint8_t* kin = static_cast<const uint8_t*>(p.k) + tile * DK * (BF ? 2 : 4);
        const uint8_t* qin = static_cast<const uint8_t*>(p.q) + tile * DK * (BF ? 2 : 4);
        auto kval = [&](int i) { return ldg1(kin, i, BF); };
        auto qval = [&](int i) { return ldg1(qin, i, BF); };
        __syncthreads();

        // the pairs' key sides through the transition, one warp per pair
        for (int l = warp; l < n; l += G::NWARPS) {
            uint8_t* a8 = sh.sa + ((h + l) % W) * DK;
            auto aval = [&](int i) { return e4m3_to_f32(a8[i]); };
            const float s = warp_canon_dot<DK>(aval, kval, lane);
            const float cs = __fmul_rn(beta, s);
            float na[DK / 32];
#pragma unroll
            for (int u = 0; u < DK / 32; u++) {
                const int i = lane + 32 * u;
                na[u] = __fmul_rn(alpha, __fmaf_rn(-cs, kval(i), aval(i)));
            }
            __syncwarp();
#pragma unroll
            for (int u = 0; u < DK / 32; u++) a8[lane + 32 * u] = f32_to_e4m3(na[u]);
        }

        // the history: a = code * (alpha * scale), r = a^T k, x = a + (beta k)(-r)^T
        float kk[8], qq[8], eta[8];
#pragma unroll
        for (int r = 0; r < 8; r++) {
            kk[r] = kval(i0 + r);
            qq[r] = qval(i0 + r);
            eta[r] = __fmul_rn(alpha, prev_scale(group ? (i0 + r) * ng + gcol : 0));
        }
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
        float x[8][8];
        {
            float2 pr[4];
#pragma unroll
            for (int c = 0; c < 4; c++) pr[c] = f2(0.0f, 0.0f);
#pragma unroll
            for (int r = 0; r < 8; r++) {
                float ar[8];
                arow(r, ar);
#pragma unroll
                for (int c = 0; c < 4; c++) pr[c] = ffma2(f2(ar[2 * c], ar[2 * c + 1]), f2(kk[r], kk[r]), pr[c]);
            }
            float p8[8], rr[8];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                p8[2 * c] = pr[c].x;
                p8[2 * c + 1] = pr[c].y;
            }
            colsum_finish<DK, DV>(p8, sh.red, sh.tot, warp, rbl, j0, rr);    // syncs: pairs propagated
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const float kap = __fmul_rn(beta, kk[r]);
                float ar[8];
                arow(r, ar);
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 x2 = ffma2(f2(kap, kap), f2(-rr[c], -rr[c + 1]), f2(ar[c], ar[c + 1]));
                    x[r][c] = x2.x;
                    x[r][c + 1] = x2.y;
                }
            }
        }
        // the oldest pair leaves a full window into the history
        const bool full = n == W;
        const int slot = full ? h : (h + n) % W;       // the step's own pair
        const int h2 = full ? (h + 1 == W ? 0 : h + 1) : h;
        const int n2 = full ? n : n + 1;
        if (full) {
            const uint8_t* a8 = sh.sa + h * DK;
            const uint8_t* b8 = sh.sb + h * DV;
            float bo[8];
#pragma unroll
            for (int c = 0; c < 8; c++) bo[c] = e4m3_to_f32(b8[j0 + c]);
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const float ao = e4m3_to_f32(a8[i0 + r]);
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 x2 = ffma2(f2(ao, ao), f2(bo[c], bo[c + 1]), f2(x[r][c], x[r][c + 1]));
                    x[r][c] = x2.x;
                    x[r][c + 1] = x2.y;
                }
            }
        }
        __syncthreads();                                   // the leaver is read
        for (int i = threadIdx.x; i < DK; i += G::NT) sh.sa[slot * DK + i] = f32_to_e4m3(__fmul_rn(beta, kval(i)));
        {
            const uint8_t* vin = static_cast<const uint8_t*>(p.v) + tile * DV * (BF ? 2 : 4);
            for (int j = threadIdx.x; j < DV; j += G::NT) sh.sb[slot * DV + j] = f32_to_e4m3(ldg1(vin, j, BF));
        }
        __syncthreads();
        // (a_l . q) of the pairs held, by age
        for (int l = warp; l < n2; l += G::NWARPS) {
            const uint8_t* a8 = sh.sa + ((h2 + l) % W) * DK;
            auto aval = [&](int i) { return e4m3_to_f32(a8[i]); };
            const float d = warp_canon_dot<DK>(aval, qval, lane);
            if (lane == 0) sh.cq[l] = d;
        }

        // the output: o = x^T q, then the pairs oldest first
        {
            float2 po2[4];
#pragma unroll
            for (int c = 0; c < 4; c++) po2[c] = f2(0.0f, 0.0f);
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int c = 0; c < 4; c++)
                    po2[c] = ffma2(f2(x[r][2 * c], x[r][2 * c + 1]), f2(qq[r], qq[r]), po2[c]);
            float po[8], oo[8];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                po[2 * c] = po2[c].x;
                po[2 * c + 1] = po2[c].y;
            }
            colsum_finish<DK, DV>(po, sh.red, sh.tot, warp, rbl, j0, oo);    // syncs: cq visible
            for (int l = 0; l < n2; l++) {
                const uint8_t* b8 = sh.sb + ((h2 + l) % W) * DV;
                const float cl = sh.cq[l];
#pragma unroll
                for (int c = 0; c < 8; c++) oo[c] = __fmaf_rn(cl, e4m3_to_f32(b8[j0 + c]), oo[c]);
            }
            if (rbl == 0 && warp == 0) {
#pragma unroll
                for (int c = 0; c < 8; c++) p.out[tile * DV + j0 + c] = oo[c];
            }
        }

        // the window back to HBM: every key side held, the new value side
        for (int l = threadIdx.x; l < n2 * (DK / 16); l += G::NT) {
            const int sl = (h2 + l / (DK / 16)) % W, part = l % (DK / 16);
            reinterpret_cast<uint4*>(At + sl * DK)[part] = reinterpret_cast<const uint4*>(sh.sa + sl * DK)[part];
        }
        for (int part = threadIdx.x; part < DV / 16; part += G::NT)
            reinterpret_cast<uint4*>(Bt + slot * DV)[part] = reinterpret_cast<const uint4*>(sh.sb + slot * DV)[part];
        if (threadIdx.x == 0) {
            P.head[tile] = h2;
            P.count[tile] = n2;
        }

        // the history requantized
        requantize<DK, DV, BITS, BDR>(p, sh.xs, sh.sprev, sbase, ct, arow, x, lane, warp, cb, i0, ng,
                                      gcol);
        __syncthreads();
    }
}

}  // namespace qs
