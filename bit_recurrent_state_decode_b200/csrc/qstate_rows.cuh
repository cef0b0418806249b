// qstate_rows.cuh -- a lean step kernel for rank-1 updates (RetNet, Mamba2,
// GLA) with round-to-nearest, one code width, no reference state and scale
// groups of 32 or 64 columns of a row, on tiles with d_v = 128.  Same
// arithmetic, order and results as step_kernel (include/qstate.h); a
// different work decomposition.
//
// Each thread owns 16 consecutive rows (two canonical row blocks of 8) x 8
// consecutive columns, so a tile takes d_k / 32 warps instead of d_k / 16 and
// the per-tile work of a thread (inputs, reductions, pipeline) is spread over
// twice the elements.  The rows are processed in two batches of 8.  A scale
// group is one row's 32 or 64 columns, held by 4 or 8 lanes of one warp: its
// maximum is reduced with shuffles inside the warp, so a batch is decayed,
// updated, scaled, rounded and stored without a CTA barrier.  The only CTA
// barrier of a tile joins the output partials of the warps; it also votes on
// the tile's input stage and is where that stage is refilled.
#pragma once

#include "qstate_kernel.cuh"

namespace qs {

template <int DK>
struct RowsGeo {
    static constexpr int DV = 128;
    static constexpr int NW = DK / 32;     // warps per tile: 32 rows each
    static constexpr int NT = 32 * NW;
    static_assert(DK == 64 || DK == 128, "d_k must be 64 or 128");
};

template <int DK>
struct __align__(16) RowsXchg {
    float red_o[RowsGeo<DK>::NW * 128];    // output partial of each warp
};

// Group maxima of 8 rows over the L consecutive lanes of a group (lp = lane's
// index in the group): a reduce-scatter, after which lane lp holds the group
// maxima of rows lp*(8/L) .. lp*(8/L) + 8/L - 1 in m[0 .. 8/L - 1].  At each
// level a lane keeps one half of its rows and sends the other half to the
// partner lane (distance o), which keeps the other half.
template <int L>
__device__ __forceinline__ void group_max_scatter(float (&m)[8], int lp) {
    static_assert(L == 1 || L == 2 || L == 4 || L == 8, "2^k lanes per group, at most 8");
    int n = 8;
#pragma unroll
    for (int o = L / 2; o >= 1; o >>= 1) {
        const bool hi = (lp & o) != 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if (j < n / 2) {
                const float keep = hi ? m[j + n / 2] : m[j];
                const float send = hi ? m[j] : m[j + n / 2];
                m[j] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, o));
            }
        }
        n >>= 1;
    }
}

// L: lanes per scale group (group = 8 L columns).  VEC: the decay is a
// per-row vector (GLA), else a scalar (RetNet gamma, Mamba2 alpha).  BF: q, k,
// v are bf16.
template <int DK, int BITS, int L, bool VEC, bool BF>
__global__ void __launch_bounds__(RowsGeo<DK>::NT, 4) rows_kernel(const StepParams p) {
    using RG = RowsGeo<DK>;
    constexpr int DV = RG::DV, NW = RG::NW, NT = RG::NT;
    constexpr int G = 8 * L, NG = DV / G, NV = 8 / L;
    constexpr int QMAX = (1 << (BITS - 1)) - 1;
    constexpr float fq = float(QMAX);
    constexpr float rq = QMAX == 7 ? 0x1.24924ap-3f : QMAX == 31 ? 0x1.08421p-5f
                       : QMAX == 127 ? 0x1.020408p-7f : 1.0f;
    constexpr int isz = BF ? 2 : 4;
    static_assert(BITS == 4 || BITS == 8, "4- or 8-bit codes");

    extern __shared__ __align__(128) uint8_t dsmem[];
    __shared__ RowsXchg<DK> xch[2];
    __shared__ __align__(8) uint64_t bars[kMaxStages];
    // non-finite flag of each tile, by tile index mod 4: tile t sets its slot
    // before and after its barrier, and thread 0 clears the slot of tile t - 1
    // right after the barrier of tile t, while tile t + 1 may already set its own
    __shared__ volatile int badf[4];
    const int S = p.nstages;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane & 15, rh = lane >> 4;
    const int j0 = cb * 8, i0 = warp * 32 + rh * 16;
    const int lp = cb % L, gbase = lane - lp, gcol = j0 / G;
    const bool sf32 = p.scale_f32 != 0;
    const bool persistent = p.scale_mode == M_PERSISTENT;
    const bool gate_bf = p.gate_bf16 != 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) mbar_init(&bars[s], 1);
        fence_barrier_init();
        badf[0] = badf[1] = badf[2] = badf[3] = 0;
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            const long long t = blockIdx.x + (long long)s * gridDim.x;
            if (t < p.ntiles) issue_tile<DK, DV, false>(p, t, dsmem + s * p.stage_bytes, &bars[s]);
        }
    }
    float g0, g1, pts;
    load_scalars(p, blockIdx.x, g0, g1, pts);

    auto prev_scale = [&](const uint8_t* st, int row) -> float {
        if (sf32) return reinterpret_cast<const float*>(st + p.off_scales)[row * NG + gcol];
        return __half2float(reinterpret_cast<const __half*>(st + p.off_scales)[row * NG + gcol]);
    };

    int it = 0, s = 0;
    uint32_t parity = 0;
    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, it++) {
        float n0, n1, nts;
        load_scalars(p, tile + gridDim.x, n0, n1, nts);
        const bool ok = mbar_wait_bounded(&bars[s], parity, p.wait_polls);
        const uint8_t* st = dsmem + s * p.stage_bytes;
        uint8_t* ct = p.codes + tile * p.tile_bytes;
        auto& xs = xch[it & 1];
        const long long sbase = tile * (long long)p.n_scales;

        // A warp whose stage did not arrive (for any lane) writes nothing of
        // the tile; the CTA vote below then gives the tile up.
        if (__all_sync(0xFFFFFFFFu, ok)) {
            float vv[8];
            ld8(st + p.off_v + j0 * isz, BF, vv);
            const float salpha = p.kind == K_RETNET ? p.gamma : g0;
            bool bad = false;
            unsigned nsat = 0;
            float po[8];
#pragma unroll
            for (int c = 0; c < 8; c++) po[c] = 0.0f;
#pragma unroll
            for (int b = 0; b < 2; b++) {
                const int ib = i0 + 8 * b;         // first row of the batch (a canonical block)
                float x[8][8], m[8], pb[8];
#pragma unroll
                for (int c = 0; c < 8; c++) pb[c] = 0.0f;
                // the batch's 8 rows of k, q and (GLA) alpha: one vector load each
                float kk[8], qq[8], al[8];
                ld8(st + p.off_k + ib * isz, BF, kk);
                ld8(st + p.off_q + ib * isz, BF, qq);
                if constexpr (VEC) {
                    ld8(st + p.off_ga + ib * (gate_bf ? 2 : 4), gate_bf, al);
                } else {
#pragma unroll
                    for (int r = 0; r < 8; r++) al[r] = salpha;
                }
                // decay, update, the block's output sums and the row maxima
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    const int row = ib + r;
                    const float kr = kk[r], qr = qq[r];
                    const float eta = __fmul_rn(al[r], prev_scale(st, row));
                    float c8[8];
                    if constexpr (BITS == 4) Decode<4>::run(st + p.off_codes + row * (DV / 2), cb, c8);
                    else Decode<8>::run(st + p.off_codes + row * DV, cb, c8);
                    float mx = 0.0f;
#pragma unroll
                    for (int c = 0; c < 8; c += 2) {
                        const float2 a2 = fmul2(f2(c8[c], c8[c + 1]), f2(eta, eta));
                        const float2 x2 = ffma2(f2(kr, kr), f2(vv[c], vv[c + 1]), a2);
                        const float2 o2 = ffma2(x2, f2(qr, qr), f2(pb[c], pb[c + 1]));
                        pb[c] = o2.x;
                        pb[c + 1] = o2.y;
                        mx = fmaxf(fmaxf(mx, fabsf(x2.x)), fabsf(x2.y));
                        x[r][c] = x2.x;
                        x[r][c + 1] = x2.y;
                    }
                    m[r] = mx;
                }
                // the thread's two row blocks, adjacent: the first level of the tree
#pragma unroll
                for (int c = 0; c < 8; c++) po[c] = b == 0 ? pb[c] : __fadd_rn(po[c], pb[c]);

                // scales: group maxima inside the warp, each lane derives NV rows
                float mg[8];
#pragma unroll
                for (int r = 0; r < 8; r++) mg[r] = m[r];
                group_max_scatter<L>(mg, lp);
                float invo[NV];
#pragma unroll
                for (int k = 0; k < NV; k++) {
                    const int row = ib + lp * NV + k;
                    const float dp = prev_scale(st, row);
                    bool sat = false;
                    float d;
                    if (persistent && !(mg[k] > __fmul_rn(fq, dp))) d = dp;
                    else d = to_stored(div_by_qmax(mg[k], fq, rq), sf32, sat);
                    invo[k] = d == 0.0f ? 0.0f : __frcp_rn(d);
                    bad |= !isfinite(mg[k]);
                    nsat += sat ? 1u : 0u;
                    store_scale(p.scales, sbase + (long long)row * NG + gcol, sf32, d);
                }
                float inv[8];
#pragma unroll
                for (int r = 0; r < 8; r++)
                    inv[r] = __shfl_sync(0xFFFFFFFFu, invo[r % NV], gbase + r / NV);

                // round and repack: the fast form needs every |x * inv| below Qmax + 1/2
                bool slow = false;
#pragma unroll
                for (int r = 0; r < 8; r++) slow |= !(__fmaf_rn(m[r], inv[r], -(fq + 0.5f)) < 0.0f);
                if (__any_sync(0xFFFFFFFFu, slow)) {
                    if (lane == 0) atomicAdd(p.counters + 3, 1ull);
                    auto no_row = [](int) { return 0.0f; };
                    round_pack_exact<DK, DV, BITS, false>(x, no_row, vv, inv, 0.0f, ct, ib, cb);
                } else {
#pragma unroll
                    for (int r = 0; r < 8; r++) {
                        float t8[8];
#pragma unroll
                        for (int c = 0; c < 8; c += 2) {
                            const float2 t2 = rtn2(f2(x[r][c], x[r][c + 1]), inv[r]);
                            t8[c] = t2.x;
                            t8[c + 1] = t2.y;
                        }
                        pack_row<DK, DV, BITS>(ct, ib + r, cb, t8);
                    }
                }
            }
            if (nsat) atomicAdd(p.counters + 1, (unsigned long long)nsat);
            if (bad) badf[it & 3] = 1;
            // the two row halves of the warp (adjacent 16-row sums), then the
            // warp's partial to shared memory
#pragma unroll
            for (int c = 0; c < 8; c++) po[c] = __fadd_rn(po[c], __shfl_xor_sync(0xFFFFFFFFu, po[c], 16));
            if (rh == 0) {
                float4* r4 = reinterpret_cast<float4*>(xs.red_o + warp * DV + j0);
                r4[0] = make_float4(po[0], po[1], po[2], po[3]);
                r4[1] = make_float4(po[4], po[5], po[6], po[7]);
            }
        }

        // the tile's barrier: votes on the stage; every thread is done with it
        if (!__syncthreads_and(ok)) {
            if (threadIdx.x == 0) {
                atomicAdd(p.counters + 2, 1ull);
                // this tile's stage and the S - 1 ahead of it may be in flight
                for (int k = 0; k < S; k++) {
                    const long long t2 = tile + (long long)k * gridDim.x;
                    if (t2 < p.ntiles)
                        (void)mbar_wait_bounded(&bars[(it + k) % S], ((it + k) / S) & 1, p.wait_polls);
                }
            }
            return;
        }
        if (threadIdx.x == 0) {
            // the previous tile's non-finite flag is complete (its outputs were
            // checked before this barrier)
            if (it > 0 && badf[(it - 1) & 3]) {
                badf[(it - 1) & 3] = 0;
                atomicAdd(p.counters, 1ull);
            }
            const long long nt = tile + (long long)S * gridDim.x;
            if (nt < p.ntiles) issue_tile<DK, DV, false>(p, nt, dsmem + s * p.stage_bytes, &bars[s]);
        }
        // output sums over the warps in row order (the rest of the tree)
        for (int j = threadIdx.x; j < DV; j += NT) {
            float t[NW];
#pragma unroll
            for (int w2 = 0; w2 < NW; w2++) t[w2] = xs.red_o[w2 * DV + j];
#pragma unroll
            for (int n = NW; n > 1; n >>= 1) {
#pragma unroll
                for (int u = 0; u < n / 2; u++) t[u] = __fadd_rn(t[2 * u], t[2 * u + 1]);
            }
            p.out[tile * DV + j] = t[0];
            if (!isfinite(t[0])) badf[it & 3] = 1;
        }
        g0 = n0;
        g1 = n1;
        pts = nts;
        if (++s == S) {
            s = 0;
            parity ^= 1u;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && it > 0 && badf[(it - 1) & 3]) atomicAdd(p.counters, 1ull);
}

}  // namespace qs
