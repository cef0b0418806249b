// qstate_kernel.cuh -- sm_100a kernels of the fused quantized recurrent-state
// decode step.  The arithmetic and its order are specified in include/qstate.h
// (recurrence: "Preserving Updates in Low-Bit Recurrent State Quantization",
// Table 1; scale modes: "When Dynamic Scaling Fails", Abstract; BDR: the
// Abstract and Figure 4 of the first page).
//
// Work decomposition.  Persistent CTAs (grid = SMs x resident CTAs) walk the
// (layer, batch, head) tiles with a grid stride, one tile per CTA at a time.
// Each CTA runs an NSTAGE-deep pipeline: one elected thread issues 1-D bulk
// copies (the TMA engine, cp.async.bulk) of a tile's packed codes, scales,
// q / k / v, GLA gate vector and yoked reference state into a shared-memory
// stage, completing on an mbarrier; the CTA computes the tile from shared
// memory and writes the new codes, scales and output straight to global
// memory.  Every wait on an mbarrier is bounded: on expiry the kernel counts a
// pipeline timeout, drains its own copies (again bounded) and returns.  A tile
// has one CTA barrier, the exchange of output partials and maxima (Gated
// DeltaNet adds one at the top and two for its column sums); the stage of the
// previous tile is refilled right after it.
//
// Each thread owns an 8 x 8 block of the tile: 8 consecutive rows (one row
// block of the canonical reduction) and 8 consecutive columns.  A warp covers
// all d_v columns of 32/(d_v/8) row blocks, so
//   - the column sums r_j, o_j are an in-thread fma chain over the block (the
//     canonical block sum), then a pairwise tree over the row blocks in row
//     order: an xor butterfly across the warp's row blocks and shared memory
//     across warps (d_v = 128), or shared memory for all of it (d_v = 64);
//   - the group maxima along d_v are an in-thread max; the per-row maxima of
//     every 8-column block go through shared memory with the output partials,
//     and each lane of a group derives the scales of 8/L of its rows and
//     broadcasts their reciprocals with shuffles.
// Element arithmetic is branch-free and uses the packed fp32x2 instructions
// of sm_100 (each lane of a pair rounds exactly as the scalar instruction).
// Codes are decoded with exponent-bias tricks (a field placed in the
// significand of 2^23 is an exact float, no int->float conversion) and
// rounded with one fma against 1.5 * 2^23 (the exact product x * inv rounded
// half to even).  No tensor cores: per tile the step is a rank-1 update and
// two matrix-vector products with no reuse.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include <type_traits>

namespace qs {

enum { K_RETNET = 0, K_MAMBA2 = 1, K_GLA = 2, K_GDN = 3 };
enum { M_DYNAMIC = 0, M_PERSISTENT = 1, M_YOKED = 2 };

constexpr int kMaxStages = 4;
// Default number of try_wait polls before a wait is declared lost (each poll
// may suspend the thread for a hardware-defined interval; this bound is
// several seconds).
constexpr uint32_t kWaitPolls = 1u << 24;

struct StepParams {
    uint8_t* codes;                 // packed codes, or the fp32 state (32-bit tiles)
    void* scales;                   // [tiles][n_scales] binary16 or binary32
    float* ref;                     // yoked reference state [tiles][d_k][d_v]
    const void* q;
    const void* k;
    const void* v;
    const void* gates;
    float* out;
    unsigned long long* counters;   // [0] non-finite tile-steps, [1] saturated scales,
                                    // [2] pipeline wait timeouts; with the taxonomy on,
                                    // [3] warp-tiles that took the element-wise rounding
                                    // path, [4..6] lost / moved / reversed elements, [7]
                                    // BDR steps applied
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
    int scalars;                    // SC_* flags: per-tile scalars the step reads
    float gamma, eps_b;
    // pipeline stage layout (byte offsets inside one stage; -1 = not staged)
    int nstages, stage_bytes;
    int off_codes, off_scales, off_q, off_k, off_v, off_ga, off_ref;
    // bounded waits: polls per wait; fault injection: tiles >= drop_from are
    // never copied (their waits run out), -1 = off
    unsigned wait_polls;
    long long drop_from;
    // 1: the tile bodies that assume every stored code is within +-Qmax may
    // run (0 for the first step after an import, which may hold -2^(b-1))
    int fast;
    // 1: classify every element of every tile-step (lost / moved / reversed)
    // into counters[4..7]; 0: nothing is computed
    int taxonomy;
    // 1: the state is kept rotated by the Hadamard matrix along d_v (the step
    // takes H v for v and emits H o_rot / d_v); 0: none
    int rotate;
    // with the taxonomy on: [tiles][d_k], per key row the squared rounding
    // error of the step, sum_j (S_hat_new - x)^2; null: not kept
    float* err_rows;
};

constexpr int kNumCounters = 8;

// per-tile scalar inputs read with plain loads: alpha (Mamba2, GDN), beta
// (GDN), and the previous scale of a per-token quantized state
enum { SC_G0 = 1, SC_G1 = 2, SC_PTS = 4 };

template <int DK, int DV>
struct Geo {
    static constexpr int CBW = DV / 8;          // column blocks per row (lanes per row)
    static constexpr int RBW = 32 / CBW;        // row blocks per warp
    static constexpr int NWARPS = DK / (8 * RBW);
    static constexpr int NT = 32 * NWARPS;
    static_assert(CBW * RBW == 32, "d_v must be 64 or 128");
    static_assert(NWARPS >= 1 && (NWARPS & (NWARPS - 1)) == 0, "warps must be a power of two");
};

constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23: integers in [2^23, 2^24)
constexpr uint32_t kMagicBits = 0x4B400000u;

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch.  A step launched with programmatic stream
// serialization may be scheduled while the previous kernel of its stream is
// still running; griddepcontrol.wait returns once that kernel has completed
// and its writes are visible (at once in a launch without the attribute), so
// every global access of the step comes after it.  launch_dependents lets the
// next such launch be scheduled onto SMs this grid no longer fills.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_addr(bar)), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> shared, completing `bytes` of transaction on bar.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity; false if it never came.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t polls) {
    for (uint32_t i = 0; i < polls; i++)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// ------------------------------------------------------------------ small loads
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

// 8 consecutive values at byte address p (16-byte aligned), f32 or bf16.
__device__ __forceinline__ void ld8(const uint8_t* p, bool bf16, float (&o)[8]) {
    if (bf16) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        bf16x2_to_f32(u.x, o[0], o[1]);
        bf16x2_to_f32(u.y, o[2], o[3]);
        bf16x2_to_f32(u.z, o[4], o[5]);
        bf16x2_to_f32(u.w, o[6], o[7]);
    } else {
        const float4 a = reinterpret_cast<const float4*>(p)[0];
        const float4 b = reinterpret_cast<const float4*>(p)[1];
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
}

__device__ __forceinline__ float ldg1(const void* base, long long idx, bool bf16) {
    if (bf16) return __uint_as_float(uint32_t(__ldg(static_cast<const uint16_t*>(base) + idx)) << 16);
    return __ldg(static_cast<const float*>(base) + idx);
}

__device__ __forceinline__ float scale_at(const void* base, long long idx, bool f32) {
    if (f32) return static_cast<const float*>(base)[idx];
    return __half2float(static_cast<const __half*>(base)[idx]);
}

// Convert a scale to its stored precision; returns the stored value widened.
__device__ __forceinline__ float to_stored(float v, bool f32, bool& saturated) {
    if (f32) return v;
    const __half h = __float2half_rn(v);
    saturated = __hisinf(h);
    return saturated ? 65504.0f : __half2float(h);
}

__device__ __forceinline__ void store_scale(void* base, long long idx, bool f32, float v) {
    if (f32) static_cast<float*>(base)[idx] = v;
    else static_cast<__half*>(base)[idx] = __float2half_rn(v);   // exact: v is a binary16 value
}

// ------------------------------------------------------------------ float2 math
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// ------------------------------------------------------------------ code decode
// Exact float code values c[8] of one thread's 8 codes of a row.  A code with
// its sign bit flipped is an unsigned field u = code + 2^(b-1); placed in the
// low byte of the float 2^23 (byte permute) it gives 2^23 + u exactly, and one
// add removes the bias.  Narrow fields that do not sit in bytes of their own
// are masked into place and XORed with 0x4B000000 plus their sign bit instead,
// giving 2^23 + u * 2^pos; one fma then scales by 2^-pos and removes the bias.
template <int BITS>
struct Decode;

template <>
struct Decode<4> {
    // byte m holds codes 2m (low nibble) and 2m+1 (high nibble): the two
    // nibble planes are split into bytes of their own
    static __device__ __forceinline__ void run(const uint8_t* row, int cb, float (&c)[8]) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(row + cb * 4) ^ 0x88888888u;
        const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
        const float2 z = f2(-8388616.0f, -8388616.0f);   // -(2^23 + 8)
        const float2 r01 = fadd2(f2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540)),
                                    __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540))), z);
        const float2 r23 = fadd2(f2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7541)),
                                    __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7541))), z);
        const float2 r45 = fadd2(f2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7542)),
                                    __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7542))), z);
        const float2 r67 = fadd2(f2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7543)),
                                    __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7543))), z);
        c[0] = r01.x; c[1] = r01.y; c[2] = r23.x; c[3] = r23.y;
        c[4] = r45.x; c[5] = r45.y; c[6] = r67.x; c[7] = r67.y;
    }
};

template <>
struct Decode<8> {
    // each byte (sign bit flipped) is permuted into the low byte of the float
    // 2^23, giving 2^23 + code + 128 exactly; one add removes the bias
    static __device__ __forceinline__ void run(const uint8_t* row, int cb, float (&c)[8]) {
        const uint2 w = *reinterpret_cast<const uint2*>(row + cb * 8);
        const uint32_t x = w.x ^ 0x80808080u, y = w.y ^ 0x80808080u;
        const float2 z = f2(-8388736.0f, -8388736.0f);   // -(2^23 + 128)
        const float2 r01 = fadd2(f2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540)),
                                    __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7541))), z);
        const float2 r23 = fadd2(f2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7542)),
                                    __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7543))), z);
        const float2 r45 = fadd2(f2(__uint_as_float(__byte_perm(y, 0x4B000000u, 0x7540)),
                                    __uint_as_float(__byte_perm(y, 0x4B000000u, 0x7541))), z);
        const float2 r67 = fadd2(f2(__uint_as_float(__byte_perm(y, 0x4B000000u, 0x7542)),
                                    __uint_as_float(__byte_perm(y, 0x4B000000u, 0x7543))), z);
        c[0] = r01.x; c[1] = r01.y; c[2] = r23.x; c[3] = r23.y;
        c[4] = r45.x; c[5] = r45.y; c[6] = r67.x; c[7] = r67.y;
    }
};

template <>
struct Decode<2> {
    static __device__ __forceinline__ void run(const uint8_t* row, int cb, float (&c)[8]) {
        const uint32_t w = *reinterpret_cast<const uint16_t*>(row + cb * 2);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float fa = __uint_as_float((w & (3u << (2 * e))) ^ (0x4B000000u | (2u << (2 * e))));
            const float fb = __uint_as_float((w & (3u << (2 * e + 2))) ^ (0x4B000000u | (2u << (2 * e + 2))));
            const float sa = __uint_as_float((127u - 2u * e) << 23);        // 4^-e
            const float sb = __uint_as_float((127u - 2u * e - 2u) << 23);   // 4^-(e+1)
            const float za = -(__uint_as_float((150u - 2u * e) << 23) + 2.0f);       // -(2^(23-2e) + 2)
            const float zb = -(__uint_as_float((150u - 2u * e - 2u) << 23) + 2.0f);
            const float2 r = ffma2(f2(fa, fb), f2(sa, sb), f2(za, zb));
            c[e] = r.x;
            c[e + 1] = r.y;
        }
    }
};

// 6-bit codes: a low-nibble plane (unsigned nibble u) and a high 2-bit plane
// (signed s); code = u + 16 s.
template <int DK, int DV>
struct Decode6 {
    static __device__ __forceinline__ void run(const uint8_t* tile, int i, int cb, float (&c)[8]) {
        const uint32_t wl = *reinterpret_cast<const uint32_t*>(tile + i * (DV / 2) + cb * 4);
        const uint32_t wh = *reinterpret_cast<const uint16_t*>(tile + DK * DV / 2 + i * (DV / 4) + cb * 2);
#pragma unroll
        for (int e = 0; e < 8; e++) {
            const uint32_t u = (wl >> (4 * e)) & 15u;
            const float fh = __uint_as_float((wh & (3u << (2 * e))) ^ (0x4B000000u | (2u << (2 * e))));
            const float sh = __fmaf_rn(fh, __uint_as_float((127u - 2u * e) << 23),
                                       -(__uint_as_float((150u - 2u * e) << 23) + 2.0f));
            c[e] = __fmaf_rn(sh, 16.0f, float(u));
        }
    }
};

// ------------------------------------------------------------------ code pack
// t[e] = 1.5 * 2^23 + code (exact): the low bits of its pattern are the code's
// two's complement.
template <int BITS>
struct Pack;

template <>
struct Pack<4> {
    // the low bytes of the even codes and of the odd codes are gathered into
    // one word each; byte m = low nibble of code 2m | low nibble of code 2m+1 << 4
    static __device__ __forceinline__ void run(uint8_t* row, int cb, const float (&t)[8]) {
        const uint32_t e01 = __byte_perm(__float_as_uint(t[0]), __float_as_uint(t[2]), 0x0040);
        const uint32_t e23 = __byte_perm(__float_as_uint(t[4]), __float_as_uint(t[6]), 0x0040);
        const uint32_t o01 = __byte_perm(__float_as_uint(t[1]), __float_as_uint(t[3]), 0x0040);
        const uint32_t o23 = __byte_perm(__float_as_uint(t[5]), __float_as_uint(t[7]), 0x0040);
        const uint32_t ev = __byte_perm(e01, e23, 0x5410), od = __byte_perm(o01, o23, 0x5410);
        *reinterpret_cast<uint32_t*>(row + cb * 4) = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
    }
};

template <>
struct Pack<8> {
    static __device__ __forceinline__ void run(uint8_t* row, int cb, const float (&t)[8]) {
        const uint32_t a = __byte_perm(__float_as_uint(t[0]), __float_as_uint(t[1]), 0x0040);
        const uint32_t b = __byte_perm(__float_as_uint(t[2]), __float_as_uint(t[3]), 0x0040);
        const uint32_t c = __byte_perm(__float_as_uint(t[4]), __float_as_uint(t[5]), 0x0040);
        const uint32_t d = __byte_perm(__float_as_uint(t[6]), __float_as_uint(t[7]), 0x0040);
        *reinterpret_cast<uint2*>(row + cb * 8) =
            make_uint2(__byte_perm(a, b, 0x5410), __byte_perm(c, d, 0x5410));
    }
};

template <>
struct Pack<2> {
    // offset code s = code + 2 in [0, 3]
    static __device__ __forceinline__ void run(uint8_t* row, int cb, const float (&t)[8]) {
        const float2 k = f2(-(kMagic - 2.0f), -(kMagic - 2.0f));
        const float2 s0 = fadd2(f2(t[0], t[4]), k), s1 = fadd2(f2(t[1], t[5]), k);
        const float2 s2 = fadd2(f2(t[2], t[6]), k), s3 = fadd2(f2(t[3], t[7]), k);
        const float2 p01 = ffma2(s1, f2(4.0f, 4.0f), s0);
        const float2 p23 = ffma2(s3, f2(4.0f, 4.0f), s2);
        float2 z = ffma2(p23, f2(16.0f, 16.0f), p01);              // 8-bit halves
        z = fadd2(z, f2(8388608.0f, 8388608.0f));
        const uint32_t w = __byte_perm(__float_as_uint(z.x), __float_as_uint(z.y), 0x0040) ^ 0xAAAAu;
        *reinterpret_cast<uint16_t*>(row + cb * 2) = uint16_t(w);
    }
};

template <int DK, int DV>
struct Pack6 {
    static __device__ __forceinline__ void run(uint8_t* tile, int i, int cb, const float (&t)[8]) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            const uint32_t u = __float_as_uint(t[e]);
            lo |= (u & 15u) << (4 * e);
            hi |= ((u >> 4) & 3u) << (2 * e);
        }
        *reinterpret_cast<uint32_t*>(tile + i * (DV / 2) + cb * 4) = lo;
        *reinterpret_cast<uint16_t*>(tile + DK * DV / 2 + i * (DV / 4) + cb * 2) = uint16_t(hi);
    }
};

// ------------------------------------------------------------------ reductions
// Column sums: p[8] holds this thread's canonical block sums (rows i0..i0+7)
// for its columns j0..j0+7.  Adjacent row blocks of the warp are joined by the
// xor butterfly over offsets CBW, 2*CBW, ..; warps by a pairwise tree.  Every
// thread gets its 8 column totals in res.
template <int DK, int DV>
__device__ __forceinline__ void colsum_finish(float (&p)[8], float* red, float* tot, int warp,
                                              int rbl, int j0, float (&res)[8]) {
    using G = Geo<DK, DV>;
#pragma unroll
    for (int off = G::CBW; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 8; c++) p[c] = __fadd_rn(p[c], __shfl_xor_sync(0xFFFFFFFFu, p[c], off));
    }
    if (rbl == 0) {
        float4* r4 = reinterpret_cast<float4*>(red + warp * DV + j0);
        r4[0] = make_float4(p[0], p[1], p[2], p[3]);
        r4[1] = make_float4(p[4], p[5], p[6], p[7]);
    }
    __syncthreads();
    if (threadIdx.x >= G::NT - DV) {       // the last warps (warp 0 refills)
        const int j = threadIdx.x - (G::NT - DV);
        float t[G::NWARPS];
#pragma unroll
        for (int w2 = 0; w2 < G::NWARPS; w2++) t[w2] = red[w2 * DV + j];
#pragma unroll
        for (int n = G::NWARPS; n > 1; n >>= 1) {
#pragma unroll
            for (int u = 0; u < n / 2; u++) t[u] = __fadd_rn(t[2 * u], t[2 * u + 1]);
        }
        tot[j] = t[0];
    }
    __syncthreads();
    const float4 a = reinterpret_cast<const float4*>(tot + j0)[0];
    const float4 b = reinterpret_cast<const float4*>(tot + j0)[1];
    res[0] = a.x; res[1] = a.y; res[2] = a.z; res[3] = a.w;
    res[4] = b.x; res[5] = b.y; res[6] = b.z; res[7] = b.w;
}

// ------------------------------------------------------------------ scales
// a flag that is either a run-time bool or a compile-time constant
__device__ __forceinline__ bool as_bool(bool b) { return b; }
template <bool B>
__device__ __forceinline__ bool as_bool(std::integral_constant<bool, B>) { return B; }

// m / Qmax correctly rounded, for m >= 0 finite or +inf and rq = RN(1 / Qmax):
// a product with the rounded reciprocal, then one correction by the exact
// remainder (Markstein's scheme for division by a constant).  For every
// non-negative binary32 m and Qmax in {1, 7, 31, 127} the result equals the
// IEEE quotient bit for bit; +inf (remainder NaN) keeps the product.
__device__ __forceinline__ float div_by_qmax(float m, float qmax, float rq) {
    const float q0 = __fmul_rn(m, rq);
    const float r = __fmaf_rn(-q0, qmax, m);
    const float q1 = __fmaf_rn(r, rq, q0);
    return r != r ? q0 : q1;
}

// ------------------------------------------------------------------ rounding
// RTN in the biased domain: t = 1.5 * 2^23 + round_half_even(x * inv).
__device__ __forceinline__ float2 rtn2(float2 x, float inv) {
    return ffma2(x, f2(inv, inv), f2(kMagic, kMagic));
}

// BDR correction of one element (branch-free).  s = a*inv - code rounded once;
// the element is reversed when sign(d) * s > eps (d = x - a != 0) and then
// moves one grid step toward its update.
__device__ __forceinline__ float bdr1(float t, float s, float d, float eps) {
    const uint32_t sg = __float_as_uint(d) & 0x80000000u;
    const float ss = __uint_as_float(__float_as_uint(s) ^ sg);
    const float step = __uint_as_float(sg | 0x3F800000u);
    const bool rev = (ss > eps) & (d != 0.0f);
    return rev ? __fadd_rn(t, step) : t;
}

// ------------------------------------------------------------------ shared state
// Partials that a tile writes before its exchange barrier and reads after it.
// They are double-buffered by tile parity: a CTA has one barrier per tile, so
// the next tile may write its partials while a slower warp still reads these.
template <int DK, int DV, bool YOKED>
struct __align__(16) Xchg {
    using G = Geo<DK, DV>;
    // output partials: one per row block when a warp holds 4 or more row
    // blocks (d_v = 64), else one per warp (row blocks joined by a shuffle)
    static constexpr int NPART = G::RBW >= 4 ? G::NWARPS * G::RBW : G::NWARPS;
    float red_o[NPART * DV];
    float wred[2][G::NWARPS];
    // per-row maxima of each 8-column block, column-block major; rows padded
    // by 4 so the lanes of a warp (different column blocks) hit different banks
    float rmax[DV / 8][DK + 4];
    float rmaxr[YOKED ? DV / 8 : 1][DK + 4];   // of the yoked reference state
};

template <int DK, int DV, bool GDN, bool YOKED, bool EXTRA = false>
struct __align__(16) Shared {
    using G = Geo<DK, DV>;
    // Gated DeltaNet column sums r = a^T k, used before the exchange barrier
    // only; the yoked reference state's sums use them first (the two sums are
    // separated by the barriers inside each)
    float red_r[GDN ? G::NWARPS * DV : 4];
    float tot_r[GDN ? DV : 4];
    Xchg<DK, DV, YOKED> x[2];
    // Hadamard-rotated states (kernels with the extra features only): H v of
    // the tile, and the output transform's exchange across warps (two
    // buffers, one per stage parity)
    float vrot[EXTRA ? DV : 4];
    float orot[2][EXTRA ? DV : 4];
};
// the partials are written and read as float4: every array starts on 16 bytes
template <int DK, int DV, bool GDN, bool YOKED, bool EXTRA>
struct SharedLayoutCheck {
    using X = Xchg<DK, DV, YOKED>;
    using S = Shared<DK, DV, GDN, YOKED, EXTRA>;
    static_assert(offsetof(X, red_o) % 16 == 0 && offsetof(X, rmax) % 16 == 0 &&
                  offsetof(X, rmaxr) % 16 == 0 && sizeof(X) % 16 == 0, "exchange layout");
    static_assert(offsetof(S, red_r) % 16 == 0 && offsetof(S, tot_r) % 16 == 0 &&
                  offsetof(S, x) % 16 == 0 && offsetof(S, vrot) % 16 == 0, "shared layout");
    static constexpr bool ok = true;
};

// 1.0f where a > b, else 0.0f (also for NaN), in one comparison
__device__ __forceinline__ float set_gt(float a, float b) {
    float r;
    asm("set.gt.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float sgnf(float x) {
    return x > 0.0f ? 1.0f : (x < 0.0f ? -1.0f : 0.0f);
}

template <int DK, int DV, int BITS>
__device__ __forceinline__ void pack_row(uint8_t* ct, int i, int cb, const float (&t8)[8]) {
    if constexpr (BITS == 4) Pack<4>::run(ct + i * (DV / 2), cb, t8);
    else if constexpr (BITS == 8) Pack<8>::run(ct + i * DV, cb, t8);
    else if constexpr (BITS == 2) Pack<2>::run(ct + i * (DV / 4), cb, t8);
    else Pack6<DK, DV>::run(ct, i, cb, t8);
}

// Round and repack a thread's 8 x 8 block, exact general path: full clamping
// of the RTN code and of the BDR step, and the update's sign taken from
// d = x - a element by element.  a holds the decayed state (BDR) or the
// updated state (RTN); with BDR the update x = fma(u_r, w_c, a) is formed
// again here.
template <int DK, int DV, int BITS, bool BDR, class URow>
__device__ __forceinline__ void round_pack_exact(const float (&a)[8][8], URow urow,
                                                 const float (&wc)[8], const float (&inv)[8],
                                                 float eps_b, uint8_t* ct, int i0, int cb) {
    constexpr float fq = float((1 << (BITS - 1)) - 1);
#pragma unroll
    for (int r = 0; r < 8; r++) {
        float t8[8];
        float ur = 0.0f;
        if constexpr (BDR) ur = urow(r);
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float2 a2 = f2(a[r][c], a[r][c + 1]);
            const float2 x2 = BDR ? ffma2(f2(ur, ur), f2(wc[c], wc[c + 1]), a2) : a2;
            float2 t2 = rtn2(x2, inv[r]);
            t2.x = fminf(fmaxf(t2.x, kMagic - fq), kMagic + fq);
            t2.y = fminf(fmaxf(t2.y, kMagic - fq), kMagic + fq);
            if constexpr (BDR) {
                const float2 d2 = ffma2(a2, f2(-1.0f, -1.0f), x2);                  // x - a
                const float2 cn = ffma2(t2, f2(-1.0f, -1.0f), f2(kMagic, kMagic));  // -code
                const float2 s2 = ffma2(a2, f2(inv[r], inv[r]), cn);
                t2.x = bdr1(t2.x, s2.x, d2.x, eps_b);
                t2.y = bdr1(t2.y, s2.y, d2.y, eps_b);
                t2.x = fminf(fmaxf(t2.x, kMagic - fq), kMagic + fq);
                t2.y = fminf(fmaxf(t2.y, kMagic - fq), kMagic + fq);
            }
            t8[c] = t2.x;
            t8[c + 1] = t2.y;
        }
        pack_row<DK, DV, BITS>(ct, i0 + r, cb, t8);
    }
}

// Fast path, taken by a warp when no element can round past the code range
// (|x * inv| < Qmax + 1/2 everywhere) and, with BDR, when every update is large
// enough that x != a exactly where u_r * w_c != 0: the sign of d = x - a is
// then sign(u_r) * sign(w_c), a rank-1 sign pattern.  A BDR step can still
// leave the range where |x * inv| > Qmax; rows flagged in `clampmask` are
// clamped after the step.
template <int DK, int DV, int BITS, bool BDR, class URow>
__device__ __forceinline__ void round_pack_fast(const float (&a)[8][8], URow urow,
                                                const float (&wc)[8], const float (&inv)[8],
                                                float eps_b, uint32_t clampmask, uint8_t* ct,
                                                int i0, int cb) {
    constexpr float fq = float((1 << (BITS - 1)) - 1);
    float sgc[8];
    if constexpr (BDR) {
#pragma unroll
        for (int c = 0; c < 8; c++) sgc[c] = sgnf(wc[c]);
    }
#pragma unroll
    for (int r = 0; r < 8; r++) {
        float t8[8];
        float ur = 0.0f, sgr = 0.0f;
        if constexpr (BDR) {
            ur = urow(r);
            sgr = sgnf(ur);
        }
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float2 a2 = f2(a[r][c], a[r][c + 1]);
            const float2 x2 = BDR ? ffma2(f2(ur, ur), f2(wc[c], wc[c + 1]), a2) : a2;
            float2 t2 = rtn2(x2, inv[r]);
            if constexpr (BDR) {
                const float2 cn = ffma2(t2, f2(-1.0f, -1.0f), f2(kMagic, kMagic));  // -code
                const float2 s2 = ffma2(a2, f2(inv[r], inv[r]), cn);                // u - code
                const float2 sg = fmul2(f2(sgr, sgr), f2(sgc[c], sgc[c + 1]));      // sign(d)
                const float2 ss = fmul2(s2, sg);
                // one grid step toward the update where ss > eps (exact: t is an
                // integer-valued float far below 2^24)
                t2 = ffma2(f2(set_gt(ss.x, eps_b), set_gt(ss.y, eps_b)), sg, t2);
            }
            t8[c] = t2.x;
            t8[c + 1] = t2.y;
        }
        if (BDR && ((clampmask >> r) & 1u)) {
#pragma unroll
            for (int c = 0; c < 8; c++) t8[c] = fminf(fmaxf(t8[c], kMagic - fq), kMagic + fq);
        }
        pack_row<DK, DV, BITS>(ct, i0 + r, cb, t8);
    }
}

// Scales of the (row, group) pairs of a thread's 8 rows, for a group of L
// lanes (L = group / 8 column blocks).  The per-row maxima of every 8-column
// block are in shared memory; lane lp of a group derives the scales of
// rows lp*nv .. lp*nv + nv - 1 of its row block (nv = 8 / min(L, 8)), stores
// them, and the reciprocals go back to the group's lanes with shuffles.
// SF32: the scales are binary32 (else binary16); sprev: the staged previous
// scales of the tile.
template <int DK, int DV, int L, bool SF32, class X, class NewScale>
__device__ __forceinline__ void group_scales(int cb, int lane, int i0, const X& sh,
                                             bool yoked, float (&inv)[8], unsigned& nsat,
                                             bool& bad, NewScale new_scale, const uint8_t* sprev,
                                             const StepParams& p, long long sbase, int ng, int gcol) {
    constexpr int Lp = L < 8 ? L : 8, nv = 8 / Lp;
    const int lp = cb % L;
    const int cb0 = cb - lp;                 // first column block of the group
    const int rbase = (lp % Lp) * nv;
    auto prev_scale = [&](int row) -> float {
        const int idx = row * ng + gcol;
        if constexpr (SF32) return reinterpret_cast<const float*>(sprev)[idx];
        else return __half2float(reinterpret_cast<const __half*>(sprev)[idx]);
    };
    float invm[nv];
#pragma unroll
    for (int k = 0; k < nv; k++) {
        const int row = i0 + rbase + k;
        float mm = 0.0f, mr = 0.0f;
#pragma unroll
        for (int b = 0; b < L; b++) {
            mm = fmaxf(mm, sh.rmax[cb0 + b][row]);
            if (yoked) mr = fmaxf(mr, sh.rmaxr[cb0 + b][row]);
        }
        bool sat;
        const float d = new_scale(mm, mr, prev_scale(row), sat, std::integral_constant<bool, SF32>{});
        invm[k] = d == 0.0f ? 0.0f : __frcp_rn(d);
        bad |= !isfinite(mm) || !isfinite(mr);
        if (lp < 8) {
            store_scale(p.scales, sbase + (long long)row * ng + gcol, SF32, d);
            nsat += sat ? 1u : 0u;
        }
    }
    if constexpr (L == 1) {
#pragma unroll
        for (int r = 0; r < 8; r++) inv[r] = invm[r];
    } else {
        const int gbase = lane - lp;
#pragma unroll
        for (int r = 0; r < 8; r++) inv[r] = __shfl_sync(0xFFFFFFFFu, invm[r % nv], gbase + r / nv);
    }
}

// ------------------------------------------------------------------ Hadamard rotation
// H x for the Sylvester Hadamard matrix of order n (entries +-1), by the
// butterfly of the specification: for h = 1, 2, 4, .. and every i with
// (i & h) == 0, (x_i, x_{i+h}) <- (x_i + x_{i+h}, x_i - x_{i+h}), one
// rounding per operation.  The pairs of one stage are independent, so any
// schedule that finishes each stage before the next gives the same bits.

// H v of a staged v (d_v values, f32 or bf16) into vrot, by warp 0: lane l
// holds elements E*l .. E*l + E - 1 (E = d_v / 32); stages below E run in the
// lane, the others pair lane l with lane l ^ (h / E).
template <int DV, bool BF>
__device__ __forceinline__ void rotate_v(const uint8_t* sv, float* vrot) {
    constexpr int E = DV / 32;
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    float x[E];
#pragma unroll
    for (int e = 0; e < E; e++) {
        const int i = E * lane + e;
        x[e] = BF ? __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(sv)[i]) << 16)
                  : reinterpret_cast<const float*>(sv)[i];
    }
#pragma unroll
    for (int h = 1; h < E; h *= 2) {
#pragma unroll
        for (int e = 0; e < E; e++)
            if ((e & h) == 0) {
                const float a = x[e], b = x[e + h];
                x[e] = __fadd_rn(a, b);
                x[e + h] = __fsub_rn(a, b);
            }
    }
#pragma unroll
    for (int h = E; h < DV; h *= 2) {
        const int o = h / E;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int e = 0; e < E; e++) {
            const float other = __shfl_xor_sync(0xFFFFFFFFu, x[e], o);
            x[e] = upper ? __fsub_rn(other, x[e]) : __fadd_rn(x[e], other);
        }
    }
#pragma unroll
    for (int e = 0; e < E; e++) vrot[E * lane + e] = x[e];
}

// H o / d_v across the DV threads that hold one output each (o of column j,
// j = the thread's index among them; they are whole warps): stages below 32
// with shuffles, the others through shared memory behind a named barrier
// (id 1) that only these DV threads join.
template <int DV>
__device__ __forceinline__ float rotate_out(float o, int j, float (*orot)[DV]) {
    const int lane = j & 31;
#pragma unroll
    for (int h = 1; h < 32 && h < DV; h *= 2) {
        const float other = __shfl_xor_sync(0xFFFFFFFFu, o, h);
        o = (lane & h) ? __fsub_rn(other, o) : __fadd_rn(o, other);
    }
    int buf = 0;
#pragma unroll
    for (int h = 32; h < DV; h *= 2) {
        orot[buf][j] = o;
        asm volatile("bar.sync 1, %0;" :: "r"(DV) : "memory");
        const float other = orot[buf][j ^ h];
        o = (j & h) ? __fsub_rn(other, o) : __fadd_rn(o, other);
        buf ^= 1;
    }
    return __fmul_rn(o, 1.0f / float(DV));
}

// ------------------------------------------------------------------ taxonomy
// The rounding taxonomy of Figure 4 of "Preserving Updates in Low-Bit
// Recurrent State Quantization" on a thread's 8 x 8 block, counted into
// counters[4..7] (lost, moved, reversed, BDR steps applied).  The decayed
// value a and the updated value x are formed again from the staged codes with
// the step's own operations and order, so the classes are those of the exact
// values the step rounded: with u = a * inv and w = x * inv (exact products),
// c = clamp(RTN(w)) and d = x - a != 0, the element is reversed when c lies
// strictly beyond u on the side away from the update (the sign of the single
// rounding of u - c is exact), else lost when c = clamp(RTN(u)), else moved.
// A BDR step is applied when d > 0 and u - c > eps_B, or d < 0 and
// u - c < -eps_B.  Diagnostic only: it runs when counters are asked for.
template <int DK, int DV, int BITS, bool BDR, class URow>
__device__ __forceinline__ void taxonomy_count(const StepParams& p, const uint8_t* st, int i0, int cb,
                                            const float (&eta)[8], URow urow,
                                            const float (&wc)[8], const float (&inv)[8],
                                            long long tile, long long sbase, int ng, int gcol) {
    constexpr float fq = float((1 << (BITS - 1)) - 1);
    using G = Geo<DK, DV>;
    unsigned nl = 0, nm = 0, nr = 0, nb = 0;
    // the step's new scales, stored by other threads of the CTA
    const bool energy = p.err_rows != nullptr;
    if (energy) __syncthreads();
#pragma unroll 1
    for (int r = 0; r < 8; r++) {
        float dnew = 0.0f, e2 = 0.0f;
        if (energy) dnew = scale_at(p.scales, p.group ? sbase + (i0 + r) * ng + gcol : sbase,
                                    p.scale_f32 != 0);
        float c8[8];
        const uint8_t* srow = st + p.off_codes;
        if constexpr (BITS == 4) Decode<4>::run(srow + (i0 + r) * (DV / 2), cb, c8);
        else if constexpr (BITS == 8) Decode<8>::run(srow + (i0 + r) * DV, cb, c8);
        else if constexpr (BITS == 2) Decode<2>::run(srow + (i0 + r) * (DV / 4), cb, c8);
        else Decode6<DK, DV>::run(srow, i0 + r, cb, c8);
        const float ur = urow(r);
#pragma unroll
        for (int c = 0; c < 8; c++) {
            const float a = __fmul_rn(c8[c], eta[r]);
            const float x = __fmaf_rn(ur, wc[c], a);
            const float d = __fsub_rn(x, a);
            const float t = fminf(fmaxf(__fmaf_rn(x, inv[r], kMagic), kMagic - fq), kMagic + fq);
            const float s = __fmaf_rn(a, inv[r], -__fsub_rn(t, kMagic));    // u - c
            const bool bdr = BDR && ((d > 0.0f && s > p.eps_b) || (d < 0.0f && s < -p.eps_b));
            if (d != 0.0f) {
                const float tu = fminf(fmaxf(__fmaf_rn(a, inv[r], kMagic), kMagic - fq), kMagic + fq);
                const bool rev = (s > 0.0f && d > 0.0f) || (s < 0.0f && d < 0.0f);
                nr += rev ? 1u : 0u;
                nl += (!rev && t == tu) ? 1u : 0u;
                nm += (!rev && t != tu) ? 1u : 0u;
                nb += bdr ? 1u : 0u;
            }
            if (energy) {
                // the code stored: the RTN code, moved one step by BDR, clamped
                const float tf = bdr ? fminf(fmaxf(__fadd_rn(t, d > 0.0f ? 1.0f : -1.0f), kMagic - fq),
                                             kMagic + fq)
                                     : t;
                const float R = __fsub_rn(__fmul_rn(__fsub_rn(tf, kMagic), dnew), x);
                e2 = __fmaf_rn(R, R, e2);
            }
        }
        if (energy) {
#pragma unroll
            for (int off = 1; off < G::CBW; off <<= 1) e2 = __fadd_rn(e2, __shfl_xor_sync(0xFFFFFFFFu, e2, off));
            if (cb == 0) p.err_rows[tile * DK + i0 + r] = e2;
        }
    }
    nl = __reduce_add_sync(0xFFFFFFFFu, nl);
    nm = __reduce_add_sync(0xFFFFFFFFu, nm);
    nr = __reduce_add_sync(0xFFFFFFFFu, nr);
    nb = __reduce_add_sync(0xFFFFFFFFu, nb);
    if ((threadIdx.x & 31) == 0) {
        if (nl) atomicAdd(p.counters + 4, (unsigned long long)nl);
        if (nm) atomicAdd(p.counters + 5, (unsigned long long)nm);
        if (nr) atomicAdd(p.counters + 6, (unsigned long long)nr);
        if (nb) atomicAdd(p.counters + 7, (unsigned long long)nb);
    }
}

// ------------------------------------------------------------------ one tile
// st: the tile's shared-memory stage; ct: its codes in global memory.
// g0, g1: scalar gates (alpha, beta) and pts: per-token previous scale,
// prefetched by the caller.  ok: this thread's stage arrived.  Without the delta
// rule or a reference state the tile has one CTA barrier, the exchange of
// output partials and maxima; it votes on ok (false is returned by every
// thread, before any global write of the tile, when one of them gave up) and
// at_barrier() runs right after it.  Gated DeltaNet and yoked tiles vote at a
// barrier of their own at the top (the caller's), before their column sums or
// their reference-state writes.
// GM: what the tile body knows at compile time.  Low two bits, the scale
// groups (GM_ANY: group read at run time; GM_TILE: one scale per tile;
// GM_ROWS: groups of >= 8 columns); GM_ALPHA: the form of the decay is known,
// a per-row vector (GLA) with GM_VEC, else a scalar (RetNet, Mamba2, GDN).
enum { GM_ANY = 0, GM_TILE = 1, GM_ROWS = 2, GM_ALPHA = 4, GM_VEC = 8 };

template <int DK, int DV, int BITS, bool GDN, bool YOKED, bool BDR, bool BF, bool EXTRA, int GM,
          class AtBarrier>
__device__ __forceinline__ bool step_tile(const StepParams& p, long long tile, const uint8_t* st,
                                          uint8_t* ct, float g0, float g1, float pts,
                                          Shared<DK, DV, GDN, YOKED, EXTRA>& sh,
                                          Xchg<DK, DV, YOKED>& xs, volatile int* badflag,
                                          bool ok, AtBarrier at_barrier) {
    using G = Geo<DK, DV>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cb = lane % G::CBW, rbl = lane / G::CBW;
    const int i0 = (warp * G::RBW + rbl) * 8, j0 = cb * 8;
    constexpr int QMAX = BITS == 32 ? 0 : (1 << (BITS - 1)) - 1;
    const bool sf32 = p.scale_f32 != 0;
    constexpr int isz = BF ? 2 : 4;
    constexpr int GMODE = GM & 3;
    const int group = GMODE == GM_TILE ? 0 : p.group;
    if (GMODE == GM_ROWS) __builtin_assume(group >= 8);
    const bool vec_alpha = (GM & GM_ALPHA) ? (GM & GM_VEC) != 0 : p.kind == K_GLA;

    // step inputs (shared-memory stage); q and k are read row by row where
    // they are used, which keeps them out of the register file
    const uint8_t* sk = st + p.off_k + i0 * isz;
    const uint8_t* sq = st + p.off_q + i0 * isz;
    // (16-byte loads of 8 bf16 or 4 fp32 rows; the unrolled uses of one
    // vector share its load)
    auto row_in = [](const uint8_t* base, int r) -> float {
        if constexpr (BF) {
            const uint4 u = reinterpret_cast<const uint4*>(base)[0];
            const uint32_t w = (r >> 1) == 0 ? u.x : (r >> 1) == 1 ? u.y : (r >> 1) == 2 ? u.z : u.w;
            return __uint_as_float((r & 1) ? (w & 0xFFFF0000u) : (w << 16));
        } else {
            const float4 f = reinterpret_cast<const float4*>(base)[r >> 2];
            return (r & 3) == 0 ? f.x : (r & 3) == 1 ? f.y : (r & 3) == 2 ? f.z : f.w;
        }
    };
    float vv[8], al[8];
    bool rotated = false;
    if constexpr (EXTRA) {
        if (p.rotate) {
            // the update's value vector of a rotated state is H v
            rotate_v<DV, BF>(st + p.off_v, sh.vrot);
            __syncthreads();
            ld8(reinterpret_cast<const uint8_t*>(sh.vrot + j0), false, vv);
            rotated = true;
        }
    }
    if (!rotated) ld8(st + p.off_v + j0 * isz, BF, vv);
    if (vec_alpha) {
        ld8(st + p.off_ga + i0 * (p.gate_bf16 ? 2 : 4), p.gate_bf16 != 0, al);
    } else {
        const float s = p.kind == K_RETNET ? p.gamma : g0;
#pragma unroll
        for (int r = 0; r < 8; r++) al[r] = s;
    }
    const float beta = GDN ? g1 : 0.0f;
    // Non-finite inputs are not checked one by one: any NaN or infinity in q,
    // k, v or the gates reaches the output o or a group maximum (0 * inf and
    // inf - inf are NaN), where it is counted.

    // group is a power of two (8 .. 128) dividing d_v
    const int gsh = group ? __ffs(group) - 1 : 0;
    const int ng = group ? DV >> gsh : 1;
    const long long sbase = tile * (long long)p.n_scales;
    const int gcol = group ? j0 >> gsh : 0;
    // previous scales of this thread's 8 rows (its group), one dtype branch
    float dprev[8];
    if constexpr (BITS == 32) {
#pragma unroll
        for (int r = 0; r < 8; r++) dprev[r] = 0.0f;
    } else if (group == 0) {
#pragma unroll
        for (int r = 0; r < 8; r++) dprev[r] = pts;
    } else if (sf32) {
        const float* sp = reinterpret_cast<const float*>(st + p.off_scales) + i0 * ng + gcol;
#pragma unroll
        for (int r = 0; r < 8; r++) dprev[r] = sp[r * ng];
    } else {
        const __half* sp = reinterpret_cast<const __half*>(st + p.off_scales) + i0 * ng + gcol;
#pragma unroll
        for (int r = 0; r < 8; r++) dprev[r] = __half2float(sp[r * ng]);
    }

    // ---- yoked reference state: stepped first; only its group maxima stay
    float mref[8];
#pragma unroll
    for (int r = 0; r < 8; r++) mref[r] = 0.0f;
    if constexpr (YOKED) {
        float ar[8][8];
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float s8[8];
            ld8(st + p.off_ref + ((i0 + r) * DV + j0) * 4, false, s8);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 v2 = fmul2(f2(s8[c], s8[c + 1]), f2(al[r], al[r]));
                ar[r][c] = v2.x;
                ar[r][c + 1] = v2.y;
            }
        }
        float e2[8];
        if constexpr (GDN) {
            float pr[8];
#pragma unroll
            for (int c = 0; c < 8; c++) pr[c] = 0.0f;
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float kr = row_in(sk, r);
                    const float2 v2 = ffma2(f2(ar[r][c], ar[r][c + 1]), f2(kr, kr),
                                            f2(pr[c], pr[c + 1]));
                    pr[c] = v2.x;
                    pr[c + 1] = v2.y;
                }
            colsum_finish<DK, DV>(pr, sh.red_r, sh.tot_r, warp, rbl, j0, e2);
#pragma unroll
            for (int c = 0; c < 8; c++) e2[c] = __fsub_rn(vv[c], e2[c]);
        }
        float* gref = p.ref + (tile * DK) * (long long)DV;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            const float kap = GDN ? __fmul_rn(beta, row_in(sk, r)) : row_in(sk, r);
            float mm = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                float2 w2;
                if constexpr (GDN) w2 = f2(e2[c], e2[c + 1]);
                else w2 = f2(vv[c], vv[c + 1]);
                const float2 v2 = ffma2(f2(kap, kap), w2, f2(ar[r][c], ar[r][c + 1]));
                ar[r][c] = v2.x;
                ar[r][c + 1] = v2.y;
                mm = fmaxf(mm, fmaxf(fabsf(v2.x), fabsf(v2.y)));
            }
            {               // the stage vote was taken at the top of the tile
                float4* dst = reinterpret_cast<float4*>(gref + (i0 + r) * DV + j0);
                dst[0] = make_float4(ar[r][0], ar[r][1], ar[r][2], ar[r][3]);
                dst[1] = make_float4(ar[r][4], ar[r][5], ar[r][6], ar[r][7]);
            }
            mref[r] = mm;
        }
    }

    // ---- 1. decay: a = code * (alpha * scale)   (32-bit state: S * alpha)
    float a[8][8];
#pragma unroll
    for (int r = 0; r < 8; r++) {
        float c8[8];
        float eta;
        if constexpr (BITS == 32) {
            ld8(st + p.off_codes + ((i0 + r) * DV + j0) * 4, false, c8);
            eta = al[r];
        } else {
            eta = __fmul_rn(al[r], dprev[r]);
            const uint8_t* srow = st + p.off_codes;
            if constexpr (BITS == 4) Decode<4>::run(srow + (i0 + r) * (DV / 2), cb, c8);
            else if constexpr (BITS == 8) Decode<8>::run(srow + (i0 + r) * DV, cb, c8);
            else if constexpr (BITS == 2) Decode<2>::run(srow + (i0 + r) * (DV / 4), cb, c8);
            else Decode6<DK, DV>::run(srow, i0 + r, cb, c8);
        }
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const float2 v2 = fmul2(f2(c8[c], c8[c + 1]), f2(eta, eta));
            a[r][c] = v2.x;
            a[r][c + 1] = v2.y;
        }
    }

    // ---- 2. update coefficients: x = fma(u_r, w_c, a), u_r = beta k_r (GDN)
    // or k_r, formed row by row
    auto urow = [&](int r) -> float {
        if constexpr (GDN) return __fmul_rn(beta, row_in(sk, r));
        else return row_in(sk, r);
    };
    float wc[8];
    if constexpr (GDN) {
        float pr[8];
#pragma unroll
        for (int c = 0; c < 8; c++) pr[c] = 0.0f;
#pragma unroll
        for (int r = 0; r < 8; r++)
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float kr = row_in(sk, r);
                const float2 v2 = ffma2(f2(a[r][c], a[r][c + 1]), f2(kr, kr), f2(pr[c], pr[c + 1]));
                pr[c] = v2.x;
                pr[c + 1] = v2.y;
            }
        colsum_finish<DK, DV>(pr, sh.red_r, sh.tot_r, warp, rbl, j0, wc);
#pragma unroll
        for (int c = 0; c < 8; c++) wc[c] = __fsub_rn(vv[c], wc[c]);       // e = v - r
    } else {
#pragma unroll
        for (int c = 0; c < 8; c++) wc[c] = vv[c];
    }

    // ---- 3. output o = x^T q and row maxima, x formed on the fly.  With one
    // scale per tile the warp maxima travel with the output partials, so the
    // tile maximum needs no barrier of its own.
    float m[8];
    float tmax = 0.0f, tref = 0.0f;
    {
        float po[8];
#pragma unroll
        for (int c = 0; c < 8; c++) po[c] = 0.0f;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float mx = 0.0f;     // max |x| of the row (three-input max)
            const float ur = urow(r), qr = row_in(sq, r);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const float2 x2 = ffma2(f2(ur, ur), f2(wc[c], wc[c + 1]), f2(a[r][c], a[r][c + 1]));
                const float2 o2 = ffma2(x2, f2(qr, qr), f2(po[c], po[c + 1]));
                po[c] = o2.x;
                po[c + 1] = o2.y;
                mx = fmaxf(fmaxf(mx, fabsf(x2.x)), fabsf(x2.y));
                if constexpr (!BDR) {        // the decayed state is not needed again
                    a[r][c] = x2.x;
                    a[r][c + 1] = x2.y;
                }
            }
            m[r] = mx;
        }
        if constexpr (G::RBW >= 4) {
            // every row block's partials go to shared memory as they are
            float4* r4 = reinterpret_cast<float4*>(xs.red_o + (warp * G::RBW + rbl) * DV + j0);
            r4[0] = make_float4(po[0], po[1], po[2], po[3]);
            r4[1] = make_float4(po[4], po[5], po[6], po[7]);
        } else {
#pragma unroll
            for (int off = G::CBW; off < 32; off <<= 1) {
#pragma unroll
                for (int c = 0; c < 8; c++) po[c] = __fadd_rn(po[c], __shfl_xor_sync(0xFFFFFFFFu, po[c], off));
            }
            if (rbl == 0) {
                float4* r4 = reinterpret_cast<float4*>(xs.red_o + warp * DV + j0);
                r4[0] = make_float4(po[0], po[1], po[2], po[3]);
                r4[1] = make_float4(po[4], po[5], po[6], po[7]);
            }
        }
        if (group != 0 && BITS != 32) {
            float4* r4 = reinterpret_cast<float4*>(&xs.rmax[cb][i0]);
            r4[0] = make_float4(m[0], m[1], m[2], m[3]);
            r4[1] = make_float4(m[4], m[5], m[6], m[7]);
            if (YOKED) {
                float4* q4 = reinterpret_cast<float4*>(&xs.rmaxr[cb][i0]);
                q4[0] = make_float4(mref[0], mref[1], mref[2], mref[3]);
                q4[1] = make_float4(mref[4], mref[5], mref[6], mref[7]);
            }
        }
        if (group == 0 && BITS != 32) {
            // the maxima are non-negative and never NaN (fmaxf drops NaN), so
            // their bit patterns order like the values: one integer warp max
            float t = m[0], tr = mref[0];
#pragma unroll
            for (int r = 1; r < 8; r++) { t = fmaxf(t, m[r]); tr = fmaxf(tr, mref[r]); }
            t = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(t)));
            if (YOKED) tr = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(tr)));
            if (lane == 0) { xs.wred[0][warp] = t; xs.wred[1][warp] = tr; }
        }
        if constexpr (GDN || YOKED) {
            __syncthreads();     // the vote was taken at the top of the tile
        } else {
            if (!__syncthreads_and(ok)) return false;
            at_barrier();
        }
        // the last DV threads sum the outputs (warp 0 refills the pipeline)
        if (threadIdx.x >= G::NT - DV) {
            // adjacent pairs, then pairs of pairs, .. over the partials in row
            // order: the canonical block tree
            constexpr int NP = Xchg<DK, DV, YOKED>::NPART;
            const int j = threadIdx.x - (G::NT - DV);
            float t[NP];
#pragma unroll
            for (int w2 = 0; w2 < NP; w2++) t[w2] = xs.red_o[w2 * DV + j];
#pragma unroll
            for (int n = NP; n > 1; n >>= 1) {
#pragma unroll
                for (int u = 0; u < n / 2; u++) t[u] = __fadd_rn(t[2 * u], t[2 * u + 1]);
            }
            float o = t[0];
            if constexpr (EXTRA) {
                if (p.rotate) o = rotate_out<DV>(o, j, sh.orot);
            }
            p.out[tile * DV + j] = o;
            if (BITS != 32 && !isfinite(o)) *badflag = 1;
        }
        if (group == 0 && BITS != 32) {
            tmax = xs.wred[0][0];
            tref = xs.wred[1][0];
#pragma unroll
            for (int w2 = 1; w2 < G::NWARPS; w2++) {
                tmax = fmaxf(tmax, xs.wred[0][w2]);
                tref = fmaxf(tref, xs.wred[1][w2]);
            }
        }
    }

    if constexpr (BITS == 32) {
        uint8_t* gs = ct;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            float x8[8];
            const float ur = urow(r);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                float2 x2 = f2(a[r][c], a[r][c + 1]);
                if constexpr (BDR)
                    x2 = ffma2(f2(ur, ur), f2(wc[c], wc[c + 1]), x2);
                x8[c] = x2.x;
                x8[c + 1] = x2.y;
            }
            float4* dst = reinterpret_cast<float4*>(gs + ((i0 + r) * DV + j0) * 4);
            dst[0] = make_float4(x8[0], x8[1], x8[2], x8[3]);
            dst[1] = make_float4(x8[4], x8[5], x8[6], x8[7]);
        }
        return true;
    } else {
        // ---- 4. scales
        const float fq = float(QMAX);
        // RN(1 / Qmax) for Qmax = 1, 7, 31, 127
        constexpr float rq = QMAX == 7 ? 0x1.24924ap-3f : QMAX == 31 ? 0x1.08421p-5f
                           : QMAX == 127 ? 0x1.020408p-7f : 1.0f;
        float inv[8];
        unsigned nsat = 0;
        // sfc: the scale dtype, a compile-time constant (row groups) or not
        auto new_scale = [&](float mm, float mr, float dp, bool& sat, auto sfc) -> float {
            const bool F = as_bool(sfc);
            sat = false;
            if constexpr (YOKED) return to_stored(div_by_qmax(mr, fq, rq), F, sat);
            if (p.scale_mode == M_PERSISTENT)
                return (mm > __fmul_rn(fq, dp)) ? to_stored(div_by_qmax(mm, fq, rq), F, sat) : dp;
            return to_stored(div_by_qmax(mm, fq, rq), F, sat);
        };
        bool bad = false;
        if (group) {
            // L = group / 8 lanes per group, and the scale dtype, fixed per call
            auto gs = [&](auto lc, auto sfc) {
                group_scales<DK, DV, decltype(lc)::value, decltype(sfc)::value>(
                    cb, lane, i0, xs, YOKED, inv, nsat, bad, new_scale, st + p.off_scales, p, sbase,
                    ng, gcol);
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
            bool sat;
            const float d = new_scale(tmax, tref, pts, sat, sf32);
            const float iv = d == 0.0f ? 0.0f : __frcp_rn(d);
#pragma unroll
            for (int r = 0; r < 8; r++) inv[r] = iv;
            bad |= !isfinite(tmax) || !isfinite(tref);
            if (threadIdx.x == G::NT - 1) {
                store_scale(p.scales, sbase, sf32, d);
                nsat += sat ? 1u : 0u;
            }
        }
        if (nsat) atomicAdd(p.counters + 1, (unsigned long long)nsat);

        // ---- 5-6. round and repack.  The fast path needs every |x * inv| below
        // Qmax + 1/2 (no RTN clamp) and, with BDR, updates large enough that
        // the sign of x - a is the sign of u_r * w_c.
        bool slow = false;
        uint32_t clampmask = 0;
        float wmin = 0.0f;
        if constexpr (BDR) {
            wmin = fabsf(wc[0]);
#pragma unroll
            for (int c = 1; c < 8; c++) wmin = fminf(wmin, fabsf(wc[c]));
        }
        if (group == 0) {
            float mt = m[0];
#pragma unroll
            for (int r = 1; r < 8; r++) mt = fmaxf(mt, m[r]);
            slow = !(__fmaf_rn(mt, inv[0], -(fq + 0.5f)) < 0.0f);
        }
        // A BDR step leaves the code range only from a code at +-Qmax toward
        // u with |u| > Qmax, and then |w| > Qmax as well (w lies beyond u).
        // With every stored code within +-Qmax (not the step after an import),
        // |u| <= Qmax |eta| inv (1 + 2^-23), eta = alpha * the previous scale.
        // A persistent scale never shrinks (inv <= RN(1 / previous scale)),
        // so with a scalar decay |alpha| <= 1 - 2^-20 every row has
        // |eta| inv <= |alpha| (1 + 2^-24)^2 < 1 - 2^-22 and |u| < Qmax:
        // then no row of the tile needs the clamp.
        bool noclamp = false;
        if constexpr (BDR && !YOKED)
            noclamp = p.fast && p.scale_mode == M_PERSISTENT && !vec_alpha &&
                      fabsf(al[0]) <= 1.0f - 0x1p-20f;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            if (group != 0) slow |= !(__fmaf_rn(m[r], inv[r], -(fq + 0.5f)) < 0.0f);
            if constexpr (BDR) {
                const float eta = __fmul_rn(al[r], dprev[r]);
                const float floor_ = fmaxf(__fmul_rn(eta, float(1 << (BITS - 1)) * 0x1p-21f), 0x1p-120f);
                slow |= !(__fmaf_rn(fabsf(urow(r)), wmin, -floor_) > 0.0f);
                if (__any_sync(0xFFFFFFFFu, __fmaf_rn(m[r], inv[r], -fq) > 0.0f)) clampmask |= 1u << r;
            }
        }
        if (noclamp) clampmask = 0;
        if (__any_sync(0xFFFFFFFFu, slow)) {
            if (EXTRA && p.taxonomy && lane == 0) atomicAdd(p.counters + 3, 1ull);
            round_pack_exact<DK, DV, BITS, BDR>(a, urow, wc, inv, p.eps_b, ct, i0, cb);
        } else {
            round_pack_fast<DK, DV, BITS, BDR>(a, urow, wc, inv, p.eps_b, clampmask, ct, i0, cb);
        }
        if (EXTRA && p.taxonomy) {
            float eta[8];
#pragma unroll
            for (int r = 0; r < 8; r++) eta[r] = __fmul_rn(al[r], dprev[r]);
            taxonomy_count<DK, DV, BITS, BDR>(p, st, i0, cb, eta, urow, wc, inv, tile, sbase, ng,
                                              gcol);
        }
        // a tile-step is counted once if an output or a group maximum was not
        // finite (the flag is collected at the next tile's barrier)
        if (bad) *badflag = 1;
        return true;
    }
}

// ------------------------------------------------------------------ producer
__device__ __forceinline__ void tile_codes(const StepParams& p, long long tile, uint8_t*& ptr,
                                           int& bits, uint32_t& bytes, int dk, int dv) {
    if (p.head_bits) {
        // tile counts fit 31 bits (checked at creation): 32-bit division
        const uint32_t t32 = uint32_t(tile), hd = uint32_t(p.heads);
        const uint32_t row = t32 / hd, h = t32 - row * hd;
        bits = p.head_bits[h];
        ptr = p.codes + (long long)row * p.row_bytes + p.head_off[h];
    } else {
        bits = p.bits;
        ptr = p.codes + tile * p.tile_bytes;
    }
    bytes = uint32_t((long long)dk * dv * bits / 8);
}

template <int DK, int DV, bool YOKED>
__device__ __forceinline__ void issue_tile(const StepParams& p, long long tile, uint8_t* st,
                                           uint64_t* bar) {
    if (p.drop_from >= 0 && tile >= p.drop_from) return;   // injected fault: never arrives
    uint8_t* cp;
    int bits;
    uint32_t cbytes;
    tile_codes(p, tile, cp, bits, cbytes, DK, DV);
    const uint32_t isz = p.qkv_bf16 ? 2 : 4, gsz = p.gate_bf16 ? 2 : 4;
    const uint32_t ssz = p.scale_f32 ? 4 : 2;
    uint32_t total = cbytes + 2 * DK * isz + DV * isz;
    const bool stage_scales = p.off_scales >= 0 && bits != 32;
    if (stage_scales) total += uint32_t(p.n_scales) * ssz;
    if (p.off_ga >= 0) total += DK * gsz;
    if (YOKED) total += DK * DV * 4;
    mbar_expect_tx(bar, total);
    bulk_g2s(st + p.off_codes, cp, cbytes, bar);
    if (stage_scales)
        bulk_g2s(st + p.off_scales,
                 static_cast<const uint8_t*>(p.scales) + tile * (long long)p.n_scales * ssz,
                 uint32_t(p.n_scales) * ssz, bar);
    bulk_g2s(st + p.off_q, static_cast<const uint8_t*>(p.q) + tile * DK * isz, DK * isz, bar);
    bulk_g2s(st + p.off_k, static_cast<const uint8_t*>(p.k) + tile * DK * isz, DK * isz, bar);
    bulk_g2s(st + p.off_v, static_cast<const uint8_t*>(p.v) + tile * DV * isz, DV * isz, bar);
    if (p.off_ga >= 0)
        bulk_g2s(st + p.off_ga, static_cast<const uint8_t*>(p.gates) + tile * DK * gsz, DK * gsz, bar);
    if (YOKED)
        bulk_g2s(st + p.off_ref, p.ref + tile * (long long)DK * DV, DK * DV * 4, bar);
}

// Scalar per-tile inputs that are too small for a bulk copy, loaded one tile
// ahead of their use.
__device__ __forceinline__ void load_scalars(const StepParams& p, long long tile, float& g0,
                                             float& g1, float& pts) {
    g0 = g1 = 0.0f;
    pts = 0.0f;
    if (tile >= p.ntiles) return;
    const int f = p.scalars;
    if (f & SC_G0) g0 = ldg1(p.gates, tile * p.n_gate, p.gate_bf16 != 0);
    if (f & SC_G1) g1 = ldg1(p.gates, tile * p.n_gate + 1, p.gate_bf16 != 0);
    if (f & SC_PTS) pts = scale_at(p.scales, tile, p.scale_f32 != 0);
}

// ------------------------------------------------------------------ kernel
// Registers are capped so that several CTAs share an SM (their barriers and
// pipeline waits then overlap); the yoked variant holds a second 8 x 8 block.
template <int DK, int DV, bool YOKED>
struct Occupancy {
    static constexpr int MIN_BLOCKS = YOKED ? 1 : (Geo<DK, DV>::NT >= 256 ? 2 : 4);
};

// BITS: the uniform code width of the object (2, 4, 6, 8, 32), or 0 when the
// width varies per head (dispatched per tile).  BF: q, k, v are bf16.
// EXTRA: the kernel also holds the rounding-taxonomy counts and the
// Hadamard-rotated layout (both switched per launch); the kernels without
// them are the ones stepped in the ordinary case.
template <int DK, int DV, int BITS, bool GDN, bool YOKED, bool BDR, bool BF, bool EXTRA>
__global__ void __launch_bounds__(Geo<DK, DV>::NT, (Occupancy<DK, DV, YOKED>::MIN_BLOCKS))
step_kernel(const StepParams p) {
    extern __shared__ __align__(128) uint8_t dsmem[];
    static_assert(SharedLayoutCheck<DK, DV, GDN, YOKED, EXTRA>::ok, "");
    __shared__ Shared<DK, DV, GDN, YOKED, EXTRA> sh;
    __shared__ __align__(8) uint64_t bars[kMaxStages];
    __shared__ volatile int badf[2];
    const int S = p.nstages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) mbar_init(&bars[s], 1);
        fence_barrier_init();
        badf[0] = badf[1] = 0;
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            const long long t = blockIdx.x + (long long)s * gridDim.x;
            if (t < p.ntiles) issue_tile<DK, DV, YOKED>(p, t, dsmem + s * p.stage_bytes, &bars[s]);
        }
    }
    float g0, g1, pts;
    load_scalars(p, blockIdx.x, g0, g1, pts);

    int it = 0;
    int s = 0;                 // stage of tile it = it % S
    uint32_t parity = 0;       // its barrier phase = (it / S) & 1
    for (long long tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, it++) {
        float n0, n1, nts;
        load_scalars(p, tile + gridDim.x, n0, n1, nts);    // next tile's scalars
        const bool ok = mbar_wait_bounded(&bars[s], parity, p.wait_polls);
        // At this tile's first barrier every thread has finished the previous
        // tile: its stage is refilled with the tile S strides ahead of it, and
        // its non-finite flag is complete.  Without the delta rule or a
        // reference state that is the exchange barrier inside step_tile; Gated
        // DeltaNet (column sums first) and yoked tiles (reference rows written
        // before the exchange) take a barrier here and refill one phase earlier.
        auto at_barrier = [&]() {
            if (threadIdx.x == 0 && it > 0) {
                if (badf[(it - 1) & 1]) {
                    badf[(it - 1) & 1] = 0;
                    atomicAdd(p.counters, 1ull);
                }
                const long long nt = tile + (long long)(S - 1) * gridDim.x;
                const int sp = s == 0 ? S - 1 : s - 1;     // stage of tile it - 1
                if (nt < p.ntiles) issue_tile<DK, DV, YOKED>(p, nt, dsmem + sp * p.stage_bytes, &bars[sp]);
            }
        };
        const uint8_t* st = dsmem + s * p.stage_bytes;
        auto& xs = sh.x[it & 1];
        volatile int* bf = &badf[it & 1];
        uint8_t* ct;
        int bits;
        uint32_t cbytes;
        tile_codes(p, tile, ct, bits, cbytes, DK, DV);
        auto run_tile_g = [&](auto gm, bool okv, auto& hook) -> bool {
            constexpr int G = decltype(gm)::value;
            if constexpr (BITS == 0) {
                switch (bits) {
                    case 2: return step_tile<DK, DV, 2, GDN, YOKED, BDR, BF, EXTRA, G>(p, tile, st, ct, g0, g1, pts, sh, xs, bf, okv, hook);
                    case 4: return step_tile<DK, DV, 4, GDN, YOKED, BDR, BF, EXTRA, G>(p, tile, st, ct, g0, g1, pts, sh, xs, bf, okv, hook);
                    case 6: return step_tile<DK, DV, 6, GDN, YOKED, BDR, BF, EXTRA, G>(p, tile, st, ct, g0, g1, pts, sh, xs, bf, okv, hook);
                    default: return step_tile<DK, DV, 8, GDN, YOKED, BDR, BF, EXTRA, G>(p, tile, st, ct, g0, g1, pts, sh, xs, bf, okv, hook);
                }
            } else {
                (void)bits;
                return step_tile<DK, DV, BITS, GDN, YOKED, BDR, BF, EXTRA, G>(p, tile, st, ct, g0, g1, pts, sh, xs, bf, okv, hook);
            }
        };
        // uniform-width objects without a reference state get a tile body for
        // each kind of scale group (one branch per tile); the others read the
        // group at run time
        auto run_tile = [&](bool okv, auto& hook) -> bool {
            if constexpr (BITS == 0 || YOKED || EXTRA) {
                return run_tile_g(std::integral_constant<int, GM_ANY>{}, okv, hook);
            } else if constexpr (GDN) {
                if (p.group == 0) return run_tile_g(std::integral_constant<int, GM_TILE>{}, okv, hook);
                return run_tile_g(std::integral_constant<int, GM_ROWS>{}, okv, hook);
            } else {
                constexpr int S_ = GM_ALPHA, V_ = GM_ALPHA | GM_VEC;
                if (p.kind == K_GLA) {
                    if (p.group == 0) return run_tile_g(std::integral_constant<int, GM_TILE | V_>{}, okv, hook);
                    return run_tile_g(std::integral_constant<int, GM_ROWS | V_>{}, okv, hook);
                }
                if (p.group == 0) return run_tile_g(std::integral_constant<int, GM_TILE | S_>{}, okv, hook);
                return run_tile_g(std::integral_constant<int, GM_ROWS | S_>{}, okv, hook);
            }
        };
        bool done;
        if constexpr (GDN || YOKED) {
            done = __syncthreads_and(ok);
            if (done) {
                at_barrier();
                auto no_op = []() {};
                run_tile(true, no_op);
            }
        } else {
            done = run_tile(ok, at_barrier);
        }
        if (!done) {
            // some thread gave up on this tile's stage (the vote is uniform)
            if (threadIdx.x == 0) {
                atomicAdd(p.counters + 2, 1ull);
                // drain this CTA's copies still in flight (tiles it .. it+S-1
                // before the first refill, it .. it+S-2 after), each wait bounded
                const int pending = it == 0 ? S : S - 1;
                for (int k = 0; k < pending; k++) {
                    const long long t2 = tile + (long long)k * gridDim.x;
                    if (t2 < p.ntiles)
                        (void)mbar_wait_bounded(&bars[(it + k) % S], ((it + k) / S) & 1,
                                                p.wait_polls);
                }
            }
            return;
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
    if (threadIdx.x == 0 && it > 0 && badf[(it - 1) & 1]) atomicAdd(p.counters, 1ull);
}

// ------------------------------------------------------------------ dequant
// S_hat = code * scale, one thread per 8-column block (reads global memory).
template <int DK, int DV>
__global__ void dequant_kernel(const StepParams p, float* S) {
    const long long nblk = p.ntiles * DK * (DV / 8);
    for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < nblk;
         b += (long long)gridDim.x * blockDim.x) {
        const long long tile = b / (DK * (DV / 8));
        const int rem = int(b % (DK * (DV / 8)));
        const int i = rem / (DV / 8), cb = rem % (DV / 8);
        uint8_t* ct;
        int bits;
        uint32_t cbytes;
        tile_codes(p, tile, ct, bits, cbytes, DK, DV);
        float* dst = S + (tile * DK + i) * (long long)DV + cb * 8;
        float c8[8];
        if (bits == 32) {
            const float* src = reinterpret_cast<const float*>(ct) + i * DV + cb * 8;
#pragma unroll
            for (int c = 0; c < 8; c++) dst[c] = src[c];
            continue;
        }
        const int group = p.group, ng = group ? DV / group : 1;
        const long long si = tile * (long long)p.n_scales + (group ? (long long)i * ng + cb * 8 / group : 0);
        const float d = scale_at(p.scales, si, p.scale_f32 != 0);
        switch (bits) {
            case 2: Decode<2>::run(ct + i * (DV / 4), cb, c8); break;
            case 4: Decode<4>::run(ct + i * (DV / 2), cb, c8); break;
            case 6: Decode6<DK, DV>::run(ct, i, cb, c8); break;
            default: Decode<8>::run(ct + i * DV, cb, c8); break;
        }
#pragma unroll
        for (int c = 0; c < 8; c++) dst[c] = __fmul_rn(c8[c], d);
    }
}

}  // namespace qs
