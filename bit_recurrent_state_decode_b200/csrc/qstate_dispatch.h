// qstate_dispatch.h -- internal: kernel table shared by the C-ABI and the
// per-shape instantiation units.
#pragma once
#include <cuda_runtime.h>

#include "qstate_kernel.cuh"

namespace qs {

struct StepEntry {
    void (*launch)(const StepParams&, int grid, int dyn_smem, cudaStream_t);
    // resident CTAs per SM with `dyn_smem` bytes of dynamic shared memory
    // (also raises the kernel's dynamic shared-memory limit to that size)
    int (*blocks_per_sm)(int dyn_smem);
    int threads;
};

// One table per (d_k, d_v, GDN?) with 96 entries, indexed by
// (((extra * 2 + yoked) * 2 + bdr) * 2 + bf16) * 6 + bits_index (see
// gen_instances.py); extra = 1: the kernels that also hold the taxonomy
// counts and the Hadamard-rotated layout.
const StepEntry* step_table_64_64_0();
const StepEntry* step_table_64_64_1();
const StepEntry* step_table_64_128_0();
const StepEntry* step_table_64_128_1();
const StepEntry* step_table_128_64_0();
const StepEntry* step_table_128_64_1();
const StepEntry* step_table_128_128_0();
const StepEntry* step_table_128_128_1();

// The row-batched kernel for rank-1 updates with round-to-nearest, one code
// width of 4 or 8 bits, scale groups of 32 or 64 columns and d_v = 128:
// 32 entries indexed by
// ((((d_k == 128) * 2 + (bits == 8)) * 2 + (group == 64)) * 2 + gla) * 2 + bf16.
const StepEntry* rows_table();

// The decode step with a Low-Rank Bypass (d_k = d_v in {64, 128}, 4- or
// 8-bit codes): 32 entries indexed by
// ((((d == 128) * 2 + (bits == 8)) * 2 + gdn) * 2 + bdr) * 2 + bf16.
struct LrbParams;
struct LrbEntry {
    void (*launch)(const StepParams&, const LrbParams&, int grid, int dyn_smem, cudaStream_t);
    int (*blocks_per_sm)(int dyn_smem);
    int threads;
};
const LrbEntry* lrb_table();

// The Gated DeltaNet decode step with a pure-write sliding window (d_k = d_v
// in {64, 128}, 4- or 8-bit codes): 16 entries indexed by
// (((d == 128) * 2 + (bits == 8)) * 2 + bdr) * 2 + bf16.
struct PwParams;
struct PwEntry {
    void (*launch)(const StepParams&, const PwParams&, int grid, int dyn_smem, cudaStream_t);
    int (*blocks_per_sm)(int dyn_smem);
    int threads;
};
const PwEntry* pw_table();

// The decode step with key-row x value-column scales: per shape 16 entries
// indexed by (((bits == 8) * 2 + gdn) * 2 + bdr) * 2 + bf16.
struct RcEntry {
    void (*launch)(const StepParams&, int grid, int dyn_smem, cudaStream_t);
    int (*blocks_per_sm)(int dyn_smem);
    void (*dequant)(const StepParams&, float* S, int grid, cudaStream_t);
    int threads;
};
const RcEntry* rc_table_64_64();
const RcEntry* rc_table_64_128();
const RcEntry* rc_table_128_64();
const RcEntry* rc_table_128_128();

// Launch a step kernel with programmatic stream serialization (the kernel
// waits for the previous kernel of the stream before any global access, and
// its prologue and scheduling overlap that kernel's tail).
template <class K>
inline void launch_pdl(K kernel, const StepParams& p, int grid, int threads, int dyn_smem,
                       cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)dyn_smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, p);
}

// 0 = per-head widths, then 2, 4, 6, 8, 32 bits; -1 if invalid
inline int bits_index(int bits) {
    switch (bits) {
        case 0: return 0;
        case 2: return 1;
        case 4: return 2;
        case 6: return 3;
        case 8: return 4;
        case 32: return 5;
        default: return -1;
    }
}

void launch_dequant(int dk, int dv, const StepParams& p, float* S, cudaStream_t st);

// Raise the kernel's dynamic shared-memory limit to at least `bytes` (never
// lower it: objects of different layouts launch the same kernel with
// different stage sizes).  Serialised by a process-wide lock; false if a
// CUDA call failed.
bool raise_dyn_smem_limit(const void* kernel, int bytes);

}  // namespace qs
