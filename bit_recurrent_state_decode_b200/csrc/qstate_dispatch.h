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

// One table per (d_k, d_v), indexed by gdn * 4 + yoked * 2 + bdr.
const StepEntry* step_table_64_64();
const StepEntry* step_table_64_128();
const StepEntry* step_table_128_64();
const StepEntry* step_table_128_128();

void launch_dequant(int dk, int dv, const StepParams& p, float* S, cudaStream_t st);

}  // namespace qs
