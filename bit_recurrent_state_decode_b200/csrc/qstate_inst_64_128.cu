// Step kernels for d_k = 64, d_v = 128: every (GDN?, yoked?, BDR?) variant.
#include "qstate_dispatch.h"

namespace qs {
namespace {

template <bool GDN, bool YOKED, bool BDR>
void launch(const StepParams& p, int grid, int dyn_smem, cudaStream_t st) {
    step_kernel<64, 128, GDN, YOKED, BDR><<<grid, Geo<64, 128>::NT, dyn_smem, st>>>(p);
}

template <bool GDN, bool YOKED, bool BDR>
int blocks_per_sm(int dyn_smem) {
    auto* k = step_kernel<64, 128, GDN, YOKED, BDR>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem) != cudaSuccess)
        return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, Geo<64, 128>::NT, dyn_smem) != cudaSuccess)
        return 0;
    return n;
}

template <bool GDN, bool YOKED, bool BDR>
constexpr StepEntry entry() {
    return StepEntry{&launch<GDN, YOKED, BDR>, &blocks_per_sm<GDN, YOKED, BDR>, Geo<64, 128>::NT};
}

const StepEntry kTable[8] = {
    entry<false, false, false>(), entry<false, false, true>(),
    entry<false, true, false>(),  entry<false, true, true>(),
    entry<true, false, false>(),  entry<true, false, true>(),
    entry<true, true, false>(),   entry<true, true, true>(),
};

}  // namespace

const StepEntry* step_table_64_128() { return kTable; }

void launch_dequant_64_128(const StepParams& p, float* S, cudaStream_t st) {
    const long long n = p.ntiles * 64 * (128 / 8);
    long long blocks = (n + 255) / 256;
    if (blocks > 65535LL * 8) blocks = 65535LL * 8;
    if (blocks < 1) blocks = 1;
    dequant_kernel<64, 128><<<(unsigned)blocks, 256, 0, st>>>(p, S);
}

}  // namespace qs
