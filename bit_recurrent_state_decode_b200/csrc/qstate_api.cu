// qstate_api.cu -- the C ABI declared in include/qstate.h: argument
// validation, device memory of a state object, kernel dispatch and the
// host-buffer step.  All compute runs in the kernels of qstate_kernel.cuh.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "qstate.h"
#include "qstate_dispatch.h"
#include "qstate_lrb.cuh"
#include "qstate_pw.cuh"
#include "qstate_rc.cuh"

namespace qs {
void launch_dequant_64_64(const StepParams&, float*, cudaStream_t);
void launch_dequant_64_128(const StepParams&, float*, cudaStream_t);
void launch_dequant_128_64(const StepParams&, float*, cudaStream_t);
void launch_dequant_128_128(const StepParams&, float*, cudaStream_t);

void launch_dequant(int dk, int dv, const StepParams& p, float* S, cudaStream_t st) {
    if (dk == 64 && dv == 64) launch_dequant_64_64(p, S, st);
    else if (dk == 64) launch_dequant_64_128(p, S, st);
    else if (dv == 64) launch_dequant_128_64(p, S, st);
    else launch_dequant_128_128(p, S, st);
}

bool raise_dyn_smem_limit(const void* kernel, int bytes) {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return false;
    if (fa.maxDynamicSharedSizeBytes >= bytes) return true;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
           cudaSuccess;
}
}  // namespace qs

struct qstate {
    qstate_layout L;
    int bits, group, scale_mode, round_mode;
    float eps_b;
    int device;
    int64_t tiles, code_bytes, scale_bytes, ref_bytes, n_scales, n_gate;
    int64_t tile_bytes, row_bytes;   // uniform tile bytes; bytes of one (layer, batch) row
    int64_t in_size, gate_size, scale_size;
    std::vector<uint8_t> head_bits;  // empty when uniform
    uint8_t* d_codes = nullptr;
    void* d_scales = nullptr;
    float* d_ref = nullptr;
    unsigned long long* d_counters = nullptr;
    long long* d_head_off = nullptr;
    unsigned char* d_head_bits = nullptr;
    const qs::StepEntry* entry = nullptr;
    int grid = 1;
    // the general kernel, when `entry` is a specialised one (the taxonomy
    // counts run in the general kernel only)
    const qs::StepEntry* entry_general = nullptr;
    const char* entry_name = "step_kernel";
    int grid_general = 1;
    bool taxonomy = false;
    int dyn_smem = 0;                 // bytes of pipeline stages per CTA
    unsigned wait_polls = qs::kWaitPolls;
    long long drop_from = -1;
    // Low-Rank Bypass (qstate_set_lrb): bypass columns, coefficients, slot
    // counts and the decay since the last merge, per tile
    // per key row the squared rounding error of the last step (allocated when
    // the taxonomy is first switched on)
    float* d_err = nullptr;
    bool lrb = false;
    int lrb_k = 0, lrb_m = 0;
    float lrb_eps = 0.0f;
    uint16_t* d_lu = nullptr;
    uint16_t* d_lw = nullptr;
    float* d_lg = nullptr;
    int* d_ln = nullptr;
    float* d_lD = nullptr;
    const qs::LrbEntry* lrb_entry = nullptr;
    int lrb_grid = 1, lrb_smem = 0;
    // key-row x value-column scales (qstate_set_rowcol): scales
    // [tiles][d_k + d_v], rho then kappa
    bool rowcol = false;
    const qs::RcEntry* rc_entry = nullptr;
    int rc_grid = 1;
    // pure-write sliding window (qstate_set_pw): the pairs, the slot of the
    // oldest pair and the pairs held, per tile
    bool pw = false;
    int pw_W = 0;
    uint8_t* d_pa = nullptr;
    uint8_t* d_pb = nullptr;
    int* d_phead = nullptr;
    int* d_pcount = nullptr;
    const qs::PwEntry* pw_entry = nullptr;
    int pw_grid = 1;
    // set by qstate_import: the next step takes the general tile bodies (an
    // imported state may hold the code -2^(bits-1), which no step produces)
    bool import_pending = false;
    qs::StepParams stage{};           // stage layout fields only
    // staging buffers of qstate_step_host (allocated by its first call): the
    // inputs in two sets used by alternate calls, copied on the object's own
    // stream so that one call's copies overlap the previous call's step
    void* st_q = nullptr;
    void* st_k = nullptr;
    void* st_v = nullptr;
    void* st_g = nullptr;
    float* st_out = nullptr;
    void* st2_q = nullptr;
    void* st2_k = nullptr;
    void* st2_v = nullptr;
    void* st2_g = nullptr;
    float* st2_out = nullptr;
    cudaStream_t h2d = nullptr;
    cudaStream_t d2h = nullptr;
    cudaEvent_t copied[2] = {nullptr, nullptr};     // inputs of set b in device memory
    cudaEvent_t consumed[2] = {nullptr, nullptr};   // the step of set b has run
    cudaEvent_t delivered[2] = {nullptr, nullptr};  // the output of set b is in host memory
    uint64_t host_calls = 0;
};

namespace {

int64_t tile_bytes_of(int bits, int dk, int dv) { return (int64_t)dk * dv * bits / 8; }

bool valid_bits(int b) { return b == 2 || b == 4 || b == 6 || b == 8 || b == 32; }

qs::StepParams params_of(const qstate* s) {
    qs::StepParams p{};
    p.codes = s->d_codes;
    p.scales = s->d_scales;
    p.ref = s->d_ref;
    p.counters = s->d_counters;
    p.head_off = s->d_head_off;
    p.head_bits = s->d_head_bits;
    p.row_bytes = s->row_bytes;
    p.tile_bytes = s->tile_bytes;
    p.ntiles = s->tiles;
    p.heads = s->L.heads;
    p.bits = s->bits;
    p.group = s->group;
    p.n_scales = (int)s->n_scales;
    p.kind = s->L.kind;
    p.scale_mode = s->scale_mode;
    p.n_gate = (int)s->n_gate;
    p.qkv_bf16 = s->L.qkv_dtype == QSTATE_BF16;
    p.gate_bf16 = s->L.gate_dtype == QSTATE_BF16;
    p.scale_f32 = s->L.scale_dtype == QSTATE_F32;
    // per-tile scalars: alpha (Mamba2, GDN), beta (GDN), the previous scale of
    // a per-token quantized state (mixed widths are never 32)
    p.scalars = 0;
    if (s->L.kind == QSTATE_MAMBA2 || s->L.kind == QSTATE_GDN) p.scalars |= qs::SC_G0;
    if (s->L.kind == QSTATE_GDN) p.scalars |= qs::SC_G1;
    if (s->group == 0 && (!s->head_bits.empty() || s->bits != 32)) p.scalars |= qs::SC_PTS;
    p.gamma = s->L.gamma;
    p.eps_b = s->eps_b;
    p.nstages = s->stage.nstages;
    p.stage_bytes = s->stage.stage_bytes;
    p.off_codes = s->stage.off_codes;
    p.off_scales = s->stage.off_scales;
    p.off_q = s->stage.off_q;
    p.off_k = s->stage.off_k;
    p.off_v = s->stage.off_v;
    p.off_ga = s->stage.off_ga;
    p.off_ref = s->stage.off_ref;
    p.wait_polls = s->wait_polls;
    p.drop_from = s->drop_from;
    p.fast = s->import_pending ? 0 : 1;
    p.taxonomy = s->taxonomy ? 1 : 0;
    p.rotate = s->L.rotation;
    p.err_rows = s->taxonomy ? s->d_err : nullptr;
    return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void free_all(qstate* s) {
    if (!s) return;
    cudaFree(s->d_codes);
    cudaFree(s->d_scales);
    cudaFree(s->d_ref);
    cudaFree(s->d_counters);
    cudaFree(s->d_head_off);
    cudaFree(s->d_head_bits);
    cudaFree(s->st_q);
    cudaFree(s->st_k);
    cudaFree(s->st_v);
    cudaFree(s->st_g);
    cudaFree(s->st_out);
    cudaFree(s->st2_q);
    cudaFree(s->st2_k);
    cudaFree(s->st2_v);
    cudaFree(s->st2_g);
    cudaFree(s->st2_out);
    for (int b = 0; b < 2; b++) {
        if (s->copied[b]) cudaEventDestroy(s->copied[b]);
        if (s->consumed[b]) cudaEventDestroy(s->consumed[b]);
        if (s->delivered[b]) cudaEventDestroy(s->delivered[b]);
    }
    if (s->h2d) cudaStreamDestroy(s->h2d);
    if (s->d2h) cudaStreamDestroy(s->d2h);
    cudaFree(s->d_err);
    cudaFree(s->d_lu);
    cudaFree(s->d_lw);
    cudaFree(s->d_lg);
    cudaFree(s->d_ln);
    cudaFree(s->d_lD);
    cudaFree(s->d_pa);
    cudaFree(s->d_pb);
    cudaFree(s->d_phead);
    cudaFree(s->d_pcount);
}

// an empty window
int zero_window(qstate* s, cudaStream_t st) {
    if (!s->pw || s->tiles == 0) return QSTATE_OK;
    const int64_t T = s->tiles, W = s->pw_W;
    if (cudaMemsetAsync(s->d_pa, 0, T * W * s->L.d_k, st) != cudaSuccess ||
        cudaMemsetAsync(s->d_pb, 0, T * W * s->L.d_v, st) != cudaSuccess ||
        cudaMemsetAsync(s->d_phead, 0, T * 4, st) != cudaSuccess ||
        cudaMemsetAsync(s->d_pcount, 0, T * 4, st) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

// decay factors a tile's bypass holds: one per key row for GLA, else one
int64_t lrb_dlen(const qstate* s) { return s->L.kind == QSTATE_GLA ? s->L.d_k : 1; }

// bypass empty, D = 1 for every tile
int zero_bypass(qstate* s, cudaStream_t st) {
    if (!s->lrb || s->tiles == 0) return QSTATE_OK;
    const int64_t K = s->lrb_k + s->lrb_m;
    if (cudaMemsetAsync(s->d_lu, 0, s->tiles * K * s->L.d_k * 2, st) != cudaSuccess ||
        cudaMemsetAsync(s->d_lw, 0, s->tiles * K * s->L.d_v * 2, st) != cudaSuccess ||
        cudaMemsetAsync(s->d_lg, 0, s->tiles * K * 4, st) != cudaSuccess ||
        cudaMemsetAsync(s->d_ln, 0, s->tiles * 2 * 4, st) != cudaSuccess)
        return QSTATE_ECUDA;
    // D = 1: copied from a host array (a copy from pageable memory has left
    // the array when the call returns)
    std::vector<float> ones((size_t)(s->tiles * lrb_dlen(s)), 1.0f);
    if (cudaMemcpyAsync(s->d_lD, ones.data(), ones.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

int zero_state(qstate* s, cudaStream_t st) {
    if (s->code_bytes && cudaMemsetAsync(s->d_codes, 0, s->code_bytes, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (s->scale_bytes && cudaMemsetAsync(s->d_scales, 0, s->scale_bytes, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (s->ref_bytes && cudaMemsetAsync(s->d_ref, 0, s->ref_bytes, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (cudaMemsetAsync(s->d_counters, 0, qs::kNumCounters * sizeof(unsigned long long), st) !=
        cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

int check_device(const qstate* s) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return QSTATE_ECUDA;
    return dev == s->device ? QSTATE_OK : QSTATE_EINVAL;
}

}  // namespace

extern "C" {

const char* qstate_error_string(int code) {
    switch (code) {
        case QSTATE_OK: return "ok";
        case QSTATE_EINVAL: return "invalid argument";
        case QSTATE_ENOMEM: return "out of memory";
        case QSTATE_ECUDA: return "CUDA runtime error";
        case QSTATE_EUNSUPPORTED: return "unsupported configuration";
        default: return "unknown error";
    }
}

int qstate_create(const qstate_layout* L, int bits, int group, qstate_scale_mode sm,
                  qstate_round_mode rm, float eps_b, qstate** out) {
    if (!L || !out) return QSTATE_EINVAL;
    *out = nullptr;
    if (L->batch < 0 || L->heads < 1 || L->layers < 1) return QSTATE_EINVAL;
    if ((int64_t)L->layers * L->batch * L->heads > INT32_MAX) return QSTATE_EINVAL;
    if (L->d_k < 8 || L->d_v < 8 || L->d_k % 8 || L->d_v % 8) return QSTATE_EINVAL;
    if (L->kind < QSTATE_RETNET || L->kind > QSTATE_GDN) return QSTATE_EINVAL;
    if (L->qkv_dtype != QSTATE_F32 && L->qkv_dtype != QSTATE_BF16) return QSTATE_EINVAL;
    if (L->gate_dtype != QSTATE_F32 && L->gate_dtype != QSTATE_BF16) return QSTATE_EINVAL;
    if (L->scale_dtype != QSTATE_F16 && L->scale_dtype != QSTATE_F32) return QSTATE_EINVAL;
    if (L->kind == QSTATE_RETNET && !std::isfinite(L->gamma)) return QSTATE_EINVAL;
    if (L->rotation != 0 && L->rotation != 1) return QSTATE_EINVAL;
    if (sm < QSTATE_DYNAMIC || sm > QSTATE_YOKED) return QSTATE_EINVAL;
    if (rm < QSTATE_RTN || rm > QSTATE_BDR) return QSTATE_EINVAL;
    if (!(eps_b >= 0.0f) || !std::isfinite(eps_b)) return QSTATE_EINVAL;
    if (group < 0 || (group && (group % 8 || L->d_v % group))) return QSTATE_EINVAL;
    std::vector<uint8_t> hb;
    if (L->head_bits) {
        hb.assign(L->head_bits, L->head_bits + L->heads);
        for (uint8_t b : hb)
            if (!(b == 2 || b == 4 || b == 6 || b == 8)) return QSTATE_EINVAL;
    } else if (!valid_bits(bits)) {
        return QSTATE_EINVAL;
    }
    if (sm == QSTATE_YOKED && hb.empty() && bits == 32) return QSTATE_EINVAL;
    if (!((L->d_k == 64 || L->d_k == 128) && (L->d_v == 64 || L->d_v == 128)))
        return QSTATE_EUNSUPPORTED;

    qstate* s = new (std::nothrow) qstate();
    if (!s) return QSTATE_ENOMEM;
    s->L = *L;
    s->L.head_bits = nullptr;
    s->bits = hb.empty() ? bits : 0;
    s->group = group;
    s->scale_mode = sm;
    s->round_mode = rm;
    s->eps_b = eps_b;
    s->head_bits = hb;
    if (cudaGetDevice(&s->device) != cudaSuccess) { delete s; return QSTATE_ECUDA; }

    const int dk = L->d_k, dv = L->d_v;
    s->tiles = (int64_t)L->layers * L->batch * L->heads;
    s->n_scales = group ? (int64_t)dk * (dv / group) : 1;
    s->n_gate = L->kind == QSTATE_RETNET ? 0 : L->kind == QSTATE_MAMBA2 ? 1
              : L->kind == QSTATE_GLA ? dk : 2;
    s->in_size = L->qkv_dtype == QSTATE_BF16 ? 2 : 4;
    s->gate_size = L->gate_dtype == QSTATE_BF16 ? 2 : 4;
    s->scale_size = L->scale_dtype == QSTATE_F32 ? 4 : 2;
    std::vector<long long> head_off;
    if (hb.empty()) {
        s->tile_bytes = tile_bytes_of(bits, dk, dv);
        s->row_bytes = s->tile_bytes * L->heads;
    } else {
        s->tile_bytes = 0;
        long long off = 0;
        for (uint8_t b : hb) { head_off.push_back(off); off += tile_bytes_of(b, dk, dv); }
        s->row_bytes = off;
    }
    s->code_bytes = s->row_bytes * (int64_t)L->layers * L->batch;
    const bool quantized = !hb.empty() || bits != 32;
    s->scale_bytes = quantized ? s->tiles * s->n_scales * s->scale_size : 0;
    s->ref_bytes = sm == QSTATE_YOKED ? s->tiles * dk * dv * 4 : 0;

    auto alloc = [&](void** p, size_t n) -> bool {
        if (!n) return true;
        return cudaMalloc(p, n) == cudaSuccess;
    };
    bool ok = alloc((void**)&s->d_codes, s->code_bytes) &&
              alloc(&s->d_scales, s->scale_bytes) &&
              alloc((void**)&s->d_ref, s->ref_bytes) &&
              alloc((void**)&s->d_counters, qs::kNumCounters * sizeof(unsigned long long));
    if (ok && !hb.empty()) {
        ok = alloc((void**)&s->d_head_off, head_off.size() * sizeof(long long)) &&
             alloc((void**)&s->d_head_bits, hb.size()) &&
             cudaMemcpy(s->d_head_off, head_off.data(), head_off.size() * sizeof(long long),
                        cudaMemcpyHostToDevice) == cudaSuccess &&
             cudaMemcpy(s->d_head_bits, hb.data(), hb.size(), cudaMemcpyHostToDevice) == cudaSuccess;
    }
    if (!ok) {
        cudaGetLastError();
        free_all(s);
        delete s;
        return QSTATE_ENOMEM;
    }

    const qs::StepEntry* tab;
    const bool gdn = L->kind == QSTATE_GDN;
    if (dk == 64 && dv == 64) tab = gdn ? qs::step_table_64_64_1() : qs::step_table_64_64_0();
    else if (dk == 64) tab = gdn ? qs::step_table_64_128_1() : qs::step_table_64_128_0();
    else if (dv == 64) tab = gdn ? qs::step_table_128_64_1() : qs::step_table_128_64_0();
    else tab = gdn ? qs::step_table_128_128_1() : qs::step_table_128_128_0();
    const int bidx = qs::bits_index(hb.empty() ? bits : 0);
    const int yk = sm == QSTATE_YOKED, bd = rm == QSTATE_BDR, bf = L->qkv_dtype == QSTATE_BF16;
    s->entry = &tab[((yk * 2 + bd) * 2 + bf) * 6 + bidx];
    // the kernel with the extra features: taxonomy counts (switched on later)
    // and the rotated layout (fixed at creation)
    s->entry_general = &tab[48 + ((yk * 2 + bd) * 2 + bf) * 6 + bidx];
    if (L->rotation) s->entry = s->entry_general;
    // rank-1 updates with round-to-nearest, one width of 4 or 8 bits, no
    // reference state, scale groups of 32 or 64 columns and d_v = 128: the
    // row-batched kernel (16 rows per thread, group maxima inside a warp)
    if (L->kind != QSTATE_GDN && rm == QSTATE_RTN && sm != QSTATE_YOKED && hb.empty() &&
        (bits == 4 || bits == 8) && dv == 128 && (group == 32 || group == 64) &&
        L->rotation == 0) {
        const int ridx = ((((dk == 128) * 2 + (bits == 8)) * 2 + (group == 64)) * 2 +
                          (L->kind == QSTATE_GLA)) * 2 + bf;
        s->entry = &qs::rows_table()[ridx];
        s->entry_name = "rows_kernel";
    }
    if (!s->entry->launch) {
        free_all(s);
        delete s;
        return QSTATE_EUNSUPPORTED;
    }

    // pipeline stage: codes | scales | q | k | v | GLA gate vector | reference
    {
        auto up16 = [](int64_t x) { return (x + 15) & ~int64_t(15); };
        int maxbits = hb.empty() ? bits : 0;
        for (uint8_t b : hb) maxbits = b > maxbits ? b : maxbits;
        qs::StepParams& g = s->stage;
        int64_t off = 0;
        g.off_codes = 0;
        off = up16(tile_bytes_of(maxbits, dk, dv));
        g.off_scales = -1;
        if (quantized && group) {
            g.off_scales = (int)off;
            off = up16(off + s->n_scales * s->scale_size);
        }
        g.off_q = (int)off;  off = up16(off + dk * s->in_size);
        g.off_k = (int)off;  off = up16(off + dk * s->in_size);
        g.off_v = (int)off;  off = up16(off + dv * s->in_size);
        g.off_ga = -1;
        if (L->kind == QSTATE_GLA) { g.off_ga = (int)off; off = up16(off + dk * s->gate_size); }
        g.off_ref = -1;
        if (sm == QSTATE_YOKED) { g.off_ref = (int)off; off = up16(off + (int64_t)dk * dv * 4); }
        g.stage_bytes = (int)off;
        // as many stages (2..4) as fit next to the kernel's static shared memory
        int ns = (int)(200 * 1024 / off);
        g.nstages = ns < 2 ? 2 : ns > qs::kMaxStages ? qs::kMaxStages : ns;
        s->dyn_smem = g.nstages * g.stage_bytes;
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, s->device);
    // resident CTAs per SM of both kernels with this stage size
    auto occupancy = [&](int& fast_sm, int& general_sm) {
        fast_sm = s->entry->blocks_per_sm(s->dyn_smem);
        general_sm = s->entry_general == s->entry ? fast_sm
                                                  : s->entry_general->blocks_per_sm(s->dyn_smem);
    };
    int per_sm, per_sm_general;
    occupancy(per_sm, per_sm_general);
    while ((per_sm < 1 || per_sm_general < 1) && s->stage.nstages > 2) {   // fewer stages
        cudaGetLastError();
        s->stage.nstages--;
        s->dyn_smem = s->stage.nstages * s->stage.stage_bytes;
        occupancy(per_sm, per_sm_general);
    }
    if (per_sm < 1 || per_sm_general < 1) {
        cudaGetLastError();
        free_all(s);
        delete s;
        return QSTATE_EUNSUPPORTED;
    }
    auto grid_of = [&](int resident) {
        long long g = (long long)sms * resident;
        if (g < 1) g = 1;
        if (s->tiles < g) g = s->tiles > 0 ? s->tiles : 1;
        return (int)g;
    };
    s->grid = grid_of(per_sm);
    s->grid_general = grid_of(per_sm_general);

    int rc = zero_state(s, nullptr);
    if (rc == QSTATE_OK && cudaDeviceSynchronize() != cudaSuccess) rc = QSTATE_ECUDA;
    if (rc != QSTATE_OK) {
        free_all(s);
        delete s;
        return rc;
    }
    *out = s;
    return QSTATE_OK;
}

int qstate_destroy(qstate* s) {
    if (!s) return QSTATE_EINVAL;
    free_all(s);
    delete s;
    return QSTATE_OK;
}

int qstate_reset(qstate* s, qstate_stream stream) {
    if (!s) return QSTATE_EINVAL;
    int rc = zero_state(s, (cudaStream_t)stream);
    if (rc == QSTATE_OK) rc = zero_bypass(s, (cudaStream_t)stream);
    if (rc == QSTATE_OK) rc = zero_window(s, (cudaStream_t)stream);
    return rc;
}

int qstate_step(qstate* s, const void* q, const void* k, const void* v, const void* gates,
                float* out, qstate_stream stream) {
    if (!s || !q || !k || !v || !out) return QSTATE_EINVAL;
    if (s->n_gate && !gates) return QSTATE_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (gates && !aligned16(gates)))
        return QSTATE_EINVAL;
    if (s->tiles == 0) return QSTATE_OK;
    int rc = check_device(s);
    if (rc != QSTATE_OK) return rc;
    qs::StepParams p = params_of(s);
    p.q = q;
    p.k = k;
    p.v = v;
    p.gates = gates;
    p.out = out;
    if (s->rowcol) {
        s->rc_entry->launch(p, s->rc_grid, 0, (cudaStream_t)stream);
        return cudaGetLastError() == cudaSuccess ? QSTATE_OK : QSTATE_ECUDA;
    }
    if (s->pw) {
        qs::PwParams Pp{s->d_pa, s->d_pb, s->d_phead, s->d_pcount, s->pw_W};
        s->pw_entry->launch(p, Pp, s->pw_grid, 0, (cudaStream_t)stream);
        return cudaGetLastError() == cudaSuccess ? QSTATE_OK : QSTATE_ECUDA;
    }
    if (s->lrb) {
        qs::LrbParams Lp{s->d_lu, s->d_lw, s->d_lg, s->d_ln, s->d_lD, s->lrb_k, s->lrb_m, s->lrb_eps};
        s->lrb_entry->launch(p, Lp, s->lrb_grid, s->lrb_smem, (cudaStream_t)stream);
        return cudaGetLastError() == cudaSuccess ? QSTATE_OK : QSTATE_ECUDA;
    }
    if (s->taxonomy)
        s->entry_general->launch(p, s->grid_general, s->dyn_smem, (cudaStream_t)stream);
    else
        s->entry->launch(p, s->grid, s->dyn_smem, (cudaStream_t)stream);
    if (cudaGetLastError() != cudaSuccess) return QSTATE_ECUDA;
    s->import_pending = false;     // every code is within +-Qmax after a step
    return QSTATE_OK;
}

int qstate_get_sizes(const qstate* s, qstate_sizes* o) {
    if (!s || !o) return QSTATE_EINVAL;
    o->tiles = s->tiles;
    o->code_bytes = s->code_bytes;
    o->scale_bytes = s->scale_bytes;
    o->ref_bytes = s->ref_bytes;
    o->n_scales = s->n_scales;
    o->n_gate = s->n_gate;
    o->q_bytes = s->tiles * s->L.d_k * s->in_size;
    o->v_bytes = s->tiles * s->L.d_v * s->in_size;
    o->gate_bytes = s->tiles * s->n_gate * s->gate_size;
    o->out_bytes = s->tiles * s->L.d_v * 4;
    return QSTATE_OK;
}

}  // extern "C"

namespace {

// The host-buffer step (qstate_step_host, qstate_step_host_pipelined): the
// inputs and outputs in two staging sets used by alternate calls; the input
// copies on the object's h2d stream, the output copy on its d2h stream, the
// step on the caller's stream.  Each copy waits only for what it reads or
// overwrites: the inputs of set b for the step two calls back (which read
// them), the step for the output copy two calls back (which read set b's
// output).  sync_out: the caller's stream also waits for this call's output
// copy (else for the previous call's).
int step_host_impl(qstate* s, const void* q, const void* k, const void* v, const void* gates,
                   float* out, cudaStream_t st, bool sync_out) {
    if (!s || !q || !k || !v || !out) return QSTATE_EINVAL;
    if (s->n_gate && !gates) return QSTATE_EINVAL;
    if (s->tiles == 0) return QSTATE_OK;
    int rc = check_device(s);
    if (rc != QSTATE_OK) return rc;
    qstate_sizes z;
    qstate_get_sizes(s, &z);
    if (!s->st_q) {
        bool ok = cudaMalloc(&s->st_q, z.q_bytes) == cudaSuccess &&
                  cudaMalloc(&s->st_k, z.q_bytes) == cudaSuccess &&
                  cudaMalloc(&s->st_v, z.v_bytes) == cudaSuccess &&
                  (!z.gate_bytes || cudaMalloc(&s->st_g, z.gate_bytes) == cudaSuccess) &&
                  cudaMalloc(&s->st2_q, z.q_bytes) == cudaSuccess &&
                  cudaMalloc(&s->st2_k, z.q_bytes) == cudaSuccess &&
                  cudaMalloc(&s->st2_v, z.v_bytes) == cudaSuccess &&
                  (!z.gate_bytes || cudaMalloc(&s->st2_g, z.gate_bytes) == cudaSuccess) &&
                  cudaMalloc((void**)&s->st_out, z.out_bytes) == cudaSuccess &&
                  cudaMalloc((void**)&s->st2_out, z.out_bytes) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&s->h2d, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&s->d2h, cudaStreamNonBlocking) == cudaSuccess;
        for (int b = 0; ok && b < 2; b++)
            ok = cudaEventCreateWithFlags(&s->copied[b], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&s->consumed[b], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&s->delivered[b], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            cudaGetLastError();
            cudaFree(s->st_q); cudaFree(s->st_k); cudaFree(s->st_v);
            cudaFree(s->st_g); cudaFree(s->st_out);
            cudaFree(s->st2_q); cudaFree(s->st2_k); cudaFree(s->st2_v); cudaFree(s->st2_g);
            cudaFree(s->st2_out);
            for (int b = 0; b < 2; b++) {
                if (s->copied[b]) cudaEventDestroy(s->copied[b]);
                if (s->consumed[b]) cudaEventDestroy(s->consumed[b]);
                if (s->delivered[b]) cudaEventDestroy(s->delivered[b]);
                s->copied[b] = s->consumed[b] = s->delivered[b] = nullptr;
            }
            if (s->h2d) cudaStreamDestroy(s->h2d);
            if (s->d2h) cudaStreamDestroy(s->d2h);
            s->h2d = s->d2h = nullptr;
            s->st_q = s->st_k = s->st_v = s->st_g = nullptr;
            s->st2_q = s->st2_k = s->st2_v = s->st2_g = nullptr;
            s->st_out = s->st2_out = nullptr;
            return QSTATE_ENOMEM;
        }
    }
    const int b = (int)(s->host_calls & 1);
    void* dq = b ? s->st2_q : s->st_q;
    void* dk = b ? s->st2_k : s->st_k;
    void* dv = b ? s->st2_v : s->st_v;
    void* dg = b ? s->st2_g : s->st_g;
    float* dout = b ? s->st2_out : s->st_out;
    if (cudaStreamWaitEvent(s->h2d, s->consumed[b], 0) != cudaSuccess ||
        cudaMemcpyAsync(dq, q, z.q_bytes, cudaMemcpyHostToDevice, s->h2d) != cudaSuccess ||
        cudaMemcpyAsync(dk, k, z.q_bytes, cudaMemcpyHostToDevice, s->h2d) != cudaSuccess ||
        cudaMemcpyAsync(dv, v, z.v_bytes, cudaMemcpyHostToDevice, s->h2d) != cudaSuccess ||
        (z.gate_bytes &&
         cudaMemcpyAsync(dg, gates, z.gate_bytes, cudaMemcpyHostToDevice, s->h2d) != cudaSuccess) ||
        cudaEventRecord(s->copied[b], s->h2d) != cudaSuccess ||
        cudaStreamWaitEvent(st, s->copied[b], 0) != cudaSuccess ||
        cudaStreamWaitEvent(st, s->delivered[b], 0) != cudaSuccess)
        return QSTATE_ECUDA;
    rc = qstate_step(s, dq, dk, dv, dg, dout, (qstate_stream)st);
    if (rc != QSTATE_OK) return rc;
    if (cudaEventRecord(s->consumed[b], st) != cudaSuccess ||
        cudaStreamWaitEvent(s->d2h, s->consumed[b], 0) != cudaSuccess ||
        cudaMemcpyAsync(out, dout, z.out_bytes, cudaMemcpyDeviceToHost, s->d2h) != cudaSuccess ||
        cudaEventRecord(s->delivered[b], s->d2h) != cudaSuccess ||
        cudaStreamWaitEvent(st, s->delivered[sync_out ? b : 1 - b], 0) != cudaSuccess)
        return QSTATE_ECUDA;
    s->host_calls++;
    return QSTATE_OK;
}

}  // namespace

extern "C" {

int qstate_step_host(qstate* s, const void* q, const void* k, const void* v, const void* gates,
                     float* out, qstate_stream stream) {
    return step_host_impl(s, q, k, v, gates, out, (cudaStream_t)stream, true);
}

int qstate_step_host_pipelined(qstate* s, const void* q, const void* k, const void* v,
                               const void* gates, float* out, qstate_stream stream) {
    return step_host_impl(s, q, k, v, gates, out, (cudaStream_t)stream, false);
}

int qstate_step_host_sync(qstate* s, qstate_stream stream) {
    if (!s) return QSTATE_EINVAL;
    if (!s->host_calls) return QSTATE_OK;
    const int last = (int)((s->host_calls - 1) & 1);
    return cudaStreamWaitEvent((cudaStream_t)stream, s->delivered[last], 0) == cudaSuccess
               ? QSTATE_OK : QSTATE_ECUDA;
}

int qstate_dequant(const qstate* s, float* S_out, qstate_stream stream) {
    if (!s || !S_out) return QSTATE_EINVAL;
    if (s->tiles == 0) return QSTATE_OK;
    int rc = check_device(s);
    if (rc != QSTATE_OK) return rc;
    if (s->rowcol)
        s->rc_entry->dequant(params_of(s), S_out, s->rc_grid, (cudaStream_t)stream);
    else
        qs::launch_dequant(s->L.d_k, s->L.d_v, params_of(s), S_out, (cudaStream_t)stream);
    return cudaGetLastError() == cudaSuccess ? QSTATE_OK : QSTATE_ECUDA;
}

int qstate_export(const qstate* s, void* codes, void* scales, float* ref, qstate_stream stream) {
    if (!s || !codes || (s->scale_bytes && !scales) || (s->ref_bytes && !ref)) return QSTATE_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    if (s->code_bytes &&
        cudaMemcpyAsync(codes, s->d_codes, s->code_bytes, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (s->scale_bytes &&
        cudaMemcpyAsync(scales, s->d_scales, s->scale_bytes, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (s->ref_bytes &&
        cudaMemcpyAsync(ref, s->d_ref, s->ref_bytes, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

int qstate_import(qstate* s, const void* codes, const void* scales, const float* ref,
                  qstate_stream stream) {
    if (!s || !codes || (s->scale_bytes && !scales) || (s->ref_bytes && !ref)) return QSTATE_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    if (s->code_bytes &&
        cudaMemcpyAsync(s->d_codes, codes, s->code_bytes, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (s->scale_bytes &&
        cudaMemcpyAsync(s->d_scales, scales, s->scale_bytes, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    if (s->ref_bytes &&
        cudaMemcpyAsync(s->d_ref, ref, s->ref_bytes, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    s->import_pending = true;
    int rc = zero_bypass(s, st);
    if (rc == QSTATE_OK) rc = zero_window(s, st);
    return rc;
}

int64_t qstate_bytes_per_step(const qstate* s) {
    if (!s) return -1;
    const int64_t dk = s->L.d_k, dv = s->L.d_v;
    const int64_t ops = s->tiles * ((2 * dk + dv) * s->in_size + s->n_gate * s->gate_size + dv * 4);
    if (s->pw) {
        // state and scales read and written; every pair read, every key side
        // and the new value side written
        const int64_t W = s->pw_W;
        return 2 * s->code_bytes + 2 * s->scale_bytes + ops +
               s->tiles * (W * (dk + dv) + W * dk + dv + 16);
    }
    if (s->lrb) {
        // averaged over a merge cycle of m steps: the state is read every step
        // and written at the merge; the columns held at the start of a step
        // (k + (m - 1) / 2 on average) are read, one column and the
        // coefficients written; the residual columns written at the merge
        const int64_t k = s->lrb_k, m = s->lrb_m;
        const int64_t col = (dk + dv) * 2 + 4;
        int64_t b = m * (s->code_bytes + s->scale_bytes) + s->code_bytes + s->scale_bytes;
        b += s->tiles * ((k * m + m * (m - 1) / 2) * col + m * col + k * col +
                         m * (8 + 8 * lrb_dlen(s)));
        return b / m + ops;
    }
    int64_t b = 2 * s->code_bytes + 2 * s->scale_bytes + 2 * s->ref_bytes;
    return b + ops;
}

int qstate_set_rowcol(qstate* s) {
    if (!s || s->rowcol || s->pw || s->lrb) return QSTATE_EINVAL;
    const int dk = s->L.d_k, dv = s->L.d_v;
    if (s->scale_mode != QSTATE_DYNAMIC || s->L.rotation || !s->head_bits.empty() ||
        !(s->bits == 4 || s->bits == 8))
        return QSTATE_EUNSUPPORTED;
    int rc = check_device(s);
    if (rc != QSTATE_OK) return rc;
    const qs::RcEntry* tab = dk == 64 ? (dv == 64 ? qs::rc_table_64_64() : qs::rc_table_64_128())
                                      : (dv == 64 ? qs::rc_table_128_64() : qs::rc_table_128_128());
    const int idx = (((s->bits == 8) * 2 + (s->L.kind == QSTATE_GDN)) * 2 +
                     (s->round_mode == QSTATE_BDR)) * 2 + (s->L.qkv_dtype == QSTATE_BF16);
    const qs::RcEntry* e = &tab[idx];
    const int per_sm = e->blocks_per_sm(0);
    if (per_sm < 1) { cudaGetLastError(); return QSTATE_EUNSUPPORTED; }
    const int64_t n_scales = dk + dv;
    const int64_t bytes = s->tiles * n_scales * s->scale_size;
    void* ns = nullptr;
    if (bytes && cudaMalloc(&ns, bytes) != cudaSuccess) { cudaGetLastError(); return QSTATE_ENOMEM; }
    cudaFree(s->d_scales);
    s->d_scales = ns;
    s->n_scales = n_scales;
    s->scale_bytes = bytes;
    s->rowcol = true;
    s->rc_entry = e;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, s->device);
    int64_t g = (int64_t)sms * per_sm;
    if (s->tiles < g) g = s->tiles > 0 ? s->tiles : 1;
    s->rc_grid = (int)g;
    rc = zero_state(s, nullptr);
    if (rc == QSTATE_OK && cudaDeviceSynchronize() != cudaSuccess) rc = QSTATE_ECUDA;
    return rc;
}

int qstate_set_pw(qstate* s, int W) {
    if (!s || s->pw || s->lrb || s->rowcol) return QSTATE_EINVAL;
    if (W < 1 || W > qs::kPwMaxW) return QSTATE_EINVAL;
    if (s->L.kind != QSTATE_GDN || s->scale_mode == QSTATE_YOKED || s->L.rotation ||
        !s->head_bits.empty() || !(s->bits == 4 || s->bits == 8) || s->L.d_k != s->L.d_v)
        return QSTATE_EUNSUPPORTED;
    int rc = check_device(s);
    if (rc != QSTATE_OK) return rc;
    const int d = s->L.d_k;
    const int idx = (((d == 128) * 2 + (s->bits == 8)) * 2 + (s->round_mode == QSTATE_BDR)) * 2 +
                    (s->L.qkv_dtype == QSTATE_BF16);
    const qs::PwEntry* e = &qs::pw_table()[idx];
    const int per_sm = e->blocks_per_sm(0);
    if (per_sm < 1) { cudaGetLastError(); return QSTATE_EUNSUPPORTED; }
    const int64_t T = s->tiles;
    auto alloc = [&](void** p, size_t n) -> bool { return !n || cudaMalloc(p, n) == cudaSuccess; };
    if (!alloc((void**)&s->d_pa, T * W * d) || !alloc((void**)&s->d_pb, T * W * d) ||
        !alloc((void**)&s->d_phead, T * 4) || !alloc((void**)&s->d_pcount, T * 4)) {
        cudaGetLastError();
        cudaFree(s->d_pa); cudaFree(s->d_pb); cudaFree(s->d_phead); cudaFree(s->d_pcount);
        s->d_pa = s->d_pb = nullptr;
        s->d_phead = s->d_pcount = nullptr;
        return QSTATE_ENOMEM;
    }
    s->pw = true;
    s->pw_W = W;
    s->pw_entry = e;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, s->device);
    int64_t g = (int64_t)sms * per_sm;
    if (T < g) g = T > 0 ? T : 1;
    s->pw_grid = (int)g;
    rc = zero_window(s, nullptr);
    if (rc == QSTATE_OK && cudaDeviceSynchronize() != cudaSuccess) rc = QSTATE_ECUDA;
    return rc;
}

int qstate_pw_export(const qstate* s, uint8_t* A, uint8_t* B, int32_t* head, int32_t* count,
                     qstate_stream stream) {
    if (!s || !s->pw || !A || !B || !head || !count) return QSTATE_EINVAL;
    if (s->tiles == 0) return QSTATE_OK;
    const int64_t T = s->tiles, W = s->pw_W;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(A, s->d_pa, T * W * s->L.d_k, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(B, s->d_pb, T * W * s->L.d_v, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(head, s->d_phead, T * 4, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(count, s->d_pcount, T * 4, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

int qstate_set_lrb(qstate* s, int k, int m, float eps_l) {
    if (!s || s->lrb || s->pw || s->rowcol) return QSTATE_EINVAL;
    if (k < 0 || k > 1 || m < 1 || k + m > qs::kLrbMaxCols) return QSTATE_EINVAL;
    if (!(eps_l >= 0.0f) || !std::isfinite(eps_l)) return QSTATE_EINVAL;
    if (s->scale_mode == QSTATE_YOKED || s->L.rotation ||
        !s->head_bits.empty() || !(s->bits == 4 || s->bits == 8) || s->L.d_k != s->L.d_v)
        return QSTATE_EUNSUPPORTED;
    int rc = check_device(s);
    if (rc != QSTATE_OK) return rc;
    const int d = s->L.d_k;
    const int kind = s->L.kind == QSTATE_GDN ? 1 : s->L.kind == QSTATE_GLA ? 2 : 0;
    const int idx = ((((d == 128) * 2 + (s->bits == 8)) * 3 + kind) * 2 +
                     (s->round_mode == QSTATE_BDR)) * 2 + (s->L.qkv_dtype == QSTATE_BF16);
    const qs::LrbEntry* e = &qs::lrb_table()[idx];
    const int smem = k == 1 ? 64 * e->threads * 4 : 0;
    const int per_sm = e->blocks_per_sm(smem);
    if (per_sm < 1) { cudaGetLastError(); return QSTATE_EUNSUPPORTED; }
    const int64_t K = k + m, T = s->tiles;
    auto alloc = [&](void** p, size_t n) -> bool { return !n || cudaMalloc(p, n) == cudaSuccess; };
    if (!alloc((void**)&s->d_lu, T * K * s->L.d_k * 2) || !alloc((void**)&s->d_lw, T * K * s->L.d_v * 2) ||
        !alloc((void**)&s->d_lg, T * K * 4) || !alloc((void**)&s->d_ln, T * 2 * 4) ||
        !alloc((void**)&s->d_lD, T * lrb_dlen(s) * 4)) {
        cudaGetLastError();
        cudaFree(s->d_lu); cudaFree(s->d_lw); cudaFree(s->d_lg); cudaFree(s->d_ln); cudaFree(s->d_lD);
        s->d_lu = s->d_lw = nullptr;
        s->d_lg = s->d_lD = nullptr;
        s->d_ln = nullptr;
        return QSTATE_ENOMEM;
    }
    s->lrb = true;
    s->lrb_k = k;
    s->lrb_m = m;
    s->lrb_eps = eps_l;
    s->lrb_entry = e;
    s->lrb_smem = smem;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, s->device);
    int64_t g = (int64_t)sms * per_sm;
    if (T < g) g = T > 0 ? T : 1;
    s->lrb_grid = (int)g;
    rc = zero_bypass(s, nullptr);
    if (rc == QSTATE_OK && cudaDeviceSynchronize() != cudaSuccess) rc = QSTATE_ECUDA;
    return rc;
}

const char* qstate_kernel(const qstate* s) {
    if (!s) return "";
    if (s->lrb) return "lrb_kernel";
    if (s->pw) return "pw_kernel";
    if (s->rowcol) return "rc_kernel";
    if (s->taxonomy || s->L.rotation) return "step_kernel";
    return s->entry_name;
}

int qstate_lrb_export(const qstate* s, uint16_t* u, uint16_t* w, float* g, int32_t* n, float* D,
                      qstate_stream stream) {
    if (!s || !s->lrb || !u || !w || !g || !n || !D) return QSTATE_EINVAL;
    if (s->tiles == 0) return QSTATE_OK;
    const int64_t K = s->lrb_k + s->lrb_m, T = s->tiles;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(u, s->d_lu, T * K * s->L.d_k * 2, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(w, s->d_lw, T * K * s->L.d_v * 2, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(g, s->d_lg, T * K * 4, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(n, s->d_ln, T * 2 * 4, cudaMemcpyDefault, st) != cudaSuccess ||
        cudaMemcpyAsync(D, s->d_lD, T * lrb_dlen(s) * 4, cudaMemcpyDefault, st) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

int qstate_debug_set(qstate* s, int64_t drop_from_tile, uint32_t wait_polls) {
    if (!s || wait_polls == 0 || drop_from_tile < -1) return QSTATE_EINVAL;
    s->drop_from = drop_from_tile;
    s->wait_polls = wait_polls;
    return QSTATE_OK;
}

int qstate_status(qstate* s, qstate_counters* o, qstate_stream stream) {
    if (!s || !o) return QSTATE_EINVAL;
    unsigned long long h[qs::kNumCounters] = {};
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(h, s->d_counters, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return QSTATE_ECUDA;
    o->nonfinite = h[0];
    o->saturated = h[1];
    o->pipeline_timeouts = h[2];
    o->exact_path_warps = h[3];
    o->lost = h[4];
    o->moved = h[5];
    o->reversed = h[6];
    o->bdr_applied = h[7];
    return QSTATE_OK;
}

int qstate_set_taxonomy(qstate* s, int on) {
    if (!s || (on != 0 && on != 1)) return QSTATE_EINVAL;
    if (on && !s->d_err && s->tiles > 0 && s->bits != 32) {
        int rc = check_device(s);
        if (rc != QSTATE_OK) return rc;
        const size_t n = (size_t)s->tiles * s->L.d_k * sizeof(float);
        if (cudaMalloc((void**)&s->d_err, n) != cudaSuccess) {
            cudaGetLastError();
            s->d_err = nullptr;
            return QSTATE_ENOMEM;
        }
        if (cudaMemset(s->d_err, 0, n) != cudaSuccess) return QSTATE_ECUDA;
    }
    s->taxonomy = on != 0;
    return QSTATE_OK;
}

int qstate_error_rows(const qstate* s, float* out, qstate_stream stream) {
    if (!s || !out || !s->d_err) return QSTATE_EINVAL;
    const size_t n = (size_t)s->tiles * s->L.d_k * sizeof(float);
    if (cudaMemcpyAsync(out, s->d_err, n, cudaMemcpyDefault, (cudaStream_t)stream) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}

}  // extern "C"
