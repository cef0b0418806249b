// qstate_static.cu -- qstate_step_host_static: the host-buffer decode step
// for callers that must not allocate device memory.
//
// qstate_step_host stages the step operands in device buffers that its first
// call allocates with cudaMalloc.  Some callers cannot allow that: a serving
// process whose device memory is all handed out by its own pool allocator,
// or a decode loop that must not stall, since cudaMalloc may synchronise the
// device and wait for work queued on other streams.  This variant stages the
// operands in one fixed array in the library's device image instead, so a
// step allocates nothing.  The array below is held on every GPU that loads
// the library until the process exits.
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "qstate.h"

namespace {

// q | k | v | gates | out of one call, each part starting on 256 bytes.
static __device__ __align__(256) unsigned char g_staging[QSTATE_STATIC_STAGING_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device address of g_staging, per device ordinal (null until set up).  In
// host code the name g_staging is only a host-side stand-in for the array:
// a kernel given it would fault, or where the GPU can reach host memory
// silently use the wrong memory.  The real address comes from
// cudaGetSymbolAddress, once per device, with that device current.
unsigned char* g_addr[kMaxDevices];

int staging_address(unsigned char** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return QSTATE_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return QSTATE_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_staging) != cudaSuccess || !p) {
            cudaGetLastError();
            return QSTATE_ECUDA;
        }
        g_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_addr[dev];
    return QSTATE_OK;
}

size_t up256(int64_t x) { return (static_cast<size_t>(x) + 255) & ~size_t(255); }

}  // namespace

extern "C" int qstate_step_host_static(qstate* s, const void* q, const void* k, const void* v,
                                       const void* gates, float* out, qstate_stream stream) {
    if (!s || !q || !k || !v || !out) return QSTATE_EINVAL;
    qstate_sizes z;
    if (qstate_get_sizes(s, &z) != QSTATE_OK) return QSTATE_EINVAL;
    if (z.n_gate && !gates) return QSTATE_EINVAL;
    if (z.tiles == 0) return QSTATE_OK;
    const size_t oq = 0, ok = oq + up256(z.q_bytes), ov = ok + up256(z.q_bytes);
    const size_t og = ov + up256(z.v_bytes), oo = og + up256(z.gate_bytes);
    const size_t need = oo + up256(z.out_bytes);
    if (need > QSTATE_STATIC_STAGING_BYTES) return QSTATE_EINVAL;   // operands too large
    unsigned char* base = nullptr;
    int rc = staging_address(&base);
    if (rc != QSTATE_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // every byte the kernel reads is copied in here and every byte of `out`
    // is written by the kernel, so nothing left by an earlier call is read
    if (cudaMemcpyAsync(base + oq, q, z.q_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(base + ok, k, z.q_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(base + ov, v, z.v_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        (z.gate_bytes &&
         cudaMemcpyAsync(base + og, gates, z.gate_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess))
        return QSTATE_ECUDA;
    rc = qstate_step(s, base + oq, base + ok, base + ov, z.gate_bytes ? base + og : nullptr,
                     reinterpret_cast<float*>(base + oo), stream);
    if (rc != QSTATE_OK) return rc;
    if (cudaMemcpyAsync(out, base + oo, z.out_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return QSTATE_ECUDA;
    return QSTATE_OK;
}
