// IF4 x IF4 linear without caller-provided workspace.
//
// if4_linear needs (M + N) * K * 2 bytes of device scratch for the two fp16
// operands it decodes before the GEMM, and takes it from the caller.  Some
// callers cannot hand out device memory at that point: a plugin running
// inside a host framework that owns every device byte through its own pool
// and offers no workspace hook, or a latency-critical path that must not
// risk the device-wide synchronisation a cudaMalloc can cause.  For them,
// if4_linear_noalloc uses a fixed scratch array that is part of this
// library's device code, so the call allocates nothing.
//
// Costs and rules of that array:
//   * it is IF4_LINEAR_NOALLOC_MAX_BYTES (32 MiB) per device; a device holds
//     it from the moment this file's device code is loaded there (at the
//     latest, the first call on that device) until the process exits;
//   * problems whose workspace exceeds it are rejected with
//     IF4_ERR_WORKSPACE before anything is enqueued;
//   * every call on a device shares the one array, and it keeps whatever the
//     last call left in it.  Nothing in it has to start at zero: the decode
//     kernels overwrite every byte a call reads before the GEMM reads it.
//     Calls whose work overlaps on the GPU (other streams, other host threads
//     without ordering) race on the array and corrupt each other's results;
//     the caller must order them, e.g. by issuing them on one stream;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it, so that
//     first call should come before any stream capture the caller starts;
//   * the cached address belongs to the device's primary context.  A
//     cudaDeviceReset ends that context and with it the array; the cache
//     cannot see that, so after a reset a process must not call
//     if4_linear_noalloc on that device again (if4_linear, with a workspace
//     from the caller, is unaffected).

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/if4.h"

namespace {

// The scratch itself.  In host code this name is only a stand-in for the
// device object, not an address a kernel may use; the device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_linear_scratch[IF4_LINEAR_NOALLOC_MAX_BYTES];

// Device address of g_linear_scratch on the current device, looked up once
// per device with that device current.
int scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[64] = {};
    static bool have[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return IF4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || p == nullptr)
            return IF4_ERR_CUDA;
        addr[dev] = p;
        have[dev] = true;
    }
    *out = addr[dev];
    return IF4_OK;
}

}  // namespace

extern "C" int if4_linear_noalloc(const uint8_t *a_codes, const uint8_t *a_scales,
                                  const float *a_ts, const uint8_t *b_codes,
                                  const uint8_t *b_scales, const float *b_ts, int64_t M,
                                  int64_t N, int64_t K, void *c, int *err_flag, void *stream)
{
    const size_t need = if4_linear_workspace_bytes(M, N, K);
    void *scratch = nullptr;
    // A problem too large for the array gets no scratch: if4_linear then
    // checks the other arguments first and refuses it with
    // IF4_ERR_WORKSPACE, so the errors come in the same order as from
    // if4_linear itself.  Invalid sizes (need == 0) are reported by the same
    // checks.
    if (need != 0 && need <= (size_t)IF4_LINEAR_NOALLOC_MAX_BYTES) {
        const int rc = scratch_address(&scratch);
        if (rc != IF4_OK) return rc;
    }
    return if4_linear(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, M, N, K, scratch,
                      scratch ? (size_t)IF4_LINEAR_NOALLOC_MAX_BYTES : 0u, c, err_flag, stream);
}
