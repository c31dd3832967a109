// pdssm_scan_fwd_noalloc: the forward scan for callers that cannot allocate
// device memory, with its scratch in a fixed device array of this library.
//
// Some callers have no way to obtain scratch memory: a host program whose
// device memory is entirely owned by another allocator, a loop that must not
// call cudaMalloc because it synchronises the device, or an environment that
// forbids allocation after start-up.  This entry point needs only the
// inputs and outputs: the workspace of pdssm_scan_fwd comes from
// kStaticScratchBytes of device memory that every GPU which loads the
// library holds until the process exits.
#include <mutex>
#include <stdio.h>

#include "common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)4 << 20;   // 4 MiB

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the static scratch array on `dev` (the current device).
// In host code the array's name is only a host-side stand-in, so the device
// address is looked up once per device and remembered for the process: the
// library must not be used on a device across cudaDeviceReset (the array of
// the new context would live elsewhere).
cudaError_t scratch_address(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (dev >= 0 && dev < kMaxDevices && g_scratch_ptr[dev]) {
        *out = g_scratch_ptr[dev];
        return cudaSuccess;
    }
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) g_scratch_ptr[dev] = ptr;
    *out = ptr;
    return cudaSuccess;
}

// The scratch of the current device, or a status (with its last-error text).
pdssm_status current_scratch(void **ws) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return pdssm::cuda_fail(e, "cudaGetDevice");
    e = scratch_address(dev, ws);
    if (e != cudaSuccess) return pdssm::cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    return PDSSM_OK;
}

}  // namespace

extern "C" {

size_t pdssm_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

pdssm_status pdssm_scan_fwd_noalloc(const pdssm_dims *dims, const int32_t *pi_dict,
                                    int64_t pi_head_stride, const int32_t *k, const void *d,
                                    const void *b, const void *c, pdssm_dtype in_dtype,
                                    const float *h0, float *y, float *h_last, int64_t chunk,
                                    void *stream) {
    // the same shape checks (and statuses) as pdssm_scan_fwd
    pdssm_status st = pdssm::check_scan_dims(dims, pi_head_stride, chunk);
    if (st != PDSSM_OK) return st;
    const size_t need = pdssm_workspace_bytes(dims, pi_head_stride, chunk, 0);
    if (need > kStaticScratchBytes) {
        char why[160];
        snprintf(why, sizeof(why), "workspace of %zu bytes exceeds the static scratch of %zu bytes",
                 need, kStaticScratchBytes);
        return pdssm::arg_fail(PDSSM_ERR_UNSUPPORTED, why);
    }
    void *ws = nullptr;
    st = current_scratch(&ws);
    if (st != PDSSM_OK) return st;
    // pdssm_scan_fwd clears the status word and overwrites every other part
    // of the workspace it reads, so what an earlier call left there is moot.
    return pdssm_scan_fwd(dims, pi_dict, pi_head_stride, k, d, b, c, in_dtype, h0, y, h_last,
                          chunk, ws, kStaticScratchBytes, stream);
}

pdssm_status pdssm_noalloc_status(void *stream) {
    void *ws = nullptr;
    const pdssm_status st = current_scratch(&ws);
    if (st != PDSSM_OK) return st;
    return pdssm_ws_status(ws, kStaticScratchBytes, stream);
}

}  // extern "C"
