// noalloc.cu -- spectra_pack_plan_noalloc: the saliency split without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory when they plan a layer: code
// running inside another framework's allocator regime or a memory pool that
// is already carved up, tools that must not perturb a process's allocation
// pattern, and hosts that simply have no cudaMalloc-capable context handy.
// For them this entry point keeps its scratch (the per-column kurtosis when
// the caller does not ask for it, the outlier count and the error word) in a
// fixed array that the library itself holds, so the call allocates nothing.
#include <cuda_runtime.h>

#include "internal.cuh"
#include "spectra.h"

namespace spectra {
namespace {

constexpr size_t kKappaBytes = (size_t)SPECTRA_NOALLOC_MAX_K * sizeof(double);
constexpr size_t kScratchBytes = kKappaBytes + 256;

// The scratch of every spectra_pack_plan_noalloc call on a device: kurtosis
// [SPECTRA_NOALLOC_MAX_K] doubles, then [0] error bits and [1] outlier count.
// Each device that loads the library keeps it until the process exits.
__device__ __align__(256) unsigned char g_plan_scratch[kScratchBytes];

// Device address of the scratch array on the current device.  The symbol's
// name in host code is only a host-side handle, so the address comes from
// cudaGetSymbolAddress, with the device current.  It is looked up on every
// call (the lookup allocates nothing): after a reset of the device's primary
// context the module is loaded again and the array may sit elsewhere, so a
// cached address could point into another allocation.
spectra_status scratch_address(unsigned char **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || !p) return SPECTRA_ERR_CUDA;
    *out = static_cast<unsigned char *>(p);
    return SPECTRA_OK;
}

}  // namespace
}  // namespace spectra

using namespace spectra;

extern "C" spectra_status spectra_pack_plan_noalloc(const uint16_t *w, const float *gain, int32_t n,
                                                    int32_t k, double tau, double *kappa_out,
                                                    int32_t *idx_out, int32_t *n_outliers_out,
                                                    void *stream) {
    if (!w || !idx_out || !n_outliers_out) return SPECTRA_ERR_INVALID_ARG;
    if (n < 1 || k < 32 || (k % 32) != 0 || (int64_t)n * (int64_t)k > ((int64_t)1 << 40))
        return SPECTRA_ERR_SHAPE;
    if (k > SPECTRA_NOALLOC_MAX_K) return SPECTRA_ERR_SHAPE;
    if (tau != tau) return SPECTRA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(w) & 15u) || (reinterpret_cast<uintptr_t>(idx_out) & 3u) ||
        (gain && (reinterpret_cast<uintptr_t>(gain) & 3u)) ||
        (kappa_out && (reinterpret_cast<uintptr_t>(kappa_out) & 7u)))
        return SPECTRA_ERR_ALIGN;
    DeviceInfo dev;
    spectra_status st = current_device(&dev);
    if (st != SPECTRA_OK) return st;
    unsigned char *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != SPECTRA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    double *kappa = kappa_out ? kappa_out : reinterpret_cast<double *>(scratch);
    int *words = reinterpret_cast<int *>(scratch + kKappaBytes);  // [0] error bits, [1] count
    // the array keeps the previous call's contents: the words must start at zero
    if (cudaMemsetAsync(words, 0, 2 * sizeof(int), s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (launch_kurtosis(w, gain, n, k, kappa, words, s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (launch_split(kappa, k, tau, idx_out, words + 1, s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    int host[2] = {0, 0};
    if (cudaMemcpyAsync(host, words, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SPECTRA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPECTRA_ERR_CUDA;
    if (host[0] & kErrNonfinite) return SPECTRA_ERR_NONFINITE;
    if (host[1] < 0 || host[1] > k) return SPECTRA_ERR_INTERNAL;
    *n_outliers_out = host[1];
    return SPECTRA_OK;
}
