// Per-device launch setup of the library's kernels, cached so that a
// steady-state call issues no CUDA API call besides its launches.
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"

namespace mtpv {

namespace {

struct SetupKey {
    const void *kernel;
    int device, threads;
    size_t smem;
    bool operator<(const SetupKey &o) const {
        return std::tie(kernel, device, threads, smem) < std::tie(o.kernel, o.device, o.threads, o.smem);
    }
};

std::mutex g_setup_mu;
std::map<SetupKey, int> g_setup;  // -> resident CTAs per SM
// largest dynamic shared memory each (kernel, device) has been opted into:
// the attribute belongs to the kernel, so it only ever grows
std::map<std::pair<const void *, int>, size_t> g_smem_optin;

}  // namespace

cudaError_t kernel_setup(const void *kernel, int threads, size_t smem, int *ctas_per_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const SetupKey key{kernel, dev, threads, smem};
    std::lock_guard<std::mutex> lock(g_setup_mu);
    auto it = g_setup.find(key);
    if (it != g_setup.end()) {
        *ctas_per_sm = it->second;
        return cudaSuccess;
    }
    size_t &optin = g_smem_optin[std::make_pair(kernel, dev)];
    if (smem > 48 * 1024 && smem > optin) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        optin = smem;
    }
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    g_setup[key] = occ;
    *ctas_per_sm = occ;
    return cudaSuccess;
}

}  // namespace mtpv
