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

struct Setup {
    int ctas_per_sm, sms;
};

std::mutex g_setup_mu;
std::map<SetupKey, Setup> g_setup;
// largest dynamic shared memory each (kernel, device) has been opted into:
// the attribute belongs to the kernel, so it only ever grows
std::map<std::pair<const void *, int>, size_t> g_smem_optin;
std::map<int, int> g_device_sms;

}  // namespace

cudaError_t kernel_setup(const void *kernel, int threads, size_t smem, int *ctas_per_sm, int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const SetupKey key{kernel, dev, threads, smem};
    std::lock_guard<std::mutex> lock(g_setup_mu);
    auto it = g_setup.find(key);
    if (it != g_setup.end()) {
        *ctas_per_sm = it->second.ctas_per_sm;
        *sms = it->second.sms;
        return cudaSuccess;
    }
    int nsm = 0;
    e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (nsm < 1) return cudaErrorInvalidDevice;
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
    g_setup[key] = Setup{occ, nsm};
    *ctas_per_sm = occ;
    *sms = nsm;
    return cudaSuccess;
}

int current_device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(g_setup_mu);
    int &n = g_device_sms[dev];
    if (n == 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    return n;
}

}  // namespace mtpv
