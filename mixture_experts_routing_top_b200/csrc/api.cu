// api.cu - status strings, ABI version and the per-device fault word.
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace moe {

// Bits set by kernels that met a fault they could not return (a bounded
// wait that expired, an index outside its range).  One word per device.
__device__ unsigned g_device_error;

namespace {
std::atomic<unsigned long long> g_launches{0};
std::mutex g_mu;
unsigned* g_err_addr[64] = {nullptr};
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

unsigned* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_addr[dev] = static_cast<unsigned*>(p);
    }
    return g_err_addr[dev];
}

// The dynamic shared-memory limit is an attribute of the kernel's instance
// on one device, so it is raised once per (kernel, device) and remembered.
bool set_smem_limit(const void* fn, size_t bytes) {
    if (bytes <= 48 * 1024) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, size_t> raised;
    std::lock_guard<std::mutex> lk(mu);
    const auto key = std::make_pair(fn, dev);
    const auto it = raised.find(key);
    if (it != raised.end() && it->second >= bytes) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
    raised[key] = bytes;
    return true;
}

}  // namespace moe

extern "C" const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_SHAPE: return "unsupported shape or alignment";
        case MOE_ERR_DTYPE: return "unsupported dtype";
        case MOE_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_UNSUPPORTED: return "device is not sm_100";
        case MOE_ERR_TIMEOUT: return "a bounded device wait expired";
        case MOE_ERR_DEVICE_INDEX: return "a kernel skipped an out-of-range index";
        default: return "unknown status";
    }
}

extern "C" int moe_abi_version(void) { return MOE_ABI_VERSION; }

extern "C" moe_status moe_device_error(int clear) {
    unsigned* p = moe::device_error_word();
    if (!p) return MOE_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (clear && v) {
        if (cudaMemset(p, 0, sizeof(unsigned)) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (v & moe::kErrTimeout) return MOE_ERR_TIMEOUT;
    if (v & moe::kErrIndex) return MOE_ERR_DEVICE_INDEX;
    return MOE_OK;
}

extern "C" uint64_t moe_kernel_launches(void) { return moe::g_launches.load(std::memory_order_relaxed); }
