// api.cu - status strings, ABI version and the per-device fault word.
#include <atomic>
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include <cuda.h>

#include "common.cuh"

namespace moe {

// Bits set by kernels that met a fault they could not return (a bounded
// wait that expired, an index outside its range).  One word per device.
__device__ unsigned g_device_error;

namespace {
std::atomic<unsigned long long> g_launches{0};
std::mutex g_mu;

using CtxGetCurrent = CUresult (*)(CUcontext*);
using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_entry(const char* name) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(fn);
}

// Unique id of the context current on this thread (0 when there is none):
// a context torn down and created again (cudaDeviceReset) gets a new id, so
// a device address cached under the old one is never used again.
unsigned long long current_context_id() {
    static const CtxGetCurrent get = driver_entry<CtxGetCurrent>("cuCtxGetCurrent");
    static const CtxGetId get_id = driver_entry<CtxGetId>("cuCtxGetId");
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get || !get_id || get(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

}  // namespace

unsigned long long context_id() { return current_context_id(); }

namespace {
CachedAddress g_err_addr[kMaxDevices];
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void* symbol_address(const void* symbol, CachedAddress* cache) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    CachedAddress& c = cache[dev];
    const unsigned long long ctx = current_context_id();
    if (c.addr && ctx != 0 && c.ctx == ctx) return c.addr;
    // first use on this device, or its context changed: look the symbol up
    // with the device current (this also creates the primary context)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
    c.addr = p;
    c.ctx = current_context_id();
    return p;
}

unsigned* device_error_word() {
    return static_cast<unsigned*>(symbol_address((const void*)&g_device_error, g_err_addr));
}

// The dynamic shared-memory limit is an attribute of the kernel's instance
// in one context, so it is raised once per (kernel, device, context) and
// remembered.
bool set_smem_limit(const void* fn, size_t bytes) {
    if (bytes <= 48 * 1024) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    static std::mutex mu;
    static std::map<std::pair<const void*, std::pair<int, unsigned long long>>, size_t> raised;
    std::lock_guard<std::mutex> lk(mu);
    const auto key = std::make_pair(fn, std::make_pair(dev, current_context_id()));
    const auto it = raised.find(key);
    if (key.second.second != 0 && it != raised.end() && it->second >= bytes) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
    raised[std::make_pair(fn, std::make_pair(dev, current_context_id()))] = bytes;
    return true;
}

int resident_ctas(const void* fn, int threads, size_t smem) {
    const char* env = getenv("LIBMOE_ONE_WAVE");
    if (env && env[0] == '0') return 1 << 30;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1 << 30;
    static std::mutex mu;
    static std::map<std::pair<std::pair<const void*, int>, std::pair<size_t, unsigned long long>>, int> known;
    std::lock_guard<std::mutex> lk(mu);
    const auto key = std::make_pair(std::make_pair(fn, threads), std::make_pair(smem, (unsigned long long)dev));
    const auto it = known.find(key);
    if (it != known.end()) return it->second;
    int per = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, threads, smem) != cudaSuccess || per < 1 ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
        (void)cudaGetLastError();
        return 1 << 30;
    }
    known[key] = per * sms;
    return per * sms;
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

extern "C" const char* moe_status_str(moe_status status) { return moe_status_string((int)status); }

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
