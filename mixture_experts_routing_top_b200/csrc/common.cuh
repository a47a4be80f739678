// common.cuh - small helpers shared by the libmoe kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/libmoe.h"

namespace moe {

// Device fault word bits (see moe_device_error).
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrIndex = 2u;

constexpr int kMaxDevices = 64;

// Device address of a __device__ variable on the current device.  In host
// code a __device__ variable's name is only a host-side stand-in, so the
// address is looked up (cudaGetSymbolAddress, with the device current) on
// first use and cached per device under the current context's unique id: a
// context created again after cudaDeviceReset gets a fresh lookup.  `cache`
// has kMaxDevices entries.  Null on a runtime error.
struct CachedAddress {
    unsigned long long ctx = 0;
    void* addr = nullptr;
};
void* symbol_address(const void* symbol, CachedAddress* cache);

// Unique id of the CUDA context current on this thread, 0 if none.
unsigned long long context_id();

// Address of the current device's fault word (defined in api.cu).
unsigned* device_error_word();

// Counts kernel launches made by the library (moe_kernel_launches).
void count_launch();

// Lets kernel fn take `bytes` of dynamic shared memory on the current device
// (no-op up to 48 KB).  False if the runtime refused.
bool set_smem_limit(const void* fn, size_t bytes);

// CTAs of kernel fn (with `threads` threads and `smem` bytes of dynamic
// shared memory each) that the current device holds at once, looked up once
// per kernel, shape and device.  A grid-strided kernel launched with at most
// this many CTAs runs in one wave and its warps share the work evenly; one
// more wave than that would leave most of the GPU idle at its end.
// LIBMOE_ONE_WAVE=0 turns the cap off (a very large number).
int resident_ctas(const void* fn, int threads, size_t smem);

// Programmatic dependent launch.  A kernel launched with programmatic
// stream serialization may start while the kernel before it in the stream
// is still running; it must call pdl_wait() before its first global memory
// access (read or write), which returns once that kernel has completed and
// its writes are visible.  Without the launch attribute pdl_wait() returns
// at once.  pdl_trigger() lets the next such kernel be scheduled now.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void raise_error(unsigned* err, unsigned bits) {
    if (err) atomicOr(err, bits);
}

__device__ __forceinline__ unsigned lane_id() {
    unsigned r;
    asm volatile("mov.u32 %0, %%laneid;" : "=r"(r));
    return r;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned r;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(r));
    return r;
}

// 16-byte vector loads/stores.  Inputs read once take the non-coherent path
// without allocating in L1; outputs are written with the streaming (.cs)
// hint so a large copy does not flush useful lines from L2.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_keep(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint4* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round-to-nearest-even packing of two floats into a bf16x2 word (lo first).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Top-KM insertion for one token's logits seen in ascending expert order:
// bv/bi hold the KM best so far, larger logit first.  A logit enters only if
// strictly larger than the current KM-th, and slides above strictly smaller
// entries only, so among equal logits the lower expert ranks first.
template <int KM>
__device__ __forceinline__ void topk_insert(float (&bv)[KM], int (&bi)[KM], float l, int e) {
    if (!(l > bv[KM - 1])) return;
    bool placed = false;
#pragma unroll
    for (int j = KM - 1; j >= 0; --j) {
        if (!placed) {
            if (j > 0 && l > bv[j - 1]) {
                bv[j] = bv[j - 1];
                bi[j] = bi[j - 1];
            } else {
                bv[j] = l;
                bi[j] = e;
                placed = true;
            }
        }
    }
}

// The same insertion without branches: every comparison is made against
// the list as it was (c[j] = l > bv[j], which, the list being sorted, holds
// for a suffix of positions), then each entry takes its upper neighbour's
// value, the new one, or keeps its own.  A lane with nothing to insert
// passes l = -inf (no comparison holds, nothing moves), so a warp can insert
// its lanes' candidates in step.
template <int KM>
__device__ __forceinline__ void topk_insert_uniform(float (&bv)[KM], int (&bi)[KM], float l, int e) {
    bool c[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) c[j] = l > bv[j];
#pragma unroll
    for (int j = KM - 1; j >= 1; --j) {
        bv[j] = c[j - 1] ? bv[j - 1] : (c[j] ? l : bv[j]);
        bi[j] = c[j - 1] ? bi[j - 1] : (c[j] ? e : bi[j]);
    }
    bv[0] = c[0] ? l : bv[0];
    bi[0] = c[0] ? e : bi[0];
}

// exp(l - m) with the rounding error of l - m carried into the result
// (TwoSum of l and -m, then exp(hi) * (1 + lo)).
__device__ __forceinline__ float exp_diff(float l, float m) {
    const float hi = __fsub_rn(l, m);
    const float bb = __fsub_rn(hi, l);
    const float lo = __fadd_rn(__fsub_rn(l, __fsub_rn(hi, bb)), __fsub_rn(-m, bb));
    const float e = expf(hi);
    return __fmaf_rn(e, lo, e);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// A kernel launch that may begin while the kernel before it in the stream
// is finishing (programmatic stream serialization); the kernel calls
// pdl_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe

// Launch-error check used right after each kernel launch in host code;
// also counts the launch.
#define MOE_LAUNCH_CHECK()                                  \
    do {                                                    \
        moe::count_launch();                                \
        if (cudaPeekAtLastError() != cudaSuccess) {         \
            (void)cudaGetLastError();                       \
            return MOE_ERR_CUDA;                            \
        }                                                   \
    } while (0)
