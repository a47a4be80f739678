// selftest.cu - a device check of the failure-detection contract: a bounded
// mbarrier wait that nobody completes gives up, records MOE_ERR_TIMEOUT in
// the per-device fault word and returns, leaving the context usable.
#include "tcgen05.cuh"

namespace moe {
namespace {

// One warp.  Lane 0 initialises an mbarrier expecting one arrival; with
// `arrive` set it makes that arrival itself (the control case), else nothing
// ever arrives.  Every lane then waits on phase 0 through the same bounded
// wait the tensor-core kernels use.  No copy or MMA is in flight, so a wait
// that gives up leaves nothing outstanding.
__global__ void bounded_wait_kernel(int arrive, long long limit_ns, int32_t* result, unsigned* err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = tc::smem_u32(&bar);
    if (threadIdx.x == 0) {
        tc::mbar_init(b, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (arrive && threadIdx.x == 0) tc::mbar_arrive(b);
    const long long t0 = tc::globaltimer();
    const bool done = tc::mbar_wait(b, 0, &abort_flag, limit_ns);
    const long long waited = tc::globaltimer() - t0;
    __syncwarp();
    if (threadIdx.x == 0) {
        if (!done) raise_error(err, kErrTimeout);
        result[0] = done ? 1 : 0;
        result[1] = (int32_t)(waited / 1000 < 0x7fffffff ? waited / 1000 : 0x7fffffff);
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_selftest_bounded_wait(int arrive, long long limit_ns, int32_t* result, moe_stream_t stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000LL || !result) return MOE_ERR_ARG;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(arrive, limit_ns, result, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
