// placement.cu - correlated expert placement and the token-shuffling statistic.
//
// "Expert Coupling in MoE Pretraining: Reducing All-to-All Overhead with
// Correlated Placement and Token Shuffling", Abstract: experts that tokens
// pick together are placed on the same GPU, and a token is moved to the GPU
// predicted to hold its next-layer experts, raising the share of
// token-expert assignments served on the token's own GPU.  On one device
// these become: a placement (group_of_expert) computed from the co-selection
// counts, a predicted home group per token from the layer-to-layer
// transition counts, and the count of assignments whose expert lies in the
// token's home group ("Expert Parallelism > Key Parameters": L/E of them
// under uniform routing with sequence-sharded homes).
//
// The pages give no placement algorithm; the one here is a plain greedy:
// each group starts from the unassigned expert with the largest off-diagonal
// co-selection mass and grows by the unassigned expert with the largest
// co-selection summed over the group's members, lower index on ties.
#include "common.cuh"

namespace moe {

// Block-wide maximum of a 64-bit key (1024 threads).
__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long v, unsigned long long* sh /*[32]*/) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) sh[wid] = v;
    __syncthreads();
    unsigned long long r = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, sh[w]);
    __syncthreads();
    return r;
}

// Key ordering "larger value first, then lower index": (value + 1) above
// bit 11 (0 marks an assigned expert), the complemented index (E <= 1024)
// in the low 11 bits.  Values are sums of counts, far below 2^52.
__device__ __forceinline__ unsigned long long pick_key(long long value, int x, bool free_) {
    if (!free_) return 0ull;
    return ((unsigned long long)(value + 1) << 11) | (unsigned long long)(2047 - x);
}

__device__ __forceinline__ int key_index(unsigned long long key) { return 2047 - (int)(key & 2047ull); }

__global__ void __launch_bounds__(1024) place_experts_kernel(const int32_t* __restrict__ cosel, int E, int G,
                                                             int32_t* __restrict__ group_of_expert) {
    __shared__ long long mass[1024], aff[1024];
    __shared__ int grp[1024];
    __shared__ unsigned long long sh[32];
    const int x = threadIdx.x;
    const bool live = x < E;
    if (live) {
        long long m = 0;
        for (int y = 0; y < E; ++y)
            if (y != x) m += cosel[(long long)x * E + y];
        mass[x] = m;
        grp[x] = -1;
    }
    __syncthreads();
    const int L = E / G;
    for (int g = 0; g < G; ++g) {
        const unsigned long long kseed = block_max_u64(live ? pick_key(mass[x], x, grp[x] < 0) : 0ull, sh);
        const int seed = key_index(kseed);
        if (live) aff[x] = cosel[(long long)x * E + seed];
        if (x == seed) grp[x] = g;
        __syncthreads();
        for (int m = 1; m < L; ++m) {
            const unsigned long long kb = block_max_u64(live ? pick_key(aff[x], x, grp[x] < 0) : 0ull, sh);
            const int best = key_index(kb);
            if (x == best) grp[x] = g;
            if (live) aff[x] += cosel[(long long)x * E + best];
            __syncthreads();
        }
    }
    if (live) group_of_expert[x] = grp[x];
}

// affinity[a][g] = sum of trans[a][b] over the experts b of group g.
__global__ void __launch_bounds__(256) group_affinity_kernel(const int32_t* __restrict__ trans, int E,
                                                             const int32_t* __restrict__ goe, int G,
                                                             long long* __restrict__ affinity, unsigned* err) {
    extern __shared__ unsigned long long acc[];          // [G]
    const int a = blockIdx.x;
    for (int g = threadIdx.x; g < G; g += blockDim.x) acc[g] = 0ull;
    __syncthreads();
    for (int b = threadIdx.x; b < E; b += blockDim.x) {
        const int g = goe[b];
        if (g < 0 || g >= G) { raise_error(err, kErrIndex); continue; }
        atomicAdd(&acc[g], (unsigned long long)(long long)trans[(long long)a * E + b]);
    }
    __syncthreads();
    for (int g = threadIdx.x; g < G; g += blockDim.x) affinity[(long long)a * G + g] = (long long)acc[g];
}

// home[t] = the group with the largest summed affinity over the token's
// layer-1 experts (lower group on ties).
__global__ void predict_home_kernel(const int32_t* __restrict__ idx1, int T, int k1, const long long* __restrict__ affinity,
                                    int E, int G, int32_t* __restrict__ home, unsigned* err) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    int best = 0;
    long long best_v = 0;
    for (int g = 0; g < G; ++g) {
        long long v = 0;
        for (int i = 0; i < k1; ++i) {
            const int a = idx1[t * k1 + i];
            if (a < 0 || a >= E) { raise_error(err, kErrIndex); continue; }
            v += affinity[(long long)a * G + g];
        }
        if (g == 0 || v > best_v) { best = g; best_v = v; }
    }
    home[t] = best;
}

// count += assignments whose expert lies in the token's home group (home
// NULL: floor(t * G / T)).
__global__ void __launch_bounds__(256) count_local_kernel(const int32_t* __restrict__ idx, int T, int k,
                                                          const int32_t* __restrict__ goe, int E, int G,
                                                          const int32_t* __restrict__ home,
                                                          unsigned long long* __restrict__ count, unsigned* err) {
    __shared__ unsigned long long sh[8];
    unsigned long long local = 0;
    const long long n = (long long)T * k;
    for (long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x; s < n; s += (long long)gridDim.x * blockDim.x) {
        const long long t = s / k;
        const int e = idx[s];
        if (e < 0 || e >= E) { raise_error(err, kErrIndex); continue; }
        const long long h = home ? (long long)home[t] : t * G / T;
        local += goe[e] == h;
    }
    local = warp_sum(local);
    if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long v = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += sh[w];
        if (v) atomicAdd(count, v);
    }
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_place_experts(const int32_t* cosel, int E, int G, int32_t* group_of_expert,
                                        moe_stream_t stream) {
    if (E < 1 || G < 1 || E % G != 0) return MOE_ERR_ARG;
    if (E > 1024) return MOE_ERR_SHAPE;
    if (!cosel || !group_of_expert) return MOE_ERR_ARG;
    place_experts_kernel<<<1, 1024, 0, (cudaStream_t)stream>>>(cosel, E, G, group_of_expert);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_group_affinity(const int32_t* trans, int E, const int32_t* group_of_expert, int G,
                                         int64_t* affinity, moe_stream_t stream) {
    if (E < 1 || G < 1) return MOE_ERR_ARG;
    if (E > 1024 || G > 1024) return MOE_ERR_SHAPE;
    if (!trans || !group_of_expert || !affinity) return MOE_ERR_ARG;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    group_affinity_kernel<<<E, 256, sizeof(unsigned long long) * G, (cudaStream_t)stream>>>(
        trans, E, group_of_expert, G, (long long*)affinity, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_predict_home(const int32_t* idx1, int T, int k1, const int64_t* affinity, int E, int G,
                                       int32_t* home, moe_stream_t stream) {
    if (T < 0 || k1 < 1 || E < 1 || G < 1) return MOE_ERR_ARG;
    if (E > 1024 || G > 1024 || k1 > 32) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    if (!idx1 || !affinity || !home) return MOE_ERR_ARG;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    predict_home_kernel<<<ceil_div(T, 256), 256, 0, (cudaStream_t)stream>>>(idx1, T, k1, (const long long*)affinity,
                                                                              E, G, home, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_count_local(const int32_t* expert_idx, int T, int k, const int32_t* group_of_expert, int E,
                                      int G, const int32_t* home, uint64_t* count, moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1 || G < 1) return MOE_ERR_ARG;
    if (E > 1024 || G > 1024 || k > 32) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    if (!expert_idx || !group_of_expert || !count) return MOE_ERR_ARG;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const long long n = (long long)T * k;
    int grid = (int)((n + 255) / 256);
    if (grid > 148 * 8) grid = 148 * 8;
    count_local_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(expert_idx, T, k, group_of_expert, E, G, home,
                                                               (unsigned long long*)count, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
