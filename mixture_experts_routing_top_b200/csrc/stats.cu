// stats.cu - routing-correlation histograms.
//
// "Expert Coupling in MoE Pretraining: Reducing All-to-All Overhead with
// Correlated Placement and Token Shuffling", Abstract: within a layer some
// expert pairs are picked jointly far more often than chance, and a token's
// expert choices in one layer are predictive of its choices in the
// following layer.  Both statistics are E x E integer histograms:
//   co-selection  cosel[a][b] += 1 for each ordered pair of a token's slots,
//   transition    trans[a][b] += 1 for each (layer-1 slot, layer-2 slot).
//
// Each CTA owns a band of rows [a0, a0 + band) of the histogram in shared
// memory (<= 64 KB), counts its share of the tokens there with shared
// atomics, and merges the non-zero bins into global memory with one atomic
// each.  Integer adds commute, so the result is exact and deterministic.
#include "common.cuh"

namespace moe {

constexpr int kHistBytes = 64 * 1024;

__global__ void __launch_bounds__(512) pair_hist_kernel(const int32_t* __restrict__ idx1, int k1,
                                                        const int32_t* __restrict__ idx2, int k2, int T, int E,
                                                        int band, int tokens_per_cta, int32_t* __restrict__ hist,
                                                        unsigned* err) {
    extern __shared__ int h[];                  // [band][E]
    const int a0 = blockIdx.y * band;
    const int a1 = min(a0 + band, E);
    const int nbins = (a1 - a0) * E;
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) h[i] = 0;
    __syncthreads();
    const long long t0 = (long long)blockIdx.x * tokens_per_cta;
    const long long t1 = min(t0 + tokens_per_cta, (long long)T);
    // one (token, slot-of-idx1) per thread iteration
    const long long n = (t1 - t0) * k1;
    for (long long q = threadIdx.x; q < n; q += blockDim.x) {
        const long long t = t0 + q / k1;
        const int a = idx1[t0 * k1 + q];
        if (a < 0 || a >= E) { raise_error(err, kErrIndex); continue; }
        if (a < a0 || a >= a1) continue;
        int* row = h + (a - a0) * E;
        const int32_t* bs = idx2 + t * k2;
        for (int j = 0; j < k2; ++j) {
            const int b = bs[j];
            if (b < 0 || b >= E) { raise_error(err, kErrIndex); continue; }
            atomicAdd(row + b, 1);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) {
        const int v = h[i];
        if (v) atomicAdd(hist + (long long)a0 * E + i, v);
    }
}

moe_status launch_pair_hist(const int32_t* idx1, int k1, const int32_t* idx2, int k2, int T, int E, int32_t* hist,
                            cudaStream_t s) {
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    int band = kHistBytes / (int)(sizeof(int) * E);
    if (band > E) band = E;
    if (band < 1) band = 1;
    const int nbands = ceil_div(E, band);
    const size_t smem = sizeof(int) * (size_t)band * E;
    // enough CTAs to fill the GPU; each keeps its band of bins in shared memory
    int tok_ctas = (148 * 4 + nbands - 1) / nbands;
    int tokens_per_cta = ceil_div(T, tok_ctas);
    if (tokens_per_cta < 256) tokens_per_cta = 256;
    tok_ctas = ceil_div(T, tokens_per_cta);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(pair_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    pair_hist_kernel<<<dim3(tok_ctas, nbands), 512, smem, s>>>(idx1, k1, idx2, k2, T, E, band, tokens_per_cta, hist, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_coselect(const int32_t* expert_idx, int T, int k, int E, int32_t* cosel,
                                   moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1) return MOE_ERR_ARG;
    if (E > 1024 || k > 32) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    if (!expert_idx || !cosel) return MOE_ERR_ARG;
    return launch_pair_hist(expert_idx, k, expert_idx, k, T, E, cosel, (cudaStream_t)stream);
}

extern "C" moe_status moe_transition(const int32_t* idx1, int k1, const int32_t* idx2, int k2, int T, int E,
                                     int32_t* trans, moe_stream_t stream) {
    if (T < 0 || k1 < 1 || k2 < 1 || E < 1) return MOE_ERR_ARG;
    if (E > 1024 || k1 > 32 || k2 > 32) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    if (!idx1 || !idx2 || !trans) return MOE_ERR_ARG;
    return launch_pair_hist(idx1, k1, idx2, k2, T, E, trans, (cudaStream_t)stream);
}
