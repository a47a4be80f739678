// route.cu - TopKRouter and ExpertChoiceRouter kernels.
//
// "How MegaDLMs Implements Mixture of Experts (MoE) Architectures",
// section "Routing Mechanisms: Top-K vs Expert Choice": the top-k router
// takes a softmax over the expert logits and keeps each token's k best
// experts with their probabilities; the expert-choice router lets every
// expert pick the tokens with the highest routing score.
#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------- top-k
// One warp per token.  Lane l holds logits e = l + 32 i (i < NV).  k rounds
// of a warp arg-max under (value desc, index asc) pick the experts; the
// top-1 value is the row maximum m.  Probabilities are exp(l - m) / sum.
// The difference l - m is split into its fp32 value and the exact rounding
// error (TwoSum, Knuth TAOCP vol. 2, 4.2.2), exp is taken of the fp32 part and
// corrected to first order by the error term, and the sum runs in fp64, so
// a gate's error is that of expf alone.
template <int NV>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                         int norm_topk, int32_t* __restrict__ expert_idx,
                                                         float* __restrict__ gate) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = warp; t < T; t += nwarps) {
        const float* row = logits + t * E;
        float v[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            int e = lane + 32 * i;
            v[i] = (e < E) ? __ldg(row + e) : 0.0f;
        }
        unsigned taken = 0;                      // bit i: v[i] already chosen (or out of range)
#pragma unroll
        for (int i = 0; i < NV; ++i)
            if (lane + 32 * i >= E) taken |= 1u << i;
        float m = 0.0f;
        float my_val = 0.0f;                     // lane j < k keeps slot j's value and index
        int my_idx = -1;
        for (int j = 0; j < k; ++j) {
            float bv = 0.0f;
            int bi = -1;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                if (taken & (1u << i)) continue;
                if (bi < 0 || v[i] > bv) { bv = v[i]; bi = lane + 32 * i; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                bool better = (oi >= 0) && (bi < 0 || ov > bv || (ov == bv && oi < bi));
                if (better) { bv = ov; bi = oi; }
            }
            if (j == 0) m = bv;
            if ((bi & 31) == lane && bi >= 0) taken |= 1u << (bi >> 5);
            if (lane == j) { my_val = bv; my_idx = bi; }
        }
        // exp(l - m) with the subtraction's rounding error folded back in
        auto expdiff = [m](float l) -> float {
            float hi = __fsub_rn(l, m);
            float bb = __fsub_rn(hi, l);                     // TwoSum(l, -m)
            float lo = __fadd_rn(__fsub_rn(l, __fsub_rn(hi, bb)), __fsub_rn(-m, bb));
            float e = expf(hi);
            return __fmaf_rn(e, lo, e);
        };
        double s = 0.0;
        if (norm_topk) {
            if (lane < k) s = (double)expdiff(my_val);
        } else {
#pragma unroll
            for (int i = 0; i < NV; ++i)
                if (lane + 32 * i < E) s += (double)expdiff(v[i]);
        }
        s = warp_sum(s);
        if (lane < k) {
            expert_idx[t * k + lane] = my_idx;
            gate[t * k + lane] = (float)((double)expdiff(my_val) / s);
        }
    }
}

// ---------------------------------------------------------- expert choice
// Scores compare as key = logit - lse, lse = m + log(sum_e exp(logit - m)),
// all in fp64 with the sum taken over e in ascending order (one thread per
// token), so the keys are those of the plain definition up to the last ulp
// of exp/log.

__global__ void ec_lse_kernel(const float* __restrict__ logits, int T, int E, double* __restrict__ lse) {
    int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const float* row = logits + (long long)t * E;
    double m = -INFINITY;
    for (int e = 0; e < E; ++e) m = fmax(m, (double)__ldg(row + e));
    double s = 0.0;
    for (int e = 0; e < E; ++e) s += exp((double)__ldg(row + e) - m);
    lse[t] = m + log(s);
}

// Order-preserving map of a double onto uint64 (larger double -> larger key).
__device__ __forceinline__ unsigned long long key_bits(double x) {
    unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// keysT[e][t] = key_bits(logit[t][e] - lse[t]), transposed through shared
// memory so that both the read and the write are coalesced.
__global__ void ec_keys_kernel(const float* __restrict__ logits, const double* __restrict__ lse, int T, int E,
                               unsigned long long* __restrict__ keysT) {
    __shared__ unsigned long long tile[32][33];
    const int t0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
    for (int r = ty; r < 32; r += 8) {
        int t = t0 + r, e = e0 + tx;
        if (t < T && e < E) tile[r][tx] = key_bits((double)logits[(long long)t * E + e] - lse[t]);
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        int e = e0 + r, t = t0 + tx;
        if (t < T && e < E) keysT[(long long)e * T + t] = tile[tx][r];
    }
}

// Block-wide exclusive scan of one int per thread (blockDim = 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, int* sh /*[32]*/) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int nw = blockDim.x >> 5;
        int w = lane < nw ? sh[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        sh[lane] = w;                               // inclusive over warps
    }
    __syncthreads();
    int base = wid ? sh[wid - 1] : 0;
    *total = sh[(blockDim.x >> 5) - 1];
    __syncthreads();
    return base + x - v;
}

// One 1024-thread CTA per expert: radix-select the C-th largest key
// (8 passes of 8 bits, stopping early once the boundary bucket is taken
// whole), then a stable compaction in token order; equal keys at the
// boundary go to the lowest token indices.  Also marks token membership
// bits for the CSR build.
__global__ void __launch_bounds__(1024) ec_select_kernel(const unsigned long long* __restrict__ keysT,
                                                         const float* __restrict__ logits, const double* __restrict__ lse,
                                                         int T, int E, int C, int32_t* __restrict__ ec_token,
                                                         float* __restrict__ ec_gate, unsigned* __restrict__ tokmask,
                                                         int mask_words) {
    __shared__ int hist[256];
    __shared__ int sh_scan[32];
    __shared__ unsigned long long s_prefix, s_mask;
    __shared__ int s_need, s_done;
    const int e = blockIdx.x;
    const unsigned long long* keys = keysT + (long long)e * T;
    if (threadIdx.x == 0) { s_prefix = 0; s_mask = 0; s_need = C; s_done = 0; }
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
        if (s_done) break;
        const int shift = 56 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        const unsigned long long prefix = s_prefix, mask = s_mask;
        for (int t = threadIdx.x; t < T; t += blockDim.x) {
            unsigned long long u = keys[t];
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255], 1);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int need = s_need, cum = 0, dgt = 255;
            for (; dgt > 0; --dgt) {
                if (cum + hist[dgt] >= need) break;
                cum += hist[dgt];
            }
            need -= cum;
            s_prefix = prefix | ((unsigned long long)dgt << shift);
            s_mask = mask | (255ull << shift);
            s_need = need;
            if (hist[dgt] == need) s_done = 1;       // the whole boundary bucket is taken
        }
        __syncthreads();
    }
    const unsigned long long prefix = s_prefix, mask = s_mask;
    const int need = s_need;
    int ties_before = 0, taken_before = 0;
    for (int t0 = 0; t0 < T; t0 += blockDim.x) {
        int t = t0 + threadIdx.x;
        int above = 0, tie = 0;
        if (t < T) {
            unsigned long long u = keys[t] & mask;
            above = u > prefix;
            tie = u == prefix;
        }
        int tie_total;
        int tie_rank = ties_before + block_exclusive_scan(tie, &tie_total, sh_scan);
        int sel = above || (tie && tie_rank < need);
        int sel_total;
        int pos = taken_before + block_exclusive_scan(sel, &sel_total, sh_scan);
        if (sel) {
            long long r = (long long)e * C + pos;
            ec_token[r] = t;
            ec_gate[r] = (float)exp((double)logits[(long long)t * E + e] - lse[t]);
            atomicOr(&tokmask[(long long)t * mask_words + (e >> 5)], 1u << (e & 31));
        }
        ties_before += tie_total;
        taken_before += sel_total;
    }
}

// tok_cnt[t] = number of experts that chose token t.
__global__ void ec_count_kernel(const unsigned* __restrict__ tokmask, int T, int mask_words, int32_t* __restrict__ cnt) {
    int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    int c = 0;
    for (int w = 0; w < mask_words; ++w) c += __popc(tokmask[(long long)t * mask_words + w]);
    cnt[t] = c;
}

// Device-wide exclusive scan of n ints, 1024 per CTA: local scans plus
// per-CTA totals, then a single-CTA scan of the totals, then the add-back.
__global__ void __launch_bounds__(1024) scan_local_kernel(const int32_t* __restrict__ in, int n, int32_t* __restrict__ out,
                                                          int32_t* __restrict__ block_tot) {
    __shared__ int sh[32];
    int i = blockIdx.x * 1024 + threadIdx.x;
    int v = i < n ? in[i] : 0;
    int tot;
    int ex = block_exclusive_scan(v, &tot, sh);
    if (i < n) out[i] = ex;
    if (threadIdx.x == 0) block_tot[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(1024) scan_totals_kernel(int32_t* __restrict__ block_tot, int nb, int32_t* __restrict__ grand) {
    __shared__ int sh[32];
    int carry = 0;
    for (int b0 = 0; b0 < nb; b0 += 1024) {
        int i = b0 + threadIdx.x;
        int v = i < nb ? block_tot[i] : 0;
        int tot;
        int ex = block_exclusive_scan(v, &tot, sh);
        if (i < nb) block_tot[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0 && grand) *grand = carry;
}

__global__ void scan_add_kernel(int32_t* __restrict__ out, int n, const int32_t* __restrict__ block_base) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] += block_base[i >> 10];
}

// tok_row[tok_ptr[t] + (#experts below e that chose t)] = row, for every row.
__global__ void ec_fill_kernel(const int32_t* __restrict__ ec_token, int E, int C, const unsigned* __restrict__ tokmask,
                               int mask_words, const int32_t* __restrict__ tok_ptr, int32_t* __restrict__ tok_row) {
    long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= (long long)E * C) return;
    int e = (int)(r / C);
    int t = ec_token[r];
    const unsigned* m = tokmask + (long long)t * mask_words;
    int below = 0;
    for (int w = 0; w < (e >> 5); ++w) below += __popc(m[w]);
    below += __popc(m[e >> 5] & ((1u << (e & 31)) - 1u));
    tok_row[tok_ptr[t] + below] = (int32_t)r;
}

}  // namespace moe

using namespace moe;

// ------------------------------------------------------------ host side

extern "C" moe_status moe_route_topk(const float* logits, int T, int E, int k, int norm_topk,
                                     int32_t* expert_idx, float* gate, moe_stream_t stream) {
    if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_ARG;
    if (k > 32 || E > 1024) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    if (!logits || !expert_idx || !gate) return MOE_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int threads = 256;
    long long warps_needed = T;
    int blocks = (int)((warps_needed + 7) / 8);
    if (blocks > 148 * 16) blocks = 148 * 16;
    const int nv = (E + 31) / 32;
#define MOE_TOPK_CASE(N) \
    case N: route_topk_kernel<N><<<blocks, threads, 0, s>>>(logits, T, E, k, norm_topk, expert_idx, gate); break;
    switch (nv <= 1 ? 1 : nv <= 2 ? 2 : nv <= 4 ? 4 : nv <= 8 ? 8 : nv <= 16 ? 16 : 32) {
        MOE_TOPK_CASE(1)
        MOE_TOPK_CASE(2)
        MOE_TOPK_CASE(4)
        MOE_TOPK_CASE(8)
        MOE_TOPK_CASE(16)
        MOE_TOPK_CASE(32)
    }
#undef MOE_TOPK_CASE
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

namespace {
struct EcWs {
    size_t lse, keys, mask, cnt, btot, total;
};
EcWs ec_layout(int T, int E) {
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    EcWs w;
    int mw = (E + 31) / 32;
    int nb = (T + 1 + 1023) / 1024;
    w.lse = 0;
    w.keys = w.lse + al(sizeof(double) * (size_t)T);
    w.mask = w.keys + al(sizeof(unsigned long long) * (size_t)T * E);
    w.cnt = w.mask + al(sizeof(unsigned) * (size_t)T * mw);
    w.btot = w.cnt + al(sizeof(int32_t) * (size_t)(T + 1));
    w.total = w.btot + al(sizeof(int32_t) * (size_t)(nb + 1));
    return w;
}
}  // namespace

extern "C" size_t moe_route_ec_workspace_bytes(int T, int E, int C) {
    (void)C;
    if (T < 0 || E < 1) return 0;
    return ec_layout(T, E).total;
}

extern "C" moe_status moe_route_ec(const float* logits, int T, int E, int C, int32_t* ec_token, float* ec_gate,
                                   int32_t* tok_ptr, int32_t* tok_row, void* workspace, size_t workspace_bytes,
                                   moe_stream_t stream) {
    if (T < 1 || E < 1 || C < 1 || C > T) return MOE_ERR_ARG;
    if (E > 1024) return MOE_ERR_SHAPE;
    if (!logits || !ec_token || !ec_gate || !tok_ptr || !tok_row) return MOE_ERR_ARG;
    EcWs L = ec_layout(T, E);
    if (!workspace || workspace_bytes < L.total || ((uintptr_t)workspace & 255)) return MOE_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    double* lse = (double*)(ws + L.lse);
    unsigned long long* keys = (unsigned long long*)(ws + L.keys);
    unsigned* mask = (unsigned*)(ws + L.mask);
    int32_t* cnt = (int32_t*)(ws + L.cnt);
    int32_t* btot = (int32_t*)(ws + L.btot);
    const int mw = (E + 31) / 32;
    if (cudaMemsetAsync(mask, 0, sizeof(unsigned) * (size_t)T * mw, s) != cudaSuccess) return MOE_ERR_CUDA;
    ec_lse_kernel<<<ceil_div(T, 128), 128, 0, s>>>(logits, T, E, lse);
    MOE_LAUNCH_CHECK();
    ec_keys_kernel<<<dim3(ceil_div(T, 32), ceil_div(E, 32)), 256, 0, s>>>(logits, lse, T, E, keys);
    MOE_LAUNCH_CHECK();
    ec_select_kernel<<<E, 1024, 0, s>>>(keys, logits, lse, T, E, C, ec_token, ec_gate, mask, mw);
    MOE_LAUNCH_CHECK();
    ec_count_kernel<<<ceil_div(T, 256), 256, 0, s>>>(mask, T, mw, cnt);
    MOE_LAUNCH_CHECK();
    // tok_ptr = exclusive scan of cnt, tok_ptr[T] = E*C
    const int n = T + 1;
    if (cudaMemsetAsync(cnt + T, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    const int nb = ceil_div(n, 1024);
    scan_local_kernel<<<nb, 1024, 0, s>>>(cnt, n, tok_ptr, btot);
    MOE_LAUNCH_CHECK();
    scan_totals_kernel<<<1, 1024, 0, s>>>(btot, nb, nullptr);
    MOE_LAUNCH_CHECK();
    scan_add_kernel<<<ceil_div(n, 256), 256, 0, s>>>(tok_ptr, n, btot);
    MOE_LAUNCH_CHECK();
    const long long rows = (long long)E * C;
    ec_fill_kernel<<<(int)((rows + 255) / 256), 256, 0, s>>>(ec_token, E, C, mask, mw, tok_ptr, tok_row);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
