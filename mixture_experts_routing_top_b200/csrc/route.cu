// route.cu - TopKRouter and ExpertChoiceRouter kernels.
//
// "How MegaDLMs Implements Mixture of Experts (MoE) Architectures",
// section "Routing Mechanisms: Top-K vs Expert Choice": the top-k router
// takes a softmax over the expert logits and keeps each token's k best
// experts with their probabilities; the expert-choice router lets every
// expert pick the tokens with the highest routing score.
#include <cstdlib>

#include "common.cuh"
#include "tcgen05.cuh"

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
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
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

// Vectorised variant for E % 4 == 0 (16-byte rows): lane l loads float4
// number l + 32 j, i.e. experts 128 j + 4 l + q.  Logits become
// order-preserving integer keys (-0 folded into +0 so that equal values tie
// exactly as floats do), and each selection round is two warp reductions:
// redux.sync max over the lanes' best keys, then redux.sync min over the
// expert indices holding that key (lowest index wins ties).  The winning
// value is recovered from its key, so no shuffles are needed.  The softmax
// denominator uses the hardware exp2 for each term, accumulated in fp64 (the
// sum is dominated by the terms nearest the maximum, where that exp is within
// a few ulp); the k gates themselves use expf with the TwoSum correction.
__device__ __forceinline__ unsigned f2key(float v) {
    unsigned u = __float_as_uint(__fadd_rn(v, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key2f(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int NV4>
__global__ void __launch_bounds__(256) route_topk_vec_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                             int norm_topk, int32_t* __restrict__ expert_idx,
                                                             float* __restrict__ gate) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    constexpr int NV = 4 * NV4;
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int E4 = E >> 2;
    for (long long t = warp; t < T; t += nwarps) {
        const uint4* row = reinterpret_cast<const uint4*>(logits + t * E);
        float v[NV];
        unsigned key[NV];
        unsigned taken = 0;
#pragma unroll
        for (int j = 0; j < NV4; ++j) {
            const int e4 = lane + 32 * j;
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (e4 < E4) w = ld_stream(row + e4);
            else taken |= 0xFu << (4 * j);
            v[4 * j + 0] = __uint_as_float(w.x);
            v[4 * j + 1] = __uint_as_float(w.y);
            v[4 * j + 2] = __uint_as_float(w.z);
            v[4 * j + 3] = __uint_as_float(w.w);
        }
#pragma unroll
        for (int i = 0; i < NV; ++i) key[i] = f2key(v[i]);
        float m = 0.0f, my_val = 0.0f;
        int my_idx = -1;
        for (int j = 0; j < k; ++j) {
            unsigned bk = 0;                     // 0 is below every real key
            int bi = -1;
#pragma unroll
            for (int i = 0; i < NV; ++i)
                if (!((taken >> i) & 1u) && (bi < 0 || key[i] > bk)) { bk = key[i]; bi = i; }
            const unsigned mk = __reduce_max_sync(0xffffffffu, bk);
            const unsigned cand = (bi >= 0 && bk == mk) ? (unsigned)(128 * (bi >> 2) + 4 * lane + (bi & 3)) : 0xFFFFFFFFu;
            const unsigned win = __reduce_min_sync(0xffffffffu, cand);
            if ((int)((win >> 2) & 31u) == lane) taken |= 1u << (4 * (win >> 7) + (win & 3u));
            const float wv = key2f(mk);
            if (j == 0) m = wv;
            if (lane == j) { my_val = wv; my_idx = (int)win; }
        }
        auto expdiff = [m](float l) -> float {
            float hi = __fsub_rn(l, m);
            float bb = __fsub_rn(hi, l);                     // TwoSum(l, -m)
            float lo = __fadd_rn(__fsub_rn(l, __fsub_rn(hi, bb)), __fsub_rn(-m, bb));
            float e = expf(hi);
            return __fmaf_rn(e, lo, e);
        };
        const float my_e = lane < k ? expdiff(my_val) : 0.0f;
        double s = 0.0;
        if (norm_topk) {
            s = (double)my_e;
        } else {
#pragma unroll
            for (int i = 0; i < NV; ++i)
                if (128 * (i >> 2) + 4 * lane + (i & 3) < E) s += (double)__expf(__fsub_rn(v[i], m));
        }
        s = warp_sum(s);
        if (lane < k) {
            expert_idx[t * k + lane] = my_idx;
            gate[t * k + lane] = (float)((double)my_e / s);
        }
    }
}

// Thread-per-token variant for k <= 8 and E % 4 == 0 (any E up to 1024).
// Each warp owns 32 consecutive tokens and walks their logits in chunks of
// 32 experts through its own shared-memory ring (cp.async, two chunks in
// flight; lanes copy 128-byte row pieces, 8 lanes per row, rows padded to
// 36 floats so that 128-bit reads of a lane's own row are conflict-free).
// Warps never wait for one another.
//
// Every lane ranks its own token by one 32-bit key per expert: the
// order-preserving image of the logit with its low `kbits` bits replaced by
// (2^kbits - 1 - expert), so keys are distinct, a larger key is a larger
// logit or, inside one bucket of 2^kbits consecutive images, a lower expert.
// The lane keeps the k + 1 best keys in a sorted list that a new key enters
// through a compare-exchange chain of integer max/min (no branch, no
// predicate per position).  Per chunk, one uniform pass marks the experts
// that can still enter the list (logit at or above the lowest float of the
// (k+1)-th key's bucket; for the first chunk at or above the lowest of
// k + 1 group maxima, which at least k + 1 of its logits reach), and the
// warp inserts the marked experts in step, one per lane per round.  At the
// end the k winners are exact unless the k-th and (k+1)-th keys share a
// bucket: then the lane ranks its row again with full comparisons (rare:
// two logits within 2^kbits units of the last place at the boundary, or
// exact ties).  Winners that share a bucket among themselves are put in
// exact order; their logits are read back for the gates.  With softmax
// gates the denominator adds the chunk's terms exp(l - m_run) relative to
// the running maximum (compensated fp32 sums per chunk, the fp64 total
// rescaled when the maximum grows); renormalised gates need only the k.
// Ties resolve as in the other variants (lower expert first, -0 == +0).
constexpr int kRowWarps = 4;                              // warps per CTA
constexpr int kRowChunk = 32;                             // experts per chunk
constexpr int kRowStride = 36;                            // floats per staged row
constexpr int kRowBufs = 3;
constexpr int kRowWarpFloats = kRowBufs * 32 * kRowStride;
constexpr int kRowSmem = kRowWarps * kRowWarpFloats * 4;  // 54 KB

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"((unsigned)__cvta_generic_to_shared(smem_dst)),
                 "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

// Order-preserving image of a float as an unsigned (a larger float, a larger
// image), -0 folded into +0 first so that the two are equal.  NaN patterns
// fall outside [image(-inf), image(+inf)].
__device__ __forceinline__ unsigned float_order_key(float v) {
    const unsigned b = __float_as_uint(__fadd_rn(v, 0.0f));
    return b ^ ((unsigned)((int)b >> 31) | 0x80000000u);
}
// The float whose image is `hk` (a bucket's lowest image); -inf at or below
// the image of -inf (the NaN patterns there, and the empty key 0).
__device__ __forceinline__ float float_of_order_key(unsigned hk) {
    if (hk <= 0x007FFFFFu) return -INFINITY;
    return __uint_as_float((hk & 0x80000000u) ? (hk ^ 0x80000000u) : ~hk);
}
// Insert x into the descending list L of distinct keys (x = 0, the empty
// key, changes nothing).  Entry j becomes max(L[j], min(L[j-1], x)): the
// entry above it if x went higher, x if x lands here, else itself - every
// entry from the old list at once, two dependent integer min/max deep.
template <int N>
__device__ __forceinline__ void key_insert(unsigned (&L)[N], unsigned x) {
#pragma unroll
    for (int j = N - 1; j >= 1; --j) L[j] = max(L[j], min(L[j - 1], x));
    L[0] = max(L[0], x);
}

template <int KM, bool NORM>
__global__ void __launch_bounds__(32 * kRowWarps, 4) route_topk_rows_kernel(const float* __restrict__ logits, int T,
                                                                            int E, int k, int kbits,
                                                                            int32_t* __restrict__ expert_idx,
                                                                            float* __restrict__ gate) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ __align__(16) float row_ring[];
    constexpr int NL = KM + 1;            // the k best keys and the next one
    const unsigned idx_max = (1u << kbits) - 1u, hi_mask = ~idx_max;
    const int lane = threadIdx.x & 31;
    float* ring = row_ring + (threadIdx.x >> 5) * kRowWarpFloats;
    const int E4 = E >> 2;
    const int nchunk = (E + kRowChunk - 1) / kRowChunk;
    const int lq = lane & 7;              // float4 slot this lane copies within a row piece
    const int lr = lane >> 3;             // first row this lane copies (then every 4th)
    const long long nwarps = (long long)gridDim.x * kRowWarps;
    for (long long w = (long long)blockIdx.x * kRowWarps + (threadIdx.x >> 5); w * 32 < T; w += nwarps) {
        const long long t0 = w * 32;
        auto issue = [&](int c) {
            if (c < nchunk) {
                const int f4 = c * (kRowChunk / 4) + lq;
                float* dst = ring + (c % kRowBufs) * (32 * kRowStride);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const long long tok = t0 + lr + 4 * u;
                    if (tok < T && f4 < E4)
                        cp_async16(&dst[(lr + 4 * u) * kRowStride + 4 * lq], logits + tok * E + 4 * f4);
                }
            }
            cp_async_commit();                 // one group per chunk slot, empty past the last chunk
        };
        unsigned L[NL];
#pragma unroll
        for (int j = 0; j < NL; ++j) L[j] = 0u;
        float m_run = -INFINITY;           // running maximum (the softmax reference)
        double s = 0.0;                    // sum of exp(l - m_run) so far
        const long long t = t0 + lane;
#pragma unroll
        for (int c = 0; c < kRowBufs - 1; ++c) issue(c);
        for (int c = 0; c < nchunk; ++c) {
            issue(c + kRowBufs - 1);           // into the slot scanned one iteration ago
            cp_async_wait<kRowBufs - 1>();     // chunk c: this lane's copies have landed
            __syncwarp();                      // ... and the other lanes' copies are visible
            const float* row = ring + (c % kRowBufs) * (32 * kRowStride) + lane * kRowStride;
            const int e0 = c * kRowChunk;
            unsigned msk = 0u;                 // this lane's candidates in the chunk
            if (t < T) {
                const int nv = min(kRowChunk, E - e0);
                // the (k+1)-th key so far: the least of the first k + 1 (a
                // minimum, not L[k], which would put L in local memory)
                unsigned lk = L[0];
#pragma unroll
                for (int j = 1; j < NL; ++j) lk = min(lk, j <= k ? L[j] : 0xFFFFFFFFu);
                float tau = float_of_order_key(lk & hi_mask);
                const float4* row4 = reinterpret_cast<const float4*>(row);
                if (c == 0 && nv == kRowChunk) {
                    // NL disjoint groups of the chunk (float4 q; the halves of the
                    // last one when NL = 9): their maxima are NL logits at or above
                    // the lowest of them, so the k + 1 best of the chunk are too
                    // (taken down to its bucket's lowest float, as the keys compare)
                    float gm[NL];
#pragma unroll
                    for (int g = 0; g < NL; ++g) gm[g] = -INFINITY;
#pragma unroll
                    for (int q = 0; q < kRowChunk / 4; ++q) {
                        const float4 a4 = row4[q];
                        if (NL > 8 && q == 7) {
                            gm[NL - 2] = fmaxf(a4.x, a4.y);
                            gm[NL - 1] = fmaxf(a4.z, a4.w);
                        } else {
                            const int g = NL > 8 ? q : q * NL / 8;
                            gm[g] = fmaxf(gm[g], fmaxf(fmaxf(a4.x, a4.y), fmaxf(a4.z, a4.w)));
                        }
                    }
                    float gmin = gm[0];
#pragma unroll
                    for (int g = 1; g < NL; ++g) gmin = fminf(gmin, gm[g]);
                    tau = float_of_order_key(float_order_key(gmin) & hi_mask);
                }
                unsigned m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int q = 0; q < kRowChunk / 4; ++q) {
                    const float4 a4 = row4[q];
                    const float v[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (4 * q + u < nv && v[u] >= tau) m4[u] |= 1u << (4 * q + u);
                }
                msk = m4[0] | m4[1] | m4[2] | m4[3];
                if (!NORM) {
                    float cm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int q = 0; q < kRowChunk / 4; ++q) {
                        const float4 a4 = row4[q];
                        const float v[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (4 * q + u < nv) cm4[u] = fmaxf(cm4[u], v[u]);
                    }
                    const float cm = fmaxf(fmaxf(cm4[0], cm4[1]), fmaxf(cm4[2], cm4[3]));
                    if (cm > m_run) {
                        s *= exp((double)m_run - (double)cm);
                        m_run = cm;
                    }
                    // four independent accumulators keep the dependency chains short
                    float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int q = 0; q < kRowChunk / 4; ++q) {
                        const float4 a4 = row4[q];
                        const float v[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (4 * q + u < nv) {
                                const float y = __fsub_rn(__expf(__fsub_rn(v[u], m_run)), cc[u]);
                                const float tt = __fadd_rn(cs[u], y);
                                cc[u] = __fsub_rn(__fsub_rn(tt, cs[u]), y);
                                cs[u] = tt;
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) s += (double)cs[u] - (double)cc[u];
                }
            }
            // the marked experts enter the list in step: each round every lane
            // inserts its next one, or the empty key once it has none left
            // (keys are distinct, so any order gives the same list); the next
            // key is read while the current one is inserted
            auto pop = [&]() -> unsigned {
                const int i = max(__ffs(msk) - 1, 0);
                const unsigned x = (float_order_key(row[i]) & hi_mask) | (idx_max - (unsigned)(e0 + i));
                const unsigned r = msk ? x : 0u;
                msk &= msk - 1;
                return r;
            };
            unsigned x = pop();
            while (__any_sync(0xffffffffu, x != 0u)) {
                const unsigned nx = pop();
                key_insert<NL>(L, x);
                x = nx;
            }
            __syncwarp();                      // slot c % kRowBufs may be refilled
        }
        cp_async_wait<0>();
        __syncwarp();                          // every lane is done with the ring
        const float* xr = logits + t * E;
        float bv[KM];
        int bi[KM];
        unsigned ka = L[0], kb = L[0];         // the k-th and (k+1)-th keys (minima, as above)
#pragma unroll
        for (int j = 1; j < NL; ++j) {
            ka = min(ka, j < k ? L[j] : 0xFFFFFFFFu);
            kb = min(kb, j <= k ? L[j] : 0xFFFFFFFFu);
        }
        // the boundary falls inside a bucket: which of its logits win is not known
        const bool amb = t < T && kb != 0u && ((ka ^ kb) & hi_mask) == 0u;
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            bi[j] = -1;
            bv[j] = -INFINITY;
            if (t < T && j < k && L[j] != 0u) {
                bi[j] = (int)(idx_max - (L[j] & idx_max));
                bv[j] = __ldg(xr + bi[j]);
            }
        }
        // Such a row: the winners above the boundary bucket stand; the other
        // places go to the bucket's logits in full order (image, then expert).
        // The warp copies the row into its ring and marks the bucket's
        // logits; the row's lane ranks those few.
        for (unsigned am = __ballot_sync(0xffffffffu, amb); am; am &= am - 1) {
            const int f = __ffs(am) - 1;
            const float4* src = reinterpret_cast<const float4*>(logits + (t0 + f) * E);
            for (int q = lane; q < E4; q += 32) reinterpret_cast<float4*>(ring)[q] = __ldg(src + q);
            const unsigned hb = __shfl_sync(0xffffffffu, kb & hi_mask, f);
            __syncwarp();
            unsigned ok[KM];
            int above = 0;                     // winners above the bucket (the list's first ones)
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                ok[j] = 0u;
                if (j < k && (L[j] & hi_mask) > hb) above = j + 1;
            }
            if (lane == f) {
#pragma unroll
                for (int j = 0; j < KM; ++j)
                    if (j >= above) bi[j] = -1;
            }
            for (int e0b = 0; e0b < E; e0b += 32) {
                const int e = e0b + lane;
                const float l = e < E ? ring[e] : 0.0f;
                const bool in = e < E && l == l && (float_order_key(l) & hi_mask) == hb;
                unsigned bm = __ballot_sync(0xffffffffu, in);
                if (lane == f) {
                    while (bm) {               // in expert order: strictly better displaces
                        const int i = __ffs(bm) - 1;
                        bm &= bm - 1;
                        unsigned u = float_order_key(ring[e0b + i]);
                        int ue = e0b + i;
                        bool placed = false;
#pragma unroll
                        for (int j = 0; j < KM; ++j) {
                            if (j >= above && (placed || u > ok[j])) {
                                placed = true;
                                const unsigned tu = ok[j];
                                const int te = bi[j];
                                ok[j] = u;
                                bi[j] = ue;
                                u = tu;
                                ue = te;
                            }
                        }
                    }
                }
            }
            if (lane == f) {
#pragma unroll
                for (int j = 0; j < KM; ++j)
                    if (j >= above) bv[j] = (j < k && bi[j] >= 0) ? ring[bi[j]] : -INFINITY;
            }
            __syncwarp();                      // the ring may be refilled
        }
        if (t < T) {
            // winners of one bucket are in expert order: put them in logit order
            bool share = false;
#pragma unroll
            for (int j = 1; j < KM; ++j)
                if (j < k && bi[j] >= 0 && ((float_order_key(bv[j]) ^ float_order_key(bv[j - 1])) & hi_mask) == 0u)
                    share = true;
            if (share) {
#pragma unroll
                for (int a = 1; a < KM; ++a) {
#pragma unroll
                    for (int b = a; b > 0; --b) {
                        if (b < k && bi[b] >= 0 && float_order_key(bv[b]) > float_order_key(bv[b - 1])) {
                            const float tv = bv[b];
                            bv[b] = bv[b - 1];
                            bv[b - 1] = tv;
                            const int ti = bi[b];
                            bi[b] = bi[b - 1];
                            bi[b - 1] = ti;
                        }
                    }
                }
            }
            const float m = bv[0];
            float ej[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) ej[j] = j < k ? exp_diff(bv[j], m) : 0.0f;
            if (NORM) {
                s = 0.0;
#pragma unroll
                for (int j = 0; j < KM; ++j) s += (double)ej[j];
            }
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j < k) {
                    expert_idx[t * k + j] = bi[j];
                    gate[t * k + j] = (float)((double)ej[j] / s);
                }
            }
        }
    }
}

// ---------------------------------------------------------- expert choice
// Scores compare as key = logit - lse, lse = m + log(sum_e exp(logit - m)),
// all in fp64 with the sum taken over e in ascending order (one thread per
// token), so the keys are those of the plain definition up to the last ulp
// of exp/log.

// Order-preserving map of a double onto uint64 (larger double -> larger key).
__device__ __forceinline__ unsigned long long key_bits(double x) {
    unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// A CTA takes `tpb` consecutive tokens (one contiguous span of logits).
// It writes each token's lse and, transposed ([e][t]), either the keys'
// selection bins (the binned selection) or the keys' high and low 32-bit
// halves (the selection from global memory, for larger T).
// Everything order-independent runs in parallel over the CTA's tokens x
// experts: the copy into shared memory, each row's max, every
// exp(l - m) in fp64; only the additions run one thread per token, over the
// experts in ascending order (the order of the logsumexp definition), from
// the staged exps.  Keys are then written transposed, keysT[e][t], with
// consecutive threads on consecutive tokens.
constexpr int kEcThreads = 256;

// Selection bins of the expert-choice keys: key = l - lse <= 0, bin =
// floor(-256 key) clamped to kEcBins - 1 (bins 1/256 wide over [-16, 0],
// every key below -16 in the last).  A larger key never has a larger bin:
// every key in a bin before the boundary bin beats every key in or after
// it, so only the boundary bin's keys are compared exactly.
constexpr int kEcBins = 4096;
__device__ __forceinline__ int ec_bin(double key) {
    const double y = -key * 256.0;
    return y >= (double)(kEcBins - 1) ? kEcBins - 1 : (y > 0.0 ? (int)y : 0);
}

__global__ void __launch_bounds__(kEcThreads) ec_lse_keys_kernel(const float* __restrict__ logits, int T, int E, int tpb,
                                                                 double* __restrict__ lse_out,
                                                                 unsigned* __restrict__ keys_hi,
                                                                 unsigned* __restrict__ keys_lo,
                                                                 uint16_t* __restrict__ bins,
                                                                 unsigned* __restrict__ tokmask, int mask_words) {
    extern __shared__ double ex[];                 // [tpb][E+1] exps (padded rows), [tpb] row max / lse, then
    const int ld = E + 1;                          // [tpb][E+1] the logits as floats (padded rows)
    double* rowv = ex + (size_t)tpb * ld;
    float* lg = reinterpret_cast<float*>(rowv + tpb);
    const long long t0 = (long long)blockIdx.x * tpb;
    const int rows = (int)min((long long)tpb, (long long)T - t0);
    const float* src = logits + t0 * E;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // the kernel before may still read the workspace
    // this CTA's tokens start with no expert's membership bit set
    for (int i = threadIdx.x; i < rows * mask_words; i += blockDim.x) tokmask[t0 * mask_words + i] = 0u;
    // logits into shared memory (read from global once) and each row's max
    // (exact in any order): one warp per row
    for (int r = wid; r < rows; r += nw) {
        float m = -INFINITY;
        for (int c = lane; c < E; c += 32) {
            const float l = __ldg(src + (long long)r * E + c);
            lg[r * ld + c] = l;
            m = fmaxf(m, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) rowv[r] = (double)m;
    }
    __syncthreads();
    // every exp(l - m) in fp64, in parallel; element f = r E + c, its row and
    // column stepped along with f (no division per element)
    const int n = rows * E;
    {
        const int dr = blockDim.x / E, dc = blockDim.x - dr * E;
        int r = threadIdx.x / E, c = threadIdx.x - r * E;
#pragma unroll 4
        for (int f = threadIdx.x; f < n; f += blockDim.x) {
            ex[r * ld + c] = exp((double)lg[r * ld + c] - rowv[r]);
            r += dr;
            c += dc;
            if (c >= E) { c -= E; ++r; }
        }
    }
    __syncthreads();
    // ascending-expert sums, one thread per token
    for (int r = threadIdx.x; r < rows; r += blockDim.x) {
        const double* er = ex + (size_t)r * ld;
        double sum = 0.0;
#pragma unroll 8
        for (int c = 0; c < E; ++c) sum += er[c];
        const double l = rowv[r] + log(sum);
        rowv[r] = l;
        lse_out[t0 + r] = l;
    }
    __syncthreads();
    // keys, transposed and coalesced, as their high and low 32-bit halves
    // (the selection reads the high halves first and the low ones rarely)
    {
        // element f = c rows + r (consecutive threads on consecutive tokens)
        const int dc = blockDim.x / rows, dr = blockDim.x - dc * rows;
        int c = threadIdx.x / rows, r = threadIdx.x - c * rows;
#pragma unroll 4
        for (int f = threadIdx.x; f < n; f += blockDim.x) {
            const double key = (double)lg[r * ld + c] - rowv[r];
            if (bins) {
                bins[(long long)c * T + t0 + r] = (uint16_t)ec_bin(key);
            } else {
                const unsigned long long kb = key_bits(key);
                keys_hi[(long long)c * T + t0 + r] = (unsigned)(kb >> 32);
                keys_lo[(long long)c * T + t0 + r] = (unsigned)kb;
            }
            c += dc;
            r += dr;
            if (r >= rows) { r -= rows; ++c; }
        }
    }
}

int ec_tokens_per_block(int E) {
    int tpb = 32;                                   // ~33 KB at E = 128: several CTAs per SM
    while (tpb > 1 && (size_t)tpb * ((E + 2) * sizeof(double) + (E + 1) * sizeof(float)) > 96 * 1024) tpb >>= 1;
    return tpb;
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

// One 1024-thread CTA per expert: radix-select the C-th largest key, then a
// stable compaction in token order (equal keys at the boundary go to the
// lowest token indices).  The leading bits all keys share (from their min
// and max) are skipped; each pass histograms the next 8 bits of the keys
// still matching the chosen prefix, with one shared-memory atomic per
// distinct digit per warp (__match_any_sync); the search stops once the
// boundary bucket is taken whole.  Also sets the token-membership bits used
// to build the token CSR.
__global__ void __launch_bounds__(1024) ec_select_kernel(const unsigned* __restrict__ keys_hi,
                                                         const unsigned* __restrict__ keys_lo, int T, int E, int C,
                                                         int32_t* __restrict__ ec_token, unsigned* __restrict__ tokmask,
                                                         int mask_words) {
    __shared__ int hist[256];
    __shared__ unsigned long long s_prefix, s_mask, s_min, s_max;
    __shared__ int s_need, s_done, s_hi;
    const int e = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const unsigned* khi = keys_hi + (long long)e * T;
    const unsigned* klo = keys_lo + (long long)e * T;
    auto key = [&](int t) -> unsigned long long { return ((unsigned long long)khi[t] << 32) | klo[t]; };
    pdl_wait();
    if (threadIdx.x == 0) { s_min = ~0ull; s_max = 0ull; }
    __syncthreads();
    unsigned long long lmin = ~0ull, lmax = 0ull;
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        const unsigned long long u = key(t);
        lmin = min(lmin, u);
        lmax = max(lmax, u);
    }
    atomicMin(&s_min, lmin);
    atomicMax(&s_max, lmax);
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long diff = s_min ^ s_max;
        s_need = C;
        if (diff == 0) {                          // every key equal: the C lowest tokens
            s_prefix = s_min; s_mask = ~0ull; s_done = 1; s_hi = -1;
        } else {
            const int hi = 63 - __clzll(diff);    // highest differing bit
            const unsigned long long low = (hi == 63) ? ~0ull : ((1ull << (hi + 1)) - 1ull);
            s_mask = ~low;
            s_prefix = s_min & ~low;
            s_done = 0;
            s_hi = hi;
        }
    }
    __syncthreads();
    while (!s_done && s_hi >= 0) {
        const int hi = s_hi;
        const int shift = max(hi - 7, 0);
        const int width = hi - shift + 1;
        const unsigned bins_mask = (1u << width) - 1u;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        const unsigned long long prefix = s_prefix, mask = s_mask;
        for (int t0 = 0; t0 < T; t0 += blockDim.x) {
            const int t = t0 + threadIdx.x;
            int digit = -1;
            if (t < T) {
                const unsigned long long u = key(t);
                if ((u & mask) == prefix) digit = (int)((u >> shift) & bins_mask);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, digit);
            if (digit >= 0 && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&hist[digit], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int need = s_need, cum = 0, dgt = (int)bins_mask;
            for (; dgt > 0; --dgt) {
                if (cum + hist[dgt] >= need) break;
                cum += hist[dgt];
            }
            need -= cum;
            const unsigned long long field = (unsigned long long)bins_mask << shift;
            s_prefix = prefix | ((unsigned long long)dgt << shift);
            s_mask = mask | field;
            s_need = need;
            if (hist[dgt] == need || shift == 0) s_done = 1;   // boundary bucket taken whole, or key fully resolved
            s_hi = shift - 1;
        }
        __syncthreads();
    }
    // stable compaction: warp w owns tokens [w*S, (w+1)*S); pass 1 counts the
    // keys above the threshold prefix and the ties per warp, one scan over
    // the 32 warps gives each warp its bases, pass 2 writes in token order.
    const unsigned long long prefix = s_prefix, mask = s_mask;
    const int need = s_need;
    __shared__ int w_above[32], w_tie[32];
    const int wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int S = (T + nw - 1) / nw;
    const int seg0 = min(wid * S, T), seg1 = min(seg0 + S, T);
    const unsigned lt = (1u << lane) - 1u;
    int n_above = 0, n_tie = 0;
    for (int c = seg0; c < seg1; c += 32) {
        const int t = c + lane;
        bool above = false, tie = false;
        if (t < seg1) {
            const unsigned long long u = key(t) & mask;
            above = u > prefix;
            tie = u == prefix;
        }
        n_above += __popc(__ballot_sync(0xffffffffu, above));
        n_tie += __popc(__ballot_sync(0xffffffffu, tie));
    }
    if (lane == 0) { w_above[wid] = n_above; w_tie[wid] = n_tie; }
    __syncthreads();
    int above_base = 0, tie_base = 0;
    for (int q = 0; q < wid; ++q) { above_base += w_above[q]; tie_base += w_tie[q]; }
    int sel_base = above_base + min(tie_base, need);
    for (int c = seg0; c < seg1; c += 32) {
        const int t = c + lane;
        bool above = false, tie = false;
        if (t < seg1) {
            const unsigned long long u = key(t) & mask;
            above = u > prefix;
            tie = u == prefix;
        }
        const unsigned tie_mask = __ballot_sync(0xffffffffu, tie);
        const int tie_rank = tie_base + __popc(tie_mask & lt);
        const bool sel = above || (tie && tie_rank < need);
        const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const long long r = (long long)e * C + sel_base + __popc(sel_mask & lt);
            ec_token[r] = t;
            atomicOr(&tokmask[(long long)t * mask_words + (e >> 5)], 1u << (e & 31));
        }
        tie_base += __popc(tie_mask);
        sel_base += __popc(sel_mask);
    }
}

// Warp 0: scanning digit bins from the top, find the bin where the running
// count first reaches `need` (nbins <= 256, 8 bins per lane, one warp scan).
// Writes the bin and the count still needed inside it.
__device__ __forceinline__ void warp_find_boundary(const int* hist, int nbins, int need, int* out_bin,
                                                   int* out_need, int* out_count) {
    const int lane = threadIdx.x & 31;
    int c[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int b = nbins - 1 - 8 * lane - j;
        c[j] = b >= 0 ? hist[b] : 0;
        sum += c[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
    const int L = hit ? __ffs(hit) - 1 : 31;
    if (lane == L) {
        int cum = incl - sum, bin = nbins - 1 - 8 * lane, cnt = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int b = nbins - 1 - 8 * lane - j;
            if (b < 0) break;
            bin = b;
            cnt = c[j];
            if (cum + c[j] >= need) break;
            cum += c[j];
        }
        *out_bin = bin;
        *out_need = need - cum;
        *out_count = cnt;
    }
}

// Binned selection (T <= kEcBinTokens): one 1024-thread CTA per expert.
// The expert's T key bins are loaded once into shared memory (two per
// 32-bit load) and counted; the boundary bin is the bin, from the best,
// where the running count reaches C.  Tokens in earlier bins are selected,
// in later bins not.  The boundary bin is taken whole when it holds exactly
// the C - (earlier) keys still needed; otherwise its tokens' exact keys
// (l - lse in fp64, recomputed from the logits and the lse as the key
// kernel computes them) decide: ranked pairwise (key descending, then token
// ascending) when the bin holds at most kEcBrute tokens, else by an 8-bit
// radix select over the 64-bit order-preserving keys (ties at the end
// resolved in token order).  Each warp owns a contiguous run of 64-token
// groups, a lane two adjacent tokens of each: one pass counts the warp's
// selected tokens and lists the boundary bin's, a second writes the rows in
// token order.  (The radix case classifies token by token, 32 tokens a
// word.)  Global loads that depend on a token (its exact key, its gate
// exp(key)) are made after the passes, all at once, so that no warp waits
// on them inside a pass.  Also sets the token-membership bits used to build
// the token CSR.
constexpr int kEcBinTokens = 65536;
constexpr int kEcBrute = 256;

__global__ void __launch_bounds__(1024) ec_select_bins_kernel(const uint16_t* __restrict__ bins,
                                                              const float* __restrict__ logits,
                                                              const double* __restrict__ lse, int T, int E, int C,
                                                              int32_t* __restrict__ ec_token,
                                                              float* __restrict__ ec_gate,
                                                              unsigned* __restrict__ tokmask, int mask_words) {
    extern __shared__ __align__(16) unsigned char ec_sm[];
    const int nwords = (T + 31) >> 5;
    const int ngroups = (T + 63) >> 6;
    int* hist = reinterpret_cast<int*>(ec_sm);                              // [kEcBins]
    unsigned long long* ckey = reinterpret_cast<unsigned long long*>(hist + kEcBins);   // [kEcBrute]
    int* ctok = reinterpret_cast<int*>(ckey + kEcBrute);                    // [kEcBrute]
    unsigned* m_sel = reinterpret_cast<unsigned*>(ctok + kEcBrute);         // [nwords] (radix case)
    unsigned* m_tie = m_sel + nwords;                                       // [nwords] (radix case)
    unsigned* chosen = m_tie + nwords;                                      // [nwords] boundary-bin tokens kept
    uint16_t* bs = reinterpret_cast<uint16_t*>(chosen + nwords);            // [64 ngroups], zero past T
    __shared__ int sh[32];
    __shared__ int s_bin, s_need, s_bcount, s_nc, s_done, s_rbin, s_rneed, s_rcount;
    __shared__ unsigned long long s_prefix, s_mask;
    __shared__ int w_sel[32], w_tie[32];
    const int e = blockIdx.x;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const unsigned lt = (1u << lane) - 1u;
    for (int i = threadIdx.x; i < kEcBins; i += blockDim.x) hist[i] = 0;
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) chosen[i] = 0u;
    if (threadIdx.x < 32) w_sel[threadIdx.x] = 0;
    __syncthreads();
    pdl_wait();                                    // the bins come from the kernel before
    const uint16_t* src = bins + (long long)e * T;
    unsigned* bs2 = reinterpret_cast<unsigned*>(bs);                        // bin pairs
    if ((T & 1) == 0) {
        // pairs of bins, 4-byte aligned (e T is even)
        const unsigned* src2 = reinterpret_cast<const unsigned*>(src);
        const int npairs = T >> 1;
        for (int p0 = 0; p0 < npairs; p0 += 16 * blockDim.x) {
            unsigned u[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int p = p0 + q * blockDim.x + threadIdx.x;
                u[q] = p < npairs ? src2[p] : 0xFFFFFFFFu;
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                if (u[q] == 0xFFFFFFFFu) continue;
                bs2[p0 + q * blockDim.x + threadIdx.x] = u[q];
                atomicAdd(&hist[u[q] & 0xFFFFu], 1);
                atomicAdd(&hist[u[q] >> 16], 1);
            }
        }
    } else {
        for (int t0 = 0; t0 < T; t0 += 8 * blockDim.x) {
            int u[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int t = t0 + q * blockDim.x + threadIdx.x;
                u[q] = t < T ? (int)src[t] : -1;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (u[q] < 0) continue;
                bs[t0 + q * blockDim.x + threadIdx.x] = (uint16_t)u[q];
                atomicAdd(&hist[u[q]], 1);
            }
        }
    }
    for (int t = T + threadIdx.x; t < 64 * ngroups; t += blockDim.x) bs[t] = 0;   // read below, never counted
    __syncthreads();
    {
        // each thread 4 consecutive bins; the one whose bins hold the C-th key finds the boundary bin
        constexpr int per = kEcBins / 1024;
        int c[per], sum = 0;
#pragma unroll
        for (int j = 0; j < per; ++j) {
            c[j] = hist[per * threadIdx.x + j];
            sum += c[j];
        }
        int total;
        int cum = block_exclusive_scan(sum, &total, sh);
        if (cum < C && cum + sum >= C) {
#pragma unroll
            for (int j = 0; j < per; ++j) {
                if (cum + c[j] >= C) {
                    s_bin = per * threadIdx.x + j;
                    s_need = C - cum;
                    s_bcount = c[j];
                    break;
                }
                cum += c[j];
            }
        }
    }
    if (threadIdx.x == 0) s_nc = 0;
    __syncthreads();
    const int bstar = s_bin;
    int need = s_need;
    const int bcount = s_bcount;
    const int mode = bcount == need ? 0 : (bcount <= kEcBrute ? 1 : 2);
    auto key_of = [&](int t) { return (double)logits[(long long)t * E + e] - lse[t]; };
    auto exact_key = [&](int t) { return key_bits(key_of(t)); };
    // the warp's groups of 64 tokens; lane l holds tokens 64 g + 2 l and 64 g + 2 l + 1
    const int gper = (ngroups + nw - 1) / nw;
    const int g0 = min(wid * gper, ngroups), g1 = min(g0 + gper, ngroups);
    if (mode != 2) {
        // mark the warp's tokens in bins before the boundary bin (and in it
        // when it is taken whole); list the boundary bin's tokens
        for (int g = g0; g < g1; ++g) {
            const unsigned pr = bs2[32 * g + lane];
            const int t = 64 * g + 2 * lane;
            const int bA = (int)(pr & 0xFFFFu), bB = (int)(pr >> 16);
            const bool okA = t < T, okB = t + 1 < T;
            // tokens before the boundary bin (and in it when it is taken whole) are chosen
            if (okA && (bA < bstar || (mode == 0 && bA == bstar))) atomicOr(&chosen[t >> 5], 1u << (t & 31));
            if (okB && (bB < bstar || (mode == 0 && bB == bstar))) atomicOr(&chosen[(t + 1) >> 5], 1u << ((t + 1) & 31));
            if (mode == 1) {
                const bool inA = okA && bA == bstar, inB = okB && bB == bstar;
                const unsigned mA = __ballot_sync(0xffffffffu, inA), mB = __ballot_sync(0xffffffffu, inB);
                if (mA | mB) {
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&s_nc, __popc(mA) + __popc(mB));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    int slot = base + __popc(mA & lt) + __popc(mB & lt);
                    if (inA) {
                        if (slot < kEcBrute) ctok[slot] = t;
                        ++slot;
                    }
                    if (inB && slot < kEcBrute) ctok[slot] = t + 1;
                }
            }
        }
        __syncthreads();
        if (mode == 1) {
            // the listed tokens' exact keys, all loads at once, then pairwise ranks
            const int nc = min(s_nc, kEcBrute);
            if ((int)threadIdx.x < nc) ckey[threadIdx.x] = exact_key(ctok[threadIdx.x]);
            __syncthreads();
            if ((int)threadIdx.x < nc) {
                const unsigned long long k0 = ckey[threadIdx.x];
                const int t = ctok[threadIdx.x];
                int rank = 0;
                for (int j = 0; j < nc; ++j) {
                    const unsigned long long kj = ckey[j];
                    rank += (kj > k0 || (kj == k0 && ctok[j] < t)) ? 1 : 0;
                }
                if (rank < need) atomicOr(&chosen[t >> 5], 1u << (t & 31));
            }
            __syncthreads();
        }
        // the chosen tokens in token order: each thread takes consecutive words
        // of the membership bits, a block scan of their counts gives its first
        // output place
        const int wpt = (nwords + (int)blockDim.x - 1) / (int)blockDim.x;
        const int w0 = min((int)threadIdx.x * wpt, nwords), w1 = min(w0 + wpt, nwords);
        int cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += __popc(chosen[w]);
        int total;
        int pos = block_exclusive_scan(cnt, &total, sh);
        for (int w = w0; w < w1; ++w) {
            unsigned m = chosen[w];
            while (m) {
                const int t = 32 * w + __ffs(m) - 1;
                m &= m - 1;
                if (pos < C) {                 // exactly C bits are set
                    const long long r = (long long)e * C + pos;
                    ec_token[r] = t;
                    atomicOr(&tokmask[(long long)t * mask_words + (e >> 5)], 1u << (e & 31));
                    ec_gate[r] = (float)exp(key_of(t));
                }
                ++pos;
            }
        }
        return;
    }
    // radix over the boundary bin's 64-bit keys, from the top byte
    if (threadIdx.x == 0) { s_prefix = 0ull; s_mask = 0ull; s_done = 0; s_rneed = need; }
    __syncthreads();
    for (int shift = 56; shift >= 0 && !s_done; shift -= 8) {
        const unsigned long long prefix = s_prefix, mask = s_mask;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int t0 = 0; t0 < T; t0 += blockDim.x) {
            const int t = t0 + threadIdx.x;
            if (t < T && bs[t] == bstar) {
                const unsigned long long k0 = exact_key(t);
                if ((k0 & mask) == prefix) atomicAdd(&hist[(int)((k0 >> shift) & 255ull)], 1);
            }
        }
        __syncthreads();
        if (wid == 0) warp_find_boundary(hist, 256, s_rneed, &s_rbin, &s_rneed, &s_rcount);
        __syncthreads();
        if (threadIdx.x == 0) {
            s_prefix = prefix | ((unsigned long long)s_rbin << shift);
            s_mask = mask | (255ull << shift);
            if (s_rcount == s_rneed) s_done = 1;
        }
        __syncthreads();
    }
    need = s_rneed;
    const unsigned long long prefix = s_prefix, mask = s_mask;
    // 1 selected, 2 at the threshold (tie order decides), 0 not
    auto classify = [&](int t) -> int {
        const int b = bs[t];
        if (b != bstar) return b < bstar ? 1 : 0;
        const unsigned long long km = exact_key(t) & mask;
        if (km != prefix) return km > prefix ? 1 : 0;
        return 2;
    };
    const int wper = (nwords + nw - 1) / nw;
    const int w0 = min(wid * wper, nwords), w1 = min(w0 + wper, nwords);
    int n_sel = 0, n_tie = 0;
    for (int w = w0; w < w1; ++w) {
        const int t = 32 * w + lane;
        const int cl = t < T ? classify(t) : 0;
        const unsigned sb = __ballot_sync(0xffffffffu, cl == 1);
        const unsigned tb = __ballot_sync(0xffffffffu, cl == 2);
        if (lane == 0) { m_sel[w] = sb; m_tie[w] = tb; }
        n_sel += __popc(sb);
        n_tie += __popc(tb);
    }
    if (lane == 0) { w_sel[wid] = n_sel; w_tie[wid] = n_tie; }
    __syncthreads();
    int sel_before = 0, tie_base = 0;
    for (int q = 0; q < wid; ++q) { sel_before += w_sel[q]; tie_base += w_tie[q]; }
    int out_base = sel_before + min(tie_base, need);
    for (int w = w0; w < w1; ++w) {
        const int t = 32 * w + lane;
        const unsigned sb = m_sel[w], tb = m_tie[w];
        const int tie_rank = tie_base + __popc(tb & lt);
        const bool sel = ((sb >> lane) & 1u) || (((tb >> lane) & 1u) && tie_rank < need);
        const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            ec_token[(long long)e * C + out_base + __popc(sel_mask & lt)] = t;
            atomicOr(&tokmask[(long long)t * mask_words + (e >> 5)], 1u << (e & 31));
        }
        tie_base += __popc(tb);
        out_base += __popc(sel_mask);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < C; j += blockDim.x) {
        const long long r = (long long)e * C + j;
        ec_gate[r] = (float)exp(key_of(ec_token[r]));
    }
}

// tok_ptr = exclusive scan over tokens of the number of experts that chose
// each token (the popcount of its membership words); tok_ptr[T] = total.
// One cluster of kScanCtas CTAs, which the hardware schedules together: CTA
// c scans tokens [c T / kScanCtas, (c + 1) T / kScanCtas), each thread a
// contiguous run of them; the CTAs' totals are exchanged through
// distributed shared memory between two cluster barriers.
constexpr int kScanCtas = 8;

__global__ void __cluster_dims__(kScanCtas, 1, 1) __launch_bounds__(1024, 1)
ec_count_scan_kernel(const unsigned* __restrict__ tokmask, int T, int mask_words, int32_t* __restrict__ tok_ptr) {
    constexpr int kCache = 16;                 // tokens per thread whose counts stay in registers
    __shared__ int sh[32];
    __shared__ int cta_total;
    pdl_trigger();
    const int c = (int)tc::cluster_rank();
    const long long t0 = (long long)T * c / kScanCtas, t1 = (long long)T * (c + 1) / kScanCtas;
    const long long per = (t1 - t0 + blockDim.x - 1) / blockDim.x;
    const long long a = min(t0 + per * threadIdx.x, t1), b = min(a + per, t1);
    pdl_wait();
    auto count = [&](long long t) {
        int n = 0;
        if (mask_words == 4) {                 // E in (96, 128]: one 16-byte load per token
            const uint4 u = reinterpret_cast<const uint4*>(tokmask)[t];
            n = __popc(u.x) + __popc(u.y) + __popc(u.z) + __popc(u.w);
        } else {
            for (int w = 0; w < mask_words; ++w) n += __popc(tokmask[t * mask_words + w]);
        }
        return n;
    };
    int cached[kCache];
    int mine = 0;
#pragma unroll
    for (int j = 0; j < kCache; ++j) {
        cached[j] = a + j < b ? count(a + j) : 0;
        mine += cached[j];
    }
    for (long long t = a + kCache; t < b; ++t) mine += count(t);
    int tot;
    const int ex = block_exclusive_scan(mine, &tot, sh);
    if (threadIdx.x == 0) cta_total = tot;
    __syncthreads();
    tc::cluster_sync();
    int v[kScanCtas];
    const uint32_t local = tc::smem_u32(&cta_total);
#pragma unroll
    for (int q = 0; q < kScanCtas; ++q) v[q] = (int)tc::ld_shared_cluster_u32(tc::map_to_rank(local, (uint32_t)q));
    int before = 0, all = 0;
#pragma unroll
    for (int q = 0; q < kScanCtas; ++q) {
        if (q < c) before += v[q];
        all += v[q];
    }
    // every CTA's reads of the others' cta_total are performed before any
    // CTA exits: a release arrive (a relaxed one may be observed while the
    // loads are still in flight, and the sums above are free to be
    // computed after it)
    tc::cluster_sync();
    int run = before + ex;
#pragma unroll
    for (int j = 0; j < kCache; ++j) {
        if (a + j < b) {
            tok_ptr[a + j] = run;
            run += cached[j];
        }
    }
    for (long long t = a + kCache; t < b; ++t) {
        tok_ptr[t] = run;
        run += count(t);
    }
    if (c == kScanCtas - 1 && threadIdx.x == 0) tok_ptr[T] = all;
}

// For every buffer row r = e*C + i holding token t:
// tok_row[tok_ptr[t] + (#experts below e that chose t)] = r, and its gate
// exp(key) when `gates` (the binned selection writes the gates itself).
__global__ void ec_fill_kernel(const int32_t* __restrict__ ec_token, int T, int E, int C,
                               const unsigned* __restrict__ tokmask, int mask_words,
                               const int32_t* __restrict__ tok_ptr, const float* __restrict__ logits,
                               const double* __restrict__ lse, int gates, float* __restrict__ ec_gate,
                               int32_t* __restrict__ tok_row) {
    long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    pdl_wait();
    if (r >= (long long)E * C) return;
    int e = (int)(r / C);
    int t = ec_token[r];
    if (gates) ec_gate[r] = (float)exp((double)logits[(long long)t * E + e] - lse[t]);
    int below = 0;
    if (mask_words == 4) {
        const uint4 u = reinterpret_cast<const uint4*>(tokmask)[t];
        const unsigned wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if (w < (e >> 5)) below += __popc(wv[w]);
            else if (w == (e >> 5)) below += __popc(wv[w] & ((1u << (e & 31)) - 1u));
        }
    } else {
        const unsigned* m = tokmask + (long long)t * mask_words;
        for (int w = 0; w < (e >> 5); ++w) below += __popc(m[w]);
        below += __popc(m[e >> 5] & ((1u << (e & 31)) - 1u));
    }
    tok_row[tok_ptr[t] + below] = (int32_t)r;
}

}  // namespace moe

using namespace moe;

// ------------------------------------------------------------ host side

namespace {
// Thread per token needs enough tokens to occupy the GPU (T threads in
// all), and pays off when the warp kernels would spend many reduction
// rounds (k >= 4); otherwise the warp-per-token kernels keep more warps in
// flight.  LIBMOE_TOPK_ROWS=0/1 forces either choice.
bool use_rows_variant(int T, int k) {
    const char* env = getenv("LIBMOE_TOPK_ROWS");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return T >= 32768 && k >= 4;
}
}  // namespace

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
    if (E % 4 == 0 && k <= 8 && ((uintptr_t)logits & 15) == 0 && use_rows_variant(T, k)) {
        for (auto fn : {route_topk_rows_kernel<1, false>, route_topk_rows_kernel<2, false>,
                        route_topk_rows_kernel<4, false>, route_topk_rows_kernel<8, false>,
                        route_topk_rows_kernel<1, true>, route_topk_rows_kernel<2, true>,
                        route_topk_rows_kernel<4, true>, route_topk_rows_kernel<8, true>})
            if (!set_smem_limit((const void*)fn, kRowSmem)) return MOE_ERR_CUDA;
        const long long warps = ((long long)T + 31) / 32;
        long long rb = (warps + kRowWarps - 1) / kRowWarps;
        const int rblocks = (int)(rb < 148 * 8 ? rb : 148 * 8);
        int kbits = 0;                                   // bits that hold an expert index
        while ((1 << kbits) < E) ++kbits;
#define MOE_TOPKR_CASE(KM)                                                                                      \
    (void)(norm_topk ? launch_pdl(route_topk_rows_kernel<KM, true>, rblocks, 32 * kRowWarps, kRowSmem, s, logits, \
                                  T, E, k, kbits, expert_idx, gate)                                             \
                     : launch_pdl(route_topk_rows_kernel<KM, false>, rblocks, 32 * kRowWarps, kRowSmem, s, logits, \
                                  T, E, k, kbits, expert_idx, gate))
        if (k <= 1) MOE_TOPKR_CASE(1);
        else if (k <= 2) MOE_TOPKR_CASE(2);
        else if (k <= 4) MOE_TOPKR_CASE(4);
        else MOE_TOPKR_CASE(8);
#undef MOE_TOPKR_CASE
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
    if (E % 4 == 0 && ((uintptr_t)logits & 15) == 0) {
        const int nv4 = (E + 127) / 128;
#define MOE_TOPKV_CASE(N) \
    case N: (void)launch_pdl(route_topk_vec_kernel<N>, blocks, threads, 0, s, logits, T, E, k, norm_topk, expert_idx, gate); break;
        switch (nv4 <= 1 ? 1 : nv4 <= 2 ? 2 : nv4 <= 4 ? 4 : 8) {
            MOE_TOPKV_CASE(1)
            MOE_TOPKV_CASE(2)
            MOE_TOPKV_CASE(4)
            MOE_TOPKV_CASE(8)
        }
#undef MOE_TOPKV_CASE
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
#define MOE_TOPK_CASE(N) \
    case N: (void)launch_pdl(route_topk_kernel<N>, blocks, threads, 0, s, logits, T, E, k, norm_topk, expert_idx, gate); break;
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
    size_t lse, keys, mask, total;
};
EcWs ec_layout(int T, int E) {
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    EcWs w;
    int mw = (E + 31) / 32;
    w.lse = 0;
    w.keys = w.lse + al(sizeof(double) * (size_t)T);              // high halves [E][T], then low halves [E][T]
    w.mask = w.keys + al(2 * sizeof(unsigned) * (size_t)T * E);
    w.total = w.mask + al(sizeof(unsigned) * (size_t)T * mw);
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
    unsigned* keys_hi = (unsigned*)(ws + L.keys);
    unsigned* keys_lo = keys_hi + (size_t)T * E;
    unsigned* mask = (unsigned*)(ws + L.mask);
    const int mw = (E + 31) / 32;
    const bool binned = T <= kEcBinTokens;
    uint16_t* bins = binned ? reinterpret_cast<uint16_t*>(keys_hi) : nullptr;   // the keys' space holds the bins
    {
        const int tpb = ec_tokens_per_block(E);
        const size_t smem = (size_t)tpb * ((E + 2) * sizeof(double) + (E + 1) * sizeof(float));
        if (!set_smem_limit((const void*)ec_lse_keys_kernel, smem)) return MOE_ERR_CUDA;
        if (launch_pdl(ec_lse_keys_kernel, ceil_div(T, tpb), kEcThreads, smem, s, logits, T, E, tpb, lse, keys_hi,
                       keys_lo, bins, mask, mw) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
    }
    cudaError_t rc;
    if (binned) {
        const size_t nwords = (size_t)(T + 31) / 32, ngroups = (size_t)(T + 63) / 64;
        const size_t smem = sizeof(int) * kEcBins + (sizeof(unsigned long long) + sizeof(int)) * kEcBrute +
                            3 * sizeof(unsigned) * nwords + sizeof(uint16_t) * 64 * ngroups;
        if (!set_smem_limit((const void*)ec_select_bins_kernel, smem)) return MOE_ERR_CUDA;
        rc = launch_pdl(ec_select_bins_kernel, E, 1024, smem, s, (const uint16_t*)bins, logits, (const double*)lse, T,
                        E, C, ec_token, ec_gate, mask, mw);
    } else {
        rc = launch_pdl(ec_select_kernel, E, 1024, 0, s, (const unsigned*)keys_hi, (const unsigned*)keys_lo, T, E, C,
                        ec_token, mask, mw);
    }
    if (rc != cudaSuccess) return MOE_ERR_CUDA;
    MOE_LAUNCH_CHECK();
    if (launch_pdl(ec_count_scan_kernel, kScanCtas, 1024, 0, s, (const unsigned*)mask, T, mw, tok_ptr) != cudaSuccess)
        return MOE_ERR_CUDA;
    MOE_LAUNCH_CHECK();
    const long long rows = (long long)E * C;
    if (launch_pdl(ec_fill_kernel, (int)((rows + 255) / 256), 256, 0, s, (const int32_t*)ec_token, T, E, C,
                   (const unsigned*)mask, mw, (const int32_t*)tok_ptr, logits, (const double*)lse, binned ? 0 : 1,
                   ec_gate, tok_row) != cudaSuccess)
        return MOE_ERR_CUDA;
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
