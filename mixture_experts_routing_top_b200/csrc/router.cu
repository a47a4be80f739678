// router.cu - the router's linear gate fused with top-k routing.
//
// "How MegaDLMs Implements Mixture of Experts (MoE) Architectures",
// "Routing Mechanisms: Top-K vs Expert Choice": the TopKRouter scores every
// expert with a linear gate over the token's hidden state, turns the scores
// into probabilities with a softmax and keeps the k most probable experts
// with their probabilities as gates.
//
// bf16: logits = x W_r^T is one persistent tcgen05 GEMM (M = 128 tokens per
// tile, N = the expert count rounded up to 16 (rows past E read as zeros),
// K = d) whose epilogue ranks each token straight out of TMEM.  One
// epilogue thread owns one token row: it walks the row's E fp32 logits in
// expert order keeping its k best (larger logit first, lower expert on
// equal logits) in registers, then forms the softmax gates exactly as the
// stand-alone top-k kernel does.  x is read once from HBM; W_r (E x d) is
// re-read per tile from L2.  A TMA warp feeds a shared-memory ring, one
// thread issues the MMAs, two TMEM accumulators let a tile's ranking overlap
// the next tile's MMAs.  Every wait is bounded (tcgen05.cuh).
//
// fp32: a plain FMA logits kernel followed by the stand-alone top-k kernel.
#include <cstdlib>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {
namespace rt {
using namespace tc;

constexpr int BM = 128;                   // tokens per tile (TMEM lanes)
constexpr int BK = 64;                    // K per stage (one 128-byte swizzle row)
constexpr int A_BYTES = BM * BK * 2;      // 16 KB
constexpr int THREADS = 192;              // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue (TMEM lane quarters)
constexpr int MAX_STAGES = 8;
constexpr int RING_BYTES = 200 * 1024;
constexpr int SMEM_BYTES = 1024 /*align slack*/ + RING_BYTES + 256 /*barriers*/;

struct RouterArgs {
    int T, d, E, n_pad, k, norm_topk, stages;
    uint32_t tmem_cols;
    float* logits;          // [T, E] fp32 out, or null
    int32_t* expert_idx;    // [T, k]
    float* gate;            // [T, k]
    unsigned* err;
};

template <int KM>
__global__ void __launch_bounds__(THREADS, 1) router_topk_kernel(const __grid_constant__ CUtensorMap map_x,
                                                                 const __grid_constant__ CUtensorMap map_w,
                                                                 RouterArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int b_bytes = a.n_pad * BK * 2;
    const int stage_bytes = A_BYTES + b_bytes;
    const int S = a.stages;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
    uint64_t* full = bars;                  // [S]
    uint64_t* empty = bars + S;             // [S]
    uint64_t* tfull = bars + 2 * S;         // [2]
    uint64_t* tempty = bars + 2 * S + 2;    // [2]
    uint64_t* drain = bars + 2 * S + 4;     // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (a.T + BM - 1) / BM;
    const int nk = a.d / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int c = 0; c < 2; ++c) {
            mbar_init(smem_u32(&tfull[c]), 1);
            mbar_init(smem_u32(&tempty[c]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(a.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, fill_parity = 0;
            for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    const uint32_t sa = smem_u32(smem + stage * stage_bytes);
                    mbar_expect_tx(fb, (uint32_t)stage_bytes);
                    issued |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    tma_load_2d(sa, &map_x, kb * BK, t * BM, fb);
                    tma_load_2d(sa + A_BYTES, &map_w, kb * BK, 0, fb);
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
            int never = 0;
            for (int st = 0; st < S; ++st)
                if (issued & (1u << st)) mbar_wait(smem_u32(&full[st]), (fill_parity >> st) & 1u, &never);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(BM, a.n_pad);
            int stage = 0, it = 0;
            uint32_t phase = 0;
            for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * a.n_pad;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * stage_bytes);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16(d_tmem, umma_desc_sw128(sa + kk * 32), umma_desc_sw128(sb + kk * 32), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    umma_commit(smem_u32(&empty[stage]));
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) { *abort_flag = 1; break; }
                umma_commit(smem_u32(&tfull[acc]));
            }
            umma_commit(smem_u32(drain));
            int never = 0;
            if (!mbar_wait(smem_u32(drain), 0, &never)) *abort_flag = 1;
        }
    } else {
        const int q = warp & 3;                 // TMEM lane quarter this warp may read
        const int r = q * 32 + lane;
        const int E = a.E, k = a.k;
        int it = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag)) { *abort_flag = 1; break; }
            tc_fence_after();
            const long long tok = (long long)t * BM + r;
            const bool valid = tok < a.T;
            const uint32_t taddr = tmem_base + acc * a.n_pad + ((uint32_t)(q * 32) << 16);
            float bv[KM];
            int bi[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) { bv[j] = -INFINITY; bi[j] = -1; }
            float* lrow = a.logits ? a.logits + tok * E : nullptr;
#pragma unroll 1
            for (int c = 0; c < a.n_pad; c += 16) {
                float v[16];
                tmem_ld16(taddr + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c + i < E) topk_insert<KM>(bv, bi, v[i], c + i);
                if (valid && lrow) {
                    float4* dst = reinterpret_cast<float4*>(lrow + c);
                    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    if (c + 16 <= E) {
                        dst[2] = make_float4(v[8], v[9], v[10], v[11]);
                        dst[3] = make_float4(v[12], v[13], v[14], v[15]);
                    }
                }
            }
            const float m = bv[0];
            double s = 0.0;
            if (!a.norm_topk) {
#pragma unroll 1
                for (int c = 0; c < a.n_pad; c += 16) {
                    float v[16];
                    tmem_ld16(taddr + c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c + i < E) s += (double)__expf(__fsub_rn(v[i], m));
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));   // accumulator free: the rest is registers only
            float ej[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                ej[j] = j < k ? exp_diff(bv[j], m) : 0.0f;
                if (a.norm_topk) s += (double)ej[j];
            }
            if (valid) {
#pragma unroll
                for (int j = 0; j < KM; ++j) {
                    if (j < k) {
                        a.expert_idx[tok * k + j] = bi[j];
                        a.gate[tok * k + j] = (float)((double)ej[j] / s);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) raise_error(a.err, kErrTimeout);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(a.tmem_cols)
                     : "memory");
    }
}

// fp32 logits: one thread per (token, expert), FMA over d in order.
__global__ void __launch_bounds__(256) router_logits_f32_kernel(const float* __restrict__ x, const float* __restrict__ W,
                                                                int T, int d, int E, float* __restrict__ logits) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)T * E) return;
    const long long t = i / E;
    const int e = (int)(i - t * E);
    const float* xr = x + t * d;
    const float* wr = W + (long long)e * d;
    float acc = 0.0f;
    for (int c = 0; c < d; ++c) acc = __fmaf_rn(xr[c], wr[c], acc);
    logits[i] = acc;
}

template <int KM>
moe_status launch_router(const CUtensorMap& mx, const CUtensorMap& mw, const RouterArgs& a, cudaStream_t s) {
    if (!set_smem_limit((const void*)router_topk_kernel<KM>, SMEM_BYTES)) return MOE_ERR_CUDA;
    const int tiles = (a.T + BM - 1) / BM;
    int grid = sm_count();
    if (tiles < grid) grid = tiles;
    const size_t smem = 1024 + (size_t)a.stages * (A_BYTES + a.n_pad * BK * 2) + 256;
    router_topk_kernel<KM><<<grid, THREADS, smem, s>>>(mx, mw, a);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

// ------------------------------------------------------ K split over a CTA pair
// With fewer 128-token tiles than half the SMs (T < 9472) the persistent
// kernel leaves SMs idle, and one SM's stream of x is too slow to cover the
// HBM.  Here each tile is one cluster of two CTAs that split K in halves:
// both accumulate their half in TMEM; once CTA 0's MMAs are done its stage
// ring is free and it tells CTA 1 (remote mbarrier arrive), CTA 1's
// epilogue copies its partial logits into that ring through distributed
// shared memory (rows padded to n_pad + 4 floats) and arrives on CTA 0's
// barrier, and CTA 0's epilogue adds the two halves (its own first, so the
// sum order is fixed) before ranking exactly as above.  All waits bounded; a
// cluster barrier at the end keeps both CTAs alive until no remote access
// can target them.  No multicast anywhere.
template <int KM>
__global__ void __launch_bounds__(THREADS, 1) router_topk_pair_kernel(const __grid_constant__ CUtensorMap map_x,
                                                                      const __grid_constant__ CUtensorMap map_w,
                                                                      RouterArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int b_bytes = a.n_pad * BK * 2;
    const int stage_bytes = A_BYTES + b_bytes;
    const int S = a.stages;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
    uint64_t* full = bars;                  // [S]
    uint64_t* empty = bars + S;             // [S]
    uint64_t* tfull = bars + 2 * S;         // accumulator ready
    uint64_t* drain = bars + 2 * S + 1;     // MMA completion before TMEM is freed
    uint64_t* rfree = bars + 2 * S + 2;     // CTA 1: CTA 0's ring may be written
    uint64_t* rready = bars + 2 * S + 3;    // CTA 0: CTA 1's partials have landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* part = reinterpret_cast<float*>(smem);   // CTA 0: [BM][n_pad + 4] partials of CTA 1
    const int pstride = a.n_pad + 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int t = blockIdx.x >> 1;
    const int nk = a.d / BK;
    const int kb0 = rank ? nk / 2 : 0, kb1 = rank ? nk : nk / 2;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), 1);
        }
        mbar_init(smem_u32(tfull), 1);
        mbar_init(smem_u32(drain), 1);
        mbar_init(smem_u32(rfree), 1);
        mbar_init(smem_u32(rready), 128);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(a.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();                         // both CTAs' barriers exist before any remote arrive
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, fill_parity = 0;
            for (int kb = kb0; kb < kb1 && !*abort_flag; ++kb) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
                    *abort_flag = 1;
                    break;
                }
                const uint32_t fb = smem_u32(&full[stage]);
                const uint32_t sa = smem_u32(smem + stage * stage_bytes);
                mbar_expect_tx(fb, (uint32_t)stage_bytes);
                issued |= 1u << stage;
                fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                tma_load_2d(sa, &map_x, kb * BK, t * BM, fb);
                tma_load_2d(sa + A_BYTES, &map_w, kb * BK, 0, fb);
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            int never = 0;
            for (int st = 0; st < S; ++st)
                if (issued & (1u << st)) mbar_wait(smem_u32(&full[st]), (fill_parity >> st) & 1u, &never);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(BM, a.n_pad);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + stage * stage_bytes);
                const uint32_t sb = sa + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_bf16(tmem_base, umma_desc_sw128(sa + kk * 32), umma_desc_sw128(sb + kk * 32), idesc,
                              (kb > kb0 || kk) ? 1u : 0u);
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (!ok) *abort_flag = 1;
            else umma_commit(smem_u32(tfull));
            umma_commit(smem_u32(drain));
            int never = 0;
            if (!mbar_wait(smem_u32(drain), 0, &never)) *abort_flag = 1;
        }
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
        const bool got = mbar_wait(smem_u32(tfull), 0, abort_flag);
        if (!got) *abort_flag = 1;
        tc_fence_after();
        if (rank == 1) {
            // copy this half's partial rows into CTA 0's (now idle) stage ring
            if (got && mbar_wait_cluster(smem_u32(rfree), 0, abort_flag)) {
                const uint32_t dst = map_to_rank(smem_u32(part + r * pstride), 0);
#pragma unroll 1
                for (int c = 0; c < a.n_pad; c += 16) {
                    float v[16];
                    tmem_ld16(taddr + c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(dst + (uint32_t)(c + i) * 4u), "f"(v[i]), "f"(v[i + 1]), "f"(v[i + 2]),
                                        "f"(v[i + 3]) : "memory");
                }
                arrive_remote(map_to_rank(smem_u32(rready), 0));
            } else {
                *abort_flag = 1;
            }
        } else {
            if (got && threadIdx.x == 64) arrive_remote(map_to_rank(smem_u32(rfree), 1));   // ring is idle
            if (got && mbar_wait_cluster(smem_u32(rready), 0, abort_flag)) {
                const int E = a.E, k = a.k;
                const long long tok = (long long)t * BM + r;
                const bool valid = tok < a.T;
                const float* prow = part + r * pstride;
                float bv[KM];
                int bi[KM];
#pragma unroll
                for (int j = 0; j < KM; ++j) { bv[j] = -INFINITY; bi[j] = -1; }
                float* lrow = a.logits ? a.logits + tok * E : nullptr;
#pragma unroll 1
                for (int c = 0; c < a.n_pad; c += 16) {
                    float v[16];
                    tmem_ld16(taddr + c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        const float4 p4 = *reinterpret_cast<const float4*>(prow + c + i);
                        v[i] = __fadd_rn(v[i], p4.x);
                        v[i + 1] = __fadd_rn(v[i + 1], p4.y);
                        v[i + 2] = __fadd_rn(v[i + 2], p4.z);
                        v[i + 3] = __fadd_rn(v[i + 3], p4.w);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c + i < E) topk_insert<KM>(bv, bi, v[i], c + i);
                    if (valid && lrow) {
                        float4* dst = reinterpret_cast<float4*>(lrow + c);
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                        if (c + 16 <= E) {
                            dst[2] = make_float4(v[8], v[9], v[10], v[11]);
                            dst[3] = make_float4(v[12], v[13], v[14], v[15]);
                        }
                    }
                }
                const float m = bv[0];
                double s = 0.0;
                if (!a.norm_topk) {
#pragma unroll 1
                    for (int c = 0; c < a.n_pad; c += 16) {
                        float v[16];
                        tmem_ld16(taddr + c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c + i < E) s += (double)__expf(__fsub_rn(__fadd_rn(v[i], prow[c + i]), m));
                    }
                }
                float ej[KM];
#pragma unroll
                for (int j = 0; j < KM; ++j) {
                    ej[j] = j < k ? exp_diff(bv[j], m) : 0.0f;
                    if (a.norm_topk) s += (double)ej[j];
                }
                if (valid) {
#pragma unroll
                    for (int j = 0; j < KM; ++j) {
                        if (j < k) {
                            a.expert_idx[tok * k + j] = bi[j];
                            a.gate[tok * k + j] = (float)((double)ej[j] / s);
                        }
                    }
                }
            } else {
                *abort_flag = 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) raise_error(a.err, kErrTimeout);
    cluster_sync();                         // no remote access may target an exited CTA
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(a.tmem_cols)
                     : "memory");
    }
}

template <int KM>
moe_status launch_router_pair(const CUtensorMap& mx, const CUtensorMap& mw, const RouterArgs& a, cudaStream_t s) {
    if (!set_smem_limit((const void*)router_topk_pair_kernel<KM>, SMEM_BYTES)) return MOE_ERR_CUDA;
    const int tiles = (a.T + BM - 1) / BM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * tiles, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = 1024 + (size_t)a.stages * (A_BYTES + a.n_pad * BK * 2) + 256;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, router_topk_pair_kernel<KM>, mx, mw, a) != cudaSuccess) {
        count_launch();
        (void)cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    count_launch();
    return MOE_OK;
}

// K split over CTA pairs when the tiles would leave more than half the SMs
// idle.  LIBMOE_ROUTER_PAIR=0/1 forces either kernel.
bool use_router_pair(int T, int d) {
    const char* env = getenv("LIBMOE_ROUTER_PAIR");
    if (d / BK < 2) return false;
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return 2 * ((T + BM - 1) / BM) <= sm_count();
}

}  // namespace rt
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_router_topk(const void* x, int dtype, int T, int d, const void* W_r, int E, int k,
                                      int norm_topk, float* logits, int32_t* expert_idx, float* gate,
                                      moe_stream_t stream) {
    if (T < 0 || d < 1 || E < 1 || k < 1 || k > E) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (E > 1024 || k > 32) return MOE_ERR_SHAPE;
    if (dtype == MOE_BF16 && (d % 64 || E % 8 || E > 256 || k > 8)) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x || !W_r || !expert_idx || !gate) return MOE_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == MOE_F32) {
        if (!logits) return MOE_ERR_ARG;
        const long long n = (long long)T * E;
        rt::router_logits_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
            (const float*)x, (const float*)W_r, T, d, E, logits);
        MOE_LAUNCH_CHECK();
        return moe_route_topk(logits, T, E, k, norm_topk, expert_idx, gate, stream);
    }
    auto a16 = [](const void* p) { return ((uintptr_t)p & 15) == 0; };
    if (!a16(x) || !a16(W_r) || (logits && !a16(logits))) return MOE_ERR_SHAPE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    if (!tc::tma_encoder_ready()) return MOE_ERR_CUDA;
    rt::RouterArgs a;
    a.T = T;
    a.d = d;
    a.E = E;
    a.n_pad = (E + 15) / 16 * 16;
    a.k = k;
    a.norm_topk = norm_topk ? 1 : 0;
    const int stage_bytes = rt::A_BYTES + a.n_pad * rt::BK * 2;
    a.stages = rt::RING_BYTES / stage_bytes;
    if (a.stages > rt::MAX_STAGES) a.stages = rt::MAX_STAGES;
    uint32_t cols = 32;
    while (cols < 2u * (uint32_t)a.n_pad) cols <<= 1;
    a.tmem_cols = cols;
    a.logits = logits;
    a.expert_idx = expert_idx;
    a.gate = gate;
    a.err = err;
    CUtensorMap mx, mw;
    if (!tc::make_bf16_map(&mx, x, T, d, rt::BM)) return MOE_ERR_CUDA;
    if (!tc::make_bf16_map(&mw, W_r, E, d, a.n_pad)) return MOE_ERR_CUDA;
    if (rt::use_router_pair(T, d)) {
        a.tmem_cols = 32;              // one accumulator
        while (a.tmem_cols < (uint32_t)a.n_pad) a.tmem_cols <<= 1;
        if (k <= 1) return rt::launch_router_pair<1>(mx, mw, a, s);
        if (k <= 2) return rt::launch_router_pair<2>(mx, mw, a, s);
        if (k <= 4) return rt::launch_router_pair<4>(mx, mw, a, s);
        return rt::launch_router_pair<8>(mx, mw, a, s);
    }
    if (k <= 1) return rt::launch_router<1>(mx, mw, a, s);
    if (k <= 2) return rt::launch_router<2>(mx, mw, a, s);
    if (k <= 4) return rt::launch_router<4>(mx, mw, a, s);
    return rt::launch_router<8>(mx, mw, a, s);
}
