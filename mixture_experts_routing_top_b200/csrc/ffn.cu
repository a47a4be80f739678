// ffn.cu - the grouped expert MLP ("MoELayer" step 2 of "How MegaDLMs
// Implements Mixture of Experts (MoE) Architectures": each expert held on
// the device runs its MLP on the rows routed to it).
//
// bf16: two persistent tcgen05 grouped GEMMs per call.
//   GEMM1  H[r, :] = act(X[r] W1[e]^T (, X[r] W3[e]^T))   (bf16 H in workspace)
//   GEMM2  Y[r, :] = H[r] W2[e]^T
// Each CTA owns one SM: a TMA warp streams 128x64 A tiles and 256x64 B tiles
// (128-byte swizzle) into a 4-stage shared-memory ring; one thread issues
// tcgen05.mma (M=128, N=256, K=16, bf16 in, fp32 accumulate in TMEM); four
// epilogue warps (one per TMEM lane quarter) drain the accumulator with tcgen05.ld, apply the
// activation and store bf16.  Two TMEM accumulators (2 x 256 columns) let
// the epilogue of one tile overlap the MMAs of the next.  For SwiGLU the B
// tile stacks 128 rows of W1 over the same 128 rows of W3, so one MMA chain
// yields both projections and silu(a) * b is formed in registers.
//
// Ragged experts: offsets[] stays on the device.  Every CTA derives the
// per-expert tile counts from it at start; tile t -> (expert, n-tile,
// m-tile), m fastest, so CTAs working at the same time share weight tiles
// through L2.  Rows of a 128-row tile past the expert's end belong to the
// next expert or lie past the buffer (TMA fills zeros); the epilogue never
// stores them.
//
// Every wait on an mbarrier is bounded (a few seconds of %globaltimer):
// on expiry the CTA records MOE_ERR_TIMEOUT in the device fault word, all
// roles leave their loops, and TMEM is still freed.
//
// fp32: a plain FMA kernel pair for small fp32 layers (no fp32-input
// tensor-core kind keeps fp32 accuracy).
#include <cstdlib>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;              // rows per tile (TMEM lanes)
constexpr int BK = 64;               // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int ACC_N = 256;           // accumulator columns per tile
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB
constexpr int B_BYTES = ACC_N * BK * 2;      // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 4;                 // one warp per TMEM lane quarter (EPI_WARPS = 8 splits the columns in half)
constexpr int THREADS = 64 + 32 * EPI_WARPS;  // warp 0 TMA, warp 1 MMA, then the epilogue warps
constexpr int MAX_E = 1024;
constexpr int OUT_CHUNK_BYTES = 32 * 64;                     // one warp's 32 rows x 32 bf16 columns
constexpr int OUT_STAGE_BYTES = EPI_WARPS * 2 * OUT_CHUNK_BYTES;   // two staging buffers per epilogue warp
constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + OUT_STAGE_BYTES + 256 /*barriers*/ +
                           4 * (MAX_E + 1);

enum { MODE_SWIGLU = 0, MODE_GELU = 1, MODE_PLAIN = 2 };


__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }
// GELU with erf by Abramowitz & Stegun, Handbook of Mathematical Functions,
// 7.1.28 (Hastings): erf(x) = 1 - (1 + a1 x + ... + a6 x^6)^-16 for x >= 0,
// |error| <= 3e-7, odd in x.  With x = |z| / sqrt(2), the exact-erf GELU
// 0.5 z (1 + erf(z / sqrt(2))) equals max(z, 0) - 0.5 |z| q(|z|)^-16 for
// either sign of z, where q(y) = 1 + b1 y + ... + b6 y^6, b_i = a_i / sqrt(2)^i.
// Branch-free: six FMAs, four squarings, one hardware reciprocal, one
// multiply, a max and a final FMA (rounded once); evaluated in fp32 the error
// of the erf part stays below 2e-6, far under the bf16 rounding of the hidden
// activations.  The GELU epilogue of a short-K GEMM is bound by instruction
// issue, where this form is cheaper than the library erf with its range split.
constexpr double kRsqrt2 = 0.70710678118654752440;
constexpr float kGb1 = (float)(7.05230784e-2 * kRsqrt2);
constexpr float kGb2 = (float)(4.22820123e-2 * kRsqrt2 * kRsqrt2);
constexpr float kGb3 = (float)(9.2705272e-3 * kRsqrt2 * kRsqrt2 * kRsqrt2);
constexpr float kGb4 = (float)(1.520143e-4 * kRsqrt2 * kRsqrt2 * kRsqrt2 * kRsqrt2);
constexpr float kGb5 = (float)(2.765672e-4 * kRsqrt2 * kRsqrt2 * kRsqrt2 * kRsqrt2 * kRsqrt2);
constexpr float kGb6 = (float)(4.30638e-5 * kRsqrt2 * kRsqrt2 * kRsqrt2 * kRsqrt2 * kRsqrt2 * kRsqrt2);

__device__ __forceinline__ float gelu_f(float z) {
    const float y = fabsf(z);
    float q = fmaf(y, kGb6, kGb5);
    q = fmaf(y, q, kGb4);
    q = fmaf(y, q, kGb3);
    q = fmaf(y, q, kGb2);
    q = fmaf(y, q, kGb1);
    q = fmaf(y, q, 1.0f);
    q *= q;
    q *= q;
    q *= q;
    q *= q;
    float r;                                      // q^-16 = 1 - erf(|z| / sqrt(2))
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(q));
    return fmaf(-0.5f * y, r, fmaxf(z, 0.0f));
}

// Store 32 consecutive bf16 values (64 bytes) of one output row.
__device__ __forceinline__ void store_row32(uint16_t* dst, const float* v) {
    uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        p[q] = w;
    }
}

// Output of one epilogue warp: its 32 rows x 32 columns per chunk.  When
// all 32 rows lie inside the expert, the chunk is packed to bf16 into one of
// the warp's two shared-memory buffers (64-byte swizzle: bank-conflict-free
// 16-byte writes) and written by one TMA store, so the stores leave the
// issue slots and the LSU; a buffer is rewritten only after the store issued
// two chunks earlier has read it.  A warp whose rows straddle the expert's
// end stores its valid rows directly: a box would overwrite the next
// expert's rows.
struct EpiOut {
    uint32_t buf;   // shared address of this warp's two buffers
    int n = 0;      // chunks staged so far

    __device__ __forceinline__ void chunk(const CUtensorMap* map, uint16_t* orow, bool valid, bool full, int grow0,
                                          int col, const float* v) {
        const int lane = threadIdx.x & 31;
        if (full) {
            if (lane == 0) bulk_wait_read1();
            __syncwarp();
            const uint32_t b = buf + (uint32_t)(n & 1) * OUT_CHUNK_BYTES + (uint32_t)lane * 64;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
                w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
                w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
                w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
                st_shared_v4(b + (uint32_t)((q ^ ((lane >> 1) & 3)) << 4), w);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(map, buf + (uint32_t)(n & 1) * OUT_CHUNK_BYTES, col, grow0);
                bulk_commit();
            }
            ++n;
        } else if (valid) {
            store_row32(orow + col, v);
        }
    }
    // every store issued by this warp has completed (before the CTA exits)
    __device__ __forceinline__ void drain() {
        if ((threadIdx.x & 31) == 0) bulk_wait0();
        __syncwarp();
    }
};

struct GemmArgs {
    const int32_t* offsets;   // [E+1] device
    int E;
    int K;                    // reduction length (multiple of 64)
    int N_out;                // output columns (multiple of 32)
    int w_rows;               // rows per expert in the B tensor(s)
    int R_max;                // rows of A / out
    uint16_t* out;            // bf16 [R_max, N_out]
    unsigned* err;
};

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                                                  const __grid_constant__ CUtensorMap map_b0,
                                                                  const __grid_constant__ CUtensorMap map_b1,
                                                                  const __grid_constant__ CUtensorMap map_out,
                                                                  GemmArgs args) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    constexpr int BN_OUT = (MODE == MODE_SWIGLU) ? 128 : 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* stage_base = smem;
    uint8_t* out_stage = smem + STAGES * STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + OUT_STAGE_BYTES);
    uint64_t* full = bars;                     // [STAGES]
    uint64_t* empty = bars + STAGES;           // [STAGES]
    uint64_t* tfull = bars + 2 * STAGES;       // [2]
    uint64_t* tempty = bars + 2 * STAGES + 2;  // [2]
    uint64_t* drain = bars + 2 * STAGES + 4;   // [1] MMA completion before TMEM is freed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* tile_prefix = reinterpret_cast<int*>(out_stage + OUT_STAGE_BYTES + 256);   // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E;
    const int n_tiles = (args.N_out + BN_OUT - 1) / BN_OUT;
    const int nk = args.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 32 * EPI_WARPS);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b0);
        if (MODE == MODE_SWIGLU) tma_prefetch_desc(&map_b1);
        tma_prefetch_desc(&map_out);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(2 * ACC_N) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    pdl_wait();                       // the offsets and operands come from the kernels before
    if (warp == 2 && lane == 0) {
        int acc = 0;
        tile_prefix[0] = 0;
        for (int e = 0; e < E; ++e) {
            int b = min(max(args.offsets[e], 0), args.R_max);
            int en = min(max(args.offsets[e + 1], 0), args.R_max);
            int cnt = max(en - b, 0);
            acc += ((cnt + BM - 1) / BM) * n_tiles;
            tile_prefix[e + 1] = acc;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_prefix[E];

    // tile -> expert, row range, n offset
    auto decode = [&](int t, int& row0, int& row_end, int& brow, int& n0) {
        int lo = 0, hi = E;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (tile_prefix[mid] <= t) lo = mid; else hi = mid - 1;
        }
        const int e = lo;
        const int b = min(max(args.offsets[e], 0), args.R_max);
        const int en = min(max(args.offsets[e + 1], 0), args.R_max);
        const int mt = (en - b + BM - 1) / BM;
        const int local = t - tile_prefix[e];
        const int n_idx = local / mt, m_idx = local - n_idx * mt;
        row0 = b + m_idx * BM;
        row_end = en;
        n0 = n_idx * BN_OUT;
        brow = e * args.w_rows + n0;
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, fill_parity = 0;     // per stage: any fill issued, parity of the last one
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                int row0, row_end, brow, n0;
                decode(t, row0, row_end, brow, n0);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    mbar_expect_tx(fb, STAGE_BYTES);
                    issued |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    tma_load_2d(sa, &map_a, kb * BK, row0, fb);
                    if (MODE == MODE_SWIGLU) {
                        tma_load_2d(sb, &map_b0, kb * BK, brow, fb);
                        tma_load_2d(sb + B_BYTES / 2, &map_b1, kb * BK, brow, fb);
                    } else {
                        tma_load_2d(sb, &map_b0, kb * BK, brow, fb);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // every issued fill has landed before the CTA may exit (immediate
            // on the normal path: the MMA thread consumed them all)
            int never = 0;
            for (int st = 0; st < STAGES; ++st)
                if (issued & (1u << st)) mbar_wait(smem_u32(&full[st]), (fill_parity >> st) & 1u, &never);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, ACC_N);
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_N;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        umma_bf16(d_tmem, umma_desc_sw128(sa + kk * 32), umma_desc_sw128(sb + kk * 32), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) { *abort_flag = 1; break; }
                umma_commit(smem_u32(&tfull[acc]));
            }
            // no tcgen05.mma of this CTA may still be running when TMEM is freed
            umma_commit(smem_u32(drain));
            int never = 0;
            if (!mbar_wait(smem_u32(drain), 0, &never)) *abort_flag = 1;
        }
    } else {
        // epilogue: warps 2.. -> TMEM lane quarter (warp % 4), column part
        const int q = warp & 3;
        const int half = (EPI_WARPS == 8) ? ((warp - 2) >> 2) : 0;
        const int r = q * 32 + lane;
        EpiOut eo{smem_u32(out_stage + (warp - 2) * 2 * OUT_CHUNK_BYTES)};
        int it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
            int row0, row_end, brow, n0;
            decode(t, row0, row_end, brow, n0);
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag)) { *abort_flag = 1; break; }
            tc_fence_after();
            const int grow = row0 + r;
            const bool valid = grow < row_end;
            const int grow0 = row0 + q * 32;
            const bool full = grow0 + 31 < row_end;
            const uint32_t taddr = tmem_base + acc * ACC_N + ((uint32_t)(q * 32) << 16);
            uint16_t* orow = args.out + (long long)grow * args.N_out;
            if (MODE == MODE_SWIGLU) {
#pragma unroll 1
                for (int c = (16 / EPI_WARPS) * half; c < (16 / EPI_WARPS) * half + 16 / EPI_WARPS; ++c) {
                    float a[32], b[32];
                    tmem_ld32(taddr + c * 32, a);
                    tmem_ld32(taddr + 128 + c * 32, b);
                    tmem_ld_wait();
                    const int col = n0 + c * 32;
                    if (col < args.N_out) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) a[i] = silu_f(a[i]) * b[i];
                        eo.chunk(&map_out, orow, valid, full, grow0, col, a);
                    }
                }
            } else {
#pragma unroll 1
                for (int c = (32 / EPI_WARPS) * half; c < (32 / EPI_WARPS) * half + 32 / EPI_WARPS; ++c) {
                    float a[32];
                    tmem_ld32(taddr + c * 32, a);
                    tmem_ld_wait();
                    const int col = n0 + c * 32;
                    if (col < args.N_out) {
                        if (MODE == MODE_GELU) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) a[i] = gelu_f(a[i]);
                        }
                        eo.chunk(&map_out, orow, valid, full, grow0, col, a);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
        }
        eo.drain();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) raise_error(args.err, kErrTimeout);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(2 * ACC_N) : "memory");
    }
}

}  // namespace tc

// ------------------------------------------------------ 2-CTA (CTA pair)
// The same grouped GEMM with tcgen05.mma.cta_group::2: a cluster of two
// CTAs on the two SMs of a TPC computes a 256-row x 256-column tile.  Each
// CTA stages its own 128 rows of A and one half of B (N rows 0-127 in the
// even CTA, 128-255 in the odd one; for SwiGLU that is the W1 tile and the
// W3 tile), so per SM a k-block costs 32 KB of shared memory instead of 48
// and six stages fit.  The even CTA's thread issues the MMAs (M=256); its
// accumulator rows live in the even CTA's TMEM, the odd half in the odd
// CTA's.  Both CTAs' TMA loads complete on the even CTA's stage barrier
// (address mapped with mapa; plain loads, no multicast); tcgen05.commit
// multicasts each stage release and each accumulator-ready signal to both
// CTAs; the odd CTA's epilogue arrives remotely on the even CTA's
// accumulator-empty barrier.  Waits are bounded as in the one-CTA kernel.
namespace tc2 {
using namespace tc;

constexpr int BM = 256;                       // rows per tile (pair)
constexpr int STAGES = 6;
constexpr int A_BYTES = 128 * BK * 2;         // 16 KB per CTA
constexpr int B_BYTES = 128 * BK * 2;         // 16 KB per CTA (half of N = 256)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + OUT_STAGE_BYTES + 256 + 4 * (MAX_E + 1);

// TMA into this CTA's shared memory, completing on the barrier at `bar_cluster`
// (a shared::cluster address: the even CTA's stage barrier).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}

// Arrives on the barrier at this shared offset in every CTA of `mask`.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t mask) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 :: "r"(bar), "h"(mask) : "memory");
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
grouped_gemm2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                     const __grid_constant__ CUtensorMap map_b1, const __grid_constant__ CUtensorMap map_out,
                     GemmArgs args) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    constexpr int BN_OUT = (MODE == MODE_SWIGLU) ? 128 : 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* stage_base = smem;
    uint8_t* out_stage = smem + STAGES * STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + OUT_STAGE_BYTES);
    uint64_t* full = bars;                     // [STAGES] (used in the even CTA)
    uint64_t* empty = bars + STAGES;           // [STAGES]
    uint64_t* tfull = bars + 2 * STAGES;       // [2]
    uint64_t* tempty = bars + 2 * STAGES + 2;  // [2] (used in the even CTA)
    uint64_t* drain = bars + 2 * STAGES + 4;   // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* tile_prefix = reinterpret_cast<int*>(out_stage + OUT_STAGE_BYTES + 256);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = args.E;
    const int n_tiles = (args.N_out + BN_OUT - 1) / BN_OUT;
    const int nk = args.K / BK;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 2 * 32 * EPI_WARPS);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b0);
        if (MODE == MODE_SWIGLU) tma_prefetch_desc(&map_b1);
        tma_prefetch_desc(&map_out);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(2 * ACC_N) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    pdl_wait();                       // the offsets and operands come from the kernels before
    if (warp == 2 && lane == 0) {
        int acc = 0;
        tile_prefix[0] = 0;
        for (int e = 0; e < E; ++e) {
            int b = min(max(args.offsets[e], 0), args.R_max);
            int en = min(max(args.offsets[e + 1], 0), args.R_max);
            int cnt = max(en - b, 0);
            acc += ((cnt + BM - 1) / BM) * n_tiles;
            tile_prefix[e + 1] = acc;
        }
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_prefix[E];
    // The last partial round of the plain (down) GEMM: its tiles are split
    // into `split` column slices of 256 / split columns (MMA N = 128 or 64),
    // so that round takes a fraction of a tile's time on more CTA pairs
    // instead of a whole tile's time on a few (896 tiles on 74 pairs: 12.1
    // rounds would run as 13).  Units [0, full_units) are whole tiles.
    int full_units = total, split = 1;
    if (MODE == MODE_PLAIN && total > 0) {
        full_units = ((total + npairs - 1) / npairs - 1) * npairs;
        const int tail = total - full_units;
        while (split < 4 && tail * split * 2 <= npairs) split *= 2;
    }
    const int units = full_units + (total - full_units) * split;

    auto decode = [&](int u, int& row0, int& row_end, int& n0, int& e_out, int& ncols) {
        int t = u, sub = 0, parts = 1;
        if (u >= full_units) {
            t = full_units + (u - full_units) / split;
            sub = (u - full_units) % split;
            parts = split;
        }
        int lo = 0, hi = E;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (tile_prefix[mid] <= t) lo = mid; else hi = mid - 1;
        }
        const int e = lo;
        const int b = min(max(args.offsets[e], 0), args.R_max);
        const int en = min(max(args.offsets[e + 1], 0), args.R_max);
        const int mt = (en - b + BM - 1) / BM;
        const int local = t - tile_prefix[e];
        const int n_idx = local / mt, m_idx = local - n_idx * mt;
        row0 = b + m_idx * BM;
        row_end = en;
        ncols = BN_OUT / parts;
        n0 = n_idx * BN_OUT + sub * ncols;
        e_out = e;
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, fill_parity = 0;
            for (int t = pair; t < units && !*abort_flag; t += npairs) {
                int row0, row_end, n0, e, ncols;
                decode(t, row0, row_end, n0, e, ncols);
                const int arow = row0 + (int)rank * 128;
                int brow;
                const CUtensorMap* bmap = &map_b0;
                if (MODE == MODE_SWIGLU) {
                    brow = e * args.w_rows + n0;
                    if (!leader) bmap = &map_b1;
                } else {
                    // each CTA holds half of the unit's columns (the 128-row box
                    // also brings rows the narrower MMAs of the last round skip)
                    brow = e * args.w_rows + n0 + (int)rank * (ncols / 2);
                }
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) { *abort_flag = 1; break; }
                    const uint32_t fb_local = smem_u32(&full[stage]);
                    const uint32_t fb = map_to_rank(fb_local, 0);
                    const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    if (leader) mbar_expect_tx(fb_local, 2 * STAGE_BYTES);
                    issued |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    tma_load_2d_pair(sa, &map_a, kb * BK, arow, fb);
                    tma_load_2d_pair(sb, bmap, kb * BK, brow, fb);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // the even CTA's own fills have landed before it may exit; the
            // odd CTA's fills complete on the even CTA's barriers, which the
            // even CTA's MMA thread consumed (or which time out)
            int never = 0;
            if (leader)
                for (int st = 0; st < STAGES; ++st)
                    if (issued & (1u << st)) mbar_wait(smem_u32(&full[st]), (fill_parity >> st) & 1u, &never);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int t = pair; t < units && !*abort_flag; t += npairs, ++it) {
                const uint32_t idesc = umma_idesc_bf16(BM, t < full_units ? ACC_N : ACC_N / split);
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait_cluster(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_N;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_cluster(smem_u32(&full[stage]), phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16_pair(d_tmem, umma_desc_sw128(sa + kk * 32), umma_desc_sw128(sb + kk * 32), idesc,
                                       (kb | kk) != 0 ? 1u : 0u);
                    umma_commit_pair(smem_u32(&empty[stage]), 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) { *abort_flag = 1; break; }
                umma_commit_pair(smem_u32(&tfull[acc]), 0x3);
            }
            umma_commit_pair(smem_u32(drain), 0x1);
            int never = 0;
            if (!mbar_wait(smem_u32(drain), 0, &never)) *abort_flag = 1;
        }
    } else {
        const int q = warp & 3;
        const int half = (EPI_WARPS == 8) ? ((warp - 2) >> 2) : 0;
        const int r = q * 32 + lane;
        const uint32_t tempty_leader0 = map_to_rank(smem_u32(&tempty[0]), 0);
        const uint32_t tempty_leader1 = map_to_rank(smem_u32(&tempty[1]), 0);
        EpiOut eo{smem_u32(out_stage + (warp - 2) * 2 * OUT_CHUNK_BYTES)};
        int it = 0;
        for (int t = pair; t < units; t += npairs, ++it) {
            int row0, row_end, n0, e, ncols;
            decode(t, row0, row_end, n0, e, ncols);
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag)) { *abort_flag = 1; break; }
            tc_fence_after();
            const int grow = row0 + (int)rank * 128 + r;
            const bool valid = grow < row_end;
            const int grow0 = row0 + (int)rank * 128 + q * 32;
            const bool full = grow0 + 31 < row_end;
            const uint32_t taddr = tmem_base + acc * ACC_N + ((uint32_t)(q * 32) << 16);
            uint16_t* orow = args.out + (long long)grow * args.N_out;
            if (MODE == MODE_SWIGLU) {
#pragma unroll 1
                for (int c = (16 / EPI_WARPS) * half; c < (16 / EPI_WARPS) * half + 16 / EPI_WARPS; ++c) {
                    float a[32], b[32];
                    tmem_ld32(taddr + c * 32, a);
                    tmem_ld32(taddr + 128 + c * 32, b);
                    tmem_ld_wait();
                    const int col = n0 + c * 32;
                    if (col < args.N_out) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) a[i] = silu_f(a[i]) * b[i];
                        eo.chunk(&map_out, orow, valid, full, grow0, col, a);
                    }
                }
            } else {
                const int per = (ncols / 32) / (EPI_WARPS / 4);   // 32-column chunks per epilogue warp
#pragma unroll 1
                for (int c = per * half; c < per * (half + 1); ++c) {
                    float a[32];
                    tmem_ld32(taddr + c * 32, a);
                    tmem_ld_wait();
                    const int col = n0 + c * 32;
                    if (col < args.N_out) {
                        if (MODE == MODE_GELU) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) a[i] = gelu_f(a[i]);
                        }
                        eo.chunk(&map_out, orow, valid, full, grow0, col, a);
                    }
                }
            }
            tc_fence_before();
            arrive_remote(acc ? tempty_leader1 : tempty_leader0);
        }
        eo.drain();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) raise_error(args.err, kErrTimeout);
    cluster_sync();                              // no remote arrival may target an exited CTA
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(2 * ACC_N) : "memory");
    }
}

}  // namespace tc2

// ------------------------------------------------------------- fp32 SIMT
// H[r, f] = act(x_r . W1[e, f] (, x_r . W3[e, f])), one thread per (r, f);
// Y[r, c] = H[r] . W2[e, c], one thread per (r, c).  e from offsets.
__device__ __forceinline__ int expert_of_row(const int32_t* __restrict__ offsets, int E, int r) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void ffn_f32_hidden_kernel(const float* __restrict__ x, int d, int F, int E, const int32_t* __restrict__ offsets,
                                      int R_max, const float* __restrict__ W1, const float* __restrict__ W3, int act,
                                      float* __restrict__ H) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int R = min(offsets[E], R_max);
    if (i >= (long long)R * F) return;
    const int r = (int)(i / F), f = (int)(i % F);
    if (r < offsets[0]) return;
    const int e = expert_of_row(offsets, E, r);
    const float* xr = x + (long long)r * d;
    const float* w1 = W1 + ((long long)e * F + f) * d;
    float a = 0.0f;
    for (int c = 0; c < d; ++c) a = __fmaf_rn(w1[c], xr[c], a);
    float h;
    if (act == MOE_ACT_SWIGLU) {
        const float* w3 = W3 + ((long long)e * F + f) * d;
        float b = 0.0f;
        for (int c = 0; c < d; ++c) b = __fmaf_rn(w3[c], xr[c], b);
        h = tc::silu_f(a) * b;
    } else {
        h = tc::gelu_f(a);
    }
    H[i] = h;
}

__global__ void ffn_f32_out_kernel(const float* __restrict__ H, int d, int F, int E, const int32_t* __restrict__ offsets,
                                   int R_max, const float* __restrict__ W2, float* __restrict__ y) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int R = min(offsets[E], R_max);
    if (i >= (long long)R * d) return;
    const int r = (int)(i / d), c = (int)(i % d);
    if (r < offsets[0]) return;
    const int e = expert_of_row(offsets, E, r);
    const float* hr = H + (long long)r * F;
    const float* w2 = W2 + ((long long)e * d + c) * F;
    float acc = 0.0f;
    for (int f = 0; f < F; ++f) acc = __fmaf_rn(w2[f], hr[f], acc);
    y[i] = acc;
}

// --------------------------------------------------------------- host side
namespace {

template <int MODE>
moe_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb0, const CUtensorMap& mb1, const CUtensorMap& mo,
                       const tc::GemmArgs& a, cudaStream_t s) {
    if (!set_smem_limit((const void*)tc::grouped_gemm_kernel<MODE>, tc::SMEM_BYTES)) return MOE_ERR_CUDA;
    const int bn_out = MODE == tc::MODE_SWIGLU ? 128 : 256;
    const long long n_tiles = (a.N_out + bn_out - 1) / bn_out;
    const long long m_tiles_max = (a.R_max + tc::BM - 1) / tc::BM + a.E;
    long long tiles_max = n_tiles * m_tiles_max;
    int grid = tc::sm_count();
    if (tiles_max < grid) grid = (int)(tiles_max > 0 ? tiles_max : 1);
    (void)launch_pdl(tc::grouped_gemm_kernel<MODE>, grid, tc::THREADS, tc::SMEM_BYTES, s, ma, mb0, mb1, mo, a);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

template <int MODE>
moe_status launch_gemm2(const CUtensorMap& ma, const CUtensorMap& mb0, const CUtensorMap& mb1, const CUtensorMap& mo,
                        const tc::GemmArgs& a, cudaStream_t s) {
    if (!set_smem_limit((const void*)tc2::grouped_gemm2_kernel<MODE>, tc2::SMEM_BYTES)) return MOE_ERR_CUDA;
    const int bn_out = MODE == tc::MODE_SWIGLU ? 128 : 256;
    const long long n_tiles = (a.N_out + bn_out - 1) / bn_out;
    const long long m_tiles_max = (a.R_max + tc2::BM - 1) / tc2::BM + a.E;
    const long long tiles_max = n_tiles * m_tiles_max;
    int pairs = tc::sm_count() / 2;
    if (tiles_max < pairs) pairs = (int)(tiles_max > 0 ? tiles_max : 1);
    (void)launch_pdl(tc2::grouped_gemm2_kernel<MODE>, 2 * pairs, tc::THREADS, tc2::SMEM_BYTES, s, ma, mb0, mb1, mo, a);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

// CTA-pair kernels when experts average at least 512 rows (256-row tiles
// waste little); one-CTA kernels otherwise.  LIBMOE_GEMM_PAIR=0/1 forces it.
bool use_pair_kernels(int R_max, int E) {
    const char* env = getenv("LIBMOE_GEMM_PAIR");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return (long long)R_max >= 512LL * E;
}

size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_expert_ffn_workspace_bytes(int R_max, int d, int F, int dtype) {
    (void)d;
    if (R_max < 0 || F < 1) return 0;
    const size_t esz = dtype == MOE_BF16 ? 2 : 4;
    return al256((size_t)R_max * F * esz) + 256;
}

extern "C" moe_status moe_expert_ffn(const void* buffer, int dtype, int R_max, int d, int F, int E,
                                     const int32_t* offsets, const void* W1, const void* W3, const void* W2, int act,
                                     void* y, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    if (R_max < 0 || d < 1 || F < 1 || E < 1) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (act != MOE_ACT_SWIGLU && act != MOE_ACT_GELU) return MOE_ERR_ARG;
    if (E > tc::MAX_E) return MOE_ERR_SHAPE;
    if (R_max == 0) return MOE_OK;
    if (!buffer || !offsets || !W1 || !W2 || !y || (act == MOE_ACT_SWIGLU && !W3)) return MOE_ERR_ARG;
    const size_t need = moe_expert_ffn_workspace_bytes(R_max, d, F, dtype);
    if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255)) return MOE_ERR_WORKSPACE;
    if (dtype == MOE_BF16) {
        if (d % 64 != 0 || F % 64 != 0) return MOE_ERR_SHAPE;
        auto al16 = [](const void* p) { return ((uintptr_t)p & 15) == 0; };
        if (!al16(buffer) || !al16(W1) || !al16(W2) || !al16(y) || (W3 && !al16(W3))) return MOE_ERR_SHAPE;
    }
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;

    if (dtype == MOE_F32) {
        float* H = (float*)workspace;
        const long long nh = (long long)R_max * F, ny = (long long)R_max * d;
        ffn_f32_hidden_kernel<<<(int)((nh + 255) / 256), 256, 0, s>>>((const float*)buffer, d, F, E, offsets, R_max,
                                                                      (const float*)W1, (const float*)W3, act, H);
        MOE_LAUNCH_CHECK();
        ffn_f32_out_kernel<<<(int)((ny + 255) / 256), 256, 0, s>>>(H, d, F, E, offsets, R_max, (const float*)W2,
                                                                   (float*)y);
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }

    // bf16 tensor-core path
    if (!tc::tma_encoder_ready()) return MOE_ERR_CUDA;
    uint16_t* H = (uint16_t*)workspace;
    CUtensorMap m_x, m_w1, m_w3, m_h, m_w2, m_hout, m_yout;
    const bool swiglu = act == MOE_ACT_SWIGLU;
    const bool pair = use_pair_kernels(R_max, E);
    // per-CTA boxes: A is always 128 rows; B is 128 rows per CTA in the pair
    // kernels, and 128 (SwiGLU halves) or 256 rows in the one-CTA kernels
    const int bbox = pair ? 128 : 256;
    if (!tc::make_bf16_map(&m_x, buffer, R_max, d, 128)) return MOE_ERR_CUDA;
    if (!tc::make_bf16_map(&m_w1, W1, (long long)E * F, d, swiglu ? 128 : bbox)) return MOE_ERR_CUDA;
    if (swiglu && !tc::make_bf16_map(&m_w3, W3, (long long)E * F, d, 128)) return MOE_ERR_CUDA;
    if (!tc::make_bf16_map(&m_h, H, R_max, F, 128)) return MOE_ERR_CUDA;
    if (!tc::make_bf16_map(&m_w2, W2, (long long)E * d, F, bbox)) return MOE_ERR_CUDA;
    if (!tc::make_store_map(&m_hout, H, R_max, F)) return MOE_ERR_CUDA;
    if (!tc::make_store_map(&m_yout, y, R_max, d)) return MOE_ERR_CUDA;

    tc::GemmArgs g1{offsets, E, d, F, F, R_max, H, err};
    if (pair) {
        moe_status st = swiglu ? launch_gemm2<tc::MODE_SWIGLU>(m_x, m_w1, m_w3, m_hout, g1, s)
                               : launch_gemm2<tc::MODE_GELU>(m_x, m_w1, m_w1, m_hout, g1, s);
        if (st != MOE_OK) return st;
        tc::GemmArgs g2{offsets, E, F, d, d, R_max, (uint16_t*)y, err};
        return launch_gemm2<tc::MODE_PLAIN>(m_h, m_w2, m_w2, m_yout, g2, s);
    }
    moe_status st = swiglu ? launch_gemm<tc::MODE_SWIGLU>(m_x, m_w1, m_w3, m_hout, g1, s)
                           : launch_gemm<tc::MODE_GELU>(m_x, m_w1, m_w1, m_hout, g1, s);
    if (st != MOE_OK) return st;
    tc::GemmArgs g2{offsets, E, F, d, d, R_max, (uint16_t*)y, err};
    return launch_gemm<tc::MODE_PLAIN>(m_h, m_w2, m_w2, m_yout, g2, s);
}
