// combine.cu - token_unpermutation: the gate-weighted sum back into token order.
//
// "How MegaDLMs Implements Mixture of Experts (MoE) Architectures",
// "MoELayer" step 3: the output sequence is rebuilt from the expert outputs.
// Each token's kept expert outputs are weighted by their gates and summed
// in fp32; "Expert Parallelism > Key Parameters": a dropped assignment
// contributes zero, and the always-on shared expert's output is added.
//
// One warp per token.  The token's (row, gate) pairs are deduplicated in
// registers first (slots that share a group-major row are read once, their
// gates summed in slot order), then either each lane streams 8-element
// vectors of every distinct row and accumulates in fp32, or (k >= 4) the
// rows are staged chunk by chunk in shared memory by the bulk-copy engine
// and summed from there in the same order.
#include <cstdlib>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {

template <bool BF16>
struct Vec8 {
    // 8 consecutive elements starting at element `e` of a row (16-byte aligned)
    static __device__ __forceinline__ void load(const void* base, long long e, float* f) {
        if (BF16) {
            uint4 v = ld_keep(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + e));
            f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
            f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
        } else {
            const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + e);
            uint4 a = ld_keep(p), b = ld_keep(p + 1);
            f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
            f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
        }
    }
    static __device__ __forceinline__ void store(void* base, long long e, const float* f) {
        if (BF16) {
            uint4 v;
            v.x = pack_bf16x2(f[0], f[1]); v.y = pack_bf16x2(f[2], f[3]);
            v.z = pack_bf16x2(f[4], f[5]); v.w = pack_bf16x2(f[6], f[7]);
            st_stream(reinterpret_cast<uint4*>(static_cast<uint16_t*>(base) + e), v);
        } else {
            uint4* p = reinterpret_cast<uint4*>(static_cast<float*>(base) + e);
            st_stream(p, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3])));
            st_stream(p + 1, make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]), __float_as_uint(f[7])));
        }
    }
};

// The same 8 elements as raw bits, loaded now and converted later, so that
// the loads of several rows can be issued before the first multiply-add.
// Rows of Y are read once per kept slot: streamed past L1.
template <bool BF16>
struct Raw8 {
    uint4 a, b;   // bf16: a holds the 8 values; fp32: a, b hold 4 each
    __device__ __forceinline__ void load(const void* base, long long e) {
        if (BF16) {
            a = ld_stream(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + e));
        } else {
            const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + e);
            a = ld_stream(p);
            b = ld_stream(p + 1);
        }
    }
    // acc[i] = fma(g, value[i], acc[i]), element by element (one rounding each)
    __device__ __forceinline__ void fma_into(float g, float* acc) const {
        float f[8];
        if (BF16) {
            f[0] = bf16_lo(a.x); f[1] = bf16_hi(a.x); f[2] = bf16_lo(a.y); f[3] = bf16_hi(a.y);
            f[4] = bf16_lo(a.z); f[5] = bf16_hi(a.z); f[6] = bf16_lo(a.w); f[7] = bf16_hi(a.w);
        } else {
            f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
            f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(g, f[i], acc[i]);
    }
};

__device__ __forceinline__ float load1(const void* base, long long e, bool bf16) {
    if (bf16) return __uint_as_float(((uint32_t) static_cast<const uint16_t*>(base)[e]) << 16);
    return static_cast<const float*>(base)[e];
}

__device__ __forceinline__ void store1(void* base, long long e, float v, bool bf16) {
    if (bf16) static_cast<__nv_bfloat16*>(base)[e] = __float2bfloat16_rn(v);
    else static_cast<float*>(base)[e] = v;
}

// A token's raw (row, gate) slots: lane j < k holds slot j; a row at or
// past R is reported and dropped.
__device__ __forceinline__ void token_slots(const int32_t* __restrict__ row_map, const float* __restrict__ gate,
                                           long long t, int k, int R, unsigned* err, int& r, float& g) {
    const int lane = threadIdx.x & 31;
    r = -1;
    g = 0.0f;
    if (lane < k) {
        r = row_map[t * k + lane];
        g = gate ? gate[t * k + lane] : 1.0f;
        if (r >= R) { raise_error(err, kErrIndex); r = -1; }
    }
}

// Per-token distinct (row, summed gate) list from the raw slots: lane j < nu
// holds entry j, entries in order of first appearance, gates of repeated
// rows summed in slot order.  Called by all 32 lanes.
__device__ __forceinline__ int dedupe_rows(int r, float g, int k, int& my_row, float& my_gate) {
    const int lane = threadIdx.x & 31;
    int nu = 0;
    my_row = -1;
    my_gate = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int rj = __shfl_sync(0xffffffffu, r, j);
        const float gj = __shfl_sync(0xffffffffu, g, j);
        if (rj < 0) continue;
        const unsigned hit = __ballot_sync(0xffffffffu, lane < nu && my_row == rj);
        const int pos = hit ? __ffs(hit) - 1 : nu;
        if (lane == pos) {
            if (hit) my_gate += gj;
            else { my_row = rj; my_gate = gj; }
        }
        if (!hit) ++nu;
    }
    return nu;
}

__device__ __forceinline__ int token_rows(const int32_t* __restrict__ row_map, const float* __restrict__ gate,
                                          long long t, int k, int R, unsigned* err, int& my_row, float& my_gate) {
    int r;
    float g;
    token_slots(row_map, gate, t, k, R, err, r, g);
    return dedupe_rows(r, g, k, my_row, my_gate);
}

template <bool IN_BF16, bool OUT_BF16, int NV>
__global__ void __launch_bounds__(256) unpermute_vec_kernel(const void* __restrict__ y, int R, int T, int d, int k,
                                                            const int32_t* __restrict__ row_map,
                                                            const float* __restrict__ gate,
                                                            const void* __restrict__ shared, void* __restrict__ out,
                                                            unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nvec = d >> 3;
    // the next token's slots are loaded while the current token's rows are summed
    int nr = -1;
    float ng = 0.0f;
    if (warp < T) token_slots(row_map, gate, warp, k, R, err, nr, ng);
    for (long long t = warp; t < T; t += nwarps) {
        int my_row;
        float my_gate;
        const int nu = dedupe_rows(nr, ng, k, my_row, my_gate);
        if (t + nwarps < T) token_slots(row_map, gate, t + nwarps, k, R, err, nr, ng);
        for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
            float acc[NV][8];
#pragma unroll
            for (int u = 0; u < NV; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            // rows two at a time: both rows' loads are in flight before the
            // first multiply-add, which still runs in first-appearance order
            for (int j = 0; j < nu; j += 2) {
                const bool two = j + 1 < nu;
                const int r0 = __shfl_sync(0xffffffffu, my_row, j);
                const float g0 = __shfl_sync(0xffffffffu, my_gate, j);
                const int r1 = __shfl_sync(0xffffffffu, my_row, two ? j + 1 : j);
                const float g1 = __shfl_sync(0xffffffffu, my_gate, two ? j + 1 : j);
                Raw8<IN_BF16> a[NV], b[NV];
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) a[u].load(y, (long long)r0 * d + 8LL * v);
                }
                if (two) {
#pragma unroll
                    for (int u = 0; u < NV; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec) b[u].load(y, (long long)r1 * d + 8LL * v);
                    }
                }
#pragma unroll
                for (int u = 0; u < NV; ++u)
                    if (v0 + u * 32 + lane < nvec) a[u].fma_into(g0, acc[u]);
                if (two) {
#pragma unroll
                    for (int u = 0; u < NV; ++u)
                        if (v0 + u * 32 + lane < nvec) b[u].fma_into(g1, acc[u]);
                }
            }
            if (shared) {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    int v = v0 + u * 32 + lane;
                    if (v < nvec) {
                        float f[8];
                        Vec8<IN_BF16>::load(shared, t * d + 8LL * v, f);
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[u][i] += f[i];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                int v = v0 + u * 32 + lane;
                if (v < nvec) Vec8<OUT_BF16>::store(out, t * d + 8LL * v, acc[u]);
            }
        }
    }
}

// Bulk-staged combine (k <= 8, 16-byte rows): a warp takes one token.  Lane 0
// brings the token's kept rows and its shared-expert row into the warp's
// shared memory column chunk by column chunk (a 9 KB stage shared by the
// rows: 1 KB per row for 8 rows and a shared row, 4 KB for two rows) with
// the bulk-copy engine, the next chunk in flight while the lanes add up the
// current one from shared memory (16-byte pieces per lane: rows in first-appearance slot
// order with their summed gates, then the shared row, in fp32 - the order of
// unpermute_vec_kernel, so the results are the same bits) and store it.  No
// per-lane global loads and few registers, so many tokens are in flight per
// SM.  UNIT: every distinct row with weight 1 (the sum of a token's group
// rows, same order and bits as unpermute_groups_kernel).  Waits bounded; on
// expiry the warp records MOE_ERR_TIMEOUT and stops.
constexpr int kCmbWarps = 4;
constexpr int kCmbStage = 9 * 1024;                    // per stage: up to 8 rows + the shared row, 1 KB each
                                                       // (fewer rows: larger chunks)
constexpr int kCmbSmem = kCmbWarps * 2 * kCmbStage;    // 72 KB

template <bool BF16>
__device__ __forceinline__ void piece_to_f32(uint4 v, float* f) {   // 16 bytes -> 8 (bf16) or 4 (fp32) values
    if (BF16) {
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
    } else {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y); f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
}

template <bool OUT_BF16, int N>
__device__ __forceinline__ void store_piece(void* out, long long e, const float* f) {   // N = 8 or 4 values
    if (OUT_BF16) {
        uint16_t* o = static_cast<uint16_t*>(out) + e;
        if (N == 8) {
            uint4 w;
            w.x = pack_bf16x2(f[0], f[1]); w.y = pack_bf16x2(f[2], f[3]);
            w.z = pack_bf16x2(f[4], f[5]); w.w = pack_bf16x2(f[6], f[7]);
            *reinterpret_cast<uint4*>(o) = w;
        } else {
            uint2 w;
            w.x = pack_bf16x2(f[0], f[1]); w.y = pack_bf16x2(f[2], f[3]);
            *reinterpret_cast<uint2*>(o) = w;
        }
    } else {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + e);
        o[0] = make_float4(f[0], f[1], f[2], f[3]);
        if (N == 8) o[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
}

// Rows of a token taken from the expert-choice CSR instead of a row map:
// tok_row[tok_ptr[t] .. tok_ptr[t+1]) with gates ec_gate[row].
struct CsrRows {
    const int32_t* tok_ptr;
    const int32_t* tok_row;
    const float* ec_gate;
};

// A token of the expert-choice combine with more than 8 rows (rare: it needs
// more than 8 experts to pick the same token): the lanes read the rows
// directly, in CSR order.
template <bool IN_BF16, bool OUT_BF16>
__device__ void ec_token_direct(const void* y, int R, int d, long long t, int p0, int p1, const CsrRows& c, void* out,
                                unsigned* err) {
    const int lane = threadIdx.x & 31;
    for (int e = lane * 8; e < d; e += 256) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int p = p0; p < p1; ++p) {
            const int r = c.tok_row[p];
            if (r < 0 || r >= R) { if (e == lane * 8) raise_error(err, kErrIndex); continue; }
            const float g = c.ec_gate[r];
            float f[8];
            Vec8<IN_BF16>::load(y, (long long)r * d + e, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(g, f[i], acc[i]);
        }
        Vec8<OUT_BF16>::store(out, t * d + e, acc);
    }
}

template <bool IN_BF16, bool OUT_BF16, bool UNIT, bool CSR>
__global__ void __launch_bounds__(32 * kCmbWarps) unpermute_bulk_kernel(const uint8_t* __restrict__ y, int R, int T,
                                                                        int d, int k,
                                                                        const int32_t* __restrict__ row_map,
                                                                        const float* __restrict__ gate,
                                                                        const uint8_t* __restrict__ shared,
                                                                        void* __restrict__ out, unsigned* err,
                                                                        CsrRows csr) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ __align__(128) uint8_t cmb_smem[];
    __shared__ __align__(8) uint64_t bars[kCmbWarps][2];
    __shared__ int no_abort;
    constexpr int ESZ = IN_BF16 ? 2 : 4;
    constexpr int N = 16 / ESZ;                        // values per 16-byte piece
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint8_t* ws = cmb_smem + (size_t)wid * 2 * kCmbStage;
    const long long row_bytes = (long long)d * ESZ;
    if (threadIdx.x == 0) no_abort = 0;
    if (lane == 0) {
        tc::mbar_init(tc::smem_u32(&bars[wid][0]), 1);
        tc::mbar_init(tc::smem_u32(&bars[wid][1]), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    uint32_t par = 0;                                  // bit st: parity of stage st's next completion
    const long long nworkers = (long long)gridDim.x * kCmbWarps;
    for (long long t = (long long)blockIdx.x * kCmbWarps + wid; t < T; t += nworkers) {
        int my_row = -1, nu;
        float my_gate = 0.0f;
        if (CSR) {                                     // lane j < nu: the token's j-th row (-1 if out of range)
            const int p0 = max(csr.tok_ptr[t], 0), p1 = min(csr.tok_ptr[t + 1], R);
            nu = max(p1 - p0, 0);
            if (nu > 8) {
                ec_token_direct<IN_BF16, OUT_BF16>(y, R, d, t, p0, p1, csr, out, err);
                continue;
            }
            if (lane < nu) {
                const int r = csr.tok_row[p0 + lane];
                if (r < 0 || r >= R) raise_error(err, kErrIndex);
                else { my_row = r; my_gate = csr.ec_gate[r]; }
            }
        } else {
            nu = token_rows(row_map, gate, t, k, R, err, my_row, my_gate);
        }
        int rr[8];
        float gg[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            rr[j] = __shfl_sync(0xffffffffu, my_row, j);
            gg[j] = __shfl_sync(0xffffffffu, my_gate, j);
        }
        const int nr = __popc(__ballot_sync(0xffffffffu, lane < nu && my_row >= 0)) + (shared ? 1 : 0);
        if (nr == 0) {                                 // every slot dropped and no shared expert: zeros
            const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (long long e = (long long)lane * N; e < d; e += 32LL * N) store_piece<OUT_BF16, N>(out, t * d + e, z);
            continue;
        }
        // chunk size for this token: the stage (9 KB) divided among its row slots, in 512-byte
        // steps, so that a token with few rows moves a few KB per wait
        const int slots = nu + (shared ? 1 : 0);
        int cb = kCmbStage / slots / 512 * 512;
        const int row_cb = (int)((row_bytes + 511) / 512 * 512);
        if (cb > row_cb) cb = row_cb;
        const int nchunk = (int)((row_bytes + cb - 1) / cb);
        auto issue = [&](int c, int st) {              // lane 0: chunk c of every row into stage st
            if (lane != 0) return;
            const long long off = (long long)c * cb;
            const uint32_t bytes = (uint32_t)min((long long)cb, row_bytes - off);
            const uint32_t bar = tc::smem_u32(&bars[wid][st]);
            const uint32_t dst = tc::smem_u32(ws + st * kCmbStage);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // earlier reads of the stage come first
            tc::mbar_expect_tx(bar, bytes * (uint32_t)nr);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < nu && rr[j] >= 0)
                    tc::bulk_load(dst + j * cb, y + (long long)rr[j] * row_bytes + off, bytes, bar);
            if (shared) tc::bulk_load(dst + nu * cb, shared + t * row_bytes + off, bytes, bar);
        };
        issue(0, 0);
        bool ok = true;
        for (int c = 0; c < nchunk; ++c) {
            const int st = c & 1;
            if (c + 1 < nchunk) issue(c + 1, st ^ 1);  // that stage's previous chunk was consumed last iteration
            const uint32_t pst = (par >> st) & 1u;
            const bool got = tc::mbar_wait(tc::smem_u32(&bars[wid][st]), pst, &no_abort);
            par ^= 1u << st;
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                if (lane == 0) {                       // loads still in flight may land: give them one more bounded wait
                    tc::mbar_wait(tc::smem_u32(&bars[wid][st]), pst, &no_abort);
                    if (c + 1 < nchunk) tc::mbar_wait(tc::smem_u32(&bars[wid][st ^ 1]), (par >> (st ^ 1)) & 1u, &no_abort);
                }
                break;
            }
            const uint8_t* stage = ws + st * kCmbStage;
#pragma unroll 2
            for (int boff = lane * 16; boff < cb; boff += 512) {       // this lane's 16-byte pieces of the chunk
                const long long e = ((long long)c * cb + boff) / ESZ;
                if (e >= d) break;
                float acc[N];
#pragma unroll
                for (int i = 0; i < N; ++i) acc[i] = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j < nu && rr[j] >= 0) {
                        float f[N];
                        piece_to_f32<IN_BF16>(*reinterpret_cast<const uint4*>(stage + j * cb + boff), f);
#pragma unroll
                        for (int i = 0; i < N; ++i) acc[i] = __fmaf_rn(UNIT ? 1.0f : gg[j], f[i], acc[i]);
                    }
                }
                if (shared) {
                    float f[N];
                    piece_to_f32<IN_BF16>(*reinterpret_cast<const uint4*>(stage + nu * cb + boff), f);
#pragma unroll
                    for (int i = 0; i < N; ++i) acc[i] += f[i];
                }
                store_piece<OUT_BF16, N>(out, t * d + e, acc);
            }
            __syncwarp();
        }
        if (!ok) {
            if (lane == 0) raise_error(err, kErrTimeout);
            return;
        }
    }
}

// Any d, any alignment: one element per lane.
__global__ void __launch_bounds__(256) unpermute_scalar_kernel(const void* __restrict__ y, bool in_bf16, int R, int T, int d,
                                                               int k, const int32_t* __restrict__ row_map,
                                                               const float* __restrict__ gate,
                                                               const void* __restrict__ shared, void* __restrict__ out,
                                                               bool out_bf16, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = warp; t < T; t += nwarps) {
        int my_row;
        float my_gate;
        const int nu = token_rows(row_map, gate, t, k, R, err, my_row, my_gate);
        for (int c0 = 0; c0 < d; c0 += 32) {
            const int c = c0 + lane;
            float acc = 0.0f;
            for (int j = 0; j < nu; ++j) {
                const int r = __shfl_sync(0xffffffffu, my_row, j);
                const float g = __shfl_sync(0xffffffffu, my_gate, j);
                if (c < d) acc = __fmaf_rn(g, load1(y, (long long)r * d + c, in_bf16), acc);
            }
            if (c < d) {
                if (shared) acc += load1(shared, t * d + c, in_bf16);
                store1(out, t * d + c, acc, out_bf16);
            }
        }
    }
}

// Expert choice: rows from the token CSR (ascending expert), gate by row.
template <bool IN_BF16, bool OUT_BF16, int NV>
__global__ void __launch_bounds__(256) unpermute_ec_vec_kernel(const void* __restrict__ y, int R, int T, int d,
                                                               const int32_t* __restrict__ tok_ptr,
                                                               const int32_t* __restrict__ tok_row,
                                                               const float* __restrict__ ec_gate,
                                                               void* __restrict__ out, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nvec = d >> 3;
    // A token's rows sit one per lane (CSR position p0 + lane), with their
    // gates.  The metadata of the warp's next token is fetched while the
    // current token's rows are summed: its CSR rows and the pointers of the
    // token after it before, its gates after (each load one step ahead of
    // its use), so the dependent pointer -> row -> gate loads stay off the
    // critical path.  Tokens with more than 32 rows take the direct loop.
    auto ptrs = [&](long long tt, int& a, int& b) {
        a = b = 0;
        if (tt < T) { a = max(tok_ptr[tt], 0); b = min(tok_ptr[tt + 1], R); }
    };
    auto row_at = [&](int a, int b) -> int { return lane < b - a ? tok_row[a + lane] : -1; };
    auto gate_of = [&](int r) -> float { return (r >= 0 && r < R) ? ec_gate[r] : 0.0f; };
    long long t = warp;
    int c0, c1, n0, n1;
    ptrs(t, c0, c1);
    int cr = row_at(c0, c1);
    ptrs(t + nwarps, n0, n1);
    float cg = gate_of(cr);
    for (; t < T; t += nwarps) {
        const int nr = row_at(n0, n1);
        int m0, m1;
        ptrs(t + 2 * nwarps, m0, m1);
        const int cnt = c1 - c0;
        if (cnt <= 32) {
            const bool in = lane < cnt;
            const bool ok = in && cr >= 0 && cr < R;
            if (in && !ok) raise_error(err, kErrIndex);
            const unsigned valid = __ballot_sync(0xffffffffu, ok);
            for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
                float acc[NV][8];
#pragma unroll
                for (int u = 0; u < NV; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
                // the valid rows two at a time (both in flight), added in CSR order
                unsigned m = valid;
                while (m) {
                    const int j0 = __ffs(m) - 1;
                    m &= m - 1;
                    const bool two = m != 0;
                    const int j1 = two ? __ffs(m) - 1 : j0;
                    if (two) m &= m - 1;
                    const int r0 = __shfl_sync(0xffffffffu, cr, j0);
                    const float g0 = __shfl_sync(0xffffffffu, cg, j0);
                    const int r1 = __shfl_sync(0xffffffffu, cr, j1);
                    const float g1 = __shfl_sync(0xffffffffu, cg, j1);
                    Raw8<IN_BF16> a[NV], b[NV];
#pragma unroll
                    for (int u = 0; u < NV; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec) a[u].load(y, (long long)r0 * d + 8LL * v);
                    }
                    if (two) {
#pragma unroll
                        for (int u = 0; u < NV; ++u) {
                            const int v = v0 + u * 32 + lane;
                            if (v < nvec) b[u].load(y, (long long)r1 * d + 8LL * v);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < NV; ++u)
                        if (v0 + u * 32 + lane < nvec) a[u].fma_into(g0, acc[u]);
                    if (two) {
#pragma unroll
                        for (int u = 0; u < NV; ++u)
                            if (v0 + u * 32 + lane < nvec) b[u].fma_into(g1, acc[u]);
                    }
                }
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) Vec8<OUT_BF16>::store(out, t * d + 8LL * v, acc[u]);
                }
            }
        } else {
            for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
                float acc[NV][8];
#pragma unroll
                for (int u = 0; u < NV; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
                for (int p = c0; p < c1; ++p) {
                    const int r = tok_row[p];
                    if (r < 0 || r >= R) { raise_error(err, kErrIndex); continue; }
                    const float g = ec_gate[r];
#pragma unroll
                    for (int u = 0; u < NV; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec) {
                            Raw8<IN_BF16> a;
                            a.load(y, (long long)r * d + 8LL * v);
                            a.fma_into(g, acc[u]);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) Vec8<OUT_BF16>::store(out, t * d + 8LL * v, acc[u]);
                }
            }
        }
        const float ng = gate_of(nr);
        c0 = n0; c1 = n1; cr = nr; cg = ng;
        n0 = m0; n1 = m1;
    }
}

__global__ void __launch_bounds__(256) unpermute_ec_scalar_kernel(const void* __restrict__ y, bool in_bf16, int R, int T, int d,
                                                                  const int32_t* __restrict__ tok_ptr,
                                                                  const int32_t* __restrict__ tok_row,
                                                                  const float* __restrict__ ec_gate,
                                                                  void* __restrict__ out, bool out_bf16, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = warp; t < T; t += nwarps) {
        const int p0 = max(tok_ptr[t], 0), p1 = min(tok_ptr[t + 1], R);
        for (int c = lane; c < d; c += 32) {
            float acc = 0.0f;
            for (int p = p0; p < p1; ++p) {
                const int r = tok_row[p];
                if (r < 0 || r >= R) { raise_error(err, kErrIndex); continue; }
                acc = __fmaf_rn(ec_gate[r], load1(y, (long long)r * d + c, in_bf16), acc);
            }
            store1(out, t * d + c, acc, out_bf16);
        }
    }
}

// ------------------------------------------- group-major expert path
// The send-once dispatcher with real experts ("Expert Coupling in MoE
// Pretraining", Abstract), each step as one GPU of an expert-parallel group
// would run it: the group-major rows (one per token and group) are copied
// to expert-major rows (the group's local permutation), the experts run,
// each token's expert outputs inside one group are pre-combined with their
// gates into that group's row, and the token's output is the sum of its
// group rows.

// dst[dst_row[s]] = src[src_row[s]] for every slot with both rows valid.
template <int NV>
__global__ void __launch_bounds__(256) copy_slot_rows_kernel(const uint4* __restrict__ src, int R_src, int vec_per_row,
                                                             const int32_t* __restrict__ src_row,
                                                             const int32_t* __restrict__ dst_row, long long S,
                                                             uint4* __restrict__ dst, int R_dst, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long s = warp; s < S; s += nwarps) {
        const int sr = src_row[s], dr = dst_row[s];
        if (sr < 0 || dr < 0) continue;
        if (sr >= R_src || dr >= R_dst) { if (lane == 0) raise_error(err, kErrIndex); continue; }
        const uint4* a = src + (long long)sr * vec_per_row;
        uint4* b = dst + (long long)dr * vec_per_row;
        for (int v0 = 0; v0 < vec_per_row; v0 += 32 * NV) {
            uint4 buf[NV];
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < vec_per_row) buf[u] = ld_stream(a + v);
            }
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < vec_per_row) st_stream(b + v, buf[u]);
            }
        }
    }
}

// y_g[r] = sum over the token's slots j with row_map_g[t, j] = r (slot order)
// of gate[t, j] * y_e[row_map_e[t, j]], fp32 accumulation, one write per
// group row.  One warp per token.
template <bool BF16, int NV>
__global__ void __launch_bounds__(256) group_precombine_kernel(const void* __restrict__ y_e, int R_e, int T, int d, int k,
                                                               const int32_t* __restrict__ row_map_e,
                                                               const int32_t* __restrict__ row_map_g,
                                                               const float* __restrict__ gate, void* __restrict__ y_g,
                                                               int R_g, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nvec = d >> 3;
    for (long long t = warp; t < T; t += nwarps) {
        int re = -1, rg = -1;
        float g = 0.0f;
        if (lane < k) {
            re = row_map_e[t * k + lane];
            rg = row_map_g[t * k + lane];
            g = gate[t * k + lane];
            if (re >= R_e || rg >= R_g) { raise_error(err, kErrIndex); re = -1; rg = -1; }
        }
        for (int j = 0; j < k; ++j) {
            const int rgj = __shfl_sync(0xffffffffu, rg, j);
            if (rgj < 0) continue;
            const unsigned earlier = __ballot_sync(0xffffffffu, lane < j && rg == rgj);
            if (earlier) continue;                          // this group row was written for an earlier slot
            for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
                float acc[NV][8];
#pragma unroll
                for (int u = 0; u < NV; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
                for (int q = j; q < k; ++q) {
                    const int rgq = __shfl_sync(0xffffffffu, rg, q);
                    const int req = __shfl_sync(0xffffffffu, re, q);
                    const float gq = __shfl_sync(0xffffffffu, g, q);
                    if (rgq != rgj || req < 0) continue;
                    float f[NV][8];
#pragma unroll
                    for (int u = 0; u < NV; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < nvec) Vec8<BF16>::load(y_e, (long long)req * d + 8LL * v, f[u]);
                    }
#pragma unroll
                    for (int u = 0; u < NV; ++u)
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[u][i] = __fmaf_rn(gq, f[u][i], acc[u][i]);
                }
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) Vec8<BF16>::store(y_g, (long long)rgj * d + 8LL * v, acc[u]);
                }
            }
        }
    }
}

// out[t] = sum of the token's distinct group rows (first-appearance order)
// plus shared[t] when given.  One warp per token.
template <bool IN_BF16, bool OUT_BF16, int NV>
__global__ void __launch_bounds__(256) unpermute_groups_kernel(const void* __restrict__ y_g, int R_g, int T, int d, int k,
                                                               const int32_t* __restrict__ row_map_g,
                                                               const void* __restrict__ shared, void* __restrict__ out,
                                                               unsigned* err) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nvec = d >> 3;
    for (long long t = warp; t < T; t += nwarps) {
        int rg = -1;
        if (lane < k) {
            rg = row_map_g[t * k + lane];
            if (rg >= R_g) { raise_error(err, kErrIndex); rg = -1; }
        }
        unsigned first = 0;                                  // slots holding a row's first appearance
        for (int j = 0; j < k; ++j) {
            const int rgj = __shfl_sync(0xffffffffu, rg, j);
            if (rgj < 0) continue;
            if (!__ballot_sync(0xffffffffu, lane < j && rg == rgj)) first |= 1u << j;
        }
        for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
            float acc[NV][8];
#pragma unroll
            for (int u = 0; u < NV; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            unsigned m = first;
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                const int r = __shfl_sync(0xffffffffu, rg, j);
                float f[NV][8];
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) Vec8<IN_BF16>::load(y_g, (long long)r * d + 8LL * v, f[u]);
                }
#pragma unroll
                for (int u = 0; u < NV; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] += f[u][i];
            }
            if (shared) {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) {
                        float f[8];
                        Vec8<IN_BF16>::load(shared, t * d + 8LL * v, f);
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[u][i] += f[i];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) Vec8<OUT_BF16>::store(out, t * d + 8LL * v, acc[u]);
            }
        }
    }
}

template <bool UNIT, bool CSR>
moe_status launch_unpermute_bulk(bool in_bf16, bool out_bf16, cudaStream_t s, const void* y, int R, int T, int d,
                                 int k, const int32_t* row_map, const float* gate, const void* shared, void* out,
                                 unsigned* err, CsrRows csr = CsrRows{nullptr, nullptr, nullptr}) {
    for (auto fn : {unpermute_bulk_kernel<true, true, UNIT, CSR>, unpermute_bulk_kernel<true, false, UNIT, CSR>,
                    unpermute_bulk_kernel<false, true, UNIT, CSR>, unpermute_bulk_kernel<false, false, UNIT, CSR>})
        if (!set_smem_limit((const void*)fn, kCmbSmem)) return MOE_ERR_CUDA;
    long long nb = ((long long)T + kCmbWarps - 1) / kCmbWarps;
    const int blocks = (int)(nb < 148 * 8 ? nb : 148 * 8);
    const uint8_t* yb = (const uint8_t*)y;
    const uint8_t* sb = (const uint8_t*)shared;
    if (in_bf16 && out_bf16)
        (void)launch_pdl(unpermute_bulk_kernel<true, true, UNIT, CSR>, blocks, 32 * kCmbWarps, kCmbSmem, s, yb, R, T, d, k, row_map, gate, sb, out, err, csr);
    else if (in_bf16)
        (void)launch_pdl(unpermute_bulk_kernel<true, false, UNIT, CSR>, blocks, 32 * kCmbWarps, kCmbSmem, s, yb, R, T, d, k, row_map, gate, sb, out, err, csr);
    else if (out_bf16)
        (void)launch_pdl(unpermute_bulk_kernel<false, true, UNIT, CSR>, blocks, 32 * kCmbWarps, kCmbSmem, s, yb, R, T, d, k, row_map, gate, sb, out, err, csr);
    else
        (void)launch_pdl(unpermute_bulk_kernel<false, false, UNIT, CSR>, blocks, 32 * kCmbWarps, kCmbSmem, s, yb, R, T, d, k, row_map, gate, sb, out, err, csr);
    return MOE_OK;
}

// Expert choice: a token has about E*C/T rows (2 at the expert-choice
// workload), too few for the staging to pay (measured 95 vs 56 us there), so
// the register kernel is the default; LIBMOE_BULK_COMBINE=1 selects the
// bulk-staged one.
bool bulk_combine_ec_enabled() {
    const char* env = getenv("LIBMOE_BULK_COMBINE");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return false;
}

// The token combine (gate-weighted rows) runs on the register kernel, which
// keeps two rows' loads in flight per warp: it measured faster than the
// bulk-staged kernel at every shape timed (k = 2: 34 vs 44 us; clustered
// top-6 with the shared row: 91 vs 116 us; top-8 group rows, T = 4096:
// 68 vs 85 us, T = 131072: 1857 vs 1894 us).  The unit-weight sum of a
// token's group rows (moe_unpermute_groups) stays on the bulk kernel, which
// is faster there (83 vs 103 us at the clustered top-6 workload, G = 8).
// LIBMOE_BULK_COMBINE=0/1 forces either kernel for both calls.
bool bulk_combine_enabled(bool unit) {
    const char* env = getenv("LIBMOE_BULK_COMBINE");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return unit;
}

int token_grid(long long T) {
    long long blocks = (T + 7) / 8;
    long long cap = 148LL * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

}  // namespace moe

using namespace moe;

// Grid of the register combines: one warp per token for fixed-size tokens
// (a finished CTA's place is taken by a fresh one: T = 131072 group rows
// 0.98 of HBM against 0.95 with one resident wave of grid-strided CTAs);
// for expert choice, whose tokens carry 0 to E rows, one resident wave of
// grid-strided warps evens the load out (0.69-0.70 against 0.60 with a warp
// per token).  `cap` is applied to the CTA count of the kernel launched.
#define MOE_LAUNCH_GRID(FN, CAP, ...) \
    (void)launch_pdl(FN, (CAP) ? min(grid, resident_ctas((const void*)FN, 256, 0)) : grid, 256, 0, s, __VA_ARGS__)
#define MOE_DISPATCH_VEC_CAP(KERNEL, NV, CAP, ...)                                                   \
    do {                                                                                             \
        if (in_bf16 && out_bf16) MOE_LAUNCH_GRID((KERNEL<true, true, NV>), CAP, __VA_ARGS__);        \
        else if (in_bf16) MOE_LAUNCH_GRID((KERNEL<true, false, NV>), CAP, __VA_ARGS__);              \
        else if (out_bf16) MOE_LAUNCH_GRID((KERNEL<false, true, NV>), CAP, __VA_ARGS__);             \
        else MOE_LAUNCH_GRID((KERNEL<false, false, NV>), CAP, __VA_ARGS__);                          \
    } while (0)
#define MOE_DISPATCH_VEC(KERNEL, NV, ...) MOE_DISPATCH_VEC_CAP(KERNEL, NV, false, __VA_ARGS__)

extern "C" moe_status moe_unpermute(const void* y, int dtype, int R, int T, int d, int k, const int32_t* row_map,
                                    const float* gate, const void* shared, void* out, int out_dtype,
                                    moe_stream_t stream) {
    if (T < 0 || d < 0 || k < 1 || R < 0) return MOE_ERR_ARG;
    if ((dtype != MOE_F32 && dtype != MOE_BF16) || (out_dtype != MOE_F32 && out_dtype != MOE_BF16)) return MOE_ERR_ARG;
    if (k > 32) return MOE_ERR_SHAPE;
    if (T == 0 || d == 0) return MOE_OK;
    if (!row_map || !gate || !out || (R > 0 && !y)) return MOE_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const bool in_bf16 = dtype == MOE_BF16, out_bf16 = out_dtype == MOE_BF16;
    const int grid = token_grid(T);
    const int in_esz = in_bf16 ? 2 : 4, out_esz = out_bf16 ? 2 : 4;
    const bool vec = (d % 8 == 0) && ((d * in_esz) % 16 == 0) && ((d * out_esz) % 16 == 0) &&
                     (y == nullptr || aligned16(y)) && aligned16(out) && (shared == nullptr || aligned16(shared));
    if (vec && k <= 8 && bulk_combine_enabled(false)) {
        const moe_status st = launch_unpermute_bulk<false, false>(in_bf16, out_bf16, s, y, R, T, d, k, row_map, gate,
                                                                  shared, out, err);
        if (st != MOE_OK) return st;
    } else if (vec) {
        const int nvec = d / 8;
        const int grid = (int)min((T + 7LL) / 8, (long long)INT_MAX);
        // two 16-byte vectors per lane per row, two rows in flight: 62 registers,
        // four 256-thread CTAs per SM (4 KB rows and up: 33.6 us against 38.4 us
        // with four vectors per lane at the Mixtral-shaped combine)
        if (nvec <= 32) MOE_DISPATCH_VEC(unpermute_vec_kernel, 1, y, R, T, d, k, row_map, gate, shared, out, err);
        else MOE_DISPATCH_VEC(unpermute_vec_kernel, 2, y, R, T, d, k, row_map, gate, shared, out, err);
    } else {
        (void)launch_pdl(unpermute_scalar_kernel, grid, 256, 0, s, y, in_bf16, R, T, d, k, row_map, gate, shared, out, out_bf16, err);
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_unpermute_ec(const void* y, int dtype, int R, int T, int d, const int32_t* tok_ptr,
                                       const int32_t* tok_row, const float* ec_gate, void* out, int out_dtype,
                                       moe_stream_t stream) {
    if (T < 0 || d < 0 || R < 0) return MOE_ERR_ARG;
    if ((dtype != MOE_F32 && dtype != MOE_BF16) || (out_dtype != MOE_F32 && out_dtype != MOE_BF16)) return MOE_ERR_ARG;
    if (T == 0 || d == 0) return MOE_OK;
    if (!tok_ptr || !tok_row || !ec_gate || !out || (R > 0 && !y)) return MOE_ERR_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const bool in_bf16 = dtype == MOE_BF16, out_bf16 = out_dtype == MOE_BF16;
    const int grid = token_grid(T);
    const int in_esz = in_bf16 ? 2 : 4, out_esz = out_bf16 ? 2 : 4;
    const bool vec = (d % 8 == 0) && ((d * in_esz) % 16 == 0) && ((d * out_esz) % 16 == 0) &&
                     (y == nullptr || aligned16(y)) && aligned16(out);
    if (vec && bulk_combine_ec_enabled()) {
        const moe_status st = launch_unpermute_bulk<false, true>(in_bf16, out_bf16, s, y, R, T, d, 0, nullptr, nullptr,
                                                                 nullptr, out, err, CsrRows{tok_ptr, tok_row, ec_gate});
        if (st != MOE_OK) return st;
    } else if (vec) {
        const int nvec = d / 8;
        const int grid = (int)min((T + 7LL) / 8, (long long)INT_MAX);
        if (nvec <= 32) MOE_DISPATCH_VEC_CAP(unpermute_ec_vec_kernel, 1, true, y, R, T, d, tok_ptr, tok_row, ec_gate, out, err);
        else MOE_DISPATCH_VEC_CAP(unpermute_ec_vec_kernel, 2, true, y, R, T, d, tok_ptr, tok_row, ec_gate, out, err);
    } else {
        (void)launch_pdl(unpermute_ec_scalar_kernel, grid, 256, 0, s, y, in_bf16, R, T, d, tok_ptr, tok_row, ec_gate, out, out_bf16, err);
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_copy_slot_rows(const void* src, int dtype, int R_src, int d, const int32_t* src_row,
                                         const int32_t* dst_row, int S, void* dst, int R_dst, moe_stream_t stream) {
    if (R_src < 0 || R_dst < 0 || d < 0 || S < 0) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (S == 0 || d == 0) return MOE_OK;
    if (!src || !src_row || !dst_row || !dst) return MOE_ERR_ARG;
    const long long row_bytes = (long long)d * (dtype == MOE_BF16 ? 2 : 4);
    if (row_bytes % 16 || !aligned16(src) || !aligned16(dst)) return MOE_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const int vpr = (int)(row_bytes / 16);
    const int grid = token_grid(S);
    if (vpr <= 32) copy_slot_rows_kernel<1><<<grid, 256, 0, s>>>((const uint4*)src, R_src, vpr, src_row, dst_row, S, (uint4*)dst, R_dst, err);
    else if (vpr <= 64) copy_slot_rows_kernel<2><<<grid, 256, 0, s>>>((const uint4*)src, R_src, vpr, src_row, dst_row, S, (uint4*)dst, R_dst, err);
    else copy_slot_rows_kernel<4><<<grid, 256, 0, s>>>((const uint4*)src, R_src, vpr, src_row, dst_row, S, (uint4*)dst, R_dst, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_group_precombine(const void* y_e, int dtype, int R_e, int T, int d, int k,
                                           const int32_t* row_map_e, const int32_t* row_map_g, const float* gate,
                                           void* y_g, int R_g, moe_stream_t stream) {
    if (R_e < 0 || R_g < 0 || T < 0 || d < 0 || k < 1) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (k > 32) return MOE_ERR_SHAPE;
    if (T == 0 || d == 0) return MOE_OK;
    if (!y_e || !row_map_e || !row_map_g || !gate || !y_g) return MOE_ERR_ARG;
    const int esz = dtype == MOE_BF16 ? 2 : 4;
    if (d % 8 || (d * esz) % 16 || !aligned16(y_e) || !aligned16(y_g)) return MOE_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const int grid = token_grid(T);
    const int nvec = d / 8;
    const bool bf16 = dtype == MOE_BF16;
#define MOE_PRE(NV)                                                                                                 \
    do {                                                                                                            \
        if (bf16) group_precombine_kernel<true, NV><<<grid, 256, 0, s>>>(y_e, R_e, T, d, k, row_map_e, row_map_g, gate, y_g, R_g, err); \
        else group_precombine_kernel<false, NV><<<grid, 256, 0, s>>>(y_e, R_e, T, d, k, row_map_e, row_map_g, gate, y_g, R_g, err); \
    } while (0)
    if (nvec <= 32) MOE_PRE(1);
    else if (nvec <= 64) MOE_PRE(2);
    else MOE_PRE(4);
#undef MOE_PRE
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

extern "C" moe_status moe_unpermute_groups(const void* y_g, int dtype, int R_g, int T, int d, int k,
                                           const int32_t* row_map_g, const void* shared, void* out, int out_dtype,
                                           moe_stream_t stream) {
    if (R_g < 0 || T < 0 || d < 0 || k < 1) return MOE_ERR_ARG;
    if ((dtype != MOE_F32 && dtype != MOE_BF16) || (out_dtype != MOE_F32 && out_dtype != MOE_BF16)) return MOE_ERR_ARG;
    if (k > 32) return MOE_ERR_SHAPE;
    if (T == 0 || d == 0) return MOE_OK;
    if (!row_map_g || !out || (R_g > 0 && !y_g)) return MOE_ERR_ARG;
    const bool in_bf16 = dtype == MOE_BF16, out_bf16 = out_dtype == MOE_BF16;
    const int in_esz = in_bf16 ? 2 : 4, out_esz = out_bf16 ? 2 : 4;
    if (d % 8 || (d * in_esz) % 16 || (d * out_esz) % 16 || (y_g && !aligned16(y_g)) || !aligned16(out) ||
        (shared && !aligned16(shared)))
        return MOE_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    if (k <= 8 && bulk_combine_enabled(true)) {
        const moe_status st = launch_unpermute_bulk<true, false>(in_bf16, out_bf16, s, y_g, R_g, T, d, k, row_map_g,
                                                                 nullptr, shared, out, err);
        if (st != MOE_OK) return st;
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
    const int grid = token_grid(T);
    const int nvec = d / 8;
    if (nvec <= 32) MOE_DISPATCH_VEC(unpermute_groups_kernel, 1, y_g, R_g, T, d, k, row_map_g, shared, out, err);
    else if (nvec <= 64) MOE_DISPATCH_VEC(unpermute_groups_kernel, 2, y_g, R_g, T, d, k, row_map_g, shared, out, err);
    else MOE_DISPATCH_VEC(unpermute_groups_kernel, 4, y_g, R_g, T, d, k, row_map_g, shared, out, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
