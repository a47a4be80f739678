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
// gates summed in slot order), then each lane streams 8-element vectors of
// every distinct row and accumulates in fp32.
#include "common.cuh"

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

__device__ __forceinline__ float load1(const void* base, long long e, bool bf16) {
    if (bf16) return __uint_as_float(((uint32_t) static_cast<const uint16_t*>(base)[e]) << 16);
    return static_cast<const float*>(base)[e];
}

__device__ __forceinline__ void store1(void* base, long long e, float v, bool bf16) {
    if (bf16) static_cast<__nv_bfloat16*>(base)[e] = __float2bfloat16_rn(v);
    else static_cast<float*>(base)[e] = v;
}

// Per-token distinct (row, summed gate) list: lane j < nu holds entry j,
// entries in order of first appearance, gates of repeated rows summed in
// slot order.  Called by all 32 lanes.
__device__ __forceinline__ int token_rows(const int32_t* __restrict__ row_map, const float* __restrict__ gate,
                                          long long t, int k, int R, unsigned* err, int& my_row, float& my_gate) {
    const int lane = threadIdx.x & 31;
    int r = -1;
    float g = 0.0f;
    if (lane < k) {
        r = row_map[t * k + lane];
        g = gate[t * k + lane];
        if (r >= R) { raise_error(err, kErrIndex); r = -1; }
    }
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

template <bool IN_BF16, bool OUT_BF16, int NV>
__global__ void __launch_bounds__(256) unpermute_vec_kernel(const void* __restrict__ y, int R, int T, int d, int k,
                                                            const int32_t* __restrict__ row_map,
                                                            const float* __restrict__ gate,
                                                            const void* __restrict__ shared, void* __restrict__ out,
                                                            unsigned* err) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nvec = d >> 3;
    for (long long t = warp; t < T; t += nwarps) {
        int my_row;
        float my_gate;
        const int nu = token_rows(row_map, gate, t, k, R, err, my_row, my_gate);
        for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
            float acc[NV][8];
#pragma unroll
            for (int u = 0; u < NV; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            for (int j = 0; j < nu; ++j) {
                const int r = __shfl_sync(0xffffffffu, my_row, j);
                const float g = __shfl_sync(0xffffffffu, my_gate, j);
                float f[NV][8];
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    int v = v0 + u * 32 + lane;
                    if (v < nvec) Vec8<IN_BF16>::load(y, (long long)r * d + 8LL * v, f[u]);
                }
#pragma unroll
                for (int u = 0; u < NV; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = __fmaf_rn(g, f[u][i], acc[u][i]);
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

// Any d, any alignment: one element per lane.
__global__ void __launch_bounds__(256) unpermute_scalar_kernel(const void* __restrict__ y, bool in_bf16, int R, int T, int d,
                                                               int k, const int32_t* __restrict__ row_map,
                                                               const float* __restrict__ gate,
                                                               const void* __restrict__ shared, void* __restrict__ out,
                                                               bool out_bf16, unsigned* err) {
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
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nvec = d >> 3;
    for (long long t = warp; t < T; t += nwarps) {
        const int p0 = max(tok_ptr[t], 0), p1 = min(tok_ptr[t + 1], R);
        for (int v0 = 0; v0 < nvec; v0 += 32 * NV) {
            float acc[NV][8];
#pragma unroll
            for (int u = 0; u < NV; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            for (int p = p0; p < p1; ++p) {
                const int r = tok_row[p];
                if (r < 0 || r >= R) { raise_error(err, kErrIndex); continue; }
                const float g = ec_gate[r];
                float f[NV][8];
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    int v = v0 + u * 32 + lane;
                    if (v < nvec) Vec8<IN_BF16>::load(y, (long long)r * d + 8LL * v, f[u]);
                }
#pragma unroll
                for (int u = 0; u < NV; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = __fmaf_rn(g, f[u][i], acc[u][i]);
            }
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                int v = v0 + u * 32 + lane;
                if (v < nvec) Vec8<OUT_BF16>::store(out, t * d + 8LL * v, acc[u]);
            }
        }
    }
}

__global__ void __launch_bounds__(256) unpermute_ec_scalar_kernel(const void* __restrict__ y, bool in_bf16, int R, int T, int d,
                                                                  const int32_t* __restrict__ tok_ptr,
                                                                  const int32_t* __restrict__ tok_row,
                                                                  const float* __restrict__ ec_gate,
                                                                  void* __restrict__ out, bool out_bf16, unsigned* err) {
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

int token_grid(long long T) {
    long long blocks = (T + 7) / 8;
    long long cap = 148LL * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

}  // namespace moe

using namespace moe;

#define MOE_DISPATCH_VEC(KERNEL, NV, ...)                                                       \
    do {                                                                                        \
        if (in_bf16 && out_bf16) KERNEL<true, true, NV><<<grid, 256, 0, s>>>(__VA_ARGS__);      \
        else if (in_bf16) KERNEL<true, false, NV><<<grid, 256, 0, s>>>(__VA_ARGS__);            \
        else if (out_bf16) KERNEL<false, true, NV><<<grid, 256, 0, s>>>(__VA_ARGS__);           \
        else KERNEL<false, false, NV><<<grid, 256, 0, s>>>(__VA_ARGS__);                        \
    } while (0)

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
    if (vec) {
        const int nvec = d / 8;
        if (nvec <= 32) MOE_DISPATCH_VEC(unpermute_vec_kernel, 1, y, R, T, d, k, row_map, gate, shared, out, err);
        else if (nvec <= 64) MOE_DISPATCH_VEC(unpermute_vec_kernel, 2, y, R, T, d, k, row_map, gate, shared, out, err);
        else MOE_DISPATCH_VEC(unpermute_vec_kernel, 4, y, R, T, d, k, row_map, gate, shared, out, err);
    } else {
        unpermute_scalar_kernel<<<grid, 256, 0, s>>>(y, in_bf16, R, T, d, k, row_map, gate, shared, out, out_bf16, err);
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
    if (vec) {
        const int nvec = d / 8;
        if (nvec <= 32) MOE_DISPATCH_VEC(unpermute_ec_vec_kernel, 1, y, R, T, d, tok_ptr, tok_row, ec_gate, out, err);
        else if (nvec <= 64) MOE_DISPATCH_VEC(unpermute_ec_vec_kernel, 2, y, R, T, d, tok_ptr, tok_row, ec_gate, out, err);
        else MOE_DISPATCH_VEC(unpermute_ec_vec_kernel, 4, y, R, T, d, tok_ptr, tok_row, ec_gate, out, err);
    } else {
        unpermute_ec_scalar_kernel<<<grid, 256, 0, s>>>(y, in_bf16, R, T, d, tok_ptr, tok_row, ec_gate, out, out_bf16, err);
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
