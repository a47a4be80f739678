// permute.cu - token_permutation on one device, and expert-choice dispatch.
//
// "How MegaDLMs Implements Mixture of Experts (MoE) Architectures",
// "MoELayer" step 1 and "Token Dispatching and Communication": token rows are
// regrouped so that each expert's tokens are contiguous.  "Expert
// Parallelism > Key Parameters", capacity_factor: an expert keeps at most
// `capacity` assignments; the rest are dropped.  "Expert Coupling in MoE
// Pretraining", Abstract: a dispatcher that ships a token to a given GPU at
// most one time - here the group-major layout, one row per (token, group).
//
// Plan (all int32, no atomics on the ordering path, so results are
// deterministic):
//   1. count:   per token block b and key (expert or group), how many slots
//               of the block carry the key  -> cnt[key][b]
//   2. scan:    per key, exclusive scan over blocks -> base[key][b], total
//   3. offsets: capacity clamp per expert, exclusive scan over keys,
//               dropped = sum(load - kept)
//   4. rank:    per block, the stable (token-order) rank of each slot among
//               the block's slots with the same key, plus base: the global
//               token-order rank.  Expert-major: row = offsets[e] + rank if
//               rank < capacity.  Group-major: kept flags first, then the
//               same count/scan/rank over the (token, group) head slots.
//   5. copy:    one token per warp, x[t] read once (16-byte vectors) and
//               written to each distinct row the token owns.
#include <mutex>

#include "common.cuh"

namespace moe {

constexpr int kTB = 256;       // tokens per block in the index kernels
constexpr int kIdxThreads = 256;

// Key of slot s.  mode 0: the expert.  mode 1: the group of the expert if
// the slot is the first kept slot of its token into that group, else -1.
__device__ __forceinline__ int slot_key(int mode, const int32_t* __restrict__ idx, const uint8_t* __restrict__ kept,
                                        const int32_t* __restrict__ goe, long long s, int k, int E, int nkeys,
                                        unsigned* err) {
    int e = idx[s];
    if (e < 0 || e >= E) { raise_error(err, kErrIndex); return -1; }
    if (mode == 0) return e;
    if (!kept[s]) return -1;
    int g = goe[e];
    if (g < 0 || g >= nkeys) { raise_error(err, kErrIndex); return -1; }
    long long t0 = (s / k) * k;
    for (long long q = t0; q < s; ++q) {
        int eq = idx[q];
        if (eq >= 0 && eq < E && kept[q] && goe[eq] == g) return -1;   // an earlier slot already owns the row
    }
    return g;
}

// 1. per-block histogram of keys, stored key-major: cnt[key * nblk + b]
__global__ void __launch_bounds__(kIdxThreads) perm_count_kernel(int mode, const int32_t* __restrict__ idx,
                                                                 const uint8_t* __restrict__ kept,
                                                                 const int32_t* __restrict__ goe, int T, int k, int E,
                                                                 int nkeys, int nblk, int32_t* __restrict__ cnt,
                                                                 unsigned* err) {
    extern __shared__ int hist[];
    for (int i = threadIdx.x; i < nkeys; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const long long s0 = (long long)blockIdx.x * kTB * k;
    const long long s1 = min((long long)(blockIdx.x + 1) * kTB, (long long)T) * k;
    for (long long s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        int key = slot_key(mode, idx, kept, goe, s, k, E, nkeys, err);
        if (key >= 0 && key < nkeys) atomicAdd(&hist[key], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nkeys; i += blockDim.x) cnt[(long long)i * nblk + blockIdx.x] = hist[i];
}

// 2. one CTA per key: exclusive scan over the blocks, total per key.
__global__ void __launch_bounds__(1024) perm_scan_blocks_kernel(const int32_t* __restrict__ cnt, int nblk,
                                                                int32_t* __restrict__ base, int32_t* __restrict__ total) {
    __shared__ int sh[32];
    const int key = blockIdx.x;
    const int32_t* c = cnt + (long long)key * nblk;
    int32_t* b = base + (long long)key * nblk;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int carry = 0;
    for (int i0 = 0; i0 < nblk; i0 += 1024) {
        int i = i0 + threadIdx.x;
        int v = i < nblk ? c[i] : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) sh[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int w = sh[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            sh[lane] = w;
        }
        __syncthreads();
        int ex = (wid ? sh[wid - 1] : 0) + x - v;
        if (i < nblk) b[i] = carry + ex;
        carry += sh[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) total[key] = carry;
}

// 3. capacity clamp (when counts != NULL), offsets over keys, dropped.
__global__ void __launch_bounds__(1024) perm_offsets_kernel(const int32_t* __restrict__ total, int nkeys,
                                                            long long cap, int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets, int32_t* __restrict__ dropped) {
    __shared__ int sh[32];
    __shared__ long long sdrop[32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int carry = 0;
    long long drop = 0;
    for (int i0 = 0; i0 < nkeys; i0 += 1024) {
        int i = i0 + threadIdx.x;
        int load = i < nkeys ? total[i] : 0;
        int kept = (int)min((long long)load, cap);
        if (i < nkeys && counts) counts[i] = kept;
        drop += load - kept;
        int v = kept, x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) sh[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int w = sh[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            sh[lane] = w;
        }
        __syncthreads();
        int ex = (wid ? sh[wid - 1] : 0) + x - v;
        if (i < nkeys && offsets) offsets[i] = carry + ex;
        carry += sh[31];
        __syncthreads();
    }
    drop = warp_sum(drop);
    if (lane == 0) sdrop[wid] = drop;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long d = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) d += sdrop[w];
        if (offsets) offsets[nkeys] = carry;
        if (dropped) *dropped = (int32_t)d;
    }
}

// 4. stable in-block ranks.  The block's slots are split into 8 contiguous
// runs, one per warp; a warp walks its run 32 slots at a time and ranks
// equal keys with __match_any_sync.  Per-warp, per-key counts are scanned
// across warps so that ranks follow slot order over the whole block.
// out_mode 0 (expert-major rows), 1 (kept flags only), 2 (group rows).
template <int OUT>
__global__ void __launch_bounds__(kIdxThreads) perm_rank_kernel(int mode, const int32_t* __restrict__ idx,
                                                                uint8_t* __restrict__ kept,
                                                                const int32_t* __restrict__ goe, int T, int k, int E,
                                                                int nkeys, int nblk, const int32_t* __restrict__ base,
                                                                long long cap, const int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ row_map, int32_t* __restrict__ row_token,
                                                                unsigned* err) {
    extern __shared__ int sm[];
    int* wcnt = sm;                              // [8][nkeys]: counts, then exclusive warp bases
    const int nw = kIdxThreads / 32;
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < nw * nkeys; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const long long s0 = (long long)blockIdx.x * kTB * k;
    const long long s1 = min((long long)(blockIdx.x + 1) * kTB, (long long)T) * k;
    const long long n = s1 - s0;
    const long long per = (n + nw - 1) / nw;
    const long long w0 = s0 + min(n, per * wid), w1 = s0 + min(n, per * (wid + 1));
    // pass 1: per-warp counts
    for (long long c = w0; c < w1; c += 32) {
        long long s = c + lane;
        int key = s < w1 ? slot_key(mode, idx, kept, goe, s, k, E, nkeys, err) : -1;
        unsigned act = __ballot_sync(0xffffffffu, key >= 0);
        unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && (peers & act & lanemask_lt()) == 0) wcnt[wid * nkeys + key] += __popc(peers & act);
        __syncwarp();
    }
    __syncthreads();
    for (int key = threadIdx.x; key < nkeys; key += blockDim.x) {
        int run = 0;
        for (int w = 0; w < nw; ++w) {
            int c = wcnt[w * nkeys + key];
            wcnt[w * nkeys + key] = run;
            run += c;
        }
    }
    __syncthreads();
    // pass 2: ranks
    for (long long c = w0; c < w1; c += 32) {
        long long s = c + lane;
        int key = s < w1 ? slot_key(mode, idx, kept, goe, s, k, E, nkeys, err) : -1;
        unsigned act = __ballot_sync(0xffffffffu, key >= 0);
        unsigned peers = __match_any_sync(0xffffffffu, key) & act;
        int rank = 0;
        if (key >= 0) rank = base[(long long)key * nblk + blockIdx.x] + wcnt[wid * nkeys + key] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (key >= 0 && (peers & lanemask_lt()) == 0) wcnt[wid * nkeys + key] += __popc(peers);
        __syncwarp();
        if (s < w1) {
            if (OUT == 0) {
                if (key >= 0 && rank < cap) {
                    int r = offsets[key] + rank;
                    row_map[s] = r;
                    row_token[r] = (int32_t)(s / k);
                } else {
                    row_map[s] = -1;
                }
            } else if (OUT == 1) {
                kept[s] = (key >= 0 && rank < cap) ? 1 : 0;
            } else {
                if (key >= 0) {
                    int r = offsets[key] + rank;
                    row_map[s] = r;
                    row_token[r] = (int32_t)(s / k);
                }
            }
        }
    }
}

// Group-major: kept slots that are not their group's head take the head's row.
__global__ void perm_group_fill_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ kept,
                                       const int32_t* __restrict__ goe, int T, int k, int E, int G,
                                       int32_t* __restrict__ row_map) {
    long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const long long s0 = t * k;
    for (int j = 0; j < k; ++j) {
        long long s = s0 + j;
        int e = idx[s];
        if (e < 0 || e >= E || !kept[s]) { row_map[s] = -1; continue; }
        int g = goe[e];
        if (g < 0 || g >= G) { row_map[s] = -1; continue; }
        for (int q = 0; q < j; ++q) {
            int eq = idx[s0 + q];
            if (eq >= 0 && eq < E && kept[s0 + q] && goe[eq] == g) { row_map[s] = row_map[s0 + q]; break; }
        }
    }
}

// 5. token-major row copy: warp per token, x[t] read once, written to each
// distinct destination row.  NV 16-byte vectors per lane are in flight.
template <int NV>
__global__ void __launch_bounds__(256) copy_rows_slots_kernel(const uint4* __restrict__ x, int T, int vec_per_row,
                                                              const int32_t* __restrict__ row_map, int k,
                                                              uint4* __restrict__ buffer) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = warp; t < T; t += nwarps) {
        // distinct destination rows of this token (lane j < k holds slot j)
        int r = -1;
        if (lane < k) {
            r = row_map[t * k + lane];
        }
        unsigned valid = __ballot_sync(0xffffffffu, r >= 0);
        // drop duplicates: keep a slot only if no lower slot has the same row
        unsigned uniq = 0;
        for (int j = 0; j < k; ++j) {
            int rj = __shfl_sync(0xffffffffu, r, j);
            if (!((valid >> j) & 1u)) continue;
            bool dup = false;
            for (int q = 0; q < j; ++q) dup |= (((uniq >> q) & 1u) && __shfl_sync(0xffffffffu, r, q) == rj);
            if (!dup) uniq |= 1u << j;
        }
        if (!uniq) continue;
        const uint4* src = x + t * (long long)vec_per_row;
        for (int v0 = 0; v0 < vec_per_row; v0 += 32 * NV) {
            uint4 buf[NV];
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                int v = v0 + u * 32 + lane;
                if (v < vec_per_row) buf[u] = ld_stream(src + v);
            }
            unsigned m = uniq;
            while (m) {
                int j = __ffs(m) - 1;
                m &= m - 1;
                int rj = __shfl_sync(0xffffffffu, r, j);
                uint4* dst = buffer + (long long)rj * vec_per_row;
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    int v = v0 + u * 32 + lane;
                    if (v < vec_per_row) st_stream(dst + v, buf[u]);
                }
            }
        }
    }
}

// Expert-choice dispatch: token CSR -> rows, each token read once.
template <int NV>
__global__ void __launch_bounds__(256) copy_rows_csr_kernel(const uint4* __restrict__ x, int T, int vec_per_row,
                                                            const int32_t* __restrict__ tok_ptr,
                                                            const int32_t* __restrict__ tok_row, int R,
                                                            uint4* __restrict__ buffer, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = warp; t < T; t += nwarps) {
        const int p0 = max(tok_ptr[t], 0), p1 = min(tok_ptr[t + 1], R);
        if (p1 <= p0) continue;
        const uint4* src = x + t * (long long)vec_per_row;
        for (int v0 = 0; v0 < vec_per_row; v0 += 32 * NV) {
            uint4 buf[NV];
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                int v = v0 + u * 32 + lane;
                if (v < vec_per_row) buf[u] = ld_stream(src + v);
            }
            for (int p = p0; p < p1; ++p) {
                const int r = tok_row[p];
                if (r < 0 || r >= R) { raise_error(err, kErrIndex); continue; }
                uint4* dst = buffer + (long long)r * vec_per_row;
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                    int v = v0 + u * 32 + lane;
                    if (v < vec_per_row) st_stream(dst + v, buf[u]);
                }
            }
        }
    }
}

int copy_grid(long long T) {
    long long warps = T;
    long long blocks = (warps + 7) / 8;
    long long cap = 148LL * 8;                    // 8 CTAs of 256 threads per SM
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace moe

using namespace moe;

namespace {
size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

struct PermWs {
    size_t cnt, base, total, kept, gcnt, gbase, gtotal, bytes;
};

PermWs perm_layout(int T, int k, int E, int G) {
    const int nblk = ceil_div(T, kTB) > 0 ? ceil_div(T, kTB) : 1;
    PermWs w;
    w.cnt = 0;
    w.base = w.cnt + al256(sizeof(int32_t) * (size_t)E * nblk);
    w.total = w.base + al256(sizeof(int32_t) * (size_t)E * nblk);
    w.kept = w.total + al256(sizeof(int32_t) * (size_t)E);
    size_t end = w.kept;
    if (G > 0) {
        w.gcnt = w.kept + al256((size_t)T * k);
        w.gbase = w.gcnt + al256(sizeof(int32_t) * (size_t)G * nblk);
        w.gtotal = w.gbase + al256(sizeof(int32_t) * (size_t)G * nblk);
        end = w.gtotal + al256(sizeof(int32_t) * (size_t)G);
    } else {
        w.gcnt = w.gbase = w.gtotal = end;
    }
    w.bytes = end;
    return w;
}

moe_status launch_copy_slots(const void* x, int T, int row_bytes, const int32_t* row_map, int k, void* buffer,
                             cudaStream_t s) {
    const int vpr = row_bytes / 16;
    const int grid = copy_grid(T);
    if (vpr <= 32) copy_rows_slots_kernel<1><<<grid, 256, 0, s>>>((const uint4*)x, T, vpr, row_map, k, (uint4*)buffer);
    else if (vpr <= 64) copy_rows_slots_kernel<2><<<grid, 256, 0, s>>>((const uint4*)x, T, vpr, row_map, k, (uint4*)buffer);
    else copy_rows_slots_kernel<4><<<grid, 256, 0, s>>>((const uint4*)x, T, vpr, row_map, k, (uint4*)buffer);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}
}  // namespace

extern "C" int64_t moe_capacity(double capacity_factor, int T, int k, int E) {
    if (capacity_factor <= 0.0 || E <= 0) return (int64_t)T * k;
    return (int64_t)ceil(capacity_factor * (double)T * (double)k / (double)E);
}

extern "C" int64_t moe_permute_max_rows(int T, int k, int E, double capacity_factor, int G) {
    if (T <= 0 || k <= 0 || E <= 0) return 0;
    if (G > 0) return (int64_t)T * (k < G ? k : G);
    int64_t cap = moe_capacity(capacity_factor, T, k, E);
    int64_t a = (int64_t)T * k, b = cap * E;
    return a < b ? a : b;
}

extern "C" size_t moe_permute_workspace_bytes(int T, int k, int E, int G) {
    if (T < 0 || k < 1 || E < 1 || G < 0) return 0;
    return perm_layout(T, k, E, G).bytes;
}

extern "C" moe_status moe_permute(const void* x, int dtype, int T, int d, const int32_t* expert_idx, int k, int E,
                                  double capacity_factor, const int32_t* group_of_expert, int G, void* buffer,
                                  int32_t* row_map, int32_t* row_token, int32_t* counts, int32_t* offsets,
                                  int32_t* dropped, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1 || k > E || d < 0) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (k > 32 || E > 1024) return MOE_ERR_SHAPE;
    if (group_of_expert && (G < 1 || G > 1024)) return (G < 1) ? MOE_ERR_ARG : MOE_ERR_SHAPE;
    if (!counts || !offsets || !dropped) return MOE_ERR_ARG;
    if (T == 0) {
        // nothing routed: zero counts, offsets, dropped
        cudaStream_t s0 = (cudaStream_t)stream;
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s0) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * ((group_of_expert ? G : E) + 1), s0) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaMemsetAsync(dropped, 0, sizeof(int32_t), s0) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!expert_idx || !row_map || !row_token) return MOE_ERR_ARG;
    if ((x == nullptr) != (buffer == nullptr)) return MOE_ERR_ARG;
    const int esz = dtype == MOE_BF16 ? 2 : 4;
    const long long row_bytes = (long long)d * esz;
    if (x && (row_bytes % 16 != 0 || ((uintptr_t)x & 15) || ((uintptr_t)buffer & 15))) return MOE_ERR_SHAPE;
    const int Gk = group_of_expert ? G : 0;
    PermWs L = perm_layout(T, k, E, Gk);
    if (!workspace || workspace_bytes < L.bytes || ((uintptr_t)workspace & 255)) return MOE_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const long long cap = moe_capacity(capacity_factor, T, k, E);
    const int nblk = ceil_div(T, kTB) > 0 ? ceil_div(T, kTB) : 1;
    char* ws = (char*)workspace;
    int32_t* cnt = (int32_t*)(ws + L.cnt);
    int32_t* base = (int32_t*)(ws + L.base);
    int32_t* total = (int32_t*)(ws + L.total);
    const int nw = kIdxThreads / 32;
    // expert pass: counts, scan, capacity
    perm_count_kernel<<<nblk, kIdxThreads, sizeof(int) * E, s>>>(0, expert_idx, nullptr, nullptr, T, k, E, E, nblk, cnt, err);
    MOE_LAUNCH_CHECK();
    perm_scan_blocks_kernel<<<E, 1024, 0, s>>>(cnt, nblk, base, total);
    MOE_LAUNCH_CHECK();
    const size_t rank_smem = sizeof(int) * (size_t)nw * (group_of_expert ? (E > G ? E : G) : E);
    if (rank_smem > 48 * 1024) {
        if (cudaFuncSetAttribute(perm_rank_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rank_smem) != cudaSuccess ||
            cudaFuncSetAttribute(perm_rank_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rank_smem) != cudaSuccess ||
            cudaFuncSetAttribute(perm_rank_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rank_smem) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (!group_of_expert) {
        perm_offsets_kernel<<<1, 1024, 0, s>>>(total, E, cap, counts, offsets, dropped);
        MOE_LAUNCH_CHECK();
        perm_rank_kernel<0><<<nblk, kIdxThreads, rank_smem, s>>>(0, expert_idx, nullptr, nullptr, T, k, E, E, nblk, base,
                                                                 cap, offsets, row_map, row_token, err);
        MOE_LAUNCH_CHECK();
    } else {
        uint8_t* kept = (uint8_t*)(ws + L.kept);
        int32_t* gcnt = (int32_t*)(ws + L.gcnt);
        int32_t* gbase = (int32_t*)(ws + L.gbase);
        int32_t* gtotal = (int32_t*)(ws + L.gtotal);
        perm_offsets_kernel<<<1, 1024, 0, s>>>(total, E, cap, counts, nullptr, dropped);
        MOE_LAUNCH_CHECK();
        perm_rank_kernel<1><<<nblk, kIdxThreads, rank_smem, s>>>(0, expert_idx, kept, nullptr, T, k, E, E, nblk, base,
                                                                 cap, nullptr, nullptr, nullptr, err);
        MOE_LAUNCH_CHECK();
        perm_count_kernel<<<nblk, kIdxThreads, sizeof(int) * G, s>>>(1, expert_idx, kept, group_of_expert, T, k, E, G,
                                                                       nblk, gcnt, err);
        MOE_LAUNCH_CHECK();
        perm_scan_blocks_kernel<<<G, 1024, 0, s>>>(gcnt, nblk, gbase, gtotal);
        MOE_LAUNCH_CHECK();
        perm_offsets_kernel<<<1, 1024, 0, s>>>(gtotal, G, (long long)T * k, nullptr, offsets, nullptr);
        MOE_LAUNCH_CHECK();
        perm_rank_kernel<2><<<nblk, kIdxThreads, rank_smem, s>>>(1, expert_idx, kept, group_of_expert, T, k, E, G, nblk,
                                                                 gbase, (long long)T * k, offsets, row_map, row_token, err);
        MOE_LAUNCH_CHECK();
        perm_group_fill_kernel<<<ceil_div(T, 256), 256, 0, s>>>(expert_idx, kept, group_of_expert, T, k, E, G, row_map);
        MOE_LAUNCH_CHECK();
    }
    if (x && d > 0) return launch_copy_slots(x, T, (int)row_bytes, row_map, k, buffer, s);
    return MOE_OK;
}

extern "C" moe_status moe_gather_rows(const void* x, int dtype, int T, int d, const int32_t* tok_ptr,
                                      const int32_t* tok_row, int R, void* buffer, moe_stream_t stream) {
    if (T < 0 || d < 0 || R < 0) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (T == 0 || d == 0) return MOE_OK;
    if (!x || !tok_ptr || !tok_row || !buffer) return MOE_ERR_ARG;
    const long long row_bytes = (long long)d * (dtype == MOE_BF16 ? 2 : 4);
    if (row_bytes % 16 || ((uintptr_t)x & 15) || ((uintptr_t)buffer & 15)) return MOE_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const int vpr = (int)(row_bytes / 16);
    const int grid = copy_grid(T);
    if (vpr <= 32) copy_rows_csr_kernel<1><<<grid, 256, 0, s>>>((const uint4*)x, T, vpr, tok_ptr, tok_row, R, (uint4*)buffer, err);
    else if (vpr <= 64) copy_rows_csr_kernel<2><<<grid, 256, 0, s>>>((const uint4*)x, T, vpr, tok_ptr, tok_row, R, (uint4*)buffer, err);
    else copy_rows_csr_kernel<4><<<grid, 256, 0, s>>>((const uint4*)x, T, vpr, tok_ptr, tok_row, R, (uint4*)buffer, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

// ------------------------------------------------ allocation-free variant
// For callers that may not allocate device memory at all: code running
// inside a host framework that owns every device byte and forbids
// allocation after start-up (an inference plugin's enqueue, a real-time
// serving loop with a pre-planned memory budget), or code that cannot
// afford cudaMalloc's implicit device synchronisation on its hot path.
// Such callers still pass their inputs and outputs; the permutation's
// scratch comes from this fixed array instead of a caller workspace.  Every
// GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_permute_noalloc_scratch[MOE_PERMUTE_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_scratch[64] = {nullptr};

// Device address of this device's scratch array.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
void* noalloc_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_scratch[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_scratch[dev] = p;
    }
    return g_noalloc_scratch[dev];
}
}  // namespace

extern "C" moe_status moe_permute_noalloc(const void* x, int dtype, int T, int d, const int32_t* expert_idx, int k,
                                          int E, double capacity_factor, const int32_t* group_of_expert, int G,
                                          void* buffer, int32_t* row_map, int32_t* row_token, int32_t* counts,
                                          int32_t* offsets, int32_t* dropped, moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1 || G < 0) return MOE_ERR_ARG;
    const size_t need = moe_permute_workspace_bytes(T, k, E, group_of_expert ? G : 0);
    if (need > (size_t)MOE_PERMUTE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
    void* scratch = noalloc_scratch_address();
    if (!scratch) return MOE_ERR_CUDA;
    // Nothing in the permutation's scratch needs to start at zero: every
    // count, base and flag it reads is written earlier in the same call, so
    // what a previous call left there is never used.
    return moe_permute(x, dtype, T, d, expert_idx, k, E, capacity_factor, group_of_expert, G, buffer, row_map,
                       row_token, counts, offsets, dropped, scratch, (size_t)MOE_PERMUTE_NOALLOC_SCRATCH_BYTES,
                       stream);
}
