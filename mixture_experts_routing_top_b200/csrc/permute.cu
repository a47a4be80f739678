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
//   1. count:   per token block b and expert, how many slots of the block
//               carry the expert -> cnt[e][b]
//   2. scan:    per expert, exclusive scan over blocks -> base[e][b], total
//   3. offsets: capacity clamp per expert, exclusive scan over experts,
//               dropped = sum(load - kept)
//      (1-3 run as one launch whose last CTA does the scans when experts x
//      blocks is small; as three launches otherwise)
//   4. rank:    per block, the stable (token-order) rank of each slot among
//               the block's slots with the same expert, plus base: the
//               global token-order rank; row = offsets[e] + rank if rank <
//               capacity.  Group-major instead: one kernel derives the kept
//               slots, each token's group heads and the per-block group
//               counts (its last CTA scanning them), one kernel ranks the
//               heads per group and gives every kept slot its head's row.
//   5. copy:    one token per warp, x[t] read once and written to each
//               distinct row the token owns - through the bulk-copy engine
//               (one bulk load into shared memory, one bulk store per row)
//               when the row fits a 32 KB slot, else in 16-byte vectors.
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {

constexpr int kTB = 256;       // tokens per block in the index kernels
constexpr int kIdxThreads = 256;

// 1. per-block histogram of experts, stored expert-major: cnt[e * nblk + b]
__global__ void __launch_bounds__(kIdxThreads) perm_count_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                                 int nblk, int tb, int32_t* __restrict__ cnt,
                                                                 unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int hist[];
    for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const long long s0 = (long long)blockIdx.x * tb * k;
    const long long s1 = min((long long)(blockIdx.x + 1) * tb, (long long)T) * k;
    for (long long s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        const int e = idx[s];
        if (e < 0 || e >= E) { raise_error(err, kErrIndex); continue; }
        atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[(long long)i * nblk + blockIdx.x] = hist[i];
}

// 2. one CTA per key: exclusive scan over the blocks, total per key.
__global__ void __launch_bounds__(1024) perm_scan_blocks_kernel(const int32_t* __restrict__ cnt, int nblk,
                                                                int32_t* __restrict__ base, int32_t* __restrict__ total) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
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
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
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

// Stable in-block ranks: the block's slots [s0, s1) are split into one
// contiguous run per warp; a warp walks its run 32 slots at a time and ranks
// equal keys with __match_any_sync; per-warp, per-key counts are scanned
// across warps so that ranks follow slot order over the whole block.
// rank = base_s[key] (the count of the key in earlier blocks) + position
// among this block's earlier slots with the same key.  key_of(s) < 0 skips a
// slot.  Called by the whole block.
template <typename KeyOf, typename OnRank>
__device__ __forceinline__ void block_stable_ranks(long long s0, long long s1, int nkeys, const int* base_s, int* wcnt,
                                                   KeyOf key_of, OnRank on_rank) {
    const int nw = blockDim.x >> 5;
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < nw * nkeys; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const long long n = s1 - s0;
    const long long per = (n + nw - 1) / nw;
    const long long w0 = s0 + min(n, per * wid), w1 = s0 + min(n, per * (wid + 1));
    for (long long c = w0; c < w1; c += 32) {
        const long long s = c + lane;
        const int key = s < w1 ? key_of(s) : -1;
        const unsigned act = __ballot_sync(0xffffffffu, key >= 0);
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && (peers & act & lanemask_lt()) == 0) wcnt[wid * nkeys + key] += __popc(peers & act);
        __syncwarp();
    }
    __syncthreads();
    for (int key = threadIdx.x; key < nkeys; key += blockDim.x) {
        int run = 0;
        for (int w = 0; w < nw; ++w) {
            const int c = wcnt[w * nkeys + key];
            wcnt[w * nkeys + key] = run;
            run += c;
        }
    }
    __syncthreads();
    for (long long c = w0; c < w1; c += 32) {
        const long long s = c + lane;
        const int key = s < w1 ? key_of(s) : -1;
        const unsigned act = __ballot_sync(0xffffffffu, key >= 0);
        const unsigned peers = __match_any_sync(0xffffffffu, key) & act;
        int rank = 0;
        if (key >= 0) rank = base_s[key] + wcnt[wid * nkeys + key] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (key >= 0 && (peers & lanemask_lt()) == 0) wcnt[wid * nkeys + key] += __popc(peers);
        __syncwarp();
        if (s < w1) on_rank(s, key, rank);
    }
}

// Each block's view of the scans, into shared memory: base_s[key] = the
// key's count in the blocks before this one; off_s[key] = exclusive scan over
// keys of the clamped totals min(total, cap).  `fused`: computed here from
// cnt[key][block] (for small keys x blocks, one pass over cnt per block);
// otherwise read from the outputs of the scan kernels (base[key][block],
// offsets).  With `fused`, block 0 also writes counts, offsets
// ([nkeys] = rows) and dropped, each when non-null.
// `blk` is the index-block whose view is taken (the calling block's own,
// unless several consumer blocks share one index block); `writer` marks the
// one block that writes counts, offsets and dropped.
__device__ void block_scan_prologue(bool fused, const int32_t* __restrict__ cnt, const int32_t* __restrict__ base,
                                    const int32_t* offsets_in, int nkeys, int nblk, long long cap,
                                    int* base_s, int* off_s, int32_t* __restrict__ counts,
                                    int32_t* offsets_out, int32_t* __restrict__ dropped, int blk, bool writer) {
    __shared__ int wsum[32];
    __shared__ long long wdrop[32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (!fused) {
        for (int key = threadIdx.x; key < nkeys; key += blockDim.x) {
            base_s[key] = base[(long long)key * nblk + blk];
            off_s[key] = offsets_in ? offsets_in[key] : 0;
        }
        __syncthreads();
        return;
    }
    // every thread reads its share of the whole keys x blocks count matrix
    // (consecutive threads on consecutive blocks: coalesced, all loads
    // independent) and adds it into the keys' totals and bases in shared
    // memory; one thread per key then applies the capacity
    for (int key = threadIdx.x; key < nkeys; key += blockDim.x) { base_s[key] = 0; off_s[key] = 0; }
    __syncthreads();
    const int n = nkeys * nblk;
#pragma unroll 4
    for (int f = threadIdx.x; f < n; f += blockDim.x) {
        const int v = cnt[f];
        if (v) {
            const int key = f / nblk, i = f - key * nblk;
            atomicAdd(&off_s[key], v);          // total, clamped and scanned below
            if (i < blk) atomicAdd(&base_s[key], v);
        }
    }
    __syncthreads();
    long long drop = 0;
    for (int key = threadIdx.x; key < nkeys; key += blockDim.x) {
        const int tot = off_s[key];
        const int kept = (int)min((long long)tot, cap);
        off_s[key] = kept;                      // scanned below
        if (writer && counts) counts[key] = kept;
        drop += tot - kept;
    }
    drop = warp_sum(drop);
    if (lane == 0) wdrop[wid] = drop;
    __syncthreads();
    int carry = 0;
    for (int k0 = 0; k0 < nkeys; k0 += blockDim.x) {
        const int key = k0 + threadIdx.x;
        const int v = key < nkeys ? off_s[key] : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        int wb = 0, tot = 0;
        for (int w = 0; w < nw; ++w) {
            if (w < wid) wb += wsum[w];
            tot += wsum[w];
        }
        if (key < nkeys) {
            off_s[key] = carry + wb + x - v;
            if (writer && offsets_out) offsets_out[key] = off_s[key];
        }
        carry += tot;
        __syncthreads();
    }
    if (writer && threadIdx.x == 0) {
        if (offsets_out) offsets_out[nkeys] = carry;
        if (dropped) {
            long long d = 0;
            for (int w = 0; w < nw; ++w) d += wdrop[w];
            *dropped = (int32_t)d;
        }
    }
    __syncthreads();
}

// Group-major, part 1 (one CTA per tb tokens): expert ranks -> kept slots;
// then, one thread per token, each kept slot's group, whether it is the
// first kept slot of its token in that group (the row's "head"), and the
// per-block head count of every group.  code[s]: group id for a head,
// -2 - j for a kept slot whose head is slot j of the same token, -1 for a
// dropped slot.  With a capacity of at least T k no slot can be dropped
// (`nodrop`): every valid slot is kept, the expert ranks are not needed, and
// the count matrix is read only for counts (each expert's total, every block
// summing the rows of its share of the experts) and dropped (zero).
__global__ void __launch_bounds__(kIdxThreads) perm_group_heads_kernel(
    const int32_t* __restrict__ idx, const int32_t* __restrict__ goe, int T, int k, int E, int G, int nblk, int tb, int fused,
    const int32_t* __restrict__ ecnt, const int32_t* __restrict__ ebase, long long cap, int nodrop,
    int32_t* __restrict__ counts, int32_t* __restrict__ dropped, int16_t* __restrict__ code, int32_t* __restrict__ gcnt,
    unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int sm[];
    int* wcnt = sm;                                          // [8][E]
    int* base_s = wcnt + (kIdxThreads / 32) * E;             // [E]
    int* off_s = base_s + E;                                 // [E]
    int* ghist = off_s + E;                                  // [G]
    int* goe_s = ghist + G;                                  // [E]
    int* keys_s = goe_s + E;                                 // [tb * k]
    uint8_t* kept_s = reinterpret_cast<uint8_t*>(keys_s + tb * k); // [tb * k]
    const long long s0 = (long long)blockIdx.x * tb * k;
    const long long s1 = min((long long)(blockIdx.x + 1) * tb, (long long)T) * k;
    for (int i = threadIdx.x; i < G; i += blockDim.x) ghist[i] = 0;
    // the block's experts and the group map into shared memory at once
    for (long long sl = s0 + threadIdx.x; sl < s1; sl += blockDim.x) keys_s[sl - s0] = idx[sl];
    for (int e = threadIdx.x; e < E; e += blockDim.x) goe_s[e] = goe[e];
    if (nodrop) {
        if (fused) {
            // nothing drops, so each expert's count is its total over the
            // blocks: every block sums the rows of its share of the experts
            // (a warp per row), so that no one block reads the whole matrix
            const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
            const int k0 = (int)((long long)E * blockIdx.x / gridDim.x);
            const int k1 = (int)((long long)E * (blockIdx.x + 1) / gridDim.x);
            for (int key = k0 + wid; key < k1; key += nw) {
                int tot = 0;
                for (int i = lane; i < nblk; i += 32) tot += ecnt[(long long)key * nblk + i];
                tot = warp_sum(tot);
                if (lane == 0) counts[key] = tot;
            }
            if (blockIdx.x == 0 && threadIdx.x == 0) *dropped = 0;
        } else if (blockIdx.x == 0) {
            block_scan_prologue(fused, ecnt, ebase, nullptr, E, nblk, cap, base_s, off_s, counts, nullptr, dropped, 0,
                                true);
        }
        __syncthreads();
        for (long long sl = s0 + threadIdx.x; sl < s1; sl += blockDim.x) {
            const int e = keys_s[sl - s0];
            const bool ok = e >= 0 && e < E;
            if (!ok) raise_error(err, kErrIndex);
            kept_s[sl - s0] = ok ? 1 : 0;
        }
    } else {
        block_scan_prologue(fused, ecnt, ebase, nullptr, E, nblk, cap, base_s, off_s, counts, nullptr, dropped,
                            (int)blockIdx.x, blockIdx.x == 0);
        block_stable_ranks(
            s0, s1, E, base_s, wcnt,
            [&](long long s) -> int {
                const int e = keys_s[s - s0];
                if (e < 0 || e >= E) { raise_error(err, kErrIndex); return -1; }
                return e;
            },
            [&](long long s, int key, int rank) { kept_s[s - s0] = (key >= 0 && rank < cap) ? 1 : 0; });
    }
    __syncthreads();
    const long long t0 = (long long)blockIdx.x * tb;
    const int ntok = (int)((s1 - s0) / k);
    for (int tl = threadIdx.x; tl < ntok; tl += blockDim.x) {
        const long long sb = (t0 + tl) * k;
        for (int j = 0; j < k; ++j) {
            const long long s = sb + j;
            int c = -1;
            if (kept_s[s - s0]) {
                const int g = goe_s[keys_s[s - s0]];
                if (g < 0 || g >= G) {
                    raise_error(err, kErrIndex);
                } else {
                    int jh = -1;
                    for (int q = 0; q < j; ++q)
                        if (kept_s[sb + q - s0] && goe_s[keys_s[sb + q - s0]] == g) { jh = q; break; }
                    if (jh < 0) { c = g; atomicAdd(&ghist[g], 1); }
                    else c = -2 - jh;
                }
            }
            code[s] = (int16_t)c;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G; i += blockDim.x) gcnt[(long long)i * nblk + blockIdx.x] = ghist[i];
}

// Group-major, part 2: head slots get stable per-group ranks (token order)
// and their rows; every other kept slot takes its head's row.
__global__ void __launch_bounds__(kIdxThreads) perm_group_rows_kernel(
    const int16_t* __restrict__ code, int T, int k, int G, int nblk, int tb, int fused, const int32_t* __restrict__ gcnt,
    const int32_t* __restrict__ gbase, const int32_t* __restrict__ goffsets_in, int32_t* __restrict__ offsets,
    int32_t* __restrict__ row_map, int32_t* __restrict__ row_token) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int sm[];
    int* wcnt = sm;                                          // [8][G]
    int* base_s = wcnt + (kIdxThreads / 32) * G;             // [G]
    int* off_s = base_s + G;                                 // [G]
    int* rows_s = off_s + G;                                 // [tb * k]
    int* codes_s = rows_s + tb * k;                          // [tb * k]
    const long long s0 = (long long)blockIdx.x * tb * k;
    const long long s1 = min((long long)(blockIdx.x + 1) * tb, (long long)T) * k;
    for (long long sl = s0 + threadIdx.x; sl < s1; sl += blockDim.x) codes_s[sl - s0] = code[sl];
    block_scan_prologue(fused, gcnt, gbase, goffsets_in, G, nblk, (long long)T * k, base_s, off_s, nullptr, offsets,
                        nullptr, (int)blockIdx.x, blockIdx.x == 0);
    block_stable_ranks(
        s0, s1, G, base_s, wcnt, [&](long long s) -> int { return codes_s[s - s0]; },
        [&](long long s, int key, int rank) {
            int r = -1;
            if (key >= 0) {
                r = off_s[key] + rank;
                row_token[r] = (int32_t)(s / k);
            }
            rows_s[s - s0] = r;
        });
    __syncthreads();
    for (long long s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        const int c = codes_s[s - s0];
        int r = -1;
        if (c >= 0) r = rows_s[s - s0];
        else if (c <= -2) r = rows_s[(s / k) * k + (-2 - c) - s0];
        row_map[s] = r;
    }
}

// 4. expert-major rows: stable ranks per expert (token order); a slot is
// kept if its rank is below the capacity, at row offsets[e] + rank.
__global__ void __launch_bounds__(kIdxThreads) perm_rank_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                                int nblk, int tb, int fused, const int32_t* __restrict__ cnt,
                                                                const int32_t* __restrict__ base, long long cap,
                                                                int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ dropped,
                                                                int32_t* __restrict__ row_map,
                                                                int32_t* __restrict__ row_token, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int sm[];
    int* wcnt = sm;                              // [8][E]
    int* base_s = wcnt + (kIdxThreads / 32) * E; // [E]
    int* off_s = base_s + E;                     // [E]
    int* keys_s = off_s + E;                     // [tb * k]
    const long long s0 = (long long)blockIdx.x * tb * k;
    const long long s1 = min((long long)(blockIdx.x + 1) * tb, (long long)T) * k;
    // the block's experts into shared memory at once (coalesced, all loads in
    // flight), so the ranking passes do not wait on a global load per step
    for (long long sl = s0 + threadIdx.x; sl < s1; sl += blockDim.x) keys_s[sl - s0] = idx[sl];
    block_scan_prologue(fused, cnt, base, offsets, E, nblk, cap, base_s, off_s, counts, offsets, dropped,
                        (int)blockIdx.x, blockIdx.x == 0);
    block_stable_ranks(
        s0, s1, E, base_s, wcnt,
        [&](long long s) -> int {
            const int e = keys_s[s - s0];
            if (e < 0 || e >= E) { raise_error(err, kErrIndex); return -1; }
            return e;
        },
        [&](long long s, int key, int rank) {
            if (key >= 0 && rank < cap) {
                const int r = off_s[key] + rank;
                row_map[s] = r;
                row_token[r] = (int32_t)(s / k);
            } else {
                row_map[s] = -1;
            }
        });
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
    pdl_wait();                                // row_map comes from the kernel before
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

// Bulk-copy variant: a warp takes one token at a time and lane 0 moves the
// row with the bulk-copy engine - one cp.async.bulk load of x[t] into the
// warp's shared-memory slot, then one cp.async.bulk store per distinct
// destination row - so a 4-16 KB row costs a handful of instructions instead
// of a 16-byte load and k 16-byte stores per lane per vector, which at these
// row sizes throttle the load/store queues.  Many warps per SM keep rows in
// flight.  No multicast.  The wait for the load is bounded; on expiry the
// warp records MOE_ERR_TIMEOUT and stops.
constexpr int kBulkWarps = 4;

__global__ void __launch_bounds__(32 * kBulkWarps) copy_rows_bulk_kernel(const uint8_t* __restrict__ x, int T,
                                                                         int row_bytes, int slot_bytes,
                                                                         const int32_t* __restrict__ row_map, int k,
                                                                         uint8_t* __restrict__ buffer, unsigned* err) {
    extern __shared__ __align__(128) uint8_t bulk_slots[];
    __shared__ __align__(8) uint64_t bars[kBulkWarps];
    __shared__ int no_abort;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t slot = tc::smem_u32(bulk_slots + (size_t)wid * slot_bytes);
    const uint32_t bar = tc::smem_u32(&bars[wid]);
    if (threadIdx.x == 0) no_abort = 0;
    if (lane == 0) tc::mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    pdl_wait();                                // row_map comes from the kernel before
    uint32_t phase = 0;
    const long long nworkers = (long long)gridDim.x * kBulkWarps;
    for (long long t = (long long)blockIdx.x * kBulkWarps + wid; t < T; t += nworkers) {
        int r = -1;
        if (lane < k) r = row_map[t * k + lane];
        const unsigned valid = __ballot_sync(0xffffffffu, r >= 0);
        unsigned uniq = 0;                     // first slot of every distinct destination row
        for (int j = 0; j < k; ++j) {
            const int rj = __shfl_sync(0xffffffffu, r, j);
            if (!((valid >> j) & 1u)) continue;
            bool dup = false;
            for (int q = 0; q < j; ++q) dup |= (((uniq >> q) & 1u) && __shfl_sync(0xffffffffu, r, q) == rj);
            if (!dup) uniq |= 1u << j;
        }
        if (!uniq) continue;
        int ok = 1;
        if (lane == 0) {
            tc::mbar_expect_tx(bar, (uint32_t)row_bytes);
            tc::bulk_load(slot, x + t * (long long)row_bytes, (uint32_t)row_bytes, bar);
            ok = tc::mbar_wait(bar, phase, &no_abort) ? 1 : 0;
        }
        phase ^= 1u;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) {
                raise_error(err, kErrTimeout);
                tc::mbar_wait(bar, phase ^ 1u, &no_abort);   // the load may still land: let it, once more bounded
            }
            break;
        }
        unsigned m = uniq;
        while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            const int rj = __shfl_sync(0xffffffffu, r, j);
            if (lane == 0) tc::bulk_store(buffer + (long long)rj * row_bytes, slot, (uint32_t)row_bytes);
        }
        if (lane == 0) {
            tc::bulk_commit();
            tc::bulk_wait_read0();             // the slot may be reloaded
        }
        __syncwarp();
    }
    if (lane == 0) tc::bulk_wait0();
}

// Expert-choice dispatch through the bulk-copy engine: the same scheme as
// copy_rows_bulk_kernel with the destinations taken from the token CSR
// (rows outside [0, R) are skipped and reported).
__global__ void __launch_bounds__(32 * kBulkWarps) copy_rows_csr_bulk_kernel(const uint8_t* __restrict__ x, int T,
                                                                             int row_bytes, int slot_bytes,
                                                                             const int32_t* __restrict__ tok_ptr,
                                                                             const int32_t* __restrict__ tok_row, int R,
                                                                             uint8_t* __restrict__ buffer,
                                                                             unsigned* err) {
    extern __shared__ __align__(128) uint8_t bulk_slots[];
    __shared__ __align__(8) uint64_t bars[kBulkWarps];
    __shared__ int no_abort;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t slot = tc::smem_u32(bulk_slots + (size_t)wid * slot_bytes);
    const uint32_t bar = tc::smem_u32(&bars[wid]);
    if (threadIdx.x == 0) no_abort = 0;
    if (lane == 0) tc::mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    uint32_t phase = 0;
    const long long nworkers = (long long)gridDim.x * kBulkWarps;
    if (lane == 0) {
        for (long long t = (long long)blockIdx.x * kBulkWarps + wid; t < T; t += nworkers) {
            const int p0 = max(tok_ptr[t], 0), p1 = min(tok_ptr[t + 1], R);
            if (p1 <= p0) continue;
            tc::mbar_expect_tx(bar, (uint32_t)row_bytes);
            tc::bulk_load(slot, x + t * (long long)row_bytes, (uint32_t)row_bytes, bar);
            const bool ok = tc::mbar_wait(bar, phase, &no_abort);
            phase ^= 1u;
            if (!ok) {
                raise_error(err, kErrTimeout);
                tc::mbar_wait(bar, phase ^ 1u, &no_abort);
                break;
            }
            for (int p = p0; p < p1; ++p) {
                const int r = tok_row[p];
                if (r < 0 || r >= R) { raise_error(err, kErrIndex); continue; }
                tc::bulk_store(buffer + (long long)r * row_bytes, slot, (uint32_t)row_bytes);
            }
            tc::bulk_commit();
            tc::bulk_wait_read0();
        }
        tc::bulk_wait0();
    }
}

// ---------------------------------------------- expert-major, two launches
// When the rows are copied in the same call, the expert-major permutation
// runs as two kernels instead of count, rank and copy:
//
//   perm_count_cluster_kernel: one cluster of kCcCtas CTAs.  The tokens are
//     cut into chunks of kRcTok; each CTA counts its run of chunks per
//     expert in shared memory and scans the counts per expert over its
//     chunks; the CTAs then read each other's per-expert totals through
//     distributed shared memory, so every CTA knows how many slots of each
//     expert precede its first chunk.  It writes chunk_base[c][e] = the
//     number of slots with expert e before chunk c (token order), and its
//     CTA 0 writes the capacity-clamped counts, the row offsets and dropped.
//   perm_rank_copy_kernel: one CTA per chunk, one warp per token.  Each warp
//     starts the bulk load of its token's row before anything else; the CTA
//     then ranks the chunk's slots (chunk_base + the stable rank inside the
//     chunk), writes row_map and row_token, and each warp stores its row to
//     the token's kept rows.
//
// A chunk's ranking work is small and overlaps its own row loads, and the
// CTAs are short (one row per warp), so no CTA waits for a separate ranking
// kernel before moving bytes and the last wave leaves no long tail.
constexpr int kRcTok = 8;                  // tokens per chunk = warps per rank-and-copy CTA
constexpr int kCcCtas = 8;                 // CTAs of the counting cluster (portable size)
constexpr int kCcThreads = 1024;
constexpr long long kCcMaxInts = 36 * 1024;   // chunk x expert counters per counting CTA

// Exclusive scan of n ints in shared memory, in place, by the whole CTA
// (each thread scans a run of ceil(n / blockDim) elements, then the runs'
// sums are scanned across the CTA).  Returns the total.  `wsum` holds 32.
__device__ int block_exclusive_scan(int* a, int n, int* wsum) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int m = (n + blockDim.x - 1) / blockDim.x;
    const int b0 = min(n, (int)threadIdx.x * m), b1 = min(n, b0 + m);
    int run = 0;
    for (int i = b0; i < b1; ++i) run += a[i];
    int x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < nw; ++w) {
        const int v = wsum[w];
        if (w < wid) before += v;
        all += v;
    }
    int acc = before + x - run;
    for (int i = b0; i < b1; ++i) {
        const int v = a[i];
        a[i] = acc;
        acc += v;
    }
    __syncthreads();
    return all;
}

__global__ void __cluster_dims__(kCcCtas, 1, 1) __launch_bounds__(kCcThreads, 1)
perm_count_cluster_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int nchunk, int cpc, long long cap,
                          int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts,
                          int32_t* __restrict__ offsets, int32_t* __restrict__ dropped, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int cc_sm[];
    const int r = (int)tc::cluster_rank();
    const int c0 = min(r * cpc, nchunk);
    const int c1 = min(c0 + cpc, nchunk);
    const int ncc = c1 - c0;
    // row stride of hist: the same in every CTA, so that tot[] sits at the
    // same offset in each (the cluster reads it there); the zero entries past
    // ncc end each row for the scan below
    const int ld = cpc + 1;
    int* hist = cc_sm;                         // [E][ld]: counts per expert and chunk, then scanned
    int* tot = hist + (size_t)E * ld;          // [E] this CTA's totals, read by the whole cluster
    int* pre = tot + E;                        // [E] slots of each expert in the lower-ranked CTAs' chunks
    int* kept_s = pre + E;                     // [E] capacity-clamped totals
    __shared__ int wsum[32];
    __shared__ long long wdrop[32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int i = threadIdx.x; i < E * ld; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int cs = kRcTok * k;                 // slots per chunk
    const long long s0 = (long long)c0 * cs;
    const long long s1 = min((long long)c1 * kRcTok, (long long)T) * k;
    {
        // slot s0 + j lies in chunk j / cs of this CTA: the chunk index and the
        // offset in it stepped along with j (no division per slot), four
        // slots' expert ids loaded before any is counted
        const int n = (int)(s1 - s0);
        const int dq = (int)blockDim.x / cs, dr = (int)blockDim.x - dq * cs;
        int q = (int)threadIdx.x / cs, rm = (int)threadIdx.x - q * cs;
        for (int j0 = threadIdx.x; j0 < n; j0 += 4 * blockDim.x) {
            int ev[4], qv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * blockDim.x;
                ev[u] = j < n ? idx[s0 + j] : -1;
                qv[u] = q;
                q += dq;
                rm += dr;
                if (rm >= cs) { rm -= cs; ++q; }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * blockDim.x;
                if (j >= n) break;
                if ((unsigned)ev[u] >= (unsigned)E) { raise_error(err, kErrIndex); continue; }
                atomicAdd(&hist[ev[u] * ld + qv[u]], 1);
            }
        }
    }
    __syncthreads();
    // one flat scan over the expert-major rows (each row ends with a zero
    // pad): entry (e, c) then counts the slots of experts < e, plus those of
    // expert e in chunks before c; the row's first entry is subtracted below
    block_exclusive_scan(hist, E * ld, wsum);
    for (int e = threadIdx.x; e < E; e += blockDim.x) tot[e] = hist[e * ld + ld - 1] - hist[e * ld];
    tc::cluster_sync();                        // every CTA's totals are complete and visible
    const uint32_t tot_addr = tc::smem_u32(tot);
    uint32_t peer[kCcCtas];
#pragma unroll
    for (int q = 0; q < kCcCtas; ++q) peer[q] = tc::map_to_rank(tot_addr, (uint32_t)q);
    long long drop = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int before = 0, all = 0;
#pragma unroll
        for (int q = 0; q < kCcCtas; ++q) {
            const int v = (int)tc::ld_shared_cluster_u32(peer[q] + 4u * (uint32_t)e);
            all += v;
            if (q < r) before += v;
        }
        pre[e] = before - hist[e * ld];        // the row's start, subtracted once here
        const int kept = (int)min((long long)all, cap);
        kept_s[e] = kept;
        if (r == 0) counts[e] = kept;
        drop += all - kept;
    }
    drop = warp_sum(drop);
    if (lane == 0) wdrop[wid] = drop;
    tc::cluster_sync();                        // the reads of the others' tot[] are performed before any CTA exits
    __syncthreads();                           // pre[], kept_s[] and wdrop[] are complete
    if (r == 0) {
        const int rows = block_exclusive_scan(kept_s, E, wsum);
        for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = kept_s[e];
        if (threadIdx.x == 0) {
            offsets[E] = rows;
            long long d = 0;
            for (int w = 0; w < nw; ++w) d += wdrop[w];
            *dropped = (int32_t)d;
        }
    }
    __syncthreads();
    {
        // element i = c E + e, its chunk and expert stepped along with i
        const int dc = (int)blockDim.x / E, de = (int)blockDim.x - dc * E;
        int c = (int)threadIdx.x / E, e = (int)threadIdx.x - c * E;
        for (int i = threadIdx.x; i < ncc * E; i += blockDim.x) {
            chunk_base[(long long)c0 * E + i] = hist[e * ld + c] + pre[e];
            c += dc;
            e += de;
            if (e >= E) { e -= E; ++c; }
        }
    }
}

__global__ void __launch_bounds__(32 * kRcTok) perm_rank_copy_kernel(
    const uint8_t* __restrict__ x, int T, int row_bytes, int slot_bytes, const int32_t* __restrict__ idx, int k, int E,
    const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets, long long cap,
    int32_t* __restrict__ row_map, int32_t* __restrict__ row_token, uint8_t* __restrict__ buffer, unsigned* err) {
    extern __shared__ __align__(128) uint8_t rc_smem[];
    __shared__ __align__(8) uint64_t bars[kRcTok];
    __shared__ int no_abort;
    int* base_s = (int*)(rc_smem + (size_t)kRcTok * slot_bytes);   // [E]
    int* off_s = base_s + E;                   // [E]
    int* wcnt = off_s + E;                     // [kRcTok][E]
    int* keys_s = wcnt + kRcTok * E;           // [kRcTok * k]
    int* rows_s = keys_s + kRcTok * k;         // [kRcTok * k]
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t slot = tc::smem_u32(rc_smem + (size_t)wid * slot_bytes);
    const uint32_t bar = tc::smem_u32(&bars[wid]);
    if (threadIdx.x == 0) no_abort = 0;
    if (lane == 0) tc::mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    pdl_wait();                                // chunk_base, offsets come from the kernel before
    const long long t0 = (long long)blockIdx.x * kRcTok;
    const int nt = (int)min((long long)kRcTok, (long long)T - t0);
    const bool mine = wid < nt;                // this warp's token exists
    if (lane == 0 && mine) {
        tc::mbar_expect_tx(bar, (uint32_t)row_bytes);
        tc::bulk_load(slot, x + (t0 + wid) * (long long)row_bytes, (uint32_t)row_bytes, bar);
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        base_s[e] = chunk_base[(long long)blockIdx.x * E + e];
        off_s[e] = offsets[e];
    }
    const long long s0 = t0 * k, s1 = (t0 + nt) * k;
    for (long long s = s0 + threadIdx.x; s < s1; s += blockDim.x) keys_s[s - s0] = idx[s];
    __syncthreads();
    block_stable_ranks(
        s0, s1, E, base_s, wcnt,
        [&](long long s) -> int {
            const int e = keys_s[s - s0];
            if ((unsigned)e >= (unsigned)E) { raise_error(err, kErrIndex); return -1; }
            return e;
        },
        [&](long long s, int key, int rank) {
            int r = -1;
            if (key >= 0 && rank < cap) {
                r = off_s[key] + rank;
                row_token[r] = (int32_t)(s / k);
            }
            row_map[s] = r;
            rows_s[s - s0] = r;
        });
    __syncthreads();
    if (!mine) return;
    const int rr = lane < k ? rows_s[wid * k + lane] : -1;
    const unsigned kept = __ballot_sync(0xffffffffu, rr >= 0);
    int ok = 1;
    if (lane == 0) ok = tc::mbar_wait(bar, 0, &no_abort) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) {
            raise_error(err, kErrTimeout);
            tc::mbar_wait(bar, 0, &no_abort);  // the load may still land: let it, once more bounded
        }
        return;
    }
    unsigned m = kept;
    while (m) {
        const int q = __ffs(m) - 1;
        m &= m - 1;
        const int rq = __shfl_sync(0xffffffffu, rr, q);
        if (lane == 0) tc::bulk_store(buffer + (long long)rq * row_bytes, slot, (uint32_t)row_bytes);
    }
    if (lane == 0 && kept) {
        tc::bulk_commit();
        tc::bulk_wait_read0();                 // the slot is read before the CTA's shared memory goes
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
    size_t cnt, base, total, code, gcnt, gbase, gtotal, cbase, bytes;
};

// Chunks per counting CTA of the two-launch expert-major path, 0 when the
// chunk x expert counters do not fit one CTA's shared memory.
int rc_chunks_per_cta(int T, int E) {
    const long long nchunk = ((long long)T + kRcTok - 1) / kRcTok;
    const long long cpc = (nchunk + kCcCtas - 1) / kCcCtas;
    if (cpc < 1 || (cpc + 1) * E > kCcMaxInts) return 0;
    return (int)cpc;
}

constexpr int kRcMaxSlot = 20 * 1024;      // row bytes (rounded to 128) the rank-and-copy CTA stages

constexpr long long kFuseLimit = 16384;   // keys x blocks each consumer block scans itself

// Tokens per block of the index kernels.  Smaller blocks (more CTAs) were
// measured slower: every block's scan prologue then reads more block counts
// (keys x blocks grows with the block count).
int perm_tokens_per_block(int) { return kTB; }

PermWs perm_layout(int T, int k, int E, int G) {
    const int tb = perm_tokens_per_block(T);
    const int nblk = ceil_div(T, tb) > 0 ? ceil_div(T, tb) : 1;
    PermWs w;
    w.cnt = 0;
    w.base = w.cnt + al256(sizeof(int32_t) * (size_t)E * nblk);
    w.total = w.base + al256(sizeof(int32_t) * (size_t)E * nblk);
    size_t end = w.total + al256(sizeof(int32_t) * (size_t)E);
    if (G > 0) {
        w.code = end;
        w.gcnt = w.code + al256(sizeof(int16_t) * (size_t)T * k);
        w.gbase = w.gcnt + al256(sizeof(int32_t) * (size_t)G * nblk);
        w.gtotal = w.gbase + al256(sizeof(int32_t) * (size_t)G * nblk);
        end = w.gtotal + al256(sizeof(int32_t) * (size_t)G);
    } else {
        w.code = w.gcnt = w.gbase = w.gtotal = end;
    }
    w.cbase = end;
    if (G == 0 && rc_chunks_per_cta(T, E) > 0)
        end = w.cbase + al256(sizeof(int32_t) * (size_t)ceil_div(T, kRcTok) * E);
    w.bytes = end;
    return w;
}

// The two-launch path wins where the ranking work is heavy: the clustered
// top-6 shape (T k = 98304) 108 -> 99 us; at the Mixtral shape (T k =
// 16384) the count and rank kernels are cheap and the separate bulk copy
// moves the rows faster (45-47 against 49-50 us), so small problems keep
// the three kernels.  LIBMOE_PERM_RANKCOPY=0/1 forces either; the tests
// run both.
constexpr long long kRankCopyMinSlots = 32768;

bool rank_copy_enabled(long long slots) {
    const char* env = getenv("LIBMOE_PERM_RANKCOPY");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return slots >= kRankCopyMinSlots;
}

// LIBMOE_BULK_COPY=0/1 forces the vectorised or the bulk-copy row copy.
bool bulk_copy_enabled() {
    const char* env = getenv("LIBMOE_BULK_COPY");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return true;
}

moe_status launch_copy_slots(const void* x, int T, int row_bytes, const int32_t* row_map, int k, void* buffer,
                             cudaStream_t s) {
    const int vpr = row_bytes / 16;
    const int grid = copy_grid(T);
    const int slot_bytes = (row_bytes + 127) / 128 * 128;
    if (bulk_copy_enabled() && slot_bytes <= 32 * 1024 && ((uintptr_t)x & 15) == 0 && ((uintptr_t)buffer & 15) == 0) {
        unsigned* err = device_error_word();
        if (!err) return MOE_ERR_CUDA;
        const size_t smem = (size_t)kBulkWarps * slot_bytes;
        if (!set_smem_limit((const void*)copy_rows_bulk_kernel, smem)) return MOE_ERR_CUDA;
        // one token per warp, as many CTAs as that takes: fresh CTAs replace
        // finished ones, which moved rows faster than a grid-strided loop
        // over fewer CTAs (T = 131072 top-8 rows: 0.94 against 0.91 of HBM
        // with 148 x 16 CTAs and 0.82 with one resident wave)
        const long long nb = ((long long)T + kBulkWarps - 1) / kBulkWarps;
        const int blocks = (int)(nb < (1LL << 30) ? nb : (1LL << 30));
        if (launch_pdl(copy_rows_bulk_kernel, blocks, 32 * kBulkWarps, smem, s, (const uint8_t*)x, T, row_bytes,
                       slot_bytes, row_map, k, (uint8_t*)buffer, err) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
    cudaError_t rc;
    if (vpr <= 32) rc = launch_pdl(copy_rows_slots_kernel<1>, grid, 256, 0, s, (const uint4*)x, T, vpr, row_map, k, (uint4*)buffer);
    else if (vpr <= 64) rc = launch_pdl(copy_rows_slots_kernel<2>, grid, 256, 0, s, (const uint4*)x, T, vpr, row_map, k, (uint4*)buffer);
    else rc = launch_pdl(copy_rows_slots_kernel<4>, grid, 256, 0, s, (const uint4*)x, T, vpr, row_map, k, (uint4*)buffer);
    if (rc != cudaSuccess) return MOE_ERR_CUDA;
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

// The argument checks of a permutation, shared by moe_permute and
// moe_permute_noalloc so that both return the same status for the same
// arguments, before any workspace question.
static moe_status permute_check_args(const void* x, int dtype, int T, int d, const int32_t* expert_idx, int k, int E,
                                     const int32_t* group_of_expert, int G, const void* buffer, const int32_t* row_map,
                                     const int32_t* row_token, const int32_t* counts, const int32_t* offsets,
                                     const int32_t* dropped) {
    if (T < 0 || k < 1 || E < 1 || k > E || d < 0) return MOE_ERR_ARG;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_ARG;
    if (k > 32 || E > 1024) return MOE_ERR_SHAPE;
    if (group_of_expert && (G < 1 || G > 1024)) return (G < 1) ? MOE_ERR_ARG : MOE_ERR_SHAPE;
    if (!counts || !offsets || !dropped) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!expert_idx || !row_map || !row_token) return MOE_ERR_ARG;
    if ((x == nullptr) != (buffer == nullptr)) return MOE_ERR_ARG;
    const long long row_bytes = (long long)d * (dtype == MOE_BF16 ? 2 : 4);
    if (x && (row_bytes % 16 != 0 || ((uintptr_t)x & 15) || ((uintptr_t)buffer & 15))) return MOE_ERR_SHAPE;
    return MOE_OK;
}

extern "C" moe_status moe_permute(const void* x, int dtype, int T, int d, const int32_t* expert_idx, int k, int E,
                                  double capacity_factor, const int32_t* group_of_expert, int G, void* buffer,
                                  int32_t* row_map, int32_t* row_token, int32_t* counts, int32_t* offsets,
                                  int32_t* dropped, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
    const moe_status bad = permute_check_args(x, dtype, T, d, expert_idx, k, E, group_of_expert, G, buffer, row_map,
                                              row_token, counts, offsets, dropped);
    if (bad != MOE_OK) return bad;
    if (T == 0) {
        // nothing routed: zero counts, offsets, dropped
        cudaStream_t s0 = (cudaStream_t)stream;
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s0) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * ((group_of_expert ? G : E) + 1), s0) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaMemsetAsync(dropped, 0, sizeof(int32_t), s0) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    const int esz = dtype == MOE_BF16 ? 2 : 4;
    const long long row_bytes = (long long)d * esz;
    const int Gk = group_of_expert ? G : 0;
    PermWs L = perm_layout(T, k, E, Gk);
    if (!workspace || workspace_bytes < L.bytes || ((uintptr_t)workspace & 255)) return MOE_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const long long cap = moe_capacity(capacity_factor, T, k, E);
    const int tb = perm_tokens_per_block(T);
    const int nblk = ceil_div(T, tb) > 0 ? ceil_div(T, tb) : 1;
    char* ws = (char*)workspace;
    int32_t* cnt = (int32_t*)(ws + L.cnt);
    int32_t* base = (int32_t*)(ws + L.base);
    int32_t* total = (int32_t*)(ws + L.total);
    const int nw = kIdxThreads / 32;
    // expert-major with rows: counting cluster, then rank and copy per chunk
    const int cpc = (!group_of_expert && x && d > 0) ? rc_chunks_per_cta(T, E) : 0;
    const int slot_bytes = (int)((row_bytes + 127) / 128 * 128);
    if (cpc > 0 && slot_bytes <= kRcMaxSlot && rank_copy_enabled((long long)T * k) && bulk_copy_enabled()) {
        const int nchunk = ceil_div(T, kRcTok);
        int32_t* cbase = (int32_t*)(ws + L.cbase);
        const size_t cc_smem = sizeof(int) * ((size_t)(cpc + 1) * E + 3 * (size_t)E);
        if (!set_smem_limit((const void*)perm_count_cluster_kernel, cc_smem)) return MOE_ERR_CUDA;
        if (launch_pdl(perm_count_cluster_kernel, kCcCtas, kCcThreads, cc_smem, s, expert_idx, T, k, E, nchunk, cpc,
                       cap, cbase, counts, offsets, dropped, err) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
        const size_t rc_smem = (size_t)kRcTok * slot_bytes +
                               sizeof(int) * ((2 + kRcTok) * (size_t)E + 2 * (size_t)kRcTok * k);
        if (!set_smem_limit((const void*)perm_rank_copy_kernel, rc_smem)) return MOE_ERR_CUDA;
        if (launch_pdl(perm_rank_copy_kernel, nchunk, 32 * kRcTok, rc_smem, s, (const uint8_t*)x, T, (int)row_bytes,
                       slot_bytes, expert_idx, k, E, (const int32_t*)cbase, (const int32_t*)offsets, cap, row_map,
                       row_token, (uint8_t*)buffer, err) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
    // 1. per-block expert counts
    if (launch_pdl(perm_count_kernel, nblk, kIdxThreads, sizeof(int) * E, s, expert_idx, T, k, E, nblk, tb, cnt, err) != cudaSuccess)
        return MOE_ERR_CUDA;
    MOE_LAUNCH_CHECK();
    // 2-3. the scans: done by every consumer block itself when experts x
    // blocks is small, else by two kernels
    const int fused_e = (long long)E * nblk <= kFuseLimit;
    int32_t* eoffsets = group_of_expert ? nullptr : offsets;
    if (!fused_e) {
        if (launch_pdl(perm_scan_blocks_kernel, E, 1024, 0, s, (const int32_t*)cnt, nblk, base, total) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
        if (launch_pdl(perm_offsets_kernel, 1, 1024, 0, s, (const int32_t*)total, E, cap, counts, eoffsets, dropped) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
    }
    if (!group_of_expert) {
        // 4. ranks and rows (its block 0 writes counts, offsets and dropped when fused)
        const size_t rank_smem = sizeof(int) * ((size_t)nw * E + 2 * (size_t)E + (size_t)tb * k);
        if (!set_smem_limit((const void*)perm_rank_kernel, rank_smem)) return MOE_ERR_CUDA;
        if (launch_pdl(perm_rank_kernel, nblk, kIdxThreads, rank_smem, s, expert_idx, T, k, E, nblk, tb, fused_e,
                       (const int32_t*)cnt, (const int32_t*)base, cap, counts, offsets, dropped, row_map, row_token,
                       err) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
    } else {
        int16_t* code = (int16_t*)(ws + L.code);
        int32_t* gcnt = (int32_t*)(ws + L.gcnt);
        int32_t* gbase = (int32_t*)(ws + L.gbase);
        int32_t* gtotal = (int32_t*)(ws + L.gtotal);
        const size_t heads_smem = sizeof(int) * ((size_t)nw * E + 3 * (size_t)E + G + (size_t)tb * k) + (size_t)tb * k;
        if (!set_smem_limit((const void*)perm_group_heads_kernel, heads_smem)) return MOE_ERR_CUDA;
        const int nodrop = cap >= (long long)T * k ? 1 : 0;
        if (launch_pdl(perm_group_heads_kernel, nblk, kIdxThreads, heads_smem, s, expert_idx, group_of_expert, T, k, E, G, nblk, tb,
                                                                        fused_e, cnt, base, cap, nodrop, counts, dropped,
                                                                        code, gcnt, err) != cudaSuccess)
            return MOE_ERR_CUDA;
        MOE_LAUNCH_CHECK();
        const int fused_g = (long long)G * nblk <= kFuseLimit;
        if (!fused_g) {
            if (launch_pdl(perm_scan_blocks_kernel, G, 1024, 0, s, (const int32_t*)gcnt, nblk, gbase, gtotal) != cudaSuccess)
                return MOE_ERR_CUDA;
            MOE_LAUNCH_CHECK();
            if (launch_pdl(perm_offsets_kernel, 1, 1024, 0, s, (const int32_t*)gtotal, G, (long long)T * k, (int32_t*)nullptr,
                           offsets, (int32_t*)nullptr) != cudaSuccess)
                return MOE_ERR_CUDA;
            MOE_LAUNCH_CHECK();
        }
        const size_t rows_smem = sizeof(int) * ((size_t)nw * G + 2 * (size_t)G + 2 * (size_t)tb * k);
        if (!set_smem_limit((const void*)perm_group_rows_kernel, rows_smem)) return MOE_ERR_CUDA;
        if (launch_pdl(perm_group_rows_kernel, nblk, kIdxThreads, rows_smem, s, code, T, k, G, nblk, tb, fused_g, gcnt, gbase, offsets,
                                                                      offsets, row_map, row_token) != cudaSuccess)
            return MOE_ERR_CUDA;
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
    const int slot_bytes = (int)((row_bytes + 127) / 128 * 128);
    if (bulk_copy_enabled() && slot_bytes <= 32 * 1024) {
        const size_t smem = (size_t)kBulkWarps * slot_bytes;
        if (!set_smem_limit((const void*)copy_rows_csr_bulk_kernel, smem)) return MOE_ERR_CUDA;
        // one token per warp (as the permutation's bulk copy): expert-choice
        // dispatch 0.74 -> 0.80 of HBM against 148 x 16 grid-strided CTAs
        const long long nb = ((long long)T + kBulkWarps - 1) / kBulkWarps;
        const int blocks = (int)(nb < (1LL << 30) ? nb : (1LL << 30));
        copy_rows_csr_bulk_kernel<<<blocks, 32 * kBulkWarps, smem, s>>>((const uint8_t*)x, T, (int)row_bytes, slot_bytes,
                                                                        tok_ptr, tok_row, R, (uint8_t*)buffer, err);
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
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
CachedAddress g_noalloc_scratch[kMaxDevices];

// Device address of this device's scratch array.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// with the device current on the first call on each device and cached; the
// cache is keyed on the context's unique id, so a context created again
// (after cudaDeviceReset) gets a fresh lookup instead of a stale address.
void* noalloc_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    CachedAddress& c = g_noalloc_scratch[dev];
    const unsigned long long ctx = context_id();
    if (c.addr && ctx != 0 && c.ctx == ctx) return c.addr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_noalloc_scratch) != cudaSuccess) return nullptr;
    c.addr = p;
    c.ctx = context_id();
    return p;
}
}  // namespace

extern "C" moe_status moe_permute_noalloc(const void* x, int dtype, int T, int d, const int32_t* expert_idx, int k,
                                          int E, double capacity_factor, const int32_t* group_of_expert, int G,
                                          void* buffer, int32_t* row_map, int32_t* row_token, int32_t* counts,
                                          int32_t* offsets, int32_t* dropped, moe_stream_t stream) {
    const moe_status bad = permute_check_args(x, dtype, T, d, expert_idx, k, E, group_of_expert, G, buffer, row_map,
                                              row_token, counts, offsets, dropped);
    if (bad != MOE_OK) return bad;
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
