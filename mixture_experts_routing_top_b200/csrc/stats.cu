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
//
// Co-selection counts every ordered pair of a token's slots, so it is
// symmetric: cosel_sym_kernel counts each unordered pair once, in the row of
// the smaller expert (the upper triangle, diagonal included), and writes it
// to both (a, b) and (b, a) when the band is merged.  That takes k(k+1)/2
// shared atomics per token instead of k^2 (36 instead of 64 at k = 8).  The
// bands are cut from the triangle so that they hold equal numbers of bins.
// Used for E >= 128 (wide histograms), where it measured faster.
#include <cstdlib>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {

constexpr int kHistBytes = 64 * 1024;

__global__ void __launch_bounds__(512) pair_hist_kernel(const int32_t* __restrict__ idx1, int k1,
                                                        const int32_t* __restrict__ idx2, int k2, int T, int E,
                                                        int band, int tokens_per_cta, int32_t* __restrict__ hist,
                                                        unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
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

// Bins of the upper triangle in rows [0, a): row r holds b in [r, E).
inline long long tri_off(long long a, long long E) { return a * E - a * (a - 1) / 2; }
__device__ __forceinline__ int tri_off_d(int a, int E) { return a * E - ((a * (a - 1)) >> 1); }   // E <= 1024

constexpr int kSymBandBytes = 72 * 1024;
constexpr int kMaxSymBands = 64;
struct SymBands {
    int start[kMaxSymBands + 1];       // band b holds rows [start[b], start[b + 1])
};

__global__ void __launch_bounds__(512) cosel_sym_kernel(const int32_t* __restrict__ idx, int k, int T, int E,
                                                        SymBands bands, int tokens_per_cta,
                                                        int32_t* __restrict__ hist, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int h[];                  // rows [a0, a1) of the upper triangle, packed
    const int a0 = bands.start[blockIdx.y];
    const int a1 = bands.start[blockIdx.y + 1];
    if (a0 >= a1) return;
    const int base = (int)tri_off_d(a0, E);
    const int nbins = (int)tri_off_d(a1, E) - base;
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) h[i] = 0;
    __syncthreads();
    // ceil(k/2) lanes per token: lane r takes slot r and slot k-1-r, so each
    // lane counts k-1 pairs (j > i) and one or two diagonal entries
    const int hk = (k + 1) >> 1;
    const int tpw = 32 / hk;                    // tokens per warp pass
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    const int tw = lane / hk;
    const int r = lane - tw * hk;
    const int i1 = r, i2 = k - 1 - r;
    const int n1 = k - 1 - i1;                  // pairs (i1, j > i1)
    const int np = i2 > i1 ? k - 1 : n1;        // ... then pairs (i2, j > i2)
    const long long t0 = (long long)blockIdx.x * tokens_per_cta;
    const long long left = (long long)T - t0;
    const int nt = left < tokens_per_cta ? (int)left : tokens_per_cta;
    const unsigned band = (unsigned)(a1 - a0);
    auto bump = [&](int lo, int hi, int v) {
        if ((unsigned)(lo - a0) < band) atomicAdd(h + (int)tri_off_d(lo, E) - base + (hi - lo), v);
    };
    if (tw < tpw) {
        for (int tt = warp * tpw + tw; tt < nt; tt += nw * tpw) {
            const int32_t* s = idx + (t0 + tt) * k;
            const int a = __ldg(s + i1);
            const int c = __ldg(s + i2);
            const bool va = (unsigned)a < (unsigned)E;
            const bool vc = (unsigned)c < (unsigned)E;
            if (!va || !vc) raise_error(err, kErrIndex);
            if (va) bump(a, a, 1);                                // the pair (i1, i1)
            if (i2 > i1 && vc) bump(c, c, 1);                     // the pair (i2, i2)
            for (int p = 0; p < np; ++p) {
                const bool first = p < n1;
                const int x = first ? a : c;
                const int j = first ? i1 + 1 + p : i2 + 1 + (p - n1);
                const int y = __ldg(s + j);
                if (!(first ? va : vc)) continue;                 // reported above
                if ((unsigned)y >= (unsigned)E) { raise_error(err, kErrIndex); continue; }
                // slots i < j: the ordered pairs (i, j) and (j, i); on one expert both land on its diagonal
                bump(min(x, y), max(x, y), x == y ? 2 : 1);
            }
        }
    }
    __syncthreads();
    for (int a = a0 + warp; a < a1; a += nw) {
        const int off = (int)tri_off_d(a, E) - base - a;
        for (int b = a + lane; b < E; b += 32) {
            const int v = h[off + b];
            if (!v) continue;
            atomicAdd(hist + (long long)a * E + b, v);
            if (b != a) atomicAdd(hist + (long long)b * E + a, v);
        }
    }
}

// Co-selection for k <= 8: thread per token.  The token's k experts are
// loaded at once into registers (independent loads, no dependent chain),
// and its k(k+1)/2 unordered slot pairs are counted in this band's packed
// upper triangle in shared memory, as in cosel_sym_kernel.  CTAs run in
// clusters of kCoselCluster: after counting, CTA r of a cluster sums rows
// a = a0 + r, a0 + r + kCoselCluster, ... over the cluster's CTAs through
// distributed shared memory and merges them with one global atomic per
// non-zero bin (two off the diagonal), so the global merge costs one pass
// per cluster instead of one per CTA.
constexpr int kCoselCluster = 8;
constexpr int kCoselBandBytes = 200 * 1024;

template <int KM>
__global__ void __cluster_dims__(kCoselCluster, 1, 1) __launch_bounds__(1024, 1)
cosel_cluster_kernel(const int32_t* __restrict__ idx, int k, int T, int E, SymBands bands, int tokens_per_cta,
                     int32_t* __restrict__ hist, unsigned* err) {
    pdl_trigger();                // the next kernel may be scheduled; it waits for this one
    pdl_wait();                   // inputs come from the kernel before
    extern __shared__ int h[];                  // rows [a0, a1) of the upper triangle, packed
    const int a0 = bands.start[blockIdx.y];
    const int a1 = bands.start[blockIdx.y + 1];
    const int base = tri_off_d(a0, E);
    const int nbins = tri_off_d(a1, E) - base;
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) h[i] = 0;
    __syncthreads();
    const unsigned band = (unsigned)(a1 - a0);
    const long long t0 = (long long)blockIdx.x * tokens_per_cta;
    const long long t1 = min(t0 + tokens_per_cta, (long long)T);
    for (long long t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int32_t* sl = idx + t * k;
        int a[KM];
#pragma unroll
        for (int i = 0; i < KM; ++i) a[i] = i < k ? __ldg(sl + i) : -1;
        bool bad = false;
#pragma unroll
        for (int i = 0; i < KM; ++i)
            if (i < k && (unsigned)a[i] >= (unsigned)E) { bad = true; a[i] = -1; }
        if (bad) raise_error(err, kErrIndex);
#pragma unroll
        for (int i = 0; i < KM; ++i) {
            if (i >= k || a[i] < 0) continue;
            if ((unsigned)(a[i] - a0) < band) atomicAdd(h + tri_off_d(a[i], E) - base, 1);   // the pair (i, i)
#pragma unroll
            for (int j = i + 1; j < KM; ++j) {
                if (j >= k || a[j] < 0) continue;
                // slots i < j: the ordered pairs (i, j) and (j, i); on one expert both land on its diagonal
                const int lo = min(a[i], a[j]), hi = max(a[i], a[j]);
                if ((unsigned)(lo - a0) < band) atomicAdd(h + tri_off_d(lo, E) - base + (hi - lo), lo == hi ? 2 : 1);
            }
        }
    }
    __syncthreads();
    tc::cluster_sync();                         // every CTA's counts are complete and visible
    const int r = (int)tc::cluster_rank();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t rbase[kCoselCluster];
#pragma unroll
    for (int q = 0; q < kCoselCluster; ++q) rbase[q] = tc::map_to_rank(tc::smem_u32(h), (uint32_t)q);
    for (int a = a0 + r + kCoselCluster * warp; a < a1; a += kCoselCluster * nw) {
        const int off = tri_off_d(a, E) - base - a;
        for (int b = a + lane; b < E; b += 32) {
            const uint32_t byte = 4u * (uint32_t)(off + b);
            int v = 0;
#pragma unroll
            for (int q = 0; q < kCoselCluster; ++q) v += (int)tc::ld_shared_cluster_u32(rbase[q] + byte);
            if (!v) continue;
            atomicAdd(hist + (long long)a * E + b, v);
            if (b != a) atomicAdd(hist + (long long)b * E + a, v);
        }
    }
    // no CTA exits while another still reads its counts: every remote load
    // above feeds the branch on its value (and the atomics) before this
    // point, so it has completed when the thread arrives, and a relaxed
    // arrive need not wait for the merge's global atomics
    tc::cluster_sync_relaxed();
}

// The symmetric kernel for E >= 128, where it measured faster (T = 131072,
// E = 256, k = 8: 48 us against 53 us); at E = 64 it was slower (15.9 us
// against 13.6 us: too few tokens per CTA to hide its longer dependent chain).
// LIBMOE_COSEL_SYM=0/1 forces the ordered-pair or the symmetric kernel.
bool cosel_sym_enabled(int E) {
    const char* env = getenv("LIBMOE_COSEL_SYM");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return E >= 128;
}

moe_status launch_cosel_sym(const int32_t* idx, int k, int T, int E, int32_t* hist, cudaStream_t s) {
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    // bands of the triangle with equal bin counts, each at most kSymBandBytes
    const long long total = tri_off(E, E);
    const long long max_bins = kSymBandBytes / (long long)sizeof(int);
    int nb = (int)((total + (max_bins - E) - 1) / (max_bins - E));
    if (nb < 1) nb = 1;
    if (nb > kMaxSymBands) return MOE_ERR_SHAPE;
    SymBands sb;
    sb.start[0] = 0;
    long long x = 0;
    for (int b = 1; b < nb; ++b) {
        const long long target = total * b / nb;
        while (tri_off(x, E) < target) ++x;
        sb.start[b] = (int)x;
    }
    sb.start[nb] = E;
    long long widest = 0;
    for (int b = 0; b < nb; ++b) {
        const long long n = tri_off(sb.start[b + 1], E) - tri_off(sb.start[b], E);
        if (n > widest) widest = n;
    }
    if (widest > max_bins) return MOE_ERR_SHAPE;
    const size_t smem = sizeof(int) * (size_t)(widest > 0 ? widest : 1);
    // one CTA per SM over all bands (fewest merge atomics; 1 to 6 CTAs per SM
    // measured 48 to 57 us at T = 131072, E = 256); at least 256 tokens each
    int tok_ctas = (148 + nb - 1) / nb;
    int tokens_per_cta = ceil_div(T, tok_ctas);
    if (tokens_per_cta < 256) tokens_per_cta = 256;
    tok_ctas = ceil_div(T, tokens_per_cta);
    if (!set_smem_limit((const void*)cosel_sym_kernel, smem)) return MOE_ERR_CUDA;
    (void)launch_pdl(cosel_sym_kernel, dim3(tok_ctas, nb), 512, smem, s, idx, k, T, E, sb, tokens_per_cta, hist, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

// Bands of the packed upper triangle with equal bin counts, each at most
// max_bytes of shared memory.  False if E is too large for kMaxSymBands.
bool make_sym_bands(int E, long long max_bytes, SymBands* sb, int* nb_out, long long* widest_out) {
    const long long total = tri_off(E, E);
    const long long max_bins = max_bytes / (long long)sizeof(int);
    int nb = (int)((total + (max_bins - E) - 1) / (max_bins - E));
    if (nb < 1) nb = 1;
    if (nb > kMaxSymBands) return false;
    sb->start[0] = 0;
    long long x = 0;
    for (int b = 1; b < nb; ++b) {
        const long long target = total * b / nb;
        while (tri_off(x, E) < target) ++x;
        sb->start[b] = (int)x;
    }
    sb->start[nb] = E;
    long long widest = 0;
    for (int b = 0; b < nb; ++b) {
        const long long n = tri_off(sb->start[b + 1], E) - tri_off(sb->start[b], E);
        if (n > widest) widest = n;
    }
    if (widest > max_bins) return false;
    *nb_out = nb;
    *widest_out = widest;
    return true;
}

// LIBMOE_COSEL_CLUSTER=0 keeps co-selection with k <= 8 on the older
// kernels; the tests run both.
bool cosel_cluster_enabled() {
    const char* env = getenv("LIBMOE_COSEL_CLUSTER");
    if (env && (env[0] == '0' || env[0] == '1')) return env[0] == '1';
    return true;
}

// How many clusters of this kernel, with this shared memory, the device runs
// at once (cached per kernel, size, device and context).  Launching more than
// that leaves the extra clusters for a second wave.
int max_active_clusters(const void* fn, size_t smem, int block) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    static std::mutex mu;
    static std::map<std::tuple<const void*, size_t, int, unsigned long long>, int> known;
    const auto key = std::make_tuple(fn, smem, dev, context_id());
    std::lock_guard<std::mutex> lk(mu);
    const auto it = known.find(key);
    if (it != known.end()) return it->second;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCoselCluster * 16);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = 1;
    }
    known[key] = n;
    return n;
}

moe_status launch_cosel_cluster(const int32_t* idx, int k, int T, int E, int32_t* hist, cudaStream_t s) {
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    SymBands sb;
    int nb = 0;
    long long widest = 0;
    if (!make_sym_bands(E, kCoselBandBytes, &sb, &nb, &widest)) return MOE_ERR_SHAPE;
    const size_t smem = sizeof(int) * (size_t)(widest > 0 ? widest : 1);
    auto fn = k <= 2 ? cosel_cluster_kernel<2> : k <= 4 ? cosel_cluster_kernel<4> : cosel_cluster_kernel<8>;
    if (!set_smem_limit((const void*)fn, smem)) return MOE_ERR_CUDA;
    // as many clusters of 8 as run at once over all bands (one wave; with one
    // CTA per SM the GPCs hold 15 at E = 256, not 148 / 8), at least 512
    // tokens per CTA
    int clusters = max_active_clusters((const void*)fn, smem, 1024) / nb;
    if (clusters < 1) clusters = 1;
    int tokens_per_cta = ceil_div(T, (long long)clusters * kCoselCluster);
    if (tokens_per_cta < 512) tokens_per_cta = 512;
    const int tok_ctas = ceil_div(ceil_div(T, tokens_per_cta), kCoselCluster) * kCoselCluster;
    (void)launch_pdl(fn, dim3(tok_ctas, nb), 1024, smem, s, idx, k, T, E, sb, tokens_per_cta, hist, err);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
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
    if (!set_smem_limit((const void*)pair_hist_kernel, smem)) return MOE_ERR_CUDA;
    (void)launch_pdl(pair_hist_kernel, dim3(tok_ctas, nbands), 512, smem, s, idx1, k1, idx2, k2, T, E, band, tokens_per_cta, hist, err);
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
    if (k <= 8 && cosel_cluster_enabled())
        return launch_cosel_cluster(expert_idx, k, T, E, cosel, (cudaStream_t)stream);
    if (cosel_sym_enabled(E)) return launch_cosel_sym(expert_idx, k, T, E, cosel, (cudaStream_t)stream);
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
