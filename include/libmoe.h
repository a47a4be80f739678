/*
 * libmoe.h - C ABI of the Mixture-of-Experts layer hot path on one B200 GPU.
 *
 * The layer, as the pages state it ("How MegaDLMs Implements Mixture of
 * Experts (MoE) Architectures", section "MoELayer"), runs three steps:
 * token permutation, expert computation, token unpermutation.  Routing comes
 * first ("Routing Mechanisms: Top-K vs Expert Choice"), capacity and
 * dropping follow "Expert Parallelism > Key Parameters", and the two routing
 * correlation statistics follow "Expert Coupling in MoE Pretraining",
 * Abstract.  One call per step:
 *
 *   moe_router_topk (x -> top-k) or
 *   moe_route_topk / moe_route_ec  ->  moe_permute / moe_gather_rows
 *   ->  moe_expert_ffn  ->  moe_unpermute / moe_unpermute_ec
 *   group-major experts: moe_copy_slot_rows, moe_group_precombine, moe_unpermute_groups
 *   beside it: moe_coselect, moe_transition
 *
 * Conventions shared by every call:
 *  - Every array argument is DEVICE memory owned by the caller, row-major,
 *    tightly packed.  The library allocates nothing: scratch comes in
 *    through an explicit workspace pointer sized by the matching
 *    *_workspace_bytes() query.  Workspace must be 256-byte aligned.
 *  - Calls are asynchronous on `stream` (NULL: the legacy default stream);
 *    results are ready when the stream reaches them.  Nothing inside a call
 *    waits on the host, so a call may be captured in a CUDA graph.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns an error status and launches nothing.  A launch
 *    failure returns MOE_ERR_CUDA.
 *  - Faults found on the device (an expert index outside [0, E), a bounded
 *    wait that gave up) cannot be returned by an asynchronous call: the
 *    kernel skips the bad element and records a code that
 *    moe_device_error() reports.
 *  - Index arrays are int32.  bf16 tensors hold raw bf16 bit patterns.
 *  - Histograms ACCUMULATE into the caller's array (zero it first), so
 *    several batches or layers can be summed.
 */
#ifndef LIBMOE_H
#define LIBMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = 1,          /* null pointer, negative size, k > E, C > T, bad dtype value, ... */
    MOE_ERR_SHAPE = 2,        /* a size the kernels do not handle (row alignment, E > 1024, k > 32, ...) */
    MOE_ERR_DTYPE = 3,        /* a dtype combination the call does not handle */
    MOE_ERR_WORKSPACE = 4,    /* workspace NULL, too small or not 256-byte aligned */
    MOE_ERR_CUDA = 5,         /* a CUDA runtime error (launch, symbol lookup) */
    MOE_ERR_UNSUPPORTED = 6,  /* the current device is not an sm_100 (B200-class) GPU */
    MOE_ERR_TIMEOUT = 7,      /* a bounded device-side wait gave up (see moe_device_error) */
    MOE_ERR_DEVICE_INDEX = 8  /* a kernel met an out-of-range index and skipped it */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_GELU = 1 } moe_act;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(int status);
/* The same, under the name the boundary's specification uses. */
const char* moe_status_str(moe_status status);

/* ABI revision of this header; bumps on any incompatible change. */
#define MOE_ABI_VERSION 1
int moe_abi_version(void);

/* Reads (and, if clear != 0, resets) the device-side fault word of the
 * current device.  Synchronises the device.  Returns MOE_OK, MOE_ERR_TIMEOUT
 * or MOE_ERR_DEVICE_INDEX (or MOE_ERR_CUDA if the read itself failed). */
moe_status moe_device_error(int clear);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all streams).  Lets a caller count the kernels a region ran. */
uint64_t moe_kernel_launches(void);

/* Device check of the failure-detection contract above (the pages have no
 * counterpart).  One warp waits on an mbarrier through the same bounded
 * wait the tensor-core kernels use, with a limit of limit_ns of
 * %globaltimer (1 us .. 1 s).  With arrive == 0 nothing ever arrives: the
 * wait gives up, the kernel records MOE_ERR_TIMEOUT in the fault word
 * (moe_device_error) and returns; with arrive != 0 the barrier is
 * completed first and no fault is recorded.  No copy or MMA is in flight,
 * so the context stays usable either way.
 *   result  [2] int32 device out: [0] = 1 if the wait completed, 0 if it
 *           gave up; [1] = microseconds spent waiting.
 * Returns MOE_ERR_ARG for a limit outside the range or a NULL result. */
moe_status moe_selftest_bounded_wait(int arrive, long long limit_ns, int32_t* result, moe_stream_t stream);

/* ------------------------------------------------------------ routing */

/* TopKRouter ("Routing Mechanisms: Top-K vs Expert Choice"): softmax over
 * each token's E router logits and its k best experts.
 *   logits      [T, E] fp32 (finite values, or -inf for a masked expert
 *               while at least k are finite; NaN gives unspecified experts)
 *   expert_idx  [T, k] int32 out: slot j = the (j+1)-th largest logit;
 *               equal logits: the lower expert index ranks first
 *   gate        [T, k] fp32 out: softmax probability of that expert; with
 *               norm_topk != 0, renormalised over the k chosen experts
 * Limits: 1 <= k <= min(E, 32), E <= 1024, T >= 0. */
moe_status moe_route_topk(const float* logits, int T, int E, int k, int norm_topk,
                          int32_t* expert_idx, float* gate, moe_stream_t stream);

/* The router's linear gate fused with moe_route_topk ("Routing Mechanisms:
 * Top-K vs Expert Choice": the TopKRouter scores each expert with a linear
 * layer over the token's hidden state, then softmax and top-k as above):
 * logits[t, e] = sum_c x[t, c] * W_r[e, c], then the top-k experts and
 * gates of each logits row, with the ranking and gates of moe_route_topk.
 *   x       [T, d] dtype;  W_r [E, d] dtype (one row per expert)
 *   logits  [T, E] fp32 out, or NULL when not wanted (bf16 only)
 *   expert_idx, gate  [T, k] out, as moe_route_topk
 * bf16: one tcgen05 GEMM (fp32 accumulation in TMEM) whose epilogue ranks
 * each token from TMEM; d % 64 == 0, E % 8 == 0, E <= 256, k <= 8, x, W_r
 * and logits 16-byte aligned.  fp32: FMA logits into `logits` (required),
 * then moe_route_topk on them; E <= 1024, k <= 32.
 * The logits' rounding differs from an fp64 evaluation by the fp32
 * accumulation error, so experts whose logits lie that close may rank
 * differently from an exact evaluation; the ranking of the returned
 * logits themselves is exact. */
moe_status moe_router_topk(const void* x, int dtype, int T, int d, const void* W_r, int E, int k, int norm_topk,
                           float* logits, int32_t* expert_idx, float* gate, moe_stream_t stream);

/* ExpertChoiceRouter (same section): each expert chooses the C tokens with
 * the highest routing score, the score being the token's softmax
 * probability for that expert, compared as log-probability
 * logit - logsumexp(token's logits) in fp64; equal scores: lower token first.
 *   ec_token [E, C] int32 out: expert e's tokens in ascending token order;
 *            buffer row e*C + i holds token ec_token[e, i]
 *   ec_gate  [E, C] fp32 out: that token's probability for expert e
 *   tok_ptr  [T + 1] int32 out, tok_row [E*C] int32 out: per-token list of
 *            the buffer rows that hold it, ascending expert (CSR)
 * Limits: 1 <= C <= T, E <= 1024.  Workspace: moe_route_ec_workspace_bytes. */
size_t moe_route_ec_workspace_bytes(int T, int E, int C);
moe_status moe_route_ec(const float* logits, int T, int E, int C,
                        int32_t* ec_token, float* ec_gate, int32_t* tok_ptr, int32_t* tok_row,
                        void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ------------------------------------------------------- permutation */

/* Capacity per expert: ceil(capacity_factor * T * k / E) computed in fp64;
 * capacity_factor <= 0 means unbounded (returns T*k).  "Expert Parallelism >
 * Key Parameters", capacity_factor. */
int64_t moe_capacity(double capacity_factor, int T, int k, int E);

/* Rows the permuted buffer needs at most: min(T*k, E*capacity) in
 * expert-major layout, T*min(k, G) in group-major layout (G > 0). */
int64_t moe_permute_max_rows(int T, int k, int E, double capacity_factor, int G);

/* token_permutation ("MoELayer" step 1; "Token Dispatching and
 * Communication"), on one device.  Each assignment (t, j) of token t to
 * expert e = expert_idx[t, j] gets a buffer row; an expert keeps its first
 * `capacity` assignments in token order and drops the rest ("Expert
 * Parallelism > Key Parameters": dropped tokens contribute zero).
 *
 * Expert-major (group_of_expert == NULL): expert e owns rows
 * [offsets[e], offsets[e] + counts[e]), tokens in ascending order.
 * Group-major (group_of_expert [E] int32 in [0, G)): one row per distinct
 * (token, group) with a kept assignment into the group, ordered by group
 * then token - the one-device form of the dispatcher that ships a token to
 * a given GPU at most one time ("Expert Coupling in MoE Pretraining",
 * Abstract).
 *
 *   x          [T, d] dtype, or NULL (indices only; buffer must then be NULL)
 *   expert_idx [T, k] int32 in [0, E), no expert twice in one token
 *   buffer     [R_max, d] dtype out (R_max = moe_permute_max_rows): buffer[r]
 *              is a byte copy of x[row_token[r]]; rows >= R are untouched
 *   row_map    [T, k] int32 out: buffer row of the assignment, -1 if dropped
 *   row_token  [R_max] int32 out: source token of each row (first R valid)
 *   counts     [E] int32 out: kept assignments per expert
 *   offsets    [E + 1] (expert-major) or [G + 1] (group-major) int32 out;
 *              R = offsets[last] rows are used (left on the device)
 *   dropped    [1] int32 out: assignments dropped by capacity
 * Row size d * sizeof(dtype) must be a multiple of 16 bytes when x != NULL.
 * Limits: 1 <= k <= 32, E <= 1024, G <= 1024.  Workspace:
 * moe_permute_workspace_bytes. */
size_t moe_permute_workspace_bytes(int T, int k, int E, int G);
moe_status moe_permute(const void* x, int dtype, int T, int d,
                       const int32_t* expert_idx, int k, int E, double capacity_factor,
                       const int32_t* group_of_expert, int G,
                       void* buffer, int32_t* row_map, int32_t* row_token,
                       int32_t* counts, int32_t* offsets, int32_t* dropped,
                       void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* moe_permute without a caller workspace, for callers that cannot allocate
 * device memory: a host framework that owns all device memory and forbids
 * allocation once running (inference plugins, serving loops with a fixed
 * memory plan), or a hot path that cannot take cudaMalloc's implicit
 * synchronisation.  The pages have no counterpart to this call; it exists
 * for deployment only.  Arguments and results are those of moe_permute.
 * Scratch: a fixed MOE_PERMUTE_NOALLOC_SCRATCH_BYTES array in device memory,
 * held by every GPU that loads the library until the process exits.
 * Limit: moe_permute_workspace_bytes(T, k, E, G) must not exceed it
 * (e.g. T = 131072, k = 8, E = 256, G = 64 needs 3.25 MiB); larger problems
 * return MOE_ERR_WORKSPACE and launch nothing; invalid arguments are
 * checked first and return what moe_permute returns for them.  The first
 * call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it for that device's context (a context
 * created again after cudaDeviceReset gets a new lookup); make that first
 * call before any stream capture.  All calls share the one
 * array, so calls whose kernels overlap on the GPU (different streams, no
 * ordering between them) race and give wrong results; serialise them. */
#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (4u << 20)
moe_status moe_permute_noalloc(const void* x, int dtype, int T, int d,
                               const int32_t* expert_idx, int k, int E, double capacity_factor,
                               const int32_t* group_of_expert, int G,
                               void* buffer, int32_t* row_map, int32_t* row_token,
                               int32_t* counts, int32_t* offsets, int32_t* dropped, moe_stream_t stream);

/* Expert-choice dispatch: buffer rows from the token CSR of moe_route_ec,
 * each token read once: buffer[tok_row[p]] = x[t] for p in
 * [tok_ptr[t], tok_ptr[t+1]).  buffer has R rows (E*C) and tok_row R
 * entries; an entry outside [0, R) is skipped and reported through
 * moe_device_error.  Row size must be a multiple of 16 bytes. */
moe_status moe_gather_rows(const void* x, int dtype, int T, int d, const int32_t* tok_ptr,
                           const int32_t* tok_row, int R, void* buffer, moe_stream_t stream);

/* ------------------------------------------------------- expert MLPs */

/* Expert computation ("MoELayer" step 2: each expert held on the device
 * runs its MLP on the rows routed to it).  Rows [offsets[e], offsets[e+1])
 * of `buffer` go through expert e:
 *   SwiGLU: h = silu(x W1[e]^T) * (x W3[e]^T),  y = h W2[e]^T
 *   GELU:   h = gelu(x W1[e]^T) (erf form),     y = h W2[e]^T
 *           (erf evaluated by Abramowitz & Stegun 7.1.28: |error| <= 2e-6 in fp32)
 * bf16: tensor-core GEMMs with fp32 accumulation; h is stored as bf16 in the
 * workspace, y as bf16.  fp32: fp32 FMA throughout (small layers).
 *   buffer  [R_max, d]; offsets [E + 1] int32 on the device, offsets[0] = 0,
 *           non-decreasing, offsets[E] <= R_max (read on the device only)
 *   W1, W3  [E, F, d] (W3 NULL for GELU);  W2 [E, d, F]
 *   y       [R_max, d] out; rows >= offsets[E] are untouched
 * A shared expert ("Expert Parallelism > Key Parameters", the always-on
 * expert) is this call with E = 1 and offsets = {0, T} over the tokens.
 * bf16 needs d % 64 == 0 and F % 64 == 0.  Workspace:
 * moe_expert_ffn_workspace_bytes. */
size_t moe_expert_ffn_workspace_bytes(int R_max, int d, int F, int dtype);
moe_status moe_expert_ffn(const void* buffer, int dtype, int R_max, int d, int F, int E,
                          const int32_t* offsets, const void* W1, const void* W3, const void* W2,
                          int act, void* y, void* workspace, size_t workspace_bytes,
                          moe_stream_t stream);

/* ----------------------------------------------------- unpermutation */

/* token_unpermutation ("MoELayer" step 3): each token's output is the sum,
 * in fp32, of its kept expert outputs weighted by their gates, plus the
 * shared expert's output (weight 1) when `shared` is not NULL.  Dropped
 * assignments (row_map = -1) contribute zero.  Slots that share a row
 * (group-major layout) are read once, their gates summed.
 *   y [R, d] dtype; row_map, gate [T, k]; shared [T, d] dtype or NULL;
 *   out [T, d] out_dtype (MOE_F32 or MOE_BF16).  A row_map entry >= R is
 *   skipped and reported through moe_device_error. */
moe_status moe_unpermute(const void* y, int dtype, int R, int T, int d, int k, const int32_t* row_map,
                         const float* gate, const void* shared, void* out, int out_dtype,
                         moe_stream_t stream);

/* Expert-choice unpermutation: out[t] = sum over the token's rows (ascending
 * expert) of ec_gate[row] * y[row]; a token no expert chose gets 0.
 *   y [R, d] with R = E*C; ec_gate [R] fp32 indexed by buffer row. */
moe_status moe_unpermute_ec(const void* y, int dtype, int R, int T, int d, const int32_t* tok_ptr,
                            const int32_t* tok_row, const float* ec_gate, void* out, int out_dtype,
                            moe_stream_t stream);

/* ------------------------------------ group-major expert path */

/* The send-once dispatcher with real experts ("Expert Coupling in MoE
 * Pretraining", Abstract: a token is shipped to a given GPU at most one
 * time, however many of its experts live there).  On one device the path is
 *   moe_permute (group-major, x)          one row per (token, group)
 *   moe_permute (expert-major, x = NULL)  the local expert rows, indices only
 *   moe_copy_slot_rows                    group rows -> expert rows
 *   moe_expert_ffn                        on the expert rows
 *   moe_group_precombine                  expert outputs -> one row per (token, group)
 *   moe_unpermute_groups                  token = sum of its group rows
 * Both permutes take the same expert_idx and capacity factor, so they keep
 * the same assignments (capacity is per expert in both layouts).
 *
 * Row copy through two row maps: for every slot s in [0, S) with
 * src_row[s] >= 0 and dst_row[s] >= 0, dst[dst_row[s]] = src[src_row[s]]
 * (a byte copy).  With src_row = the group-major row_map and dst_row = the
 * expert-major row_map ([T, k], S = T*k) this is each group's local
 * permutation to its experts; a destination row reached from several slots
 * must get the same source row (as here: one slot per expert row).
 *   src [R_src, d], dst [R_dst, d], dtype; row size a multiple of 16 bytes.
 *   A row >= R_src or >= R_dst is skipped and reported through
 *   moe_device_error. */
moe_status moe_copy_slot_rows(const void* src, int dtype, int R_src, int d, const int32_t* src_row,
                              const int32_t* dst_row, int S, void* dst, int R_dst, moe_stream_t stream);

/* Pre-combine inside a group (same Abstract, the receiving side of the
 * send-once dispatcher): y_g[r] = sum over the slots j of token t with
 * row_map_g[t, j] = r, in slot order, of gate[t, j] * y_e[row_map_e[t, j]],
 * accumulated in fp32 and stored once in dtype.  Slots with
 * row_map_g = -1 (dropped) are skipped.
 *   y_e [R_e, d] (expert rows, moe_expert_ffn output); y_g [R_g, d] out;
 *   row_map_e, row_map_g, gate [T, k].  d % 8 == 0, k <= 32.  Entries past
 *   R_e or R_g are skipped and reported through moe_device_error. */
moe_status moe_group_precombine(const void* y_e, int dtype, int R_e, int T, int d, int k,
                                const int32_t* row_map_e, const int32_t* row_map_g, const float* gate,
                                void* y_g, int R_g, moe_stream_t stream);

/* Token output from its group rows: out[t] = sum, in fp32 and in the order
 * the rows first appear among the token's slots, of its distinct group rows
 * y_g[row_map_g[t, j]] (unit weight: the gates were applied by
 * moe_group_precombine), plus shared[t] when not NULL; a token with every
 * slot dropped gets shared[t] or 0.
 *   y_g [R_g, d] dtype; shared [T, d] dtype or NULL; out [T, d] out_dtype.
 *   d % 8 == 0, k <= 32. */
moe_status moe_unpermute_groups(const void* y_g, int dtype, int R_g, int T, int d, int k,
                                const int32_t* row_map_g, const void* shared, void* out, int out_dtype,
                                moe_stream_t stream);

/* -------------------------------------------- routing statistics */

/* Expert pair co-selection ("Expert Coupling in MoE Pretraining",
 * Abstract: pairs of experts a token selects together), on the routing
 * decisions before capacity: cosel[a][b] += 1 for every ordered pair of
 * slots (i, j) of a token with a = expert_idx[t, i], b = expert_idx[t, j].
 * The diagonal is each expert's load.  cosel [E, E] int32, accumulated.
 * An index outside [0, E) is skipped with every pair it is part of, and
 * sets MOE_ERR_DEVICE_INDEX in the fault word.  E <= 1024, k <= 32. */
moe_status moe_coselect(const int32_t* expert_idx, int T, int k, int E, int32_t* cosel,
                        moe_stream_t stream);

/* Layer-to-layer expert transitions (same Abstract: a token's expert
 * choices in one layer are predictive of its choices in the next):
 * trans[a][b] += 1 for every a among idx1[t, :k1] and b among idx2[t, :k2].
 * trans [E, E] int32, accumulated.  Out-of-range indices as for
 * moe_coselect.  E <= 1024, k1, k2 <= 32. */
moe_status moe_transition(const int32_t* idx1, int k1, const int32_t* idx2, int k2, int T, int E,
                          int32_t* trans, moe_stream_t stream);

/* ------------------------------- placement and token shuffling */

/* Correlated expert placement ("Expert Coupling in MoE Pretraining",
 * Abstract: experts often picked together go to the same GPU).  The pages
 * give no algorithm; this is a greedy on the co-selection counts cosel
 * [E, E] (as moe_coselect produces): each of the G groups (L = E/G experts)
 * starts from the unassigned expert with the largest off-diagonal
 * co-selection mass and grows by the unassigned expert with the largest
 * co-selection summed over the group's members (column reads cosel[x][m]);
 * lower index on ties.  group_of_expert [E] int32 out, in [0, G).  One CTA.
 * Limits: G divides E, E <= 1024. */
moe_status moe_place_experts(const int32_t* cosel, int E, int G, int32_t* group_of_expert, moe_stream_t stream);

/* Affinity of each expert's next-layer traffic to each group (same Abstract:
 * tokens are moved to the GPU predicted to hold their next-layer experts):
 * affinity[a][g] = sum over experts b of group g of trans[a][b], with trans
 * the layer-to-layer transition counts [E, E] of moe_transition.
 * affinity [E, G] int64 out.  Limits: E, G <= 1024. */
moe_status moe_group_affinity(const int32_t* trans, int E, const int32_t* group_of_expert, int G,
                              int64_t* affinity, moe_stream_t stream);

/* Predicted home group of each token: the group with the largest affinity
 * summed over the token's layer-1 experts idx1 [T, k1] (lower group on
 * ties).  home [T] int32 out.  Limits: k1 <= 32, E, G <= 1024. */
moe_status moe_predict_home(const int32_t* idx1, int T, int k1, const int64_t* affinity, int E, int G,
                            int32_t* home, moe_stream_t stream);

/* Assignments served on the token's own GPU: count += the slots of
 * expert_idx [T, k] whose expert's group equals the token's home group;
 * home [T] (moe_predict_home) or NULL for the sequence-sharded home
 * floor(t * G / T) ("Expert Parallelism > Key Parameters": L/E of the
 * assignments under uniform routing).  count [1] uint64, accumulated. */
moe_status moe_count_local(const int32_t* expert_idx, int T, int k, const int32_t* group_of_expert, int E, int G,
                           const int32_t* home, uint64_t* count, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBMOE_H */
