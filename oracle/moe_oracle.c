/*
 * moe_oracle.c - the CPU oracle for the MoE layer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this code; the library's product path never
 * calls it.  It shares no code with the CUDA library: plain, slow,
 * single-threaded C, double precision, loops written straight from the
 * definitions so that each can be checked against the pages by eye.
 *
 * Sources (page title, then section):
 *  [MegaDLMs]  "How MegaDLMs Implements Mixture of Experts (MoE) Architectures"
 *              - "MoELayer" (permutation -> expert computation -> unpermutation),
 *              - "Routing Mechanisms: Top-K vs Expert Choice" (TopKRouter,
 *                ExpertChoiceRouter), "Activation Checkpointing and
 *                Constraints" (no token dropping).
 *  [Coupling]  "Expert Coupling in MoE Pretraining: Reducing All-to-All
 *              Overhead with Correlated Placement and Token Shuffling" - Abstract
 *              (expert pairs chosen by the same token, layer-to-layer
 *              prediction, a dispatcher that ships a token to a given GPU
 *              at most one time).
 *  [EPKey]     "Expert Parallelism > Key Parameters" (top_k, capacity_factor,
 *              dropped tokens contribute zero, shared expert, L/E local share).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - top-k ties: the lower expert index wins; selection uses the raw fp32
 *    logits (softmax is strictly increasing within a row, so the chosen set
 *    is the same as on the probabilities).
 *  - gates are the softmax probabilities of the chosen experts; with
 *    norm_topk they are renormalised over the chosen k.
 *  - capacity = ceil(cf * T * k / E); cf <= 0 means unbounded.  An expert
 *    keeps its first `capacity` assignments in slot order (token order).
 *  - expert-choice scores are the per-token softmax; an expert takes the C
 *    tokens with the largest log-probability, lower token index on ties.
 *  - shared expert output is added with weight 1.
 *
 * All arrays are row-major.  bf16 values are passed as uint16 bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum { ORC_SWIGLU = 0, ORC_GELU = 1 };

/* ---------------------------------------------------------------- helpers */

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 value (ties to even), returned as a
 * double.  bf16 has an 8-bit significand: scale x so that the bits to keep
 * form an integer, round that integer half-to-even with rint(), scale back. */
static double round_to_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int ex;
    frexp(x, &ex);                 /* |x| in [2^(ex-1), 2^ex) */
    if (ex < -125) ex = -125;      /* below the normal range: fixed spacing 2^-133 */
    double scale = ldexp(1.0, 8 - ex);
    double r = rint(x * scale) / scale;   /* rint: round half to even (default mode) */
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, r);
    return r;
}

static double load_elem(const void* p, int dtype, int64_t i) {
    if (dtype == ORC_BF16) return bf16_bits_to_double(((const uint16_t*)p)[i]);
    return (double)((const float*)p)[i];
}

/* ------------------------------------------------ router linear gate */
/* [MegaDLMs] "Routing Mechanisms": the TopKRouter's scores are a linear
 * layer over the token's hidden state, one output per expert:
 * logits[t][e] = sum_c x[t][c] * W_r[e][c] (c ascending, double).
 * x: [T, d], W_r: [E, d] (dtype); logits: [T, E] doubles. */
void oracle_router_logits(const void* x, int dtype, int64_t T, int d, const void* W_r, int E, double* logits) {
    for (int64_t t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += load_elem(x, dtype, t * d + c) * load_elem(W_r, dtype, (int64_t)e * d + c);
            logits[t * E + e] = acc;
        }
}

/* ------------------------------------------------------- TopKRouter */
/* [MegaDLMs] "Routing Mechanisms": softmax over the expert logits, then the
 * top-k experts of each token; returns the probability weights (gates) and
 * the routing map (expert indices).  Slot j holds the (j+1)-th best expert
 * under (logit descending, expert index ascending). */
int oracle_route_topk(const float* logits, int64_t T, int E, int k, int norm_topk,
                      int32_t* expert_idx, float* gate) {
    if (k < 1 || k > E) return 1;
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * (int64_t)E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: lower index wins ties */
            }
            taken[best] = 1;
            expert_idx[t * k + j] = best;
        }
        /* softmax probabilities, in double */
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) if ((double)l[e] > m) m = (double)l[e];
        double denom = 0.0;
        if (norm_topk) {
            for (int j = 0; j < k; ++j) denom += exp((double)l[expert_idx[t * k + j]] - m);
        } else {
            for (int e = 0; e < E; ++e) denom += exp((double)l[e] - m);
        }
        for (int j = 0; j < k; ++j)
            gate[t * k + j] = (float)(exp((double)l[expert_idx[t * k + j]] - m) / denom);
    }
    free(taken);
    return 0;
}

/* ---------------------------------------------------- capacity */
/* [EPKey] "capacity_factor": each expert is given capacity_factor times the
 * average load T*k/E (rounded up to whole rows).  cf <= 0: unbounded, the
 * no-dropping mode of [MegaDLMs] "Activation Checkpointing and Constraints". */
int64_t oracle_capacity(double capacity_factor, int64_t T, int k, int E) {
    if (capacity_factor <= 0.0) return T * (int64_t)k;
    return (int64_t)ceil(capacity_factor * (double)T * (double)k / (double)E);
}

/* ------------------------------------------- token_permutation */
/* [MegaDLMs] "MoELayer" step 1 and "Token Dispatching": tokens are placed
 * into per-expert buckets.  [EPKey]: assignments beyond an expert's capacity
 * are dropped (row_map = -1).  Expert-major layout, packed: expert e owns
 * rows [offsets[e], offsets[e] + counts[e]) in ascending token order.
 *
 * Group-major layout (group_of_expert != NULL): [Coupling] Abstract, the
 * dispatcher that ships a token to a given GPU at most one time, on one
 * device: one row per distinct (token, group) with at least one kept assignment into that
 * group, ordered by group then token; every kept slot of the token into that
 * group maps to the row.  offsets has G+1 entries.
 *
 * Outputs: row_map [T*k], row_token [T*k] (first R used), counts [E] (kept),
 * load [E] (before capacity), offsets [E+1] or [G+1], *dropped, returns R. */
int64_t oracle_permute(const int32_t* expert_idx, int64_t T, int k, int E, int64_t capacity,
                       const int32_t* group_of_expert, int G,
                       int32_t* row_map, int32_t* row_token, int32_t* counts, int32_t* load,
                       int32_t* offsets, int64_t* dropped) {
    const int64_t S = T * (int64_t)k;
    unsigned char* kept = (unsigned char*)malloc((size_t)(S > 0 ? S : 1));
    for (int e = 0; e < E; ++e) load[e] = 0;
    /* rank of each slot among its expert's slots in slot (= token) order */
    for (int64_t s = 0; s < S; ++s) {
        int e = expert_idx[s];
        int64_t rank = load[e]++;
        kept[s] = rank < capacity;
    }
    int64_t drop = 0;
    for (int e = 0; e < E; ++e) {
        counts[e] = (int32_t)(load[e] < capacity ? load[e] : capacity);
        drop += load[e] - counts[e];
    }
    *dropped = drop;
    int64_t R = 0;
    if (group_of_expert == NULL) {
        int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
        offsets[0] = 0;
        for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
        for (int e = 0; e < E; ++e) pos[e] = offsets[e];
        for (int64_t s = 0; s < S; ++s) {
            if (!kept[s]) { row_map[s] = -1; continue; }
            int64_t r = pos[expert_idx[s]]++;
            row_map[s] = (int32_t)r;
            row_token[r] = (int32_t)(s / k);
        }
        R = offsets[E];
        free(pos);
    } else {
        for (int64_t s = 0; s < S; ++s) row_map[s] = -1;
        for (int g = 0; g < G; ++g) {
            offsets[g] = (int32_t)R;
            for (int64_t t = 0; t < T; ++t) {
                int has = 0;
                for (int j = 0; j < k; ++j) {
                    int64_t s = t * k + j;
                    if (kept[s] && group_of_expert[expert_idx[s]] == g) {
                        row_map[s] = (int32_t)R;
                        has = 1;
                    }
                }
                if (has) { row_token[R] = (int32_t)t; ++R; }
            }
        }
        offsets[G] = (int32_t)R;
    }
    free(kept);
    return R;
}

/* buffer[r] = x[row_token[r]], byte for byte. */
void oracle_gather_rows(const void* x, int64_t row_bytes, const int32_t* row_token, int64_t R, void* buffer) {
    for (int64_t r = 0; r < R; ++r)
        memcpy((char*)buffer + r * row_bytes, (const char*)x + (int64_t)row_token[r] * row_bytes, (size_t)row_bytes);
}

/* -------------------------------------------------- expert FFN */
/* [MegaDLMs] "MoELayer" step 2: each expert on the device runs on its rows;
 * the experts are MLPs.  SwiGLU MLP: h = silu(W1 x) * (W3 x), y = W2 h;
 * GELU MLP: h = gelu(W1 x), y = W2 h, gelu(z) = z * Phi(z) (erf form).
 * [EPKey] "shared expert": the same MLP applied to every token.
 * For bf16 activations h is rounded to bf16 before W2 (h is a bf16 tensor),
 * and y is rounded to bf16; fp32 activations are not rounded.
 *
 * x: [n, d] rows; row_expert[i]: the expert of row i; W1/W3: [E, F, d];
 * W2: [E, d, F]; y: [n, d] doubles (already rounded to the activation dtype). */
static double silu(double z) { return z / (1.0 + exp(-z)); }
static double gelu(double z) { return 0.5 * z * (1.0 + erf(z / sqrt(2.0))); }

void oracle_expert_ffn_rows(const void* x, int dtype, int64_t n, int d, int F,
                            const int32_t* row_expert, const void* W1, const void* W3,
                            const void* W2, int act, double* y) {
    double* xr = (double*)malloc(sizeof(double) * (size_t)d);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    for (int64_t i = 0; i < n; ++i) {
        const int64_t e = row_expert[i];
        for (int c = 0; c < d; ++c) xr[c] = load_elem(x, dtype, i * d + c);
        for (int f = 0; f < F; ++f) {
            const int64_t wrow = (e * F + f) * (int64_t)d;
            double a = 0.0;
            for (int c = 0; c < d; ++c) a += load_elem(W1, dtype, wrow + c) * xr[c];
            double v;
            if (act == ORC_SWIGLU) {
                double b = 0.0;
                for (int c = 0; c < d; ++c) b += load_elem(W3, dtype, wrow + c) * xr[c];
                v = silu(a) * b;
            } else {
                v = gelu(a);
            }
            h[f] = (dtype == ORC_BF16) ? round_to_bf16(v) : v;
        }
        for (int c = 0; c < d; ++c) {
            const int64_t wrow = (e * d + c) * (int64_t)F;
            double acc = 0.0;
            for (int f = 0; f < F; ++f) acc += load_elem(W2, dtype, wrow + f) * h[f];
            y[i * d + c] = (dtype == ORC_BF16) ? round_to_bf16(acc) : acc;
        }
    }
    free(xr);
    free(h);
}

/* ---------------------------------------------- token_unpermutation */
/* [MegaDLMs] "MoELayer" step 3: the output sequence is rebuilt from the
 * expert outputs, each token's expert outputs weighted by its gates and
 * summed (slot order j = 0..k-1).  [EPKey]: a dropped assignment
 * (row_map = -1) contributes zero.  shared (may be NULL): [T, d], weight 1.
 * Y: [R, d] (dtype); out: [T, d] doubles. */
void oracle_unpermute(const void* Y, int dtype, int64_t T, int d, int k, const int32_t* row_map,
                      const float* gate, const void* shared, double* out) {
    for (int64_t t = 0; t < T; ++t) {
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int32_t r = row_map[t * k + j];
                if (r < 0) continue;
                acc += (double)gate[t * k + j] * load_elem(Y, dtype, (int64_t)r * d + c);
            }
            if (shared) acc += load_elem(shared, dtype, t * d + c);
            out[t * d + c] = acc;
        }
    }
}

/* ------------------------------------------- group-major expert path */
/* [Coupling] Abstract: the dispatcher ships a token to a given GPU at most
 * one time.  With real experts behind it, each GPU receives one row per
 * (token, group), runs the token's experts that it holds, and returns one
 * row: the gate-weighted sum of those experts' outputs.  The token's output
 * is the sum of its returned rows - the same sum as the plain unpermutation,
 * grouped by GPU.  The returned row is a tensor of the activation dtype, so
 * for bf16 it is rounded to bf16 (as the expert outputs are).  */

/* dst[dst_row[s]] = src[src_row[s]] byte for byte, for every slot with both
 * rows valid (>= 0). */
void oracle_copy_slot_rows(const void* src, int64_t row_bytes, const int32_t* src_row, const int32_t* dst_row,
                           int64_t S, void* dst) {
    for (int64_t s = 0; s < S; ++s) {
        if (src_row[s] < 0 || dst_row[s] < 0) continue;
        memcpy((char*)dst + (int64_t)dst_row[s] * row_bytes, (const char*)src + (int64_t)src_row[s] * row_bytes,
               (size_t)row_bytes);
    }
}

/* P[r] for each group row r = sum over the slots j of its token with
 * row_map_g[t, j] = r (slot order) of gate[t, j] * Y_e[row_map_e[t, j]];
 * rounded to bf16 when dtype is bf16.  Rows no slot maps to are left as
 * they are.  Y_e: [R_e, d] dtype; P: [R_g, d] doubles. */
void oracle_group_precombine(const void* Y_e, int dtype, int64_t T, int d, int k, const int32_t* row_map_e,
                             const int32_t* row_map_g, const float* gate, double* P) {
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            const int32_t r = row_map_g[t * k + j];
            if (r < 0) continue;
            int first = 1;                       /* has an earlier slot of t already produced row r? */
            for (int i = 0; i < j; ++i)
                if (row_map_g[t * k + i] == r) first = 0;
            if (!first) continue;
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int q = j; q < k; ++q) {
                    if (row_map_g[t * k + q] != r) continue;
                    acc += (double)gate[t * k + q] * load_elem(Y_e, dtype, (int64_t)row_map_e[t * k + q] * d + c);
                }
                P[(int64_t)r * d + c] = (dtype == ORC_BF16) ? round_to_bf16(acc) : acc;
            }
        }
    }
}

/* out[t] = sum of the token's distinct group rows (each once, in the order
 * they first appear among its slots) + shared[t] (weight 1, may be NULL).
 * Y_g: [R_g, d] dtype; out: [T, d] doubles. */
void oracle_unpermute_groups(const void* Y_g, int dtype, int64_t T, int d, int k, const int32_t* row_map_g,
                             const void* shared, double* out) {
    for (int64_t t = 0; t < T; ++t) {
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                const int32_t r = row_map_g[t * k + j];
                if (r < 0) continue;
                int first = 1;
                for (int i = 0; i < j; ++i)
                    if (row_map_g[t * k + i] == r) first = 0;
                if (first) acc += load_elem(Y_g, dtype, (int64_t)r * d + c);
            }
            if (shared) acc += load_elem(shared, dtype, t * d + c);
            out[t * d + c] = acc;
        }
    }
}

/* ---------------------------------------------- ExpertChoiceRouter */
/* [MegaDLMs] "Routing Mechanisms": the selection is inverted, every expert
 * picking the tokens that score highest for it.  Scores: per-token softmax over experts,
 * compared through key = logit - logsumexp (same order as the probability,
 * computed in double, sum over e in ascending order).  Expert e keeps the C
 * tokens with the largest key (lower token index on equal keys), stored in
 * ascending token order: rows e*C .. e*C+C-1.  gate = exp(key).
 * Token CSR: tok_ptr [T+1]; tok_row lists each token's rows by ascending e. */
static const double* g_keys;   /* single-threaded qsort context */
static int g_E, g_e;

static int cmp_key_desc(const void* a, const void* b) {
    int32_t ta = *(const int32_t*)a, tb = *(const int32_t*)b;
    double ka = g_keys[(int64_t)ta * g_E + g_e], kb = g_keys[(int64_t)tb * g_E + g_e];
    if (ka > kb) return -1;
    if (ka < kb) return 1;
    return (ta > tb) - (ta < tb);
}

static int cmp_int_asc(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

int oracle_route_ec(const float* logits, int64_t T, int E, int C,
                    int32_t* ec_token, float* ec_gate, int32_t* tok_ptr, int32_t* tok_row) {
    if (C < 1 || C > T) return 1;
    double* key = (double*)malloc(sizeof(double) * (size_t)(T * E));
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * (int64_t)E;
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) if ((double)l[e] > m) m = (double)l[e];
        double s = 0.0;
        for (int e = 0; e < E; ++e) s += exp((double)l[e] - m);
        double lse = m + log(s);
        for (int e = 0; e < E; ++e) key[t * E + e] = (double)l[e] - lse;
    }
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
    g_keys = key;
    g_E = E;
    for (int e = 0; e < E; ++e) {
        for (int64_t t = 0; t < T; ++t) order[t] = (int32_t)t;
        g_e = e;
        qsort(order, (size_t)T, sizeof(int32_t), cmp_key_desc);
        qsort(order, (size_t)C, sizeof(int32_t), cmp_int_asc);
        for (int i = 0; i < C; ++i) {
            ec_token[(int64_t)e * C + i] = order[i];
            ec_gate[(int64_t)e * C + i] = (float)exp(key[(int64_t)order[i] * E + e]);
        }
    }
    /* token CSR, experts ascending */
    int32_t* cnt = (int32_t*)calloc((size_t)T, sizeof(int32_t));
    for (int64_t r = 0; r < (int64_t)E * C; ++r) cnt[ec_token[r]]++;
    tok_ptr[0] = 0;
    for (int64_t t = 0; t < T; ++t) tok_ptr[t + 1] = tok_ptr[t] + cnt[t];
    for (int64_t t = 0; t < T; ++t) cnt[t] = 0;
    for (int e = 0; e < E; ++e)
        for (int i = 0; i < C; ++i) {
            int64_t r = (int64_t)e * C + i;
            int32_t t = ec_token[r];
            tok_row[tok_ptr[t] + cnt[t]++] = (int32_t)r;
        }
    free(cnt);
    free(order);
    free(key);
    return 0;
}

/* Expert-choice unpermutation: y[t] = sum over the token's rows (ascending
 * expert) of ec_gate[row] * Y[row]; tokens no expert chose get 0. */
void oracle_unpermute_ec(const void* Y, int dtype, int64_t T, int d, const int32_t* tok_ptr,
                         const int32_t* tok_row, const float* ec_gate, double* out) {
    for (int64_t t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int32_t p = tok_ptr[t]; p < tok_ptr[t + 1]; ++p) {
                int32_t r = tok_row[p];
                acc += (double)ec_gate[r] * load_elem(Y, dtype, (int64_t)r * d + c);
            }
            out[t * d + c] = acc;
        }
}

/* ------------------------------------------------ co-selection */
/* [Coupling] Abstract: pairs of experts that one token picks jointly.
 * cosel[a][b] += 1 for every ordered pair of the token's slots (a from slot
 * i, b from slot j); the diagonal (i == j) is each expert's load.  Counts are
 * accumulated into cosel [E, E] and use the routing decisions before
 * capacity. */
void oracle_coselect(const int32_t* expert_idx, int64_t T, int k, int E, int32_t* cosel) {
    for (int64_t t = 0; t < T; ++t)
        for (int i = 0; i < k; ++i)
            for (int j = 0; j < k; ++j)
                cosel[(int64_t)expert_idx[t * k + i] * E + expert_idx[t * k + j]] += 1;
}

/* ------------------------------------------ layer transition */
/* [Coupling] Abstract: a token's expert choices in one layer are predictive
 * of its choices in the following layer.  trans[a][b] += 1 for every a among the
 * token's layer-1 experts and b among its layer-2 experts (accumulated). */
void oracle_transition(const int32_t* idx1, int k1, const int32_t* idx2, int k2, int64_t T, int E,
                       int32_t* trans) {
    for (int64_t t = 0; t < T; ++t)
        for (int i = 0; i < k1; ++i)
            for (int j = 0; j < k2; ++j)
                trans[(int64_t)idx1[t * k1 + i] * E + idx2[t * k2 + j]] += 1;
}

/* -------------------------------------------- local share (statistic) */
/* [EPKey] "num_local_experts": with L of E experts local, L/E of token-expert
 * pairs route locally under uniform routing.  Token t's home group is
 * floor(t * G / T); returns the fraction of slots whose expert lies in it. */
double oracle_local_fraction(const int32_t* expert_idx, int64_t T, int k, const int32_t* group_of_expert, int G) {
    int64_t local = 0;
    for (int64_t t = 0; t < T; ++t) {
        int64_t home = t * G / T;
        for (int j = 0; j < k; ++j)
            if (group_of_expert[expert_idx[t * k + j]] == home) ++local;
    }
    return T > 0 ? (double)local / (double)(T * k) : 0.0;
}

/* Exposed for the pin tests of the activation helpers. */
double oracle_silu(double z) { return silu(z); }
double oracle_gelu(double z) { return gelu(z); }
double oracle_round_bf16(double x) { return round_to_bf16(x); }

/* -------------------------------------------- correlated placement */
/* [Coupling] Abstract: experts that tokens often pick together are placed on
 * the same GPU.  The pages give no algorithm; this is a plain greedy reading
 * on the co-selection counts C (symmetric, E x E) for G groups of L = E/G:
 * each group starts from the unassigned expert with the largest off-diagonal
 * co-selection mass and grows by the unassigned expert with the largest
 * summed co-selection with the group's members; ties go to the lower index.
 * Returns 0, or 1 if G does not divide E. */
int oracle_place_experts(const int32_t* cosel, int E, int G, int32_t* group_of_expert) {
    if (G < 1 || E % G != 0) return 1;
    const int L = E / G;
    int64_t* mass = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    int64_t* aff = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    for (int x = 0; x < E; ++x) {
        group_of_expert[x] = -1;
        for (int y = 0; y < E; ++y)
            if (y != x) mass[x] += cosel[(int64_t)x * E + y];
    }
    for (int g = 0; g < G; ++g) {
        int seed = -1;
        for (int x = 0; x < E; ++x)
            if (group_of_expert[x] < 0 && (seed < 0 || mass[x] > mass[seed])) seed = x;
        group_of_expert[seed] = g;
        for (int x = 0; x < E; ++x) aff[x] = cosel[(int64_t)x * E + seed];
        for (int m = 1; m < L; ++m) {
            int best = -1;
            for (int x = 0; x < E; ++x)
                if (group_of_expert[x] < 0 && (best < 0 || aff[x] > aff[best])) best = x;
            group_of_expert[best] = g;
            for (int x = 0; x < E; ++x) aff[x] += cosel[(int64_t)x * E + best];
        }
    }
    free(mass);
    free(aff);
    return 0;
}

/* ------------------------------------------ token shuffling statistic */
/* [Coupling] Abstract: a token is moved to the GPU predicted to hold its
 * next-layer experts.  Prediction from the layer-to-layer transition counts
 * M: affinity[a][g] = sum of M[a][b] over the experts b of group g. */
void oracle_group_affinity(const int32_t* trans, int E, const int32_t* group_of_expert, int G, int64_t* affinity) {
    for (int64_t i = 0; i < (int64_t)E * G; ++i) affinity[i] = 0;
    for (int a = 0; a < E; ++a)
        for (int b = 0; b < E; ++b)
            affinity[(int64_t)a * G + group_of_expert[b]] += trans[(int64_t)a * E + b];
}

/* A token's predicted home group: the group with the largest summed affinity
 * over its layer-1 experts (lower group on ties). */
void oracle_predict_home(const int32_t* idx1, int64_t T, int k1, const int64_t* affinity, int G, int32_t* home) {
    for (int64_t t = 0; t < T; ++t) {
        int best = 0;
        int64_t best_v = 0;
        for (int g = 0; g < G; ++g) {
            int64_t v = 0;
            for (int i = 0; i < k1; ++i) v += affinity[(int64_t)idx1[t * k1 + i] * G + g];
            if (g == 0 || v > best_v) { best = g; best_v = v; }
        }
        home[t] = best;
    }
}

/* Slots served on the token's own GPU: assignments whose expert lies in the
 * token's home group; home == NULL means the sequence-sharded home
 * floor(t * G / T) ([EPKey] L/E baseline; [Coupling] 12.5% on one node). */
int64_t oracle_count_local(const int32_t* expert_idx, int64_t T, int k, const int32_t* group_of_expert, int G,
                           const int32_t* home) {
    int64_t local = 0;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t h = home ? home[t] : t * G / T;
        for (int j = 0; j < k; ++j)
            if (group_of_expert[expert_idx[t * k + j]] == h) ++local;
    }
    return local;
}
