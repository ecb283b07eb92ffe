/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for the MoE
 * routing hot path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline leg load it; the product path never does, and
 * this file shares no code, header, table or helper with the CUDA library.
 *
 * Every function follows the plain definition of its step, in double
 * precision unless the step itself is defined in fp32 (selection keys,
 * combine weights, the bias step, the FP8 encoding).  There is no blocking,
 * fusion or reordering: loops run in the index order of the definition.
 * OpenMP only splits independent tokens across threads; no token's
 * arithmetic depends on the split.
 *
 * Sources (web pages on MoE load balancing):
 *  [ENT] "MoE Routing Entropy vs Expert Saturation: Optimizing DeepSeek V4
 *        Load Balancing" (dailyaiworld.com): softmax and Shannon-entropy
 *        equations (section "The Mathematics: Router Entropy and Gating
 *        Imbalance"), the DynamicEntropyMoERouter (section "Concrete
 *        Implementation"), the 1.25 capacity factor (section "Production
 *        Testing: The All-Gather Deadlock").
 *  [HD]  "DeepSeek V4 MoE load balancing" (blog.hotdry.top): sigmoid affinity
 *        and weighted combine (section "Token routing and Top-K selection"),
 *        per-expert bias used for routing only and its direction of update
 *        (section "Auxiliary-loss-free load balancing"), redundant experts,
 *        FP8 dispatch / BF16 combine (section "DeepEP").
 *  [GL]  "DeepSeek-V3 Group-Limited Expert Routing" (cnnetsun.cn): 256 experts
 *        in 8 groups, best 4 groups, then top-8 among their 128 experts
 *        (section 1, and the Gate description in section 3).
 *  [MIN] "A minimal experiment in expert-load imbalance" (tech-blog-chi):
 *        total / max / max-over-mean imbalance / fixed capacity = max * N
 *        (sections "Run the example" and "Expected output").
 *
 * Readings where the pages leave a step open (each one is also listed in
 * the design notes): group score = sum of the group's top-n (n = 2) biased
 * keys; groups outside the kept set are excluded (not zeroed); ties go to
 * the lower index; combine weights use the unbiased scores; the bias step is
 * b -= u * sign(c_e - T*K/N) with sign(0) = 0; the order of rows inside an
 * expert segment is ascending flat (t,k); FP8 is e4m3 with one fp32 scale
 * per row and 128-channel block, scale = amax / 448.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ---------------------------------------------------------------------------
 * Gate logits [ENT] "The Mathematics": h_i = x . W_g, with the gate an
 * nn.Linear(hidden, N, bias=False) ([ENT] "Concrete Implementation"), so
 * W is stored [N, d] and h[t,e] = sum_j x[t,j] * W[e,j].  A per-expert logit
 * offset (workload recipe: celebrity experts, Zipf popularity) is added.
 * Inputs are the exact bf16/fp32 values widened to float; the sum is double,
 * in j order.
 * ------------------------------------------------------------------------- */
void oracle_logits(const float* x, const float* W, const float* off,
                   int64_t T, int64_t d, int64_t N, double* h) {
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        for (int64_t e = 0; e < N; ++e) {
            double acc = 0.0;
            for (int64_t j = 0; j < d; ++j)
                acc += (double)x[t * d + j] * (double)W[e * d + j];
            if (off) acc += (double)off[e];
            h[t * N + e] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Affinity scores, computed in double and rounded once to fp32.
 *  fn 0: softmax over the N experts ([ENT] "The Mathematics", softmax
 *        equation), evaluated as exp(h - max) / sum exp(h - max).
 *  fn 1: sigmoid 1 / (1 + exp(-h)) ([HD] "Token routing": sigmoid gating so a
 *        token may go to several experts without mutual exclusion).
 * ------------------------------------------------------------------------- */
void oracle_scores(const double* h, int64_t T, int64_t N, int fn, float* s) {
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        const double* row = h + t * N;
        if (fn == 0) {
            double mx = row[0];
            for (int64_t e = 1; e < N; ++e) if (row[e] > mx) mx = row[e];
            double den = 0.0;
            for (int64_t e = 0; e < N; ++e) den += exp(row[e] - mx);
            for (int64_t e = 0; e < N; ++e) s[t * N + e] = (float)(exp(row[e] - mx) / den);
        } else {
            for (int64_t e = 0; e < N; ++e) s[t * N + e] = (float)(1.0 / (1.0 + exp(-row[e])));
        }
    }
}

/* (key desc, index asc): the total order used for every "top" choice. */
static int beats(float ka, int ia, float kb, int ib) {
    return (ka > kb) || (ka == kb && ia < ib);
}

/* ---------------------------------------------------------------------------
 * Selection, on fp32 scores s[T,N] and an optional fp32 bias b[N].
 *  1. key_e = fp32(s_e + b_e)     ([HD] "Auxiliary-loss-free load balancing":
 *                                  the bias joins the affinity for the
 *                                  routing decision only)
 *  2. n_groups > 1: group score = fp32 sum, largest first, of the group's
 *     group_topn largest keys; keep the topk_groups best groups by
 *     (score desc, group asc); experts of the other groups are not
 *     candidates ([GL] section 1 and section 3).
 *  3. The K best candidates by (key desc, index asc), output in that order
 *     ([ENT] "Concrete Implementation", torch.topk).
 *  4. Weights from the UNBIASED scores: renorm ? s_k / sum_k' s_k' : s_k,
 *     times route_scale, each op rounded to fp32; the sum runs in k order
 *     ([ENT] "Concrete Implementation", renormalisation of the top-K weights).
 * Returns 0, or -1 on an invalid configuration.
 * ------------------------------------------------------------------------- */
int oracle_select(const float* s, const float* bias, int64_t T, int N, int K,
                  int n_groups, int topk_groups, int group_topn, int renorm,
                  float route_scale, int32_t* idx, float* w) {
    if (N <= 0 || K <= 0 || K > N || n_groups <= 0 || N % n_groups) return -1;
    const int gsize = N / n_groups;
    if (n_groups > 1 && (topk_groups <= 0 || topk_groups > n_groups ||
                         topk_groups * gsize < K || group_topn <= 0 || group_topn > gsize))
        return -1;
    int64_t t;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (t = 0; t < T; ++t) {
        float* key = (float*)malloc(sizeof(float) * (size_t)N);
        int* cand = (int*)malloc(sizeof(int) * (size_t)N);
        int* gkeep = (int*)malloc(sizeof(int) * (size_t)n_groups);
        float* gs = (float*)malloc(sizeof(float) * (size_t)n_groups);
        float* tmp = (float*)malloc(sizeof(float) * (size_t)gsize);
        int* taken = (int*)malloc(sizeof(int) * (size_t)N);
        if (!key || !cand || !gkeep || !gs || !tmp || !taken) { bad |= 1; goto next; }

        for (int e = 0; e < N; ++e) {
            float b = bias ? bias[e] : 0.0f;
            key[e] = s[t * N + e] + b; /* one fp32 add */
        }
        for (int g = 0; g < n_groups; ++g) gkeep[g] = 1;
        if (n_groups > 1) {
            for (int g = 0; g < n_groups; ++g) {
                /* group_topn largest keys of the group, by repeated maximum */
                for (int i = 0; i < gsize; ++i) tmp[i] = key[g * gsize + i];
                float sum = 0.0f;
                for (int r = 0; r < group_topn; ++r) {
                    int best = 0;
                    for (int i = 1; i < gsize; ++i) if (tmp[i] > tmp[best]) best = i;
                    sum = (r == 0) ? tmp[best] : sum + tmp[best];
                    tmp[best] = -INFINITY;
                }
                gs[g] = sum;
            }
            for (int g = 0; g < n_groups; ++g) {
                int rank = 0; /* how many groups beat group g */
                for (int h2 = 0; h2 < n_groups; ++h2)
                    if (h2 != g && beats(gs[h2], h2, gs[g], g)) ++rank;
                gkeep[g] = rank < topk_groups;
            }
        }
        for (int e = 0; e < N; ++e) { cand[e] = gkeep[e / gsize]; taken[e] = 0; }

        float ssum = 0.0f;
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < N; ++e) {
                if (!cand[e] || taken[e]) continue;
                if (best < 0 || beats(key[e], e, key[best], best)) best = e;
            }
            taken[best] = 1;
            idx[t * K + k] = best;
            ssum = (k == 0) ? s[t * N + best] : ssum + s[t * N + best];
        }
        for (int k = 0; k < K; ++k) {
            float sk = s[t * N + idx[t * K + k]];
            float v = renorm ? sk / ssum : sk;
            w[t * K + k] = v * route_scale;
        }
    next:
        free(key); free(cand); free(gkeep); free(gs); free(tmp); free(taken);
    }
    return bad ? -1 : 0;
}

/* ---------------------------------------------------------------------------
 * Load histogram: c_e = #{(t,k) : slot(t,k) = e}  ([ENT] "Concrete
 * Implementation", bincount of the selected experts).  A negative slot is an
 * assignment dropped by the capacity limit ([ENT] "Production Testing") and
 * counts nowhere.
 * ------------------------------------------------------------------------- */
int oracle_histogram(const int32_t* slot, int64_t A, int n_slots, int64_t* counts) {
    for (int e = 0; e < n_slots; ++e) counts[e] = 0;
    for (int64_t a = 0; a < A; ++a) {
        if (slot[a] < 0) continue;
        if (slot[a] >= n_slots) return -1;
        counts[slot[a]] += 1;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Load statistics from a histogram, all in double.
 *  out[0] total      = sum c                       [MIN] "Run the example"
 *  out[1] max        = max c                       [MIN]
 *  out[2] mean       = total / n_slots             [MIN]; also the target
 *                                                  load T*K/N of [ENT]
 *  out[3] imbalance  = max / mean, 0 if mean == 0  [MIN]
 *  out[4] std / mean (population std, 0 if mean == 0)
 *                                                  [HD] "Deployment
 *                                                  parameters and monitoring"
 *  out[5] H_load     = -sum_{c>0} p log2 p, p = c / total
 *                                                  [ENT] entropy equation
 *  out[6] capacity_fixed = max * n_slots           [MIN]
 *  out[7] capacity_125   = 1.25 * mean             [ENT] "Production Testing"
 * ------------------------------------------------------------------------- */
void oracle_load_stats(const int64_t* counts, int n_slots, double* out) {
    double total = 0.0, mx = 0.0;
    for (int e = 0; e < n_slots; ++e) {
        total += (double)counts[e];
        if ((double)counts[e] > mx) mx = (double)counts[e];
    }
    double mean = n_slots > 0 ? total / (double)n_slots : 0.0;
    double var = 0.0;
    for (int e = 0; e < n_slots; ++e) {
        double dlt = (double)counts[e] - mean;
        var += dlt * dlt;
    }
    var = n_slots > 0 ? var / (double)n_slots : 0.0;
    double H = 0.0;
    for (int e = 0; e < n_slots; ++e) {
        if (counts[e] > 0) {
            double p = (double)counts[e] / total;
            H -= p * log2(p);
        }
    }
    out[0] = total;
    out[1] = mx;
    out[2] = mean;
    out[3] = mean > 0.0 ? mx / mean : 0.0;
    out[4] = mean > 0.0 ? sqrt(var) / mean : 0.0;
    out[5] = H;
    out[6] = mx * (double)n_slots;
    out[7] = 1.25 * mean;
}

/* ---------------------------------------------------------------------------
 * Score entropy ([ENT] "Concrete Implementation", compute_routing_entropy):
 * H_score = -sum_e m_e log2 m_e with m_e = mean_t p[t,e].  p is the softmax
 * itself (fn 0) or, for sigmoid scores, each token's scores divided by their
 * sum (fn 1).  The page's +1e-9 is dropped; 0 log 0 = 0.
 * ------------------------------------------------------------------------- */
double oracle_score_entropy(const float* s, int64_t T, int N, int fn) {
    double* m = (double*)calloc((size_t)N, sizeof(double));
    if (!m) return NAN;
    for (int64_t t = 0; t < T; ++t) {
        double rs = 1.0;
        if (fn == 1) {
            rs = 0.0;
            for (int e = 0; e < N; ++e) rs += (double)s[t * N + e];
        }
        for (int e = 0; e < N; ++e) m[e] += (double)s[t * N + e] / rs;
    }
    double H = 0.0;
    for (int e = 0; e < N; ++e) {
        double me = m[e] / (double)T;
        if (me > 0.0) H -= me * log2(me);
    }
    free(m);
    return H;
}

/* ---------------------------------------------------------------------------
 * Redundant experts ([HD] "Auxiliary-loss-free load balancing": hot experts
 * are replicated for prefill; [GL] section 2: 32 redundant experts).
 * The n_rep hottest experts by (count desc, index asc) get replica slots
 * N, N+1, ... in that order; replica_slot[e] = -1 for the others.
 * ------------------------------------------------------------------------- */
void oracle_replica_plan(const int64_t* counts, int N, int n_rep, int32_t* replica_slot) {
    for (int e = 0; e < N; ++e) replica_slot[e] = -1;
    int* used = (int*)calloc((size_t)N, sizeof(int));
    for (int j = 0; j < n_rep && j < N; ++j) {
        int best = -1;
        for (int e = 0; e < N; ++e) {
            if (used[e]) continue;
            if (best < 0 || counts[e] > counts[best]) best = e;
        }
        used[best] = 1;
        replica_slot[best] = N + j;
    }
    free(used);
}

/* A token t routed to a replicated expert goes to the replica when t is odd,
 * to the original when t is even (alternation by token index). */
void oracle_apply_replicas(const int32_t* idx, int64_t T, int K,
                           const int32_t* replica_slot, int32_t* slot) {
    for (int64_t t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            int32_t e = idx[t * K + k];
            int32_t r = (replica_slot && e >= 0) ? replica_slot[e] : -1;
            slot[t * K + k] = (r >= 0 && (t & 1)) ? r : e;
        }
}

/* ---------------------------------------------------------------------------
 * Expert-contiguous layout ([HD] "DeepEP": dispatch sends each token to its
 * experts, combine brings the results back).  offsets = exclusive prefix of
 * counts (n_slots + 1 entries); walking the flat assignments a = t*K + k in
 * ascending order, pos[a] = offsets[e] + rank[a] with rank[a] the number of
 * earlier assignments to the same slot; row_src[pos[a]] = t.  A dropped
 * assignment (negative slot) gets rank = pos = -1 and no row.
 * ------------------------------------------------------------------------- */
void oracle_positions(const int32_t* slot, int64_t T, int K, const int64_t* counts,
                      int n_slots, int64_t* offsets, int64_t* pos, int64_t* rank,
                      int64_t* row_src) {
    offsets[0] = 0;
    for (int e = 0; e < n_slots; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t* seen = (int64_t*)calloc((size_t)n_slots, sizeof(int64_t));
    for (int64_t a = 0; a < T * K; ++a) {
        int32_t e = slot[a];
        if (e < 0) { rank[a] = -1; pos[a] = -1; continue; }
        rank[a] = seen[e];
        pos[a] = offsets[e] + seen[e];
        seen[e] += 1;
        row_src[pos[a]] = a / K;
    }
    free(seen);
}

/* rows[pos[t,k]] = x[t]: a byte copy of each token row, K times (dropped
 * assignments, pos < 0, copy nothing). */
void oracle_dispatch_rows(const uint8_t* x, int64_t T, int64_t row_bytes, int K,
                          const int64_t* pos, uint8_t* rows) {
    for (int64_t t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k)
            if (pos[t * K + k] >= 0) memcpy(rows + pos[t * K + k] * row_bytes, x + t * row_bytes, (size_t)row_bytes);
}

/* ---------------------------------------------------------------------------
 * FP8 E4M3 encoding, written from the OCP 8-bit floating point format
 * definition: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; largest finite 448 = 1.75 * 2^8; smallest
 * normal 2^-6; subnormals m/8 * 2^-6; smallest subnormal 2^-9.
 * Round to nearest, ties to even, saturating to +-448 ("satfinite").
 *
 * Method: for |v| in the normal range with unbiased exponent E (-6..8) the
 * representable spacing is 2^(E-3); below 2^-6 it is 2^-9.  Divide by the
 * spacing (exact: a power of two), round to nearest-even with rint() in
 * double (default rounding mode), and rebuild the code.  A carry into the
 * next binade is handled because the rebuilt value is re-encoded from its
 * integer multiple of the spacing.
 * ------------------------------------------------------------------------- */
uint8_t oracle_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int E;
    if (a < ldexp(1.0, -6)) {
        E = -6; /* subnormal spacing 2^-9 */
    } else {
        E = (int)floor(log2(a));
        /* guard against log2 rounding at exact powers of two */
        if (ldexp(1.0, E) > a) E -= 1;
        if (ldexp(1.0, E + 1) <= a) E += 1;
    }
    double q = rint(a / ldexp(1.0, E - 3)); /* integer multiple of the spacing */
    double val = q * ldexp(1.0, E - 3);
    if (val >= 448.0) return (uint8_t)(sign | 0x7E);
    if (val == 0.0) return sign;
    if (val < ldexp(1.0, -6)) {
        /* subnormal: exponent field 0, mantissa = val / 2^-9 */
        int m = (int)(val / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    int e2 = (int)floor(log2(val));
    if (ldexp(1.0, e2) > val) e2 -= 1;
    if (ldexp(1.0, e2 + 1) <= val) e2 += 1;
    int m = (int)(val / ldexp(1.0, e2 - 3)) - 8; /* 1.mmm * 2^e2 */
    return (uint8_t)(sign | ((e2 + 7) << 3) | m);
}

float oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 0xF && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Per row and per block of 128 channels ([HD] "DeepEP": FP8 dispatch):
 * amax = max |v| (fp32), inv = amax > 0 ? fp32(448 / amax) : 0,
 * q = e4m3(fp32(v * inv)), scale = fp32(amax / 448). */
void oracle_fp8_rows(const float* rows, int64_t R, int64_t d, uint8_t* q, float* scales) {
    const int64_t nb = d / 128;
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < R; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* v = rows + r * d + b * 128;
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i) {
                float av = fabsf(v[i]);
                if (av > amax) amax = av;
            }
            float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
            for (int i = 0; i < 128; ++i) {
                float p = v[i] * inv;
                q[r * d + b * 128 + i] = oracle_e4m3_encode(p);
            }
            scales[r * nb + b] = amax / 448.0f;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Combine ([HD] "Token routing": expert outputs are summed weighted by their
 * affinity; "DeepEP": combine returns them to the token's place):
 * out[t] = sum_k w[t,k] * y[pos[t,k]], in double, k order; dropped
 * assignments (pos < 0) contribute nothing.
 * ------------------------------------------------------------------------- */
void oracle_combine(const float* y, const int64_t* pos, const float* w, int64_t T,
                    int K, int64_t d, double* out) {
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t)
        for (int64_t j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                if (pos[t * K + k] >= 0) acc += (double)w[t * K + k] * (double)y[pos[t * K + k] * d + j];
            out[t * d + j] = acc;
        }
}

/* ---------------------------------------------------------------------------
 * Bias update ([HD] "Auxiliary-loss-free load balancing": lower the bias of
 * overloaded experts, raise it for underloaded ones).
 *  mode 0 (sign rule): sgn = sign(c_e - total/N) decided exactly on integers
 *         (c_e * N vs total); b_e = fp32(b_e - fp32(u * sgn)).
 *  mode 1 (the DynamicEntropyMoERouter rule of [ENT] "Concrete
 *         Implementation"): target = total / N, err = c_e - target,
 *         b_e -= u * sign(err) * (|err| / target), every op in fp32 in that
 *         order (u plays the role of bias_decay).
 * ------------------------------------------------------------------------- */
void oracle_bias_update(const int64_t* counts, int N, int64_t total, float u, int mode,
                        float* bias) {
    for (int e = 0; e < N; ++e) {
        if (mode == 0) {
            int64_t lhs = counts[e] * (int64_t)N;
            int sgn = (lhs > total) - (lhs < total);
            float step = u * (float)sgn;
            bias[e] = bias[e] - step;
        } else {
            float target = (float)((double)total / (double)N);
            float err = (float)counts[e] - target;
            float sgn = (float)((err > 0.0f) - (err < 0.0f));
            float a = u * sgn;
            float r = fabsf(err) / target;
            bias[e] = bias[e] - a * r;
        }
    }
}

/* ---------------------------------------------------------------------------
 * "Forcible load balancing" (MindIE expert_parallelism_load_balancer page:
 * the top-k outputs are replaced by fake ones that balance the experts
 * exactly, an upper bound for balance).  Reading: expert (t*K + k) mod N in
 * round-robin order, equal weights route_scale / K.
 * ------------------------------------------------------------------------- */
void oracle_route_balanced(int64_t T, int K, int N, float route_scale, int32_t* idx, float* w) {
    for (int64_t t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            idx[t * K + k] = (int32_t)((t * K + k) % N);
            w[t * K + k] = route_scale / (float)K;
        }
}

/* ---------------------------------------------------------------------------
 * Bias update on a smoothed load ("DeepSeek V4 MoE load balancing",
 * aux-loss-free section: a moving average smooths the load statistics).
 *   ema_e = fp32(fp32(alpha * ema_e) + fp32((1 - alpha) * c_e))
 *   mean  = fp32(total / N)
 *   b_e   = fp32(b_e - fp32(u * sign(ema_e - mean)))      (sign(0) = 0)
 * every op a single fp32 rounding, in that order.
 * ------------------------------------------------------------------------- */
void oracle_bias_update_ema(const int64_t* counts, int N, int64_t total, float u, float alpha,
                            float* ema, float* bias) {
    const float mean = (float)((double)total / (double)N);
    const float beta = 1.0f - alpha;
    for (int e = 0; e < N; ++e) {
        float a = alpha * ema[e];
        float c = beta * (float)counts[e];
        ema[e] = a + c;
        float sgn = (float)((ema[e] > mean) - (ema[e] < mean));
        float step = u * sgn;
        bias[e] = bias[e] - step;
    }
}

/* ---------------------------------------------------------------------------
 * Capacity-limited routing ([ENT] "Production Testing": a hard token capacity
 * per expert, 1.25 * T*K/N, with the excess routed to secondary candidate
 * experts by the bias-adjusted ranking).
 *  1. Candidates of token t: the experts of its kept groups (selection step
 *     2), ranked by (key desc, index asc) with key = fp32(s + b); the first K
 *     are the selection's choice, in its order.
 *  2. Primary pass, flat order a = t*K + k: an assignment is accepted while
 *     its expert has accepted fewer than C; otherwise it overflows.
 *  3. Reroute pass: token t's j-th overflowed slot (counting in k order) takes
 *     candidate K + j, if the token has that many.  In flat order again, a
 *     rerouted assignment is accepted while its expert holds fewer than C in
 *     all (primaries and earlier reroutes).  Anything else is dropped:
 *     idx -1, weight 0.  One reroute round; a second overflow is a drop.
 *  4. Weights from the unbiased scores of the token's final experts:
 *     renorm ? s / (sum over its kept slots in k order) : s, times
 *     route_scale, each op rounded to fp32 (a token with every slot dropped
 *     gets zero weights).
 * info[0] = overflowed primaries, info[1] = accepted reroutes, info[2] =
 * dropped assignments.  Returns 0, or -1 on an invalid configuration.
 * ------------------------------------------------------------------------- */
typedef struct { float key; int e; } cap_cand;

static int cap_cand_cmp(const void* a, const void* b) {
    const cap_cand* x = (const cap_cand*)a;
    const cap_cand* y = (const cap_cand*)b;
    if (beats(x->key, x->e, y->key, y->e)) return -1;
    if (beats(y->key, y->e, x->key, x->e)) return 1;
    return 0;
}

int oracle_route_capacity(const float* s, const float* bias, int64_t T, int N, int K,
                          int n_groups, int topk_groups, int group_topn, int renorm,
                          float route_scale, int64_t C, int32_t* idx, float* w, int64_t* info) {
    if (N <= 0 || K <= 0 || K > N || n_groups <= 0 || N % n_groups || C < 0) return -1;
    const int gsize = N / n_groups;
    if (n_groups > 1 && (topk_groups <= 0 || topk_groups > n_groups ||
                         topk_groups * gsize < K || group_topn <= 0 || group_topn > gsize))
        return -1;
    /* ranked candidates: second[t*K + j] = candidate K + j, or -1 */
    int32_t* second = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * K + 1));
    int64_t* used = (int64_t*)calloc((size_t)N, sizeof(int64_t));
    int32_t* fin = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * K + 1));
    if (!second || !used || !fin) { free(second); free(used); free(fin); return -1; }
    int64_t t;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (t = 0; t < T; ++t) {
        float* key = (float*)malloc(sizeof(float) * (size_t)N);
        float* gs = (float*)malloc(sizeof(float) * (size_t)n_groups);
        float* tmp = (float*)malloc(sizeof(float) * (size_t)gsize);
        cap_cand* cand = (cap_cand*)malloc(sizeof(cap_cand) * (size_t)N);
        if (!key || !gs || !tmp || !cand) { bad |= 1; goto next; }
        for (int e = 0; e < N; ++e) key[e] = s[t * N + e] + (bias ? bias[e] : 0.0f);
        int nc = 0;
        for (int g = 0; g < n_groups; ++g) {
            int keep = 1;
            if (n_groups > 1) {
                /* group scores as in the selection, then this group's rank */
                for (int h2 = 0; h2 < n_groups; ++h2) {
                    for (int i = 0; i < gsize; ++i) tmp[i] = key[h2 * gsize + i];
                    float sum = 0.0f;
                    for (int r = 0; r < group_topn; ++r) {
                        int best = 0;
                        for (int i = 1; i < gsize; ++i) if (tmp[i] > tmp[best]) best = i;
                        sum = (r == 0) ? tmp[best] : sum + tmp[best];
                        tmp[best] = -INFINITY;
                    }
                    gs[h2] = sum;
                }
                int rank = 0;
                for (int h2 = 0; h2 < n_groups; ++h2)
                    if (h2 != g && beats(gs[h2], h2, gs[g], g)) ++rank;
                keep = rank < topk_groups;
            }
            if (keep)
                for (int i = 0; i < gsize; ++i) {
                    cand[nc].key = key[g * gsize + i];
                    cand[nc].e = g * gsize + i;
                    ++nc;
                }
        }
        qsort(cand, (size_t)nc, sizeof(cap_cand), cap_cand_cmp);
        for (int k = 0; k < K; ++k) {
            idx[t * K + k] = cand[k].e;
            second[t * K + k] = (K + k < nc) ? cand[K + k].e : -1;
        }
    next:
        free(key); free(gs); free(tmp); free(cand);
    }
    if (bad) { free(second); free(used); free(fin); return -1; }

    int64_t n_over = 0, n_rer = 0, n_drop = 0;
    /* 2. primary pass */
    for (int64_t a = 0; a < T * K; ++a) {
        const int32_t e = idx[a];
        if (used[e] < C) { used[e] += 1; fin[a] = e; }
        else { fin[a] = -2; ++n_over; } /* -2: overflowed, to reroute */
    }
    /* 3. reroute pass */
    for (int64_t tt = 0; tt < T; ++tt) {
        int j = 0;
        for (int k = 0; k < K; ++k) {
            const int64_t a = tt * K + k;
            if (fin[a] != -2) continue;
            const int32_t e2 = second[tt * K + j];
            ++j;
            if (e2 >= 0 && used[e2] < C) { used[e2] += 1; fin[a] = e2; ++n_rer; }
            else { fin[a] = -1; ++n_drop; }
        }
    }
    /* 4. weights */
    for (int64_t tt = 0; tt < T; ++tt) {
        float ssum = 0.0f;
        int first = 1;
        for (int k = 0; k < K; ++k) {
            const int32_t e = fin[tt * K + k];
            if (e < 0) continue;
            ssum = first ? s[tt * N + e] : ssum + s[tt * N + e];
            first = 0;
        }
        for (int k = 0; k < K; ++k) {
            const int32_t e = fin[tt * K + k];
            idx[tt * K + k] = e;
            if (e < 0) { w[tt * K + k] = 0.0f; continue; }
            const float sk = s[tt * N + e];
            const float v = renorm ? sk / ssum : sk;
            w[tt * K + k] = v * route_scale;
        }
    }
    info[0] = n_over; info[1] = n_rer; info[2] = n_drop;
    free(second); free(used); free(fin);
    return 0;
}
