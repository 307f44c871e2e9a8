/*
 * CPU oracle of the sparse Mixture-of-Experts layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this code.  It shares no code,
 * header or table with the CUDA library; both read the same seeded inputs.
 *
 * Plain, slow, obviously correct: every quantity is computed in double from
 * the exactly stored inputs (bf16 and fp32 values convert to double without
 * error), one definition at a time, in the order the pages state it.  The
 * only concession to speed is an OpenMP loop over independent tokens or rows,
 * which does not change any arithmetic.
 *
 * Sources (web pages on sparse MoE):
 *  - "LLM from scratch", ch. 36 (faketrader.github.io, 27-mixture-experts):
 *    notation table (36.1); routing, softmax and top-k (36.1 "dense and
 *    sparse mixture"); the two weight normalisations (36.2); dispatch,
 *    combine and capacity (36.3); load statistics and the N=4, E_r=3, k=2
 *    worked example (36.4); Algorithm 36.1 (sparse expert forward with an
 *    explicit capacity rule); shared expert (36.6); router layout (36.8).
 *  - auturnal.com review "sparse-mixture-experts" (equations block):
 *    C_e = ceil(c T k / E), O = sum_e max(0, L_e - C_e), rho_max.
 *  - vegetog.com "MoE token routing", sections 2-3: router shapes, the
 *    4-expert renormalisation example, the SwiGLU expert.
 *  - jeefy.top WDMoE note: token latency t = t_up + t_comp + t_down and the
 *    weight-latency-ratio (WLR) pruning rule with threshold theta.
 *
 * Layout: weights are stored output-major ("K-major"): W_r is [E_r, d],
 * W_g and W_u are [E_r, d_f, d], W_d is [E_r, d, d_f].  The pages write the
 * transposes (x W with W in R^{d x E_r}); ch. 36.8 notes that the [out, in]
 * storage is only a transposition convention.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DT_F32 0
#define DT_BF16 1
#define NORM_RENORM 0
#define NORM_FULLPROB 1
#define NORM_WLR 2

static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double load(const void* p, int dtype, size_t i) {
    return dtype == DT_BF16 ? bf16_value(((const uint16_t*)p)[i]) : (double)((const float*)p)[i];
}

/* Round a double to the nearest bf16 value (8 significant bits), ties to
 * even: the storage precision of the expert hidden activation h in the bf16
 * layer (fp32 exponent range; subnormals use the fixed spacing 2^-133). */
double oracle_round_bf16(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    double a = fabs(v);
    double q;
    if (a < 0x1.0p-126) {
        q = nearbyint(v * 0x1.0p133) * 0x1.0p-133;
    } else {
        int e;
        frexp(a, &e);                       /* a = m 2^e, m in [0.5, 1) */
        double ulp = ldexp(1.0, e - 8);     /* 8 significant bits */
        q = nearbyint(v / ulp) * ulp;       /* default rounding: ties to even */
        if (fabs(q) > 0x1.fe0000p127) q = v > 0 ? INFINITY : -INFINITY;
    }
    return q;
}

/* SiLU(z) = z / (1 + e^{-z})  (vegetog sec. 3, SwiGLU expert). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * Router, softmax, top-k and weights for every token (ch. 36.1-36.2;
 * Algorithm 36.1 first two steps; WDMoE WLR rule).
 *
 *  g_te = sum_i x_ti W_r[e,i] + b_e                      (router scores G)
 *  p_te = exp(g_te - max_j g_tj) / sum_j exp(...)         (stable softmax)
 *  S_t  = first k experts in the order (g descending, expert index ascending)
 *  weights, by norm:
 *    RENORM   a_te = p_te / sum_{j in S_t} p_tj
 *    FULLPROB a_te = p_te                        (Switch: full-expert prob)
 *    WLR      over the current set S (initially S_t), WLR_e = p_e / t_e; while
 *             |S| >= 2 and min WLR / (min WLR + max WLR) <= theta, drop the
 *             expert with the smallest WLR (on equal WLR the higher index);
 *             then a_e = softmax over {g_e : e in S} = p_e / sum_S p; an
 *             expert with infinite latency (disconnected) gets weight 0.
 *
 * Outputs per token t (rank order j = 0..k-1):
 *  ids[t*k+j]  chosen expert, -1 if pruned (WLR) or the token is invalid
 *  w[t*k+j]    weight a_te (0 for -1 entries)
 *  margin[t]   g_(k) - g_(k+1) in the sorted order (+inf when k == E_r)
 *  wlr_gap[t]  min |ratio - theta| over the WLR tests made (+inf otherwise)
 *  invalid[t]  1 when a score (or a chosen expert's latency) is not a finite
 *              positive number: Algorithm 36.1 treats non-finite scores as an
 *              input failure that does not enter the sort.
 *  logits      optional [N, E_r] copy of g.
 */
int oracle_route(int64_t N, int d, int E, int k, int norm, double theta, int dtype,
                 const void* x, const void* W_r, const float* b_r, const float* lat,
                 double* logits, int32_t* ids, double* w, double* margin, double* wlr_gap,
                 uint8_t* invalid) {
    if (N < 0 || d < 1 || E < 1 || k < 1 || k > E) return 1;
    if (norm == NORM_WLR && !lat) return 1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < N; ++t) {
        double* g = (double*)malloc(sizeof(double) * E);
        double* p = (double*)malloc(sizeof(double) * E);
        int* order = (int*)malloc(sizeof(int) * E);
        int bad = 0;
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int i = 0; i < d; ++i)
                s += load(x, dtype, (size_t)t * d + i) * load(W_r, dtype, (size_t)e * d + i);
            if (b_r) s += (double)b_r[e];
            g[e] = s;
            if (!isfinite(s)) bad = 1;
            if (logits) logits[t * E + e] = s;
        }
        /* insertion sort of expert indices: score descending, index ascending */
        for (int e = 0; e < E; ++e) order[e] = e;
        if (!bad) {
            for (int a = 1; a < E; ++a) {
                int cur = order[a], b = a - 1;
                while (b >= 0 && (g[order[b]] < g[cur] || (g[order[b]] == g[cur] && order[b] > cur))) {
                    order[b + 1] = order[b];
                    --b;
                }
                order[b + 1] = cur;
            }
        }
        if (!bad && norm == NORM_WLR) {
            for (int j = 0; j < k; ++j) {
                double te = (double)lat[t * E + order[j]];
                if (!(te > 0.0) || isnan(te)) bad = 1;
            }
        }
        wlr_gap[t] = INFINITY;
        if (bad) {
            invalid[t] = 1;
            margin[t] = NAN;
            for (int j = 0; j < k; ++j) { ids[t * k + j] = -1; w[t * k + j] = 0.0; }
            free(g); free(p); free(order);
            continue;
        }
        invalid[t] = 0;
        margin[t] = k < E ? g[order[k - 1]] - g[order[k]] : INFINITY;
        double gmax = g[order[0]], z = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp(g[e] - gmax); z += p[e]; }
        for (int e = 0; e < E; ++e) p[e] /= z;

        int* active = (int*)malloc(sizeof(int) * k);
        for (int j = 0; j < k; ++j) active[j] = 1;
        if (norm == NORM_WLR) {
            int n_active = k;
            while (n_active >= 2) {
                int jmin = -1, jmax = -1;
                double vmin = 0.0, vmax = 0.0;
                for (int j = 0; j < k; ++j) {
                    if (!active[j]) continue;
                    int e = order[j];
                    double v = p[e] / (double)lat[t * E + e];
                    if (jmin < 0 || v < vmin || (v == vmin && e > order[jmin])) { jmin = j; vmin = v; }
                    if (jmax < 0 || v > vmax) { jmax = j; vmax = v; }
                }
                double ratio = vmin / (vmin + vmax);
                double gap = fabs(ratio - theta);
                if (gap < wlr_gap[t]) wlr_gap[t] = gap;
                if (ratio <= theta) { active[jmin] = 0; --n_active; }
                else break;
            }
        }
        double ssel = 0.0;
        for (int j = 0; j < k; ++j) if (active[j]) ssel += p[order[j]];
        for (int j = 0; j < k; ++j) {
            int e = order[j];
            if (!active[j]) { ids[t * k + j] = -1; w[t * k + j] = 0.0; continue; }
            ids[t * k + j] = e;
            if (norm == NORM_FULLPROB) w[t * k + j] = p[e];
            else w[t * k + j] = p[e] / ssel;
            if (norm == NORM_WLR && isinf((double)lat[t * E + e])) w[t * k + j] = 0.0;
        }
        free(active);
        free(g); free(p); free(order);
    }
    return 0;
}

/*
 * Capacity check and token-order acceptance (Algorithm 36.1, steps 3-4;
 * ch. 36.3 "capacity and overflow"; review equations for O).
 *
 * Tokens are visited t = 0..N-1 in order; for each requested path (t, e)
 * (ids >= 0) the requested load L_e grows by one; if the counter c_e < C the
 * path is accepted into slot c_e and c_e grows, otherwise it is rejected.
 *
 * Outputs: slot[t*k+j] (slot index, -1 if rejected or not requested),
 * L[e] requested, acc[e] accepted, and counters
 *  cnt[0] requested = sum_e L_e       cnt[1] accepted        cnt[2] rejected
 *  cnt[3] O = sum_e max(0, L_e - C)   cnt[4] tokens with >= 1 rejected path
 *  cnt[5] tokens with >= 1 request and every requested path rejected
 *  cnt[6] max_e L_e
 */
int oracle_dispatch(int64_t N, int k, int E, int64_t C, const int32_t* ids, int32_t* slot,
                    int64_t* L, int64_t* acc, int64_t* cnt) {
    if (N < 0 || k < 1 || E < 1 || C < 1) return 1;
    for (int e = 0; e < E; ++e) { L[e] = 0; acc[e] = 0; }
    for (int i = 0; i < 7; ++i) cnt[i] = 0;
    for (int64_t t = 0; t < N; ++t) {
        int req = 0, rej = 0;
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            if (e < 0) { slot[t * k + j] = -1; continue; }
            ++req;
            L[e] += 1;
            if (acc[e] < C) { slot[t * k + j] = (int32_t)acc[e]; acc[e] += 1; }
            else { slot[t * k + j] = -1; ++rej; }
        }
        if (rej > 0) cnt[4] += 1;
        if (req > 0 && rej == req) cnt[5] += 1;
    }
    for (int e = 0; e < E; ++e) {
        cnt[0] += L[e];
        cnt[1] += acc[e];
        cnt[3] += L[e] > C ? L[e] - C : 0;
        if (L[e] > cnt[6]) cnt[6] = L[e];
    }
    cnt[2] = cnt[0] - cnt[1];
    return 0;
}

/*
 * Acceptance by gate weight ("LLM from scratch" ch. 36.3, on how the
 * acceptance rule makes outputs depend on the batch: besides
 * first-come-first-served the page names ordering by gate weight, under which
 * the low-weight paths are the ones that lose their computation).  Read here
 * as: among the paths that request expert e, the C with the largest routing
 * weight w[t*k+j] (a_te) are accepted; equal weights go to the earlier token.
 * Accepted paths take slots in token order (slot = number of accepted paths
 * of e from earlier tokens), so only which paths are accepted differs from
 * oracle_dispatch.  Outputs and counters as oracle_dispatch.
 */
typedef struct { int32_t e; int64_t t; int j; double w; } prio_req;

static int prio_cmp(const void* pa, const void* pb) {
    const prio_req* a = (const prio_req*)pa;
    const prio_req* b = (const prio_req*)pb;
    if (a->e != b->e) return a->e < b->e ? -1 : 1;
    if (a->w != b->w) return a->w > b->w ? -1 : 1;  /* larger weight first */
    if (a->t != b->t) return a->t < b->t ? -1 : 1;  /* then the earlier token */
    return 0;
}

int oracle_dispatch_priority(int64_t N, int k, int E, int64_t C, const int32_t* ids, const double* w,
                             int32_t* slot, int64_t* L, int64_t* acc, int64_t* cnt) {
    if (N < 0 || k < 1 || E < 1 || C < 1) return 1;
    for (int e = 0; e < E; ++e) { L[e] = 0; acc[e] = 0; }
    for (int i = 0; i < 7; ++i) cnt[i] = 0;
    int64_t nreq = 0;
    for (int64_t i = 0; i < N * k; ++i)
        if (ids[i] >= 0) ++nreq;
    prio_req* r = (prio_req*)malloc(sizeof(prio_req) * (size_t)(nreq > 0 ? nreq : 1));
    char* ok = (char*)calloc((size_t)(N * k > 0 ? N * k : 1), 1);
    if (!r || !ok) { free(r); free(ok); return 2; }
    int64_t n = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int j = 0; j < k; ++j) {
            const int e = ids[t * k + j];
            if (e < 0) continue;
            r[n].e = e; r[n].t = t; r[n].j = j; r[n].w = w[t * k + j];
            ++n;
            L[e] += 1;
        }
    qsort(r, (size_t)n, sizeof(prio_req), prio_cmp);
    /* the first C entries of each expert's run are accepted */
    int64_t run = 0;
    for (int64_t i = 0; i < n; ++i) {
        run = (i > 0 && r[i].e == r[i - 1].e) ? run + 1 : 0;
        if (run < C) ok[r[i].t * k + r[i].j] = 1;
    }
    for (int64_t t = 0; t < N; ++t) {
        int req = 0, rej = 0;
        for (int j = 0; j < k; ++j) {
            const int e = ids[t * k + j];
            if (e < 0) { slot[t * k + j] = -1; continue; }
            ++req;
            if (ok[t * k + j]) { slot[t * k + j] = (int32_t)acc[e]; acc[e] += 1; }
            else { slot[t * k + j] = -1; ++rej; }
        }
        if (rej > 0) cnt[4] += 1;
        if (req > 0 && rej == req) cnt[5] += 1;
    }
    for (int e = 0; e < E; ++e) {
        cnt[0] += L[e];
        cnt[1] += acc[e];
        cnt[3] += L[e] > C ? L[e] - C : 0;
        if (L[e] > cnt[6]) cnt[6] = L[e];
    }
    cnt[2] = cnt[0] - cnt[1];
    free(r);
    free(ok);
    return 0;
}

/*
 * Token-order acceptance for one shard of a routing group split over ranks in
 * token order (rank 0's tokens first).  base[e] = requests for expert e made
 * by the tokens of earlier ranks.  A request is the base[e] + j-th request for
 * e in the whole group (j = earlier requests for e in this shard) and is
 * accepted iff that number is < C, exactly as Algorithm 36.1 decides on the
 * concatenated batch.  slot[] receives that group-wide slot (or -1); L and
 * acc are this shard's requested and accepted counts; cnt as oracle_dispatch
 * but for this shard's requests, except cnt[3] (O) and cnt[6] (max load),
 * which are left 0 (they need the group-wide loads).
 */
int oracle_dispatch_ranked(int64_t N, int k, int E, int64_t C, const int32_t* ids,
                           const int64_t* base, int32_t* slot, int64_t* L, int64_t* acc,
                           int64_t* cnt) {
    if (N < 0 || k < 1 || E < 1 || C < 1) return 1;
    for (int e = 0; e < E; ++e) { L[e] = 0; acc[e] = 0; }
    for (int i = 0; i < 7; ++i) cnt[i] = 0;
    for (int64_t t = 0; t < N; ++t) {
        int req = 0, rej = 0;
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            if (e < 0) { slot[t * k + j] = -1; continue; }
            ++req;
            int64_t c = base[e] + L[e];
            L[e] += 1;
            if (c < C) { slot[t * k + j] = (int32_t)c; acc[e] += 1; }
            else { slot[t * k + j] = -1; ++rej; }
        }
        if (rej > 0) cnt[4] += 1;
        if (req > 0 && rej == req) cnt[5] += 1;
    }
    for (int e = 0; e < E; ++e) { cnt[0] += L[e]; cnt[1] += acc[e]; }
    cnt[2] = cnt[0] - cnt[1];
    return 0;
}

/*
 * Combine weights under an overflow policy ("LLM from scratch" ch. 36.3: the
 * handling of a rejected path is part of the model definition; ch. 36.4
 * worked example, both outcomes).  policy 0: a rejected path contributes 0
 * and the other paths keep a_te (Algorithm 36.1).  policy 1: for a token
 * that lost some but not all paths, its accepted paths are rescaled to sum to
 * one: wc = a_te / sum over its accepted paths of a.  wc is 0 for rejected or
 * unrequested paths.
 */
int oracle_reject_weights(int64_t N, int k, int policy, const int32_t* ids, const double* w,
                          const int32_t* slot, double* wc) {
    for (int64_t t = 0; t < N; ++t) {
        int req = 0, rej = 0;
        double acc_sum = 0.0;
        for (int j = 0; j < k; ++j) {
            if (ids[t * k + j] < 0) continue;
            ++req;
            if (slot[t * k + j] < 0) ++rej;
            else acc_sum += w[t * k + j];
        }
        for (int j = 0; j < k; ++j) {
            int i = (int)(t * k + j);
            if (ids[i] < 0 || slot[i] < 0) { wc[i] = 0.0; continue; }
            wc[i] = (policy == 1 && rej > 0 && rej < req) ? w[i] / acc_sum : w[i];
        }
    }
    return 0;
}

/*
 * Rerouting as an overflow policy ("LLM from scratch" ch. 36.3, capacity and
 * overflow: handling a path past capacity is part of the model definition;
 * besides zeroing it, a rejected path may be rerouted, which calls another
 * expert's parameters; the same section notes that other experts' free slots
 * do not stand in for the full expert's function; vegetog "MoE token routing"
 * sec. 5: an over-capacity token is dropped from that expert's branch or
 * rerouted, depending on the implementation).  The pages do not say to which
 * expert or with what weight.  Reading taken here:
 *
 *  - A token's rerouting candidates are its experts of ranks k, k+1, ...,
 *    k+X-1 in the router's order (score descending, ties to the lower index),
 *    i.e. the experts it would have chosen next.
 *  - A candidate carries the weight the router's normalisation gives it
 *    against the token's chosen set S (the same factor as the token's other
 *    paths): p_e / sum_{S} p under renormalisation, p_e under the full
 *    probability.  (WLR pruning is not combined with rerouting.)
 *  - Round 0 is Algorithm 36.1: first-choice requests in token order, the
 *    first C per expert accepted.  Rerouting then fills the slots left free,
 *    in rounds r = 1, 2, ...: each path still without an expert takes its
 *    token's next unused candidate whose expert was not full at the start of
 *    the round (a token's paths in rank order take consecutive candidates);
 *    the round's offers are accepted in token order while the expert has a
 *    free slot (slot = rows already accepted by that expert).  A path that is
 *    refused tries its token's next candidate in the next round; rounds stop
 *    when no path makes an offer.  A path that finds no free expert adds 0.
 *  - An expert's rows are its first-choice rows in token order, then each
 *    round's rerouted rows in token order.
 */

/* cand[t*X+q] = the token's expert of rank k+q (-1 past E_r or for an
 * invalid token), cand_w its weight as above.  logits [N, E] in double (the
 * router scores); ids/w the router's records.  norm: renorm or full
 * probability only. */
int oracle_reroute_candidates(int64_t N, int E, int k, int X, int norm, const double* logits,
                              const int32_t* ids, const uint8_t* invalid, int32_t* cand, double* cand_w) {
    if (N < 0 || E < 1 || k < 1 || k > E || X < 1) return 1;
    if (norm != NORM_RENORM && norm != NORM_FULLPROB) return 1;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t t = 0; t < N; ++t) {
        const double* g = logits + t * E;
        for (int q = 0; q < X; ++q) { cand[t * X + q] = -1; cand_w[t * X + q] = 0.0; }
        if (invalid[t]) continue;
        int* order = (int*)malloc(sizeof(int) * E);
        double* p = (double*)malloc(sizeof(double) * E);
        for (int e = 0; e < E; ++e) order[e] = e;
        for (int a = 1; a < E; ++a) {
            int cur = order[a], b = a - 1;
            while (b >= 0 && (g[order[b]] < g[cur] || (g[order[b]] == g[cur] && order[b] > cur))) {
                order[b + 1] = order[b];
                --b;
            }
            order[b + 1] = cur;
        }
        double gmax = g[order[0]], z = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp(g[e] - gmax); z += p[e]; }
        for (int e = 0; e < E; ++e) p[e] /= z;
        double ssel = 0.0;
        for (int j = 0; j < k; ++j)
            if (ids[t * k + j] >= 0) ssel += p[ids[t * k + j]];
        for (int q = 0; q < X && k + q < E; ++q) {
            int e = order[k + q];
            cand[t * X + q] = e;
            cand_w[t * X + q] = norm == NORM_FULLPROB ? p[e] : p[e] / ssel;
        }
        free(order);
        free(p);
    }
    return 0;
}

/* Token-order acceptance with rerouting of the rejected paths (rounds as
 * above).  Outputs: slot [N,k] first-choice slot (-1 if rejected or not
 * requested), as oracle_dispatch; rr_e [N,k] expert a rejected path was
 * rerouted to (-1: none), rr_slot [N,k] its slot there, rr_q [N,k] the
 * candidate index used; L [E] first-choice requested loads; acc [E] rows per
 * expert (first-choice plus rerouted); counters
 *  cnt[0] requested   cnt[1] paths given a slot (first choice or rerouted)
 *  cnt[2] requested - cnt[1]   cnt[3] O = sum_e max(0, L_e - C)
 *  cnt[4] tokens with >= 1 requested path left without an expert
 *  cnt[5] tokens with >= 1 request and every requested path without an expert
 *  cnt[6] max_e L_e   cnt[7] rerouted paths  cnt[8] rounds that made offers */
int oracle_dispatch_reroute(int64_t N, int k, int E, int64_t C, int X, const int32_t* ids,
                            const int32_t* cand, int32_t* slot, int32_t* rr_e, int32_t* rr_slot,
                            int32_t* rr_q, int64_t* L, int64_t* acc, int64_t* cnt) {
    if (N < 0 || k < 1 || E < 1 || C < 1 || X < 1) return 1;
    int64_t base_cnt[7];
    int rc = oracle_dispatch(N, k, E, C, ids, slot, L, acc, base_cnt);
    if (rc) return rc;
    for (int64_t i = 0; i < N * k; ++i) { rr_e[i] = -1; rr_slot[i] = -1; rr_q[i] = -1; }
    int* next = (int*)calloc((size_t)(N > 0 ? N : 1), sizeof(int));     /* next unused candidate per token */
    int64_t* full_at_start = (int64_t*)malloc(sizeof(int64_t) * E);
    int32_t* offer = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N * k > 0 ? N * k : 1));
    int rounds = 0;
    for (;;) {
        for (int e = 0; e < E; ++e) full_at_start[e] = acc[e] >= C;
        int64_t n_offers = 0;
        for (int64_t t = 0; t < N; ++t) {
            for (int j = 0; j < k; ++j) {
                int64_t i = t * k + j;
                offer[i] = -1;
                if (ids[i] < 0 || slot[i] >= 0 || rr_e[i] >= 0) continue;
                while (next[t] < X && cand[t * X + next[t]] >= 0 && full_at_start[cand[t * X + next[t]]]) ++next[t];
                if (next[t] < X && cand[t * X + next[t]] >= 0) {
                    offer[i] = next[t];
                    ++next[t];
                    ++n_offers;
                }
            }
        }
        if (n_offers == 0) break;
        ++rounds;
        for (int64_t t = 0; t < N; ++t) {
            for (int j = 0; j < k; ++j) {
                int64_t i = t * k + j;
                if (offer[i] < 0) continue;
                int e = cand[t * X + offer[i]];
                if (acc[e] < C) {
                    rr_e[i] = e;
                    rr_slot[i] = (int32_t)acc[e];
                    rr_q[i] = offer[i];
                    acc[e] += 1;
                }
            }
        }
    }
    for (int i = 0; i < 9; ++i) cnt[i] = 0;
    for (int64_t t = 0; t < N; ++t) {
        int req = 0, lost = 0;
        for (int j = 0; j < k; ++j) {
            int64_t i = t * k + j;
            if (ids[i] < 0) continue;
            ++req;
            if (slot[i] < 0 && rr_e[i] < 0) ++lost;
            if (rr_e[i] >= 0) cnt[7] += 1;
        }
        if (lost > 0) cnt[4] += 1;
        if (req > 0 && lost == req) cnt[5] += 1;
    }
    for (int e = 0; e < E; ++e) {
        cnt[0] += L[e];
        cnt[1] += acc[e];
        cnt[3] += L[e] > C ? L[e] - C : 0;
        if (L[e] > cnt[6]) cnt[6] = L[e];
    }
    cnt[2] = cnt[0] - cnt[1];
    cnt[8] = rounds;
    free(next);
    free(full_at_start);
    free(offer);
    return 0;
}

/*
 * One SwiGLU expert on a list of token rows (vegetog sec. 3):
 *   E(x) = [SiLU(x W_gate) (.) (x W_up)] W_down
 * with W_gate, W_up stored [d_f, d] and W_down stored [d, d_f].  When
 * round_h is set, the hidden activation h is rounded to bf16 (the storage
 * precision of h in the bf16 layer) before the down projection.
 * out[r*d + o] = E(x_{rows[r]})_o.
 */
int oracle_swiglu_rows(int d, int d_f, int dtype, int round_h, const void* x, const int64_t* rows,
                       int64_t M, const void* Wg, const void* Wu, const void* Wd, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M; ++r) {
        int64_t t = rows[r];
        double* xt = (double*)malloc(sizeof(double) * d);
        double* h = (double*)malloc(sizeof(double) * d_f);
        for (int i = 0; i < d; ++i) xt[i] = load(x, dtype, (size_t)t * d + i);
        for (int j = 0; j < d_f; ++j) {
            double gs = 0.0, us = 0.0;
            for (int i = 0; i < d; ++i) {
                gs += xt[i] * load(Wg, dtype, (size_t)j * d + i);
                us += xt[i] * load(Wu, dtype, (size_t)j * d + i);
            }
            double hv = silu(gs) * us;
            h[j] = round_h ? oracle_round_bf16(hv) : hv;
        }
        for (int o = 0; o < d; ++o) {
            double s = 0.0;
            for (int j = 0; j < d_f; ++j) s += h[j] * load(Wd, dtype, (size_t)o * d_f + j);
            out[r * d + o] = s;
        }
        free(xt);
        free(h);
    }
    return 0;
}

/*
 * The same SwiGLU expert on M input rows given directly in double (for Soft
 * MoE, whose expert inputs are mixtures of token rows, not token rows):
 * out[r*d + o] = E(X_r)_o.
 */
int oracle_swiglu_dense(int d, int d_f, int dtype, int round_h, const double* X, int64_t M, const void* Wg,
                        const void* Wu, const void* Wd, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M; ++r) {
        const double* xt = X + r * d;
        double* h = (double*)malloc(sizeof(double) * d_f);
        for (int j = 0; j < d_f; ++j) {
            double gs = 0.0, us = 0.0;
            for (int i = 0; i < d; ++i) {
                gs += xt[i] * load(Wg, dtype, (size_t)j * d + i);
                us += xt[i] * load(Wu, dtype, (size_t)j * d + i);
            }
            double hv = silu(gs) * us;
            h[j] = round_h ? oracle_round_bf16(hv) : hv;
        }
        for (int o = 0; o < d; ++o) {
            double s = 0.0;
            for (int j = 0; j < d_f; ++j) s += h[j] * load(Wd, dtype, (size_t)o * d_f + j);
            out[r * d + o] = s;
        }
        free(h);
    }
    return 0;
}

/*
 * Combine (ch. 36.3, Algorithm 36.1 step 6): for every accepted record
 * (t, e, slot c, a_te), Y_t += a_te * H_e[c].  H is given per expert as a
 * pointer table Hs[e] -> [rows, d] with row c = slot c.  Y is overwritten
 * (starts at 0).  Rejected or pruned paths add nothing and the remaining
 * weights are not renormalised (Algorithm 36.1, reject rule).
 */
int oracle_combine(int64_t N, int k, int d, const int32_t* ids, const double* w, const int32_t* slot,
                   const double* const* Hs, double* Y) {
    for (int64_t t = 0; t < N; ++t) {
        for (int o = 0; o < d; ++o) Y[t * d + o] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            int c = slot[t * k + j];
            if (e < 0 || c < 0) continue;
            for (int o = 0; o < d; ++o) Y[t * d + o] += w[t * k + j] * Hs[e][(size_t)c * d + o];
        }
    }
    return 0;
}

/*
 * Output rows for a chosen set of tokens, given the routing records: for
 * token t, Y_t = sum over its accepted paths of a_te E_e(x_t), plus the shared
 * expert F_sh(x_t) with weight 1 when present (ch. 36.6 shared expert;
 * DeepSeek-V3 form y = FFN_shared(x) + sum_i g_i FFN_i(x)).
 * Tokens are processed one by one, so any sample of a large batch can be
 * checked.  Wg/Wu/Wd are the stacked expert weights; Ws_* may be NULL.
 */
int oracle_forward_rows(int d, int d_f, int E, int k, int dtype, int d_f_sh, const void* x,
                        const int32_t* ids, const double* w, const int32_t* slot,
                        const int64_t* tokens, int64_t T, const void* Wg, const void* Wu,
                        const void* Wd, const void* Wsg, const void* Wsu, const void* Wsd, double* Y) {
    int round_h = dtype == DT_BF16;
    size_t esz = dtype == DT_BF16 ? 2 : 4;
    (void)E;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < T; ++r) {
        int64_t t = tokens[r];
        double* o = (double*)malloc(sizeof(double) * d);
        for (int i = 0; i < d; ++i) Y[r * d + i] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            if (e < 0 || slot[t * k + j] < 0) continue;
            const char* g = (const char*)Wg + (size_t)e * d_f * d * esz;
            const char* u = (const char*)Wu + (size_t)e * d_f * d * esz;
            const char* dn = (const char*)Wd + (size_t)e * d * d_f * esz;
            oracle_swiglu_rows(d, d_f, dtype, round_h, x, &t, 1, g, u, dn, o);
            for (int i = 0; i < d; ++i) Y[r * d + i] += w[t * k + j] * o[i];
        }
        if (d_f_sh > 0 && Wsg) {
            oracle_swiglu_rows(d, d_f_sh, dtype, round_h, x, &t, 1, Wsg, Wsu, Wsd, o);
            for (int i = 0; i < d; ++i) Y[r * d + i] += o[i];
        }
        free(o);
    }
    return 0;
}

/*
 * The whole layer (Algorithm 36.1, generalised by the normalisation mode, the
 * overflow policy of oracle_reject_weights and an optional shared expert): route, token-order acceptance with capacity C,
 * each expert evaluated only on its accepted slots, weighted combine, plus
 * the shared expert.  Y is [N, d] in double.
 */
int oracle_forward(int64_t N, int d, int d_f, int E, int k, int norm, double theta, int dtype,
                   int64_t C, int d_f_sh, int reject_policy, int accept_order, const void* x,
                   const void* W_r, const float* b_r,
                   const float* lat, const void* Wg, const void* Wu, const void* Wd,
                   const void* Wsg, const void* Wsu, const void* Wsd, double* Y, int32_t* ids,
                   double* w, int32_t* slot, double* margin, double* wlr_gap, uint8_t* invalid,
                   int64_t* L, int64_t* acc, int64_t* cnt) {
    if (N == 0) {
        for (int e = 0; e < E; ++e) { L[e] = 0; acc[e] = 0; }
        for (int i = 0; i < 7; ++i) cnt[i] = 0;
        return 0;
    }
    int rc = oracle_route(N, d, E, k, norm, theta, dtype, x, W_r, b_r, lat, 0, ids, w, margin,
                          wlr_gap, invalid);
    if (rc) return rc;
    rc = accept_order == 1 ? oracle_dispatch_priority(N, k, E, C, ids, w, slot, L, acc, cnt)
                           : oracle_dispatch(N, k, E, C, ids, slot, L, acc, cnt);
    if (rc) return rc;
    int round_h = dtype == DT_BF16;
    size_t esz = dtype == DT_BF16 ? 2 : 4;
    double** Hs = (double**)calloc(E, sizeof(double*));
    for (int e = 0; e < E; ++e) {
        int64_t M = acc[e];
        if (M == 0) continue;
        int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * M);
        for (int64_t t = 0; t < N; ++t)
            for (int j = 0; j < k; ++j)
                if (ids[t * k + j] == e && slot[t * k + j] >= 0) rows[slot[t * k + j]] = t;
        Hs[e] = (double*)malloc(sizeof(double) * M * d);
        oracle_swiglu_rows(d, d_f, dtype, round_h, x, rows, M, (const char*)Wg + (size_t)e * d_f * d * esz,
                           (const char*)Wu + (size_t)e * d_f * d * esz,
                           (const char*)Wd + (size_t)e * d * d_f * esz, Hs[e]);
        free(rows);
    }
    double* wc = (double*)malloc(sizeof(double) * N * k);
    oracle_reject_weights(N, k, reject_policy, ids, w, slot, wc);
    oracle_combine(N, k, d, ids, wc, slot, (const double* const*)Hs, Y);
    free(wc);
    for (int e = 0; e < E; ++e) free(Hs[e]);
    free(Hs);
    if (d_f_sh > 0 && Wsg) {
        int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * N);
        for (int64_t t = 0; t < N; ++t) rows[t] = t;
        double* S = (double*)malloc(sizeof(double) * N * d);
        oracle_swiglu_rows(d, d_f_sh, dtype, round_h, x, rows, N, Wsg, Wsu, Wsd, S);
        for (int64_t i = 0; i < N * d; ++i) Y[i] += S[i];
        free(S);
        free(rows);
    }
    return 0;
}
