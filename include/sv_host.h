/*
 * sv_host.h -- host-side (CPU) components that feed and steer batched
 * speculative-sampling verification: model-free drafters, the fan-out
 * prefetcher, the draft-length controller and the request budgets.
 *
 * They run on the CPU next to the rollout loop and exchange only token ids
 * and the per-request outcome (j accepted drafts, then token b) that
 * spec_verify returns, so they are plain C functions over host arrays.  No
 * function here touches a GPU.  Every handle is owned by the caller: create
 * it, use it from one thread at a time, destroy it.  Functions taking a
 * handle do nothing (and return a negative value where they return one) when
 * it is NULL.  Token ids are int32 and may be any value; sequence lengths are
 * int64.
 *
 * Sources (web pages, cited by title and section):
 *  [NG-TABLE]  "AI 开始抄自己的作业——而且抄得理直气壮" (zhichai.net), section
 *              "📓 NgramRL：每道题配一本活页草稿本": one n-gram table per prompt,
 *              n <= 6, the current tail of the generation is the key, the
 *              table proposes k = 16 tokens; it lives in host memory and holds
 *              the rollouts of the most recent W training steps (W = 4 is
 *              enough, more than 16 hurts).
 *  [NG-FETCH]  same page, section "🚰 真正的瓶颈不在算法，在流水线": while the
 *              GPU verifies, the CPU prepares drafts for the likely outcomes
 *              (j, b); a causal sliding window gives P(j) and, per branch j, a
 *              coverage profile c_j(f); a budget of N = 16 candidates goes
 *              greedily to the largest expected coverage; the all-accepted
 *              branch needs one candidate; a miss falls back to a synchronous
 *              lookup.
 *  [DAS-TREE]  "distribution-aware speculative decoding" (shilu.ai, Together AI
 *              blog), section "Adaptive suffix tree drafter": a suffix tree
 *              over a sliding window of recent trajectories; the longest match
 *              of the current context; candidate next tokens scored by their
 *              frequency in the matched subtree, the top one drafted; verified
 *              tokens are inserted at once; the tree is built per problem and
 *              freed after each training step.
 *  [DAS-LEN]   same page, section "Length-aware scheduling": long requests are
 *              spread across ranks; inside a GPU, requests are classed Long /
 *              Medium / Short from rollout history, with an aggressive, a
 *              moderate and no speculation budget; the classes are updated at
 *              run time.
 *  [ER-LEN]    the qunfachuanzhen.com article on EfficientRollout (FuriosaAI and
 *              UC Berkeley; the page has no title line, its lead paragraph is
 *              "一个每天都在上演的低效故事"), section "四、自适应草稿长度": draft
 *              lengths {5, 7, 9, 11}, start at the shortest; after each step
 *              measure the block efficiency (verified tokens per draft-verify
 *              cycle); move up after two consecutive steps near the current
 *              length's limit, down when it stays too low; waiting two steps
 *              keeps a one-step blip from moving it.
 *  [ER-SWITCH] same page, section "三、聪明的开关": speculation is switched on
 *              only when the predicted speedup exceeds 1.05, and then stays on
 *              until the batch ends.
 *  [ER-ROOF]   same section: the speedup comes from a roofline model (each
 *              step bound by compute or by memory bandwidth; with many
 *              sequences in flight the GPU is compute-bound and drafting plus
 *              verifying loses, with few it is memory-bound and idle compute
 *              makes verification cheap), calibrated once per model and
 *              hardware by fitting its parameters to run times measured at
 *              several batch sizes and sequence lengths.
 */
#ifndef SV_HOST_H
#define SV_HOST_H

#include <stddef.h>
#include <stdint.h>

#include "spec_verify.h" /* SV_API */

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------------
 * Per-prompt n-gram drafter [NG-TABLE].
 *
 * Each prompt has its own table; a rollout added during step s belongs to
 * step s, and beginning step s evicts the rollouts of steps <= s - window.
 * Drafting looks up the longest n (max_n down to 1) such that the last n
 * context tokens occur in the prompt's retained rollouts followed by at least
 * one more token; among those occurrences it takes the most recent one (the
 * latest step, then the latest rollout, then the latest position) and copies
 * up to k tokens that follow it in that rollout.
 */
typedef struct sv_ngram sv_ngram;

/* max_n in [1, 16], window >= 1; NULL on bad arguments. */
SV_API sv_ngram *sv_ngram_create(int32_t max_n, int32_t window);
SV_API void sv_ngram_destroy(sv_ngram *t);
/* Start the next training step (the first call starts step 0). */
SV_API void sv_ngram_begin_step(sv_ngram *t);
/* Add a finished rollout of prompt_id to the current step.  Returns 0, or -1
 * on bad arguments (n < 0, tokens NULL with n > 0). */
SV_API int32_t sv_ngram_add(sv_ngram *t, int64_t prompt_id, const int32_t *tokens, int64_t n);
/* Draft up to k tokens continuing context[0..n) into out[0..k); returns the
 * number written (0 when nothing matches). */
SV_API int32_t sv_ngram_draft(const sv_ngram *t, int64_t prompt_id, const int32_t *context,
                              int64_t n, int32_t k, int32_t *out);
/* Ranked candidates for the next token after context[0..n): the distinct
 * tokens that follow an occurrence of the longest matching n-gram, by
 * number of occurrences (ties: the more recent occurrence first); at most
 * f written to out, count returned. */
SV_API int32_t sv_ngram_candidates(const sv_ngram *t, int64_t prompt_id, const int32_t *context,
                                   int64_t n, int32_t f, int32_t *out);
/* Rollouts and tokens currently retained (for tests and memory accounting). */
SV_API int64_t sv_ngram_rollouts(const sv_ngram *t);
SV_API int64_t sv_ngram_tokens(const sv_ngram *t);

/* ------------------------------------------------------------------------
 * Suffix drafter with frequency scoring [DAS-TREE].
 *
 * For every problem, every context of length d <= max_depth that occurs in
 * the problem's trajectories maps to the counts of the tokens that follow it
 * (the frequencies in the subtree below the matched node of a suffix tree cut
 * at depth max_depth + 1).  Drafting repeats k times: find the longest
 * d <= max_depth whose last-d-token context has a count table, append its
 * most frequent next token (ties: the lowest id), stop when nothing matches.
 * sv_suffix_append extends a live trajectory and counts the new contexts at
 * once, so verified tokens are visible to the next draft.
 */
typedef struct sv_suffix sv_suffix;

/* max_depth in [1, 64]; NULL on bad arguments. */
SV_API sv_suffix *sv_suffix_create(int32_t max_depth);
SV_API void sv_suffix_destroy(sv_suffix *t);
/* Drop every trajectory and count (the end of a training step). */
SV_API void sv_suffix_clear(sv_suffix *t);
/* Append tokens[0..m) to trajectory seq_id of problem_id (created empty on
 * first use).  Returns 0 or -1 on bad arguments. */
SV_API int32_t sv_suffix_append(sv_suffix *t, int64_t problem_id, int64_t seq_id, const int32_t *tokens,
                                int64_t m);
/* Draft up to k tokens continuing context[0..n); returns the number written. */
SV_API int32_t sv_suffix_draft(const sv_suffix *t, int64_t problem_id, const int32_t *context, int64_t n,
                               int32_t k, int32_t *out);
/* Ranked next-token candidates after context[0..n) from the longest match
 * (by count, ties: lowest id); at most f written, count returned. */
SV_API int32_t sv_suffix_candidates(const sv_suffix *t, int64_t problem_id, const int32_t *context,
                                    int64_t n, int32_t f, int32_t *out);

/* ------------------------------------------------------------------------
 * Batched drafting straight into the verification inputs.
 *
 * One call drafts for a whole batch and writes the drafted-id and length
 * arrays of spec_verify's one-hot path (no draft logits).  Request b
 * continues ctx[ctx_off[b] .. ctx_off[b+1]) of prompt (problem) ids[b] and
 * drafts up to cap_b = min(k_max, max_lens[b]) tokens (k_max alone when
 * max_lens is NULL; a cap from the draft-length controller or the request
 * budgets goes there).  The result is exactly what the single-request draft
 * call returns with k = cap_b:
 *   out_tokens[b][0 .. m_b)      the drafted ids;
 *   out_tokens[b][m_b .. k_max)  -1;
 *   out_lens[b] = m_b.
 * A request with no match gets m_b = 0, which spec_verify treats as no
 * speculation (one token drawn from target row 0).
 *
 * Layouts: ids[B]; ctx_off[B+1], non-decreasing from ctx_off[0] >= 0, with
 * ctx holding at least ctx_off[B] tokens; max_lens[B] or NULL; out_tokens
 * [B][k_max] row-major; out_lens[B].  All host memory, owned by the caller.
 * The table is only read, so requests run concurrently on up to n_threads
 * host threads (0 = one per hardware thread; small batches use fewer).  The
 * table must not be modified during the call.  Returns 0, or -1 on bad
 * arguments (NULL pointers, B < 0, k_max outside [0, SV_MAX_K], decreasing
 * offsets, a negative cap, n_threads < 0); nothing is written then.
 */
SV_API int32_t sv_ngram_draft_batch(const sv_ngram *t, int32_t B, const int64_t *ids, const int32_t *ctx,
                                    const int64_t *ctx_off, int32_t k_max, const int32_t *max_lens,
                                    int32_t n_threads, int32_t *out_tokens, int32_t *out_lens);
SV_API int32_t sv_suffix_draft_batch(const sv_suffix *t, int32_t B, const int64_t *ids, const int32_t *ctx,
                                     const int64_t *ctx_off, int32_t k_max, const int32_t *max_lens,
                                     int32_t n_threads, int32_t *out_tokens, int32_t *out_lens);

/* ------------------------------------------------------------------------
 * Fan-out prefetch budget [NG-FETCH].
 *
 * Observations are verification outcomes: j in [0, k] accepted drafts and the
 * rank of the emitted token b among the drafter's ranked candidates for
 * branch j (0 = top candidate, -1 = not among the first fmax).  Only the last
 * `window` observations count (causal sliding window).  Estimates:
 *   P(j)    = share of the window with outcome j;
 *   c_j(f)  = share of branch-j observations whose rank is < f, f = 0..fmax
 *             (c_j(0) = 0); a branch without observations uses the profile
 *             pooled over all branches.
 * sv_prefetch_allocate spends `budget` candidates one at a time on the
 * branch with the largest gain P(j) (c_j(f_j + 1) - c_j(f_j)) (ties: the
 * lower j), never beyond fmax per branch, and stops early when no gain is
 * positive; out_f[j] = candidates for branch j.  Returns the expected
 * coverage sum_j P(j) c_j(f_j).  An empty window allocates nothing (every
 * outcome then takes the synchronous lookup).
 */
typedef struct sv_prefetch sv_prefetch;

/* k >= 0 drafts per step, fmax >= 1, window >= 1; NULL on bad arguments. */
SV_API sv_prefetch *sv_prefetch_create(int32_t k, int32_t fmax, int32_t window);
SV_API void sv_prefetch_destroy(sv_prefetch *p);
/* Record one outcome; returns 0 or -1 (j outside [0, k], rank < -1). */
SV_API int32_t sv_prefetch_observe(sv_prefetch *p, int32_t j, int32_t b_rank);
/* P_j[0..k] and coverage[(k+1) x (fmax+1)] (row j, column f); either may be
 * NULL.  Returns the number of observations in the window. */
SV_API int32_t sv_prefetch_estimates(const sv_prefetch *p, double *P_j, double *coverage);
SV_API double sv_prefetch_allocate(const sv_prefetch *p, int32_t budget, int32_t *out_f);

/* ------------------------------------------------------------------------
 * Fan-out prefetch of the next draft [NG-FETCH].
 *
 * While the GPU verifies draft d[0..L) of a request that continues
 * context[0..n), the host drafts ahead for the outcomes the budget covers.
 * After outcome (j, b) -- j drafts accepted, b the emitted token -- the
 * request continues context + d[0..j) + b.  Branch j takes the f[j]
 * top-ranked candidates b for the token after context + d[0..j) (the
 * sv_ngram_candidates ranking, the same ranking whose rank of the actual b
 * feeds sv_prefetch_observe), and each (j, b) gets the next draft
 * sv_ngram_draft(context + d[0..j) + b, k).  Entries are written in order of
 * j, then candidate rank:
 *   out_j[e], out_b[e], out_tokens[e][0..k) (-1 padded), out_lens[e];
 * at most max_entries of them.  f[0..L] (from sv_prefetch_allocate with this
 * request's L as k) may ask for more candidates than a branch has; such a
 * branch gets what exists.  Returns the entry count, or -1 on bad arguments
 * (NULL pointers, n < 0, L < 0, L > SV_MAX_K, a negative f[j], k outside
 * [0, SV_MAX_K], max_entries < 0).  All arrays are host memory owned by the
 * caller; the table is only read.
 *
 * When verification reports (j, b), sv_prefetch_find returns the entry that
 * holds its next draft (a hit) or -1 (a miss: draft synchronously).
 */
SV_API int32_t sv_ngram_prefetch(const sv_ngram *t, int64_t prompt_id, const int32_t *context, int64_t n,
                                 const int32_t *draft, int32_t L, const int32_t *f, int32_t k,
                                 int32_t max_entries, int32_t *out_j, int32_t *out_b, int32_t *out_tokens,
                                 int32_t *out_lens);
/* The entry e < count with out_j[e] == j and out_b[e] == b, or -1. */
SV_API int32_t sv_prefetch_find(const int32_t *out_j, const int32_t *out_b, int32_t count, int32_t j, int32_t b);

/* ------------------------------------------------------------------------
 * Adaptive draft length [ER-LEN].
 *
 * Candidate lengths ascending (e.g. 5, 7, 9, 11); the controller starts at
 * the first.  Each training step reports its block efficiency tau (verified
 * tokens per draft-verify cycle, at most k + 1 for draft length k).  With
 * r = tau / (k + 1): `patience` consecutive steps with r >= up_frac move to
 * the next longer length, `patience` consecutive steps with r < down_frac
 * move to the next shorter one; a move resets both streaks.  Defaults (a
 * reading; the page gives no numbers): up_frac 0.7, down_frac 0.4,
 * patience 2.
 */
typedef struct sv_draft_len sv_draft_len;

/* n_lengths in [1, 64], lengths strictly ascending and >= 1, 0 <= down_frac
 * <= up_frac <= 1, patience >= 1; NULL on bad arguments. */
SV_API sv_draft_len *sv_draft_len_create(const int32_t *lengths, int32_t n_lengths, double up_frac,
                                         double down_frac, int32_t patience);
SV_API void sv_draft_len_destroy(sv_draft_len *c);
SV_API int32_t sv_draft_len_current(const sv_draft_len *c);
/* Report one step's block efficiency; returns the length for the next step. */
SV_API int32_t sv_draft_len_update(sv_draft_len *c, double block_efficiency);
/* Block efficiency of a batch of outcomes: mean of (accept_len + 1) over the
 * entries with accept_len >= 0 (invalid requests, -1 / -2, are skipped);
 * NaN when none is valid. */
SV_API double sv_block_efficiency(const int32_t *accept_len, int64_t n);

/* Speculation switch [ER-SWITCH]: returns 1 once any predicted speedup has
 * exceeded the threshold (1.05 on the page) since *state was set to 0, and
 * keeps returning 1 until the caller resets *state for the next batch. */
SV_API int32_t sv_spec_switch(int32_t *state, double predicted_speedup, double threshold);

/* ------------------------------------------------------------------------
 * Roofline predictor behind the switch [ER-ROOF].
 *
 * A forward step of a decoder over B sequences, q new tokens each, with n
 * tokens already cached per sequence, is either compute- or memory-bound:
 *   flops(B, q, n) = 2 N B q + 4 L d B q n        (weights; attention over n)
 *   bytes(B, q, n) = N w + 2 L h d_h e B n        (weights once; K and V read)
 *   T(B, q, n)     = max(flops / pi, bytes / beta) + tau
 * (a reading: the page names the two ceilings and a calibration, not the
 * terms).  pi, beta and tau are calibrated once per model and machine from
 * measured step times (sv_roofline_fit).  A speculative cycle with draft
 * length k drafts k tokens one at a time and verifies k + 1 positions in one
 * target step; with per-token acceptance alpha it yields
 *   E = (1 - alpha^(k+1)) / (1 - alpha)  tokens   (E = k + 1 at alpha = 1),
 * so the predicted speedup over plain decoding is
 *   S = E T_t(B, 1, n) / (k T_d(B, 1, n) + T_t(B, k + 1, n)),
 * which sv_spec_switch compares with 1.05.
 */
typedef struct {
    double params;        /* N: weights */
    double weight_bytes;  /* w: bytes per weight as stored (2 for bf16; ~0.56 for 4-bit with group scales) */
    int32_t layers;       /* L */
    int32_t width;        /* d: query heads x head dim */
    int32_t kv_heads;     /* h */
    int32_t head_dim;     /* d_h */
    double kv_bytes;      /* e: bytes per cached K or V element */
} sv_arch;

typedef struct {
    double flops_per_s;   /* pi */
    double bytes_per_s;   /* beta */
    double overhead_s;    /* tau */
} sv_roofline;

/* flops and bytes of one step; 0, or -1 on bad arguments (NULL, a negative
 * or non-finite count, an architecture with a non-positive field). */
SV_API int32_t sv_roofline_work(const sv_arch *a, double B, double q, double n, double *flops, double *bytes);
/* T(B, q, n) in seconds; NaN on bad arguments. */
SV_API double sv_roofline_time(const sv_arch *a, const sv_roofline *r, double B, double q, double n);
/* Calibrate pi, beta, tau on m >= 3 measured steps (B[i], q[i], n[i],
 * seconds[i] > 0): minimises the squared relative error
 * sum_i ((T_i - seconds_i) / seconds_i)^2.  For fixed pi and beta the best
 * tau >= 0 has a closed form; pi and beta are searched on a 41 x 41 log10
 * grid from one decade below to three above the largest flops and bytes per
 * measured second, then seven more times on a 10x finer grid spanning two
 * steps of the previous one either side of its best point.  Writes the fit
 * and, if rms_rel is not NULL,
 * the root-mean-square relative error.  Returns 0, or -1 on bad arguments. */
SV_API int32_t sv_roofline_fit(const sv_arch *a, int32_t m, const double *B, const double *q, const double *n,
                               const double *seconds, sv_roofline *out, double *rms_rel);
/* Predicted speedup S of speculative decoding (above); NaN on bad
 * arguments (alpha outside [0, 1], k < 1, B <= 0, n < 0). */
SV_API double sv_spec_speedup(const sv_arch *target, const sv_roofline *rt, const sv_arch *draft,
                              const sv_roofline *rd, double B, int32_t k, double alpha, double n);

/* ------------------------------------------------------------------------
 * Length-aware budgets [DAS-LEN].
 *
 * sv_length_classes: classes from predicted lengths (e.g. the mean rollout
 * length of the prompt so far): the n requests sorted by predicted length,
 * longest first (ties: lower index first); the first n/3 (integer division)
 * are Long (class 2), the last n/3 Short (class 0), the rest Medium
 * (class 1).  budgets are the draft lengths per class {Short, Medium, Long}
 * (Short 0 skips speculation); out_budget[i] = budgets[class].  Returns 0, or
 * -1 on bad arguments.
 *
 * sv_interleave_ranks: spreads requests over world_size ranks: sorted by
 * predicted length, longest first (ties: lower index first), dealt
 * round-robin, so every rank gets an equal share of the long ones.
 */
SV_API int32_t sv_length_classes(const double *predicted_len, int64_t n, const int32_t budgets[3],
                                 int32_t *out_class, int32_t *out_budget);
SV_API int32_t sv_interleave_ranks(const double *predicted_len, int64_t n, int32_t world_size,
                                   int32_t *out_rank);

#ifdef __cplusplus
}
#endif

#endif /* SV_HOST_H */
