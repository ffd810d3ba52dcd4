/*
 * spec_verify.h -- C ABI of the B200 (sm_100a) speculative-sampling
 * verification library (libspecverify.so).
 *
 * What it computes.  For each request b of a batch, a drafter proposed
 * L_b <= k_max tokens x_0 .. x_{L_b-1}.  The target model's logits for the
 * L_b + 1 positions (and, for a model drafter, the draft model's logits for
 * the L_b drafted positions) are given.  The library runs the lossless
 * verification rule described on the pages:
 *
 *   - temperature softmax of every used row: p_i = softmax(Z_i / T),
 *     q_i = softmax(Y_i / T) (or q_i = one-hot at x_i when there are no draft
 *     logits -- n-gram / suffix-tree drafters supply ids only);
 *   - draft i is accepted with probability min(1, p_i(x_i) / q_i(x_i)), in
 *     order, stopping at the first rejection ("AI 开始抄自己的作业——而且抄得理直气壮",
 *     zhichai.net, section "⚡ 投机解码：让草稿先跑，考官殿后"; and
 *     "今热点：让AI草稿模型学会"照镜子"" (001ce.com), section
 *     "先搞懂投机解码在干什么");
 *   - on a rejection at position j the token is redrawn from the residual
 *     distribution normalise(max(0, p_j - q_j)) (same NgramRL section);
 *   - when every draft is accepted, a bonus token is drawn from p at row
 *     L_b (same page, section "🚰 真正的瓶颈不在算法，在流水线": the step's
 *     outcome is the pair (j, b));
 *   - greedy mode replaces sampling by prefix matching against the target's
 *     argmax ("NgramRL：用Rollout历史加速RL后训练的推测解码新方案",
 *     kongchang.com, section "一个被忽视的草稿源", glossary entry), ties going
 *     to the lowest index.
 *
 * Readings where the pages are silent: uniforms[b][i] (i < L_b) is the
 * acceptance draw of draft i and accept iff u < a; uniforms[b][k_max] drives
 * the final draw; the draw picks the smallest token t whose running weight
 * sum exceeds u * W (W = total weight); a zero residual mass (only possible
 * when p == q) falls back to drawing from p_j.
 *
 * Layouts (all row-major, "elements" are of the logit dtype):
 *   target_logits  [B][k_max+1][row_stride]   rows 0..L_b are read
 *   draft_logits   [B][k_max][row_stride]     rows 0..L_b-1 are read; NULL = one-hot q
 *   draft_tokens   [B][k_max] int32           entries 0..L_b-1 are read
 *   draft_lens     [B] int32 in [0, k_max]    NULL = every request uses k_max
 *   uniforms       [B][k_max+1] float32 in [0, 1)
 *   out_accept_len [B] int32                  j, the number of accepted drafts
 *   out_tokens     [B][k_max+1] int32         x_0..x_{j-1}, then the drawn token at
 *                                             index j, then -1 up to index k_max
 * Padded rows (beyond L_b) and columns V..row_stride-1 are never read, so
 * they may hold anything (NaN included).
 *
 * Ownership and execution.  Every pointer argument of spec_verify,
 * spec_verify_ex and spec_verify_stats is DEVICE memory owned by the caller
 * (spec_verify_host takes host buffers, see there).  The library allocates
 * nothing.  Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL
 * = legacy default stream) as a chain of kernels -- a control-word reset, row
 * statistics, the acceptance scan and (sampling only) the final draw, plus
 * the selection of residual draws when draft logits are given; results are
 * valid once the stream has reached the call's end.  The workspace (per-piece row statistics and
 * the queue of draws) needs no initialisation and holds nothing between
 * calls; two calls that run concurrently need separate workspaces.
 * The host keeps one small per-device cache of SM count and kernel
 * attributes.
 *
 * Errors.  Argument errors are found on the host before anything is
 * enqueued and return SV_EINVAL (NULL required pointer, B < 0, k_max < 0,
 * V < 1, row_stride < V, greedy off with temperature <= 0 or non-finite,
 * uniforms NULL with greedy off, workspace too small) or SV_EUNSUPPORTED
 * (k_max > SV_MAX_K, V > SV_MAX_V, unknown dtype).  A failed launch returns
 * SV_ECUDA.  Values that can only be checked on the device never cause an
 * out-of-bounds access: a request whose draft_lens entry is outside
 * [0, k_max] or whose first L_b drafted ids are outside [0, V) gets
 * out_accept_len = -1 and out_tokens all -1; a request whose statistics or
 * final draw were lost to a device-side wait timeout gets out_accept_len = -2
 * and out_tokens all -1 (tests make a wait run out through
 * sv_options.lost_copy_request / lost_draw_request).  NaN or +inf logits in
 * rows that are read give unspecified (but in-bounds) results.
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SV_API __attribute__((visibility("default")))
#else
#define SV_API
#endif

#define SV_ABI_VERSION 3
#define SV_MAX_K 1024      /* largest supported k_max */
#define SV_MAX_V 393216    /* largest supported vocabulary (96 pieces of 16 KiB in fp32) */

typedef enum { SV_F32 = 0, SV_BF16 = 1 } sv_dtype;

typedef enum {
    SV_OK = 0,
    SV_EINVAL = 1,
    SV_ECUDA = 2,
    SV_EUNSUPPORTED = 3,
    SV_ESCRATCH = 4    /* spec_verify_static_scratch: problem larger than its fixed scratch area */
} sv_status;

/* Problem shape.  row_stride is in elements between consecutive rows
 * (>= V); 0 means V. */
typedef struct {
    int32_t B;
    int32_t k_max;
    int32_t V;
    int32_t dtype; /* sv_dtype of both logit tensors */
    int64_t row_stride;
} sv_shape;

/* Which row-statistics kernel to run (spec_verify_ex).  AUTO picks the TMA
 * bulk-copy pipeline when every row start is 16-byte aligned, else scalar
 * loads. */
typedef enum {
    SV_STATS_AUTO = 0,
    SV_STATS_TMA = 1,    /* cp.async.bulk + mbarrier ring; needs 16-byte aligned rows */
    SV_STATS_VEC16 = 2,  /* 16-byte vector loads; needs 16-byte aligned rows */
    SV_STATS_SCALAR = 3  /* element loads; any alignment */
} sv_stats_kernel;

typedef struct {
    int32_t stats_kernel;      /* sv_stats_kernel */
    int32_t wait_timeout_us;   /* bound on each device-side barrier wait; 0 = 2 s */
    void *event_stats_begin;   /* cudaEvent_t recorded just before the row-statistics kernel, or NULL */
    void *event_stats_end;     /* cudaEvent_t recorded just after it, or NULL */
    /* Fault injection for tests of the wait bound; 0 = off.  A value r > 0
     * names request b = r - 1 (0 <= b < B): the bulk-copy statistics kernel
     * then never issues the copy of the first piece of b's target row 0.
     * The wait on that stage runs out after wait_timeout_us, and b
     * gets out_accept_len = -2 (so may other requests whose statistics fell
     * to the same CTA after it); the call itself still returns SV_OK and the
     * context stays usable.  Needs the bulk-copy kernel (SV_STATS_TMA, or
     * AUTO on aligned rows): with any other kernel, SV_EUNSUPPORTED. */
    int32_t lost_copy_request;
    /* Fault injection for tests of the draw kernel's wait bound; 0 = off.  A
     * value r > 0 names request b = r - 1: if b needs a sampled draw, the
     * draw kernel never issues the copy of the first piece it stages for b,
     * so its bounded wait runs out after wait_timeout_us; b (and any later
     * draw of the same CTA) gets out_accept_len = -2, the call returns SV_OK
     * and the context stays usable.  No effect on calls without a draw
     * (greedy, statistics). */
    int32_t lost_draw_request;
    /* How a sampling call makes its final draws (sv_draw_path).  AUTO: one
     * thread-block cluster per request when the batch's clusters fit on the
     * GPU at once (small batches: the scan and the draw in one kernel), else
     * the scan kernel, the draw kernel over a queue of pieces and the
     * residual selection kernel.  The outputs are the same either way. */
    int32_t draw_path;
    int32_t reserved[5];       /* must be zero */
} sv_options;

typedef enum {
    SV_DRAW_AUTO = 0,
    SV_DRAW_QUEUE = 1,    /* scan kernel, draw kernel, selection kernel */
    SV_DRAW_CLUSTER = 2   /* one cluster of up to 16 CTAs per request */
} sv_draw_path;

/* Bytes of device workspace spec_verify / spec_verify_stats need for this
 * shape (0 on an invalid shape). */
SV_API size_t spec_verify_workspace_bytes(const sv_shape *shape);

/* One verification step for the whole batch (see the top of this file).
 * greedy != 0 selects prefix matching against the target argmax; then
 * draft_logits, uniforms and temperature are ignored and may be NULL / 0. */
SV_API sv_status spec_verify(const sv_shape *shape, const void *target_logits,
                      const void *draft_logits, const int32_t *draft_tokens,
                      const int32_t *draft_lens, const float *uniforms,
                      float temperature, int32_t greedy,
                      int32_t *out_accept_len, int32_t *out_tokens,
                      void *workspace, size_t workspace_bytes, void *stream);

/* spec_verify with launch options (kernel choice, timing events, wait
 * bound); opts == NULL is spec_verify. */
SV_API sv_status spec_verify_ex(const sv_shape *shape, const void *target_logits,
                         const void *draft_logits, const int32_t *draft_tokens,
                         const int32_t *draft_lens, const float *uniforms,
                         float temperature, int32_t greedy,
                         int32_t *out_accept_len, int32_t *out_tokens,
                         void *workspace, size_t workspace_bytes, void *stream,
                         const sv_options *opts);

/* Diagnostic / test hook running the same row-statistics kernel: per used
 * row the natural-log log-sum-exp of Z/T (out_lse_target [B][k_max+1]) and
 * Y/T (out_lse_draft [B][k_max], may be NULL), and p_i(x_i), q_i(x_i)
 * (out_p, out_q [B][k_max]; q = 1 without draft logits).  Entries of rows a
 * request does not use are NaN; invalid requests get NaN everywhere. */
SV_API sv_status spec_verify_stats(const sv_shape *shape, const void *target_logits,
                            const void *draft_logits,
                            const int32_t *draft_tokens,
                            const int32_t *draft_lens, float temperature,
                            float *out_lse_target, float *out_lse_draft,
                            float *out_p, float *out_q, void *workspace,
                            size_t workspace_bytes, void *stream,
                            const sv_options *opts);

/* Acceptance simulation over a batch of drafted sequences, for training-time
 * use: the same row-statistics pass and acceptance rule as spec_verify,
 * without the final draw ("今热点：让AI草稿模型学会"照镜子"：训练时就知道自己会不会被
 * 打回", sections "VAT怎么把"验收规则"塞进训练里" and "第二件事，改权重分配的锚点":
 * the verification is simulated with the probability-ratio rule, everything
 * from the first rejection on is marked rejected, and the per-position loss
 * weights keep full weight up to the first rejection and start the decay
 * curve there).  Inputs are those of spec_verify; uniforms may be NULL.
 *
 *   out_accept_prob [B][k_max]  a_i = min(1, p_i(x_i) / q_i(x_i)) for i < L_b,
 *                               NaN for i >= L_b (q = 1 without draft logits);
 *   out_expected_len [B]        E[j] = sum_{m=1..L_b} prod_{l<m} a_l, the
 *                               expected number of accepted drafts;
 *   out_first_reject [B]        (needs uniforms, else must be NULL) the first
 *                               i < L_b with !(u_i < a_i), else L_b -- the j
 *                               spec_verify returns for the same inputs;
 *   out_weights [B][k_max]      (needs uniforms, else must be NULL) 1 for
 *                               i <= j, decay^(i - j) for j < i < L_b, 0 for
 *                               i >= L_b; decay in [0, 1] (0.8 is the fixed
 *                               per-position curve of the EAGLE-3 recipe the
 *                               page cites, 0 the hard cut-off of its
 *                               ablation).
 *
 * out_accept_prob and out_expected_len are required.  A request with an
 * invalid length or drafted id gets out_first_reject = -1 and NaN elsewhere;
 * one whose statistics were lost to a wait timeout gets -2.  Same ownership,
 * stream and workspace rules as spec_verify_stats. */
SV_API sv_status spec_verify_accept_sim(const sv_shape *shape, const void *target_logits,
                                        const void *draft_logits,
                                        const int32_t *draft_tokens,
                                        const int32_t *draft_lens, const float *uniforms,
                                        float temperature, float decay,
                                        float *out_accept_prob, float *out_expected_len,
                                        int32_t *out_first_reject, float *out_weights,
                                        void *workspace, size_t workspace_bytes,
                                        void *stream);

/* Bytes of caller-provided device staging memory spec_verify_host needs. */
SV_API size_t spec_verify_host_staging_bytes(const sv_shape *shape, int32_t has_draft,
                                      int32_t has_lens);

/* End-to-end form taking HOST buffers (same layouts as spec_verify): copies
 * the inputs into `device_staging` (cudaMemcpyAsync on `stream`), verifies,
 * and copies out_accept_len / out_tokens back to the host buffers.  Of the
 * logits only the rows the method reads are copied when h_draft_lens is
 * given: target rows 0..L_b and draft rows 0..L_b-1 of each request (L_b
 * clamped to [0, k_max]), one copy per contiguous run; the staging rows
 * past them keep their old contents and are never read.  The
 * copies are asynchronous only when the host buffers are page-locked;
 * results are valid after the stream is synchronised.  `device_staging`
 * (spec_verify_host_staging_bytes) and `workspace` are caller-owned device
 * memory; the library allocates nothing. */
SV_API sv_status spec_verify_host(const sv_shape *shape, const void *h_target_logits,
                           const void *h_draft_logits,
                           const int32_t *h_draft_tokens,
                           const int32_t *h_draft_lens, const float *h_uniforms,
                           float temperature, int32_t greedy,
                           int32_t *h_out_accept_len, int32_t *h_out_tokens,
                           void *device_staging, size_t staging_bytes,
                           void *workspace, size_t workspace_bytes,
                           void *stream);

/* Static description of a status code. */
SV_API const char *spec_verify_status_string(sv_status status);

/* The draw path (sv_draw_path) that SV_DRAW_AUTO takes for a sampling call
 * of this shape on the current device: SV_DRAW_CLUSTER or SV_DRAW_QUEUE; -1
 * on an invalid shape or a CUDA error.  No work is enqueued. */
SV_API int32_t spec_verify_auto_draw_path(const sv_shape *shape);

/* SV_ABI_VERSION of the built library. */
SV_API int32_t spec_verify_abi_version(void);

/* Allocation-free form of spec_verify, for callers that cannot hand the
 * library any device memory of its own: code running while a stream is being
 * captured into a CUDA graph (allocating then breaks or invalidates the
 * capture), plain C hosts or runtimes that have no device allocator at hand,
 * and services that reserve all device memory up front and forbid ad-hoc
 * allocations.  The pages describe nothing like it; it exists only for those
 * callers.
 *
 * It runs exactly the kernels of spec_verify, but their scratch (the
 * row-statistics partials, spec_verify_workspace_bytes(shape) bytes) lives in
 * one fixed array of SV_STATIC_SCRATCH_BYTES bytes inside the library
 * instead of a caller-provided workspace.  Every GPU that loads the library
 * holds that array until the process exits.  Inputs and outputs are still the
 * caller's device buffers, as for spec_verify.
 *
 * - Shapes whose workspace would exceed SV_STATIC_SCRATCH_BYTES are rejected
 *   with SV_ESCRATCH before anything is enqueued; use spec_verify then.
 * - The library calls no cudaMalloc / cudaFree or any allocating routine.  The
 *   first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it together
 *   with the id of the device's current context; make that first call on a
 *   device before capturing a stream.  If the context is replaced (for
 *   example cudaDeviceReset, then new work on the device), the next call sees
 *   a different context id and looks the address up again, so it never uses
 *   an address of a destroyed context; make that call before any capture too.
 * - All calls share the one array and it keeps the last call's contents (no
 *   part of it needs to start at zero).  Calls whose work overlaps on the GPU
 *   (different streams, or different host threads, without ordering between
 *   them) race on it and give wrong results; order them on one stream.
 */
#define SV_STATIC_SCRATCH_BYTES (1u << 20)
SV_API sv_status spec_verify_static_scratch(const sv_shape *shape,
                                            const void *target_logits,
                                            const void *draft_logits,
                                            const int32_t *draft_tokens,
                                            const int32_t *draft_lens,
                                            const float *uniforms,
                                            float temperature, int32_t greedy,
                                            int32_t *out_accept_len,
                                            int32_t *out_tokens, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H */
