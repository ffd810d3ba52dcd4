// sv_fused.cuh -- the whole sampling step in one persistent launch.
//
// The work of K1 (row statistics) and K2 (scan and draw) runs through the
// same bulk-copy ring, in one grid of resident CTAs:
//
//  * stats items (row, chunk) as in K1, handed out in request order through a
//    global ticket; every consumer warp stores its own (m, s) partial per item,
//    so a row has C x W partials (W consumer warps) and no warp ever waits for
//    another;
//  * the warp that stores the last partial of request b (a per-request
//    counter) runs b's scan at once: it merges the partials, takes p and q at
//    the drafted ids, finds j, writes the accepted prefix, and enqueues b's
//    draw tasks:
//      - residual draw: C tasks, one per chunk, over target and draft row j;
//      - bonus or one-hot draw: the chunk that holds u*W (chosen from the
//        partials), one task;
//  * a draw task streams its chunk through the ring, each warp storing the
//    weight sums of its 32-vector segments; the warp that finishes the
//    request's last task picks the chunk (residual), then the segment, vector
//    and element, and writes the drawn token.
//
// Draw tasks take priority over stats items, so a request's draw runs soon
// after its rows were streamed, mostly from L2.  The producer lane of every
// CTA claims work.  Nothing waits on another CTA for correctness:
//  * a CTA out of stats items polls for draw tasks (with back-off) only until
//    every request is done;
//  * the warp that enqueues tasks belongs to a CTA whose producer keeps
//    claiming, so no task is left behind.
// Waits: the ring's mbarriers and a claimed task slot whose enqueuer is still
// writing it, all bounded by timeout_ns.  After a timeout the CTA stops, and
// the last CTA to exit marks every request left unfinished with -2.
//
// The rule each step follows is that of K1 / K2 (sv_row_stats.cuh,
// sv_verify_draw.cuh) and the pages cited there.
#pragma once

#include "sv_common.cuh"
#include "sv_row_stats.cuh"
#include "sv_verify_draw.cuh"

namespace sv {

// Counters of one launch (zeroed by the host before the launch).
struct FusedState {
    int32_t stats_next;      // next stats ticket
    int32_t dispatch;        // draw tasks handed out so far (task n goes to CTA n % grid)
    int32_t unused;
    int32_t requests_done;   // requests whose outputs are final
    int32_t ctas_exited;
    int32_t error;           // a bounded wait ran out somewhere
    int32_t pad[2];
};

// Per-request record written by the scan for the draw tasks.
struct FusedReq {
    float lse_p, lse_q;      // row j, log2 domain (lse_q: residual only)
    float local_target;      // bonus / one-hot: u*W minus the chunks before kstar
    float ustar;
    int32_t j, mode, kstar, zero_at;
    int32_t ntasks;          // draw tasks of this request
    int32_t pad[3];
};

struct FusedParams {
    const unsigned char* target;   // [B][k_max+1][row_stride]
    const unsigned char* draft;    // [B][k_max][row_stride] or null (one-hot q)
    const int32_t* tokens;         // [B][k_max]
    const int32_t* lens;           // [B] or null
    const float* uniforms;         // [B][k_max+1]
    int32_t* out_len;
    int32_t* out_tokens;
    float2* partials;              // [B][2k_max+1][C][W]
    FusedState* state;             // zeroed
    int32_t* done_items;           // [B] zeroed: warp-items stored
    int32_t* draw_done;            // [B] zeroed: warp-tasks finished
    int32_t* final_flag;           // [B] zeroed: outputs written
    int32_t* mbox_ready;           // [grid][mbox_slots] zeroed: a task was posted
    int32_t* mbox_task;            // [grid][mbox_slots] (b * C + chunk) * P + piece
    FusedReq* req;                 // [B]
    float* segs;                   // [B][C][nseg_max]
    float* piece_tot;              // [B][C][P][W] per-warp sums of a draw task's segments
    int32_t B, k_max, V;
    int64_t row_stride;
    int32_t C, CE, nseg_max;
    int32_t P;                     // draw pieces (one ring stage each) per chunk
    int32_t mbox_slots;            // ceil(B*C*P / grid) + 1 task slots per CTA
    float scale;                   // log2(e) / T
    uint64_t timeout_ns;
};

// Workspace carve-up (all parts 256-byte aligned); W consumer warps.
struct FusedLayout {
    size_t partials, state, done_items, draw_done, final_flag, mbox_ready, mbox_task, req, segs, piece_tot, total;
    size_t zero_begin, zero_end;   // the span the host zeroes before a launch
};

__host__ __device__ inline size_t fused_align(size_t n) { return (n + 255) & ~size_t(255); }

// Largest grid of the fused launch; the mailboxes hold B*C*P + 2*kMaxFusedGrid
// slots, enough for grid * (ceil(B*C*P / grid) + 1) whenever grid <= kMaxFusedGrid.
constexpr int kMaxFusedGrid = 1024;

__host__ __device__ inline FusedLayout fused_layout(int B, int k_max, int C, int W, int nseg_max, int P) {
    FusedLayout l;
    size_t o = 0;
    l.partials = o;    o += fused_align(sizeof(float2) * size_t(B) * (2 * size_t(k_max) + 1) * C * W);
    l.state = o;       o += fused_align(sizeof(FusedState));
    l.done_items = o;  o += fused_align(4 * size_t(B));
    l.draw_done = o;   o += fused_align(4 * size_t(B));
    l.final_flag = o;  o += fused_align(4 * size_t(B));
    const size_t mbox = size_t(B) * C * P + 2 * size_t(kMaxFusedGrid);
    l.mbox_ready = o;  o += fused_align(4 * mbox);
    l.zero_begin = l.state;
    l.zero_end = o;
    l.mbox_task = o;   o += fused_align(4 * mbox);
    l.req = o;         o += fused_align(sizeof(FusedReq) * size_t(B));
    l.segs = o;        o += fused_align(4 * size_t(B) * C * nseg_max);
    l.piece_tot = o;   o += fused_align(4 * size_t(B) * C * P * W);
    l.total = o;
    return l;
}

// Stage metadata of the fused ring.
struct FusedMeta {
    const unsigned char* tail;  // stats: ragged-tail elements of the row's last chunk
    int64_t partial_idx;        // stats: (b * (2k+1) + slot) * C + c
    int32_t elem0;              // stats: row index of the first element; draw: first vector of the piece
    int32_t n_bytes;            // bytes per row delivered by the bulk copies
    int32_t tail_n;             // stats
    int32_t flags;              // kFirst | kLast | kDraw | kResid | kDone
    int32_t b, c;               // request, chunk
    // draw pieces: row j's statistics and the request's task count
    float lse_p, lse_q;
    int32_t j, zero_at, ntasks;
};
constexpr int kFirst = 1, kLast = 2, kDraw = 4, kResid = 8, kDone = 16;
constexpr int kPieceBytes = 8192;                 // per row and stage of a draw task
constexpr int kPieceVecsF = kPieceBytes / 16;     // 512 vectors = 16 segments

// ring | metas | barriers | misc | row prefix [B+1] | per-warp segment sums [W][nseg_max]
template <int kConsumerWarps, int kStages>
struct FusedSmem {
    static constexpr size_t kMetaOff = size_t(kStages) * kStageBytes;
    static constexpr size_t kBarOff = kMetaOff + sizeof(FusedMeta) * kStages;
    static constexpr size_t kMiscOff = kBarOff + 16 * kStages;                            // full[], empty[]
    static constexpr size_t kRowOff = kMiscOff + 4 * 64;                                   // misc ints
    __host__ __device__ static size_t seg_off(int B) { return (kRowOff + 4 * size_t(B + 1) + 15) & ~size_t(15); }
    __host__ __device__ static size_t bytes(int B, int nseg_max) {
        return seg_off(B) + 4 * size_t(kConsumerWarps) * nseg_max;
    }
};

__device__ __forceinline__ int ld_acquire_s32(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int ld_relaxed_s32(const int32_t* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_s32(int32_t* p, int v) {
    asm volatile("st.relaxed.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_release_s32(int32_t* p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void nap(uint32_t ns) { asm volatile("nanosleep.u32 %0;" ::"r"(ns)); }
// Counter increment with release (this thread's earlier writes are visible
// before it) and acquire (the last arriver sees everyone's writes) semantics;
// much cheaper than a sequentially consistent fence around a plain atomic.
__device__ __forceinline__ int atom_add_acq_rel(int32_t* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Pieces of chunk c (the last chunk of a row can be shorter).
__device__ __forceinline__ int fused_pieces(const FusedParams& p, int c, int per_vec) {
    const int n = min(p.V - c * p.CE, p.CE);
    const int nvec = (n + per_vec - 1) / per_vec;
    return (nvec + kPieceVecsF - 1) / kPieceVecsF;
}

// Post the pieces of chunks c0 .. c0+nc-1 of request b as draw tasks: task
// number t (one global counter) goes to CTA t % grid, into its slot t / grid,
// so no CTA competes for a task and a request's pieces land on many CTAs.
// Returns the number of tasks posted.
template <typename T>
__device__ inline int fused_post(const FusedParams& p, int b, int c0, int nc) {
    constexpr int PV = Logit<T>::kPerVec;
    int total = 0;
    for (int c = c0; c < c0 + nc; ++c) total += fused_pieces(p, c, PV);
    const int t0 = atomicAdd(&p.state->dispatch, total);
    const int G = int(gridDim.x);
    int t = t0;
    for (int c = c0; c < c0 + nc; ++c) {
        const int np = fused_pieces(p, c, PV);
        for (int k = 0; k < np; ++k, ++t) p.mbox_task[(t % G) * p.mbox_slots + t / G] = (b * p.C + c) * p.P + k;
    }
    // one release fence orders the tasks (and the request record) before
    // every flag below
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    for (t = t0; t < t0 + total; ++t) st_relaxed_s32(p.mbox_ready + (t % G) * p.mbox_slots + t / G, 1);
    return total;
}

// Request b's outputs are final (lane 0 of the calling warp).
__device__ inline void fused_request_done(const FusedParams& p, int b) {
    st_release_s32(p.final_flag + b, 1);
    atomicAdd(&p.state->requests_done, 1);
}

// Warp-cooperative log2-sum-exp of up to kRows partial rows of request b at
// once: lane l holds partial l of each row (C x W <= 32 partials per row), so
// every row costs one round trip and the rows' loads are in flight together.
// Returns row r's value in every lane through out[r]; *lost (warp-uniform)
// when a partial is NaN (its statistics were lost to a timeout).
template <int kW, int kRows>
__device__ inline void warp_rows_lse(const FusedParams& p, int b, const int (&slots)[kRows], int nrows,
                                     float (&out)[kRows], bool* lost) {
    const int lane = threadIdx.x & 31;
    const int cw = p.C * kW;
    float2 v[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        v[r] = make_float2(-INFINITY, 0.f);
        if (r < nrows && lane < cw)
            v[r] = __ldcg(p.partials + ((int64_t(b) * (2 * p.k_max + 1) + slots[r]) * p.C) * kW + lane);
    }
    bool bad = false;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        bad |= isnan(v[r].x) || isnan(v[r].y);
        float m = v[r].x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = m == -INFINITY ? 0.f : v[r].y * ex2_approx(v[r].x - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        out[r] = m + log2f(sum);
    }
    if (__any_sync(0xffffffffu, bad)) *lost = true;
}

template <int kW>
__device__ inline float warp_row_lse(const FusedParams& p, int b, int slot, bool* lost) {
    const int slots[1] = {slot};
    float out[1];
    warp_rows_lse<kW, 1>(p, b, slots, 1, out, lost);
    return out[0];
}

// ---------------------------------------------------------------------------
// Scan of request b, run by one warp.
template <typename T, int kW>
__device__ void fused_scan(const FusedParams& p, int b) {
    const int lane = threadIdx.x & 31;
    const int K = p.k_max;
    const int64_t es = Logit<T>::kSize;
    const bool has_draft = p.draft != nullptr;
    const int32_t* x = p.tokens + int64_t(b) * K;
    int32_t* out_tok = p.out_tokens + int64_t(b) * (K + 1);
    const float* u = p.uniforms + int64_t(b) * (K + 1);
    const int L = p.lens ? __ldg(p.lens + b) : K;
    bool invalid = L < 0 || L > K;
    bool lost = false;
    int first = invalid ? 0 : L;
    if (!invalid) {
        // positions in blocks of 32: lane l takes position i0 + l
        for (int i0 = 0; i0 <= L; i0 += 32) {
            const int i = i0 + lane;
            const bool mine = i < L;   // a drafted position of this lane
            int xi = 0;
            float z = 0.f, y = 0.f;
            if (mine) {
                xi = __ldg(x + i);
                if (xi < 0 || xi >= p.V) {
                    invalid = true;
                } else {
                    z = Logit<T>::load(p.target + (int64_t(b) * (K + 1) + i) * p.row_stride * es, xi);
                    if (has_draft) y = Logit<T>::load(p.draft + (int64_t(b) * K + i) * p.row_stride * es, xi);
                }
            }
            // the statistics of this block's target rows (and draft rows): 8 rows
            // per pass, 4 lanes per row, each lane merging up to 8 of the row's
            // C x W partials with all its loads in flight
            const int nt = min(32, L + 1 - i0);           // target rows i0 .. i0+nt-1 (row L included)
            const int nd = has_draft ? max(0, min(32, L - i0)) : 0;
            const int cw = p.C * kW;
            const int sub = lane & 3, rp = lane >> 2;
            float lse_t = 0.f, lse_d = 0.f;
            for (int q0 = 0; q0 < nt + nd; q0 += 8) {
                const int q = q0 + rp;                     // this lane group's row of the pass
                const int slot = q < nt ? i0 + q : K + 1 + i0 + (q - nt);
                float2 v[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const int e = sub + 4 * t;
                    v[t] = (q < nt + nd && e < cw)
                               ? __ldcg(p.partials + ((int64_t(b) * (2 * K + 1) + slot) * p.C) * kW + e)
                               : make_float2(-INFINITY, 0.f);
                }
                float m = -INFINITY;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (isnan(v[t].x) || isnan(v[t].y)) lost = true;
                    m = fmaxf(m, v[t].x);
                }
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
                float sum = 0.f;
                if (m != -INFINITY) {
#pragma unroll
                    for (int t = 0; t < 8; ++t) sum += v[t].y * ex2_approx(v[t].x - m);
                }
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                const float lse_row = m + log2f(sum);      // in the 4 lanes of row q
                // hand each position's rows to its lane
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float val = __shfl_sync(0xffffffffu, lse_row, 4 * r);
                    const int qq = q0 + r;
                    if (qq < nt && qq == lane) lse_t = val;
                    if (qq >= nt && qq < nt + nd && qq - nt == lane) lse_d = val;
                }
            }
            if (mine && xi >= 0 && xi < p.V) {
                const float pi = exp2f(z * p.scale - lse_t);
                const float qi = has_draft ? exp2f(y * p.scale - lse_d) : 1.f;
                if (!(__ldg(u + i) < accept_prob(pi, qi)) && i < first) first = i;
            }
        }
    }
    invalid = __any_sync(0xffffffffu, invalid);
    lost = __any_sync(0xffffffffu, lost);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    if (invalid || lost) {
        for (int i = lane; i <= K; i += 32) out_tok[i] = -1;
        if (lane == 0) {
            p.out_len[b] = invalid ? -1 : -2;
            fused_request_done(p, b);
        }
        return;
    }
    const int j = first;
    for (int i = lane; i <= K; i += 32) {
        if (i < j) out_tok[i] = __ldg(x + i);
        else if (i > j) out_tok[i] = -1;
    }
    // row j: statistics, draw mode and the chunk weights of a bonus / one-hot draw
    bool dummy = false;
    FusedReq r;
    r.j = j;
    r.mode = j == L ? kBonus : (has_draft ? kResidual : kOneHot);
    {
        const int slots[2] = {j, K + 1 + j};
        float out[2];
        warp_rows_lse<kW, 2>(p, b, slots, r.mode == kResidual ? 2 : 1, out, &dummy);
        r.lse_p = out[0];
        r.lse_q = r.mode == kResidual ? out[1] : 0.f;
    }
    r.ustar = __ldg(u + K);
    r.zero_at = r.mode == kOneHot ? __ldg(x + j) : -1;
    r.kstar = 0;
    r.local_target = 0.f;
    r.ntasks = 0;
    if (r.mode != kResidual) {
        // lane c: chunk c's share of p_j, merged over its W partials
        const float2* part = p.partials + ((int64_t(b) * (2 * K + 1) + j) * p.C) * kW;
        float Wc = 0.f;
        if (lane < p.C)
            for (int w = 0; w < kW; ++w) {
                const float2 v = __ldcg(part + lane * kW + w);
                Wc += v.y * exp2f(v.x - r.lse_p);
            }
        if (r.mode == kOneHot) {
            const unsigned char* trow = p.target + (int64_t(b) * (K + 1) + j) * p.row_stride * es;
            const float pj = exp2f(Logit<T>::load(trow, r.zero_at) * p.scale - r.lse_p);
            if (lane == r.zero_at / p.CE) Wc = fmaxf(0.f, Wc - pj);
        }
        float total = Wc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        if (!(total > 0.f)) {  // p_j has no mass left outside x_j: draw from p_j
            r.mode = kBonus;
            r.zero_at = -1;
            Wc = 0.f;
            if (lane < p.C)
                for (int w = 0; w < kW; ++w) {
                    const float2 v = __ldcg(part + lane * kW + w);
                    Wc += v.y * exp2f(v.x - r.lse_p);
                }
            total = Wc;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        }
        const float target = r.ustar * total;
        const float wi = warp_scan_incl(Wc);
        const unsigned cross = __ballot_sync(0xffffffffu, Wc > 0.f && wi > target);
        const unsigned pos = __ballot_sync(0xffffffffu, Wc > 0.f);
        const int cstar = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : 0);
        const float before = __shfl_sync(0xffffffffu, wi - Wc, cstar);
        r.kstar = cstar;
        r.local_target = cross ? fmaxf(0.f, target - before) : INFINITY;
        r.ntasks = 0;
    }
    if (lane == 0) {
        p.out_len[b] = j;
        constexpr int PV = Logit<T>::kPerVec;
        if (r.mode == kResidual) {
            for (int c = 0; c < p.C; ++c) r.ntasks += fused_pieces(p, c, PV);
        } else {
            r.ntasks = fused_pieces(p, r.kstar, PV);
        }
        p.req[b] = r;   // published by the release stores of the posts
        if (r.mode == kResidual) fused_post<T>(p, b, 0, p.C);
        else fused_post<T>(p, b, r.kstar, 1);
    }
}

// ---------------------------------------------------------------------------
// Final selection of request b, run by one warp; s_seg is this warp's own
// nseg_max floats of shared memory.
template <typename T, int kW>
__device__ void fused_select(const FusedParams& p, int b, float* s_seg) {
    const int lane = threadIdx.x & 31;
    const int K = p.k_max;
    const int64_t es = Logit<T>::kSize;
    constexpr int PV = Logit<T>::kPerVec;
    FusedReq r;
    {
        const int32_t* src = reinterpret_cast<const int32_t*>(p.req + b);
        int32_t* dst = reinterpret_cast<int32_t*>(&r);
#pragma unroll
        for (int i = 0; i < int(sizeof(FusedReq) / 4); ++i) dst[i] = __ldcg(src + i);
    }
    const bool resid = r.mode == kResidual;
    WeightRow wr;
    wr.trow = p.target + (int64_t(b) * (K + 1) + r.j) * p.row_stride * es;
    wr.drow = resid ? p.draft + (int64_t(b) * K + r.j) * p.row_stride * es : nullptr;
    wr.scale = p.scale;
    wr.lse_p = r.lse_p;
    wr.lse_q = r.lse_q;
    wr.zero_at = r.zero_at;
    const float* segs_b = p.segs + int64_t(b) * p.C * p.nseg_max;
    auto nseg_of = [&](int c) {
        const int n = min(p.V - c * p.CE, p.CE);
        return ((n + PV - 1) / PV + kSegVecs - 1) / kSegVecs;
    };
    int kstar = r.kstar;
    float target = r.local_target;
    bool fallback = false;
    if (resid) {
        // chunk c's residual weight (lane c): its pieces' per-warp totals, in
        // piece then warp order
        float W = 0.f;
        if (lane < p.C) {
            const int n = fused_pieces(p, lane, PV) * kW;
            const float* pt = p.piece_tot + (int64_t(b) * p.C + lane) * p.P * kW;
#pragma unroll 8
            for (int i = 0; i < n; ++i) W += __ldcg(pt + i);
        }
        float total = W;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        const float t = r.ustar * total;
        const float wi = warp_scan_incl(W);
        const unsigned cross = __ballot_sync(0xffffffffu, W > 0.f && wi > t);
        const unsigned pos = __ballot_sync(0xffffffffu, W > 0.f);
        if (!pos) {
            fallback = true;   // no residual mass (p == q numerically): draw from p_j
        } else {
            kstar = cross ? __ffs(cross) - 1 : 31 - __clz(pos);
            const float before = __shfl_sync(0xffffffffu, wi - W, kstar);
            target = cross ? fmaxf(0.f, t - before) : INFINITY;
        }
    }
    int token;
    if (fallback) {
        // inverse CDF of p_j over the whole row, 32 elements at a time
        float W = 0.f;
        for (int e = lane; e < p.V; e += 32) W += draw_weight<false>(wr, Logit<T>::load(wr.trow, e), 0.f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        const float t = r.ustar * W;
        float acc = 0.f;
        token = -1;
        int last = -1;
        for (int e0 = 0; e0 < p.V && token < 0; e0 += 32) {
            const int e = e0 + lane;
            const float w = e < p.V ? draw_weight<false>(wr, Logit<T>::load(wr.trow, e), 0.f) : 0.f;
            const float incl = acc + warp_scan_incl(w);
            const unsigned cr = __ballot_sync(0xffffffffu, w > 0.f && incl > t);
            const unsigned ps = __ballot_sync(0xffffffffu, w > 0.f);
            if (ps) last = e0 + 31 - __clz(ps);
            if (cr) token = e0 + __ffs(cr) - 1;
            acc = __shfl_sync(0xffffffffu, incl, 31);
        }
        if (token < 0) token = last >= 0 ? last : 0;
    } else {
        const int n = min(p.V - kstar * p.CE, p.CE);
        const int ns = nseg_of(kstar);
#pragma unroll 8
        for (int s = lane; s < ns; s += 32) s_seg[s] = __ldcg(segs_b + kstar * p.nseg_max + s);
        __syncwarp();
        token = draw_select<T>(wr, resid, kstar * p.CE, n, s_seg, target);
        if (token < 0) token = kstar * p.CE;
    }
    if (lane == 0) {
        p.out_tokens[int64_t(b) * (K + 1) + r.j] = token;
        fused_request_done(p, b);
    }
}

// ---------------------------------------------------------------------------

template <typename T, int kConsumerWarps, int kStages>
__global__ void __launch_bounds__((kConsumerWarps + 1) * 32, TmaCtasPerSm<T>::value)
verify_fused_kernel(const FusedParams p) {
    constexpr int kW = kConsumerWarps;
    constexpr int kConsumers = kConsumerWarps * 32;
    constexpr int kThreads = kConsumers + 32;
    constexpr int kVecPerThread = (kStageBytes / 16 + kConsumers - 1) / kConsumers;
    constexpr int kDrawVecPerThread = kPieceVecsF / kConsumers;
    static_assert(kPieceVecsF % kConsumers == 0, "draw pieces split evenly over the consumers");
    static_assert(2 * kPieceBytes <= kStageBytes, "a draw stage holds a piece of two rows");
    using Lay = FusedSmem<kConsumerWarps, kStages>;
    constexpr int PV = Logit<T>::kPerVec;
    constexpr int ES = Logit<T>::kSize;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* stage_buf = smem;
    FusedMeta* meta = reinterpret_cast<FusedMeta*>(smem + Lay::kMetaOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* empty = full + kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff);
    int* scan_scratch = reinterpret_cast<int*>(smem + Lay::kMiscOff) + 8;   // 32 ints (row prefix scan)
    int* row_start = reinterpret_cast<int*>(smem + Lay::kRowOff);
    float* s_seg_all = reinterpret_cast<float*>(smem + Lay::seg_off(p.B));

    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    StatsParams sp{};
    sp.target = p.target;
    sp.draft = p.draft;
    sp.lens = p.lens;
    sp.b0 = 0;
    sp.nB = p.B;
    sp.k_max = p.k_max;
    sp.V = p.V;
    sp.row_stride = p.row_stride;
    sp.C = p.C;
    sp.CE = p.CE;
    sp.use_draft = p.draft != nullptr ? 1 : 0;
    build_row_prefix<kThreads>(sp, row_start, scan_scratch);  // ends with __syncthreads
    const int64_t total_items = (int64_t)row_start[p.B] * p.C;

    if (tid >= kConsumers) {
        // ----------------------------- producer warp -----------------------------
        const int lane = tid - kConsumers;
        int slot = 0;
        uint32_t phase = 0;
        bool wrapped = false;
        uint32_t last_phase[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_phase[s] = 0xffffffffu;
        // one stage: wait for the slot, fill meta, arm the barrier and copy
        auto put = [&](const FusedMeta& m, const unsigned char* src0, const unsigned char* src1, int bytes) {
            bool ok = true;
            if (wrapped) ok = mbar_wait_bounded(empty + slot, phase ^ 1u, p.timeout_ns);
            if (!ok || *abort_flag) {
                *abort_flag = 1;
                return false;
            }
            meta[slot] = m;
            last_phase[slot] = phase;
            if (bytes > 0 && src0) {
                mbar_arrive_expect_tx(full + slot, static_cast<uint32_t>(bytes * (src1 ? 2 : 1)));
                bulk_copy_g2s(stage_buf + size_t(slot) * kStageBytes, src0, static_cast<uint32_t>(bytes), full + slot);
                if (src1)
                    bulk_copy_g2s(stage_buf + size_t(slot) * kStageBytes + kPieceBytes, src1,
                                  static_cast<uint32_t>(bytes), full + slot);
            } else {
                mbar_arrive(full + slot);
            }
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1u;
                wrapped = true;
            }
            return true;
        };
        if (lane == 0) {
            bool stop = false;
            int64_t next = atomicAdd(&p.state->stats_next, 1);
            uint64_t idle_since = 0;
            uint32_t backoff = 32;
            // this CTA's mailbox: the next slot to serve, and its flag loaded
            // (relaxed) while the previous stats item was being issued, so
            // looking for a draw task costs no round trip
            int32_t* my_ready = p.mbox_ready + int64_t(blockIdx.x) * p.mbox_slots;
            const int32_t* my_task = p.mbox_task + int64_t(blockIdx.x) * p.mbox_slots;
            int mslot = 0;
            int pf_ready = 0;   // my_ready[mslot] as loaded (relaxed) some time ago
            auto prefetch = [&]() { pf_ready = mslot < p.mbox_slots ? ld_relaxed_s32(my_ready + mslot) : 0; };
            // issue one posted draw piece if the prefetched flag shows one
            auto serve = [&]() {
                if (pf_ready == 0 || mslot >= p.mbox_slots) return false;
                fence_acquire_gpu();   // the relaxed flag load above becomes an acquire
                const int task = __ldcg(my_task + mslot);
                ++mslot;
                const int piece = task % p.P, bc = task / p.P;
                const int b = bc / p.C, c = bc - b * p.C;
                const int j = __ldcg(&p.req[b].j);
                const bool resid = __ldcg(&p.req[b].mode) == kResidual;
                const float lse_p = __ldcg(&p.req[b].lse_p), lse_q = __ldcg(&p.req[b].lse_q);
                const int zero_at = __ldcg(&p.req[b].zero_at), ntasks = __ldcg(&p.req[b].ntasks);
                const unsigned char* trow = p.target + (int64_t(b) * (p.k_max + 1) + j) * p.row_stride * ES;
                const unsigned char* drow = resid ? p.draft + (int64_t(b) * p.k_max + j) * p.row_stride * ES : nullptr;
                const int e0 = c * p.CE;
                const int n = min(p.V - e0, p.CE);
                const int tma_bytes = (n * ES) & ~15;   // whole vectors; a partial last one is read element-wise
                const int off = piece * kPieceBytes;
                const int bytes = max(0, min(kPieceBytes, tma_bytes - off));
                FusedMeta m{};
                m.elem0 = piece * kPieceVecsF;
                m.n_bytes = bytes;
                m.flags = kDraw | (resid ? kResid : 0) | kFirst | kLast;
                m.b = b;
                m.c = c;
                m.lse_p = lse_p;
                m.lse_q = lse_q;
                m.j = j;
                m.zero_at = zero_at;
                m.ntasks = ntasks;
                const int64_t src_off = int64_t(e0) * ES + off;
                if (!put(m, bytes > 0 ? trow + src_off : nullptr, (bytes > 0 && resid) ? drow + src_off : nullptr,
                         bytes))
                    stop = true;
                prefetch();
                return true;
            };
            prefetch();
            while (!stop) {
                // 1. a draw piece posted to this CTA
                if (serve()) {
                    idle_since = 0;
                    backoff = 32;
                    continue;
                }
                // 2. the next stats item (posted pieces are served between its stages)
                if (next < total_items) {
                    idle_since = 0;
                    const int64_t item = next;
                    next = atomicAdd(&p.state->stats_next, 1);
                    const ItemDesc d = decode_item<T>(sp, row_start, item);
                    const int64_t bytes_all = int64_t(d.e1 - d.e0) * ES;
                    const int64_t tma_bytes = bytes_all & ~int64_t(15);
                    const int tail_n = static_cast<int>((bytes_all - tma_bytes) / ES);
                    const int nsub = tma_bytes == 0 ? 1 : static_cast<int>((tma_bytes + kStageBytes - 1) / kStageBytes);
                    const unsigned char* src0 = d.row + int64_t(d.e0) * ES;
                    const int b = static_cast<int>(d.partial_idx / (int64_t(2 * p.k_max + 1) * p.C));
                    for (int sub = 0; sub < nsub && !stop; ++sub) {
                        const int64_t off = int64_t(sub) * kStageBytes;
                        const int64_t left = tma_bytes - off;
                        const int n = static_cast<int>(left < kStageBytes ? left : int64_t(kStageBytes));
                        FusedMeta m{};
                        m.tail = tail_n ? src0 + tma_bytes : nullptr;
                        m.partial_idx = d.partial_idx;
                        m.elem0 = d.e0 + static_cast<int>(off / ES);
                        m.n_bytes = n > 0 ? n : 0;
                        m.tail_n = tail_n;
                        m.flags = (sub == 0 ? kFirst : 0) | (sub == nsub - 1 ? kLast : 0);
                        m.b = b;
                        if (!put(m, n > 0 ? src0 + off : nullptr, nullptr, n > 0 ? n : 0)) stop = true;
                        prefetch();
                        while (!stop && serve()) {}
                    }
                    continue;
                }
                // 3. nothing to do now: done when every request is final;
                // otherwise poll (bounded) for tasks that running CTAs enqueue
                if (ld_relaxed_s32(&p.state->requests_done) >= p.B) break;
                const uint64_t now = global_timer_ns();
                if (idle_since == 0) idle_since = now;
                else if (now - idle_since > p.timeout_ns) break;
                nap(backoff);
                backoff = backoff < 1024 ? backoff * 2 : 1024;
                prefetch();
            }
            // tell the consumers there is no more work
            FusedMeta m{};
            m.flags = kDone;
            (void)put(m, nullptr, nullptr, 0);
        }
        __syncwarp();
        named_barrier_sync(2, kThreads);
        if (lane == 0 && *abort_flag) {
            for (int s = 0; s < kStages; ++s)
                if (last_phase[s] != 0xffffffffu) (void)mbar_wait_bounded(full + s, last_phase[s], p.timeout_ns);
        }
        if (lane == 0) {
            // the last CTA out marks requests that never finished (a timeout)
            if (atom_add_acq_rel(&p.state->ctas_exited, 1) == int(gridDim.x) - 1 &&
                ld_acquire_s32(&p.state->requests_done) < p.B) {
                for (int b = 0; b < p.B; ++b)
                    if (ld_acquire_s32(p.final_flag + b) == 0) {
                        for (int i = 0; i <= p.k_max; ++i) p.out_tokens[int64_t(b) * (p.k_max + 1) + i] = -1;
                        p.out_len[b] = -2;
                    }
            }
        }
        return;
    }

    // ------------------------------- consumer warps -------------------------------
    // Warps never wait for one another: each stores its own partials and
    // segment sums and counts its own completions.
    const int lane = tid & 31, warp = tid >> 5;
    float* s_seg = s_seg_all + warp * p.nseg_max;
    Acc<false> acc;
    acc.reset();
    int slot = 0;
    uint32_t phase = 0;
    WeightRow wr{};
    float task_sum = 0.f;   // this warp's share of the current draw task (lane 0)
    for (;;) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(full + slot, phase, p.timeout_ns));
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) atomicExch(&p.state->error, 1);
            break;
        }
        const FusedMeta m = meta[slot];
        const unsigned char* buf = stage_buf + size_t(slot) * kStageBytes;
        if (m.flags & kDone) break;
        if (!(m.flags & kDraw)) {
            // ---------------- stats stage (as K1) ----------------
            if (m.flags & kFirst) acc.reset();
            const int nvec = m.n_bytes >> 4;
            uint4 vv[kVecPerThread];
            if (nvec == kVecPerThread * kConsumers) {
#pragma unroll
                for (int k = 0; k < kVecPerThread; ++k) vv[k] = ld_shared_v4(buf + 16 * (tid + k * kConsumers));
                fold_vectors<T, kVecPerThread>(acc, vv, p.scale);
            } else {
#pragma unroll
                for (int k = 0; k < kVecPerThread; ++k) {
                    const int v = tid + k * kConsumers;
                    vv[k] = v < nvec ? ld_shared_v4(buf + 16 * v) : make_uint4(0, 0, 0, 0);
                }
                const int nv = nvec > tid ? (nvec - tid + kConsumers - 1) / kConsumers : 0;
                fold_vectors_count<T, kVecPerThread>(acc, vv, nv, p.scale);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);
            if (++slot == kStages) { slot = 0; phase ^= 1u; }
            if (m.flags & kLast) {
                if (m.tail && tid < m.tail_n) acc.fold1(Logit<T>::load(m.tail, tid) * p.scale);
                const MS v = warp_merge_ms_maxfirst(acc.ms);
                int scan_now = 0;
                if (lane == 0) {
                    p.partials[m.partial_idx * kW + warp] = make_float2(v.m, v.s);
                    const int items = (row_start[m.b + 1] - row_start[m.b]) * p.C * kW;
                    scan_now = atom_add_acq_rel(p.done_items + m.b, 1) == items - 1;
                }
                if (__shfl_sync(0xffffffffu, scan_now, 0)) {
                    fence_acquire_gpu();   // every lane reads the other warps' partials
                    fused_scan<T, kW>(p, m.b);
                }
            }
        } else {
            // ---------------- draw stage ----------------
            const bool resid = (m.flags & kResid) != 0;
            if (m.flags & kFirst) {
                task_sum = 0.f;
                wr.trow = p.target + (int64_t(m.b) * (p.k_max + 1) + m.j) * p.row_stride * ES;
                wr.drow = resid ? p.draft + (int64_t(m.b) * p.k_max + m.j) * p.row_stride * ES : nullptr;
                wr.scale = p.scale;
                wr.lse_p = m.lse_p;
                wr.lse_q = m.lse_q;
                wr.zero_at = m.zero_at;
            }
            const int e0 = m.c * p.CE;
            const int n = min(p.V - e0, p.CE);
            const int nfull = n / PV, nvec = (n + PV - 1) / PV;
            float segsum[kDrawVecPerThread];
#pragma unroll
            for (int i = 0; i < kDrawVecPerThread; ++i) {
                const int lv = tid + i * kConsumers;     // vector within the piece
                const int v = m.elem0 + lv;              // vector within the chunk
                float w[PV];
                float sum = 0.f;
                if (v < nfull) {
                    const uint4 tz = ld_shared_v4(buf + 16 * lv);
                    if (resid) {
                        const uint4 ty = ld_shared_v4(buf + kPieceBytes + 16 * lv);
                        sum = vector_weights<T, true>(wr, tz, ty, e0 + v * PV, w);
                    } else {
                        sum = vector_weights<T, false>(wr, tz, tz, e0 + v * PV, w);
                    }
                } else if (v < nvec) {
                    sum = resid ? tail_weights<T, true>(wr, e0 + v * PV, n - v * PV, w)
                                : tail_weights<T, false>(wr, e0 + v * PV, n - v * PV, w);
                }
                segsum[i] = sum;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);
            if (++slot == kStages) { slot = 0; phase ^= 1u; }
            float* segs_bc = p.segs + (int64_t(m.b) * p.C + m.c) * p.nseg_max;
#pragma unroll
            for (int i = 0; i < kDrawVecPerThread; ++i) {
                float s = segsum[i];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                const int v0 = m.elem0 + i * kConsumers + warp * 32;   // first vector of this warp's segment
                if (lane == 0 && v0 < nvec) segs_bc[v0 / kSegVecs] = s;
                task_sum += s;
            }
            if (m.flags & kLast) {
                int select_now = 0;
                if (lane == 0) {
                    p.piece_tot[((int64_t(m.b) * p.C + m.c) * p.P + m.elem0 / kPieceVecsF) * kW + warp] = task_sum;
                    select_now = atom_add_acq_rel(p.draw_done + m.b, 1) == m.ntasks * kW - 1;
                }
                if (__shfl_sync(0xffffffffu, select_now, 0)) {
                    fence_acquire_gpu();
                    fused_select<T, kW>(p, m.b, s_seg);
                }
            }
        }
    }
    named_barrier_sync(2, kThreads);
}

}  // namespace sv
