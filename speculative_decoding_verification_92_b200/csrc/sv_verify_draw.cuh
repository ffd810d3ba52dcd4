// sv_verify_draw.cuh -- K2b, the final draw (residual / bonus / one-hot),
// and K2c, the selection of residual draws.
//
// The scan kernel queued one draw per sampling request: a residual draw
// (rejection with draft logits) as P tasks, one per piece of the row pair,
// and a bonus or one-hot draw as one task.  K2b is a persistent grid of
// resident CTAs; CTA x takes tasks x, x + G, x + 2G, ...; the single-piece
// draws, whose chain is longest, take the last CTAs of the first round, and
// the residual pieces fill the other tasks in queue order, so one draw's
// pieces run on P different CTAs at once (TaskMap).  Each task stages its piece(s) in shared memory with 1-D bulk copies
// (double-buffered: the next task's copies, and the queue entry of the one
// after, are in flight while the current task is computed) and computes the
// draw weights
//     residual: w_v = max(0, p_j(v) - q_j(v))     ("AI 开始抄自己的作业——而且抄得理直气壮",
//               section "⚡ 投机解码：让草稿先跑，考官殿后": the redraw comes from the
//               target with the draft's share taken out);
//     bonus:    w_v = p_L(v)                      (same page, section
//               "🚰 真正的瓶颈不在算法，在流水线": all drafts accepted -> the next
//               position's token);
//     one-hot:  w_v = p_j(v), 0 at the drafted id (max(0, p - 1) there),
// with p_j(v) = 2^(z_v * log2(e)/T - lse_j), and one weight sum per segment of
// 32 16-byte vectors.
//
// The token is the smallest v whose running weight sum exceeds u*W (u* =
// uniforms[b][k_max], W the total); it is found piece -> segment -> vector ->
// element:
//   * residual: each K2b task stores its piece's 32 segment sums; K2c (one
//     warp per residual draw, after K2b) picks the piece and the segment from
//     the stored sums, re-reads that one segment of both rows (one vector per
//     lane) and picks the vector and element.  Nothing waits on another CTA.
//   * bonus: the piece was chosen by the scan kernel from the row-statistics
//     partials; the task picks segment, vector and element in shared memory.
//   * one-hot: the task computes the exact weight of the piece holding the
//     drafted id (the partials cannot give it without cancellation), takes
//     the other pieces' weights from the partials, picks the piece, and
//     selects in it (loading it first unless it is the drafted id's piece).
// Rounding that leaves u*W past every step at some level takes the last
// block with positive weight there, so a zero-weight token is never drawn.
// A zero residual mass (p == q numerically) draws from p_j instead.
//
// Waits: only on a CTA's own bulk copies, bounded by timeout_ns; after a
// timeout the CTA reports its remaining draws with out_accept_len = -2.
#pragma once

#include "sv_common.cuh"
#include "sv_verify_scan.cuh"

#ifndef SV_DRAW_CTAS_PER_SM
#define SV_DRAW_CTAS_PER_SM 3
#endif

namespace sv {

struct DrawParams {
    int32_t B;
    const unsigned char* target;
    const unsigned char* draft;
    const float2* partials;      // [B][2k+1][P] row-statistics partials
    const int32_t* ctrl;         // [0] residual draws, [1] single-piece draws
    const DrawReq* res_req;
    const DrawReq* one_req;
    int32_t* res_lost;           // [B] per residual draw: set when one of its pieces was lost to a timeout
    float* seg;                  // [B][P][32] segment sums of residual draws (by queue slot)
    int32_t* out_len;
    int32_t* out_tokens;
    int32_t k_max;
    int32_t V;
    int64_t row_stride;
    int32_t P;
    int32_t PE;
    float scale;
    int32_t rows_aligned;        // every row starts on a 16-byte boundary: pieces are staged by bulk copies
    uint64_t timeout_ns;         // bound on each wait for a staged piece
    int32_t lost_draw_b;         // test fault injection: the first staging for this request's draw is
                                 // never issued (its wait runs out); -1 = off
};

constexpr int kDrawThreads = 256;
constexpr int kDrawWarps = kDrawThreads / 32;
constexpr int kDrawCtasPerSm = SV_DRAW_CTAS_PER_SM;
constexpr int kSegVecs = 32;                                  // vectors per segment: one warp-wide load
constexpr int kPieceVecs = kPieceBytes / 16;                  // 1024
constexpr int kSegsPerPiece = kPieceVecs / kSegVecs;          // 32
constexpr int kVecsPerThread = kPieceVecs / kDrawThreads;     // 4
static_assert(kSegsPerPiece == 32, "one segment sum per lane");
static_assert(kPieceVecs % kDrawThreads == 0, "a piece must split evenly over the threads");
// Dynamic shared memory: two buffers, each a target piece and a draft piece.
constexpr size_t kDrawBufBytes = 2 * size_t(kPieceBytes);
constexpr size_t kDrawSmemBytes = 2 * kDrawBufBytes;

// Everything a weight computation needs about row j.
struct WeightRow {
    const unsigned char* trow;   // target row j
    const unsigned char* drow;   // draft row j (residual only)
    float scale, lse_p, lse_q;   // log2 domain
    int zero_at;                 // row index whose weight is 0 (one-hot), or -1
    int mode;
};

// Up to PV logits of one row starting at element idx0 (count < PV: the rest
// are -inf), from shared memory when `sm` is given, else from global memory
// (16-byte load when `vec_ok` and the vector is whole).
// kGeneric: `sm` is a generic address (another CTA's shared memory in the
// cluster) rather than this CTA's.
template <typename T, bool kGeneric = false>
__device__ __forceinline__ void load_vec(const unsigned char* sm, const unsigned char* row, int idx0, int count,
                                         bool vec_ok, float (&z)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    if (sm) {
        if constexpr (kGeneric) Logit<T>::unpack(*reinterpret_cast<const uint4*>(sm), z);
        else Logit<T>::unpack(ld_shared_v4(sm), z);
    } else if (vec_ok && count == PV) {
        Logit<T>::unpack(ld_global_stream_v4(row + int64_t(idx0) * Logit<T>::kSize), z);
    } else {
#pragma unroll
        for (int i = 0; i < PV; ++i) z[i] = i < count ? Logit<T>::load(row, idx0 + i) : -INFINITY;
    }
}

// Draw weights of the (up to PV) elements of one vector starting at row
// index idx0; returns their sum, added in element order.
template <typename T>
__device__ __forceinline__ float vec_weights(const WeightRow& r, const float (&z)[Logit<T>::kPerVec],
                                             const float (&y)[Logit<T>::kPerVec], int idx0, int count,
                                             float (&w)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
        float wi = 0.f;
        if (i < count) {
            wi = ex2_approx(fmaf(z[i], r.scale, -r.lse_p));
            if (r.mode == kResidual) wi = fmaxf(0.f, wi - ex2_approx(fmaf(y[i], r.scale, -r.lse_q)));
            if (idx0 + i == r.zero_at) wi = 0.f;  // max(0, p - 1) = 0 at the drafted id
        }
        w[i] = wi;
        sum += wi;
    }
    return sum;
}

// Weights of vector v of piece pc (elements [e0, e0 + n) of the row), from
// the staged copy when it holds the vector, else from global memory.
template <typename T, bool kGeneric = false>
__device__ __forceinline__ float piece_vec_weights(const WeightRow& r, const unsigned char* tbuf,
                                                   const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0,
                                                   int n, int v, float (&w)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    const int idx0 = e0 + v * PV;
    const int count = min(PV, n - v * PV);
    float z[PV], y[PV];
    const bool staged = v < nstaged_vec;
    load_vec<T, kGeneric>(staged ? tbuf + 16 * v : nullptr, r.trow, idx0, count, vec_ok, z);
    if (r.mode == kResidual) load_vec<T, kGeneric>(staged ? dbuf + 16 * v : nullptr, r.drow, idx0, count, vec_ok, y);
#pragma unroll
    for (int i = 0; i < PV; ++i)
        if (r.mode != kResidual) y[i] = 0.f;
    return vec_weights<T>(r, z, y, idx0, count, w);
}

// Sum of the draw weights of one whole staged vector (PV elements from row
// index idx0), for a draw of mode kMode; every element weight is computed
// exactly as vec_weights computes it (the selection recomputes them there).
// A one-hot vector holding the drafted id goes through vec_weights, so the
// drafted id's weight is left out rather than subtracted.
template <typename T, int kMode>
__device__ __forceinline__ float vec_sum_staged(const WeightRow& r, const unsigned char* tp, const unsigned char* dp,
                                                int idx0) {
    constexpr int PV = Logit<T>::kPerVec;
    float z[PV], y[PV];
    Logit<T>::unpack(ld_shared_v4(tp), z);
    if constexpr (kMode == kResidual) Logit<T>::unpack(ld_shared_v4(dp), y);
    if constexpr (kMode == kOneHot) {
        if (static_cast<unsigned>(r.zero_at - idx0) < static_cast<unsigned>(PV)) {
            float w[PV];
#pragma unroll
            for (int i = 0; i < PV; ++i) y[i] = 0.f;
            return vec_weights<T>(r, z, y, idx0, PV, w);
        }
    }
    const float nlp = -r.lse_p, nlq = -r.lse_q;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int i = 0; i < PV; i += 2) {
        float w0 = ex2_approx(fmaf(z[i], r.scale, nlp));
        float w1 = ex2_approx(fmaf(z[i + 1], r.scale, nlp));
        if constexpr (kMode == kResidual) {
            w0 = fmaxf(0.f, w0 - ex2_approx(fmaf(y[i], r.scale, nlq)));
            w1 = fmaxf(0.f, w1 - ex2_approx(fmaf(y[i + 1], r.scale, nlq)));
        }
        s0 += w0;
        s1 += w1;
    }
    return s0 + s1;
}

// All threads: the 32 segment sums of one piece into s_seg (ends with
// __syncthreads).  Thread t handles vectors t + 256 k, so warp w at step k
// covers segment w + 8 k.  Whole staged vectors take the fast path; the
// ragged end of a row and unstaged (unaligned) rows take the general one.
template <typename T, int kMode>
__device__ __forceinline__ void piece_segments_mode(const WeightRow& r, const unsigned char* tbuf,
                                                    const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0,
                                                    int n, float* s_seg) {
    constexpr int PV = Logit<T>::kPerVec;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = (n + PV - 1) / PV;
    float sum[kVecsPerThread];
    if (nstaged_vec == kPieceVecs) {
        // a whole staged piece: every vector on the fast path, all in flight
#pragma unroll
        for (int k = 0; k < kVecsPerThread; ++k) {
            const int v = threadIdx.x + k * kDrawThreads;
            sum[k] = vec_sum_staged<T, kMode>(r, tbuf + 16 * v, kMode == kResidual ? dbuf + 16 * v : nullptr,
                                              e0 + v * PV);
        }
    } else {
#pragma unroll
        for (int k = 0; k < kVecsPerThread; ++k) {
            const int v = threadIdx.x + k * kDrawThreads;
            sum[k] = 0.f;
            if (v < nstaged_vec) {
                sum[k] = vec_sum_staged<T, kMode>(r, tbuf + 16 * v, kMode == kResidual ? dbuf + 16 * v : nullptr,
                                                  e0 + v * PV);
            } else if (v < nvec) {
                float w[PV];
                sum[k] = piece_vec_weights<T>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, v, w);
            }
        }
    }
    // four independent warp sums, interleaved
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < kVecsPerThread; ++k) sum[k] += __shfl_xor_sync(0xffffffffu, sum[k], o);
    if (lane == 0) {
#pragma unroll
        for (int k = 0; k < kVecsPerThread; ++k) s_seg[warp + kDrawWarps * k] = sum[k];
    }
    __syncthreads();
}

template <typename T>
__device__ __forceinline__ void piece_segments(const WeightRow& r, const unsigned char* tbuf,
                                               const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0,
                                               int n, float* s_seg) {
    if (r.mode == kResidual) piece_segments_mode<T, kResidual>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, s_seg);
    else if (r.mode == kOneHot) piece_segments_mode<T, kOneHot>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, s_seg);
    else piece_segments_mode<T, kBonus>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, s_seg);
}

// One warp: inside a piece (elements [e0, e0 + n) of row j) whose segment
// sums are seg[0..32), the element at which the running weight first exceeds
// `target` -- segment (scan over lanes), vector (one vector per lane, a scan
// over lanes) and element.  Returns the row index (same in every lane), or -1
// when the piece has no positive weight.
template <typename T, bool kGeneric = false>
__device__ __forceinline__ int select_in_piece_body(const WeightRow& r, const float* seg, const unsigned char* tbuf,
                                                    const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0,
                                                    int n, float target) {
    constexpr int PV = Logit<T>::kPerVec;
    const int lane = threadIdx.x & 31;
    float one[1] = {seg[lane]};
    float t_seg;
    const int s = warp_pick<1>(one, kSegsPerPiece, target, &t_seg);
    if (s < 0) return -1;
    const int v = s * kSegVecs + lane;
    const int nvec = (n + PV - 1) / PV;
    float w[PV];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < PV; ++i) w[i] = 0.f;
    if (v < nvec) sum = piece_vec_weights<T, kGeneric>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, v, w);
    const float lv = warp_scan_incl(sum);
    const unsigned cross = __ballot_sync(0xffffffffu, sum > 0.f && lv > t_seg);
    const unsigned pos = __ballot_sync(0xffffffffu, sum > 0.f);
    const int lsel = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : -1);
    if (lsel < 0) return -1;
    int found = -1, last = -1;
    if (lane == lsel) {
        const float t2 = cross ? t_seg : INFINITY;
        float run = lv - sum;
#pragma unroll
        for (int i = 0; i < PV; ++i) {
            if (w[i] > 0.f && found < 0) {
                last = i;
                run += w[i];
                if (run > t2) found = i;
            }
        }
        found = e0 + v * PV + (found >= 0 ? found : last);
    }
    return __shfl_sync(0xffffffffu, found, lsel);
}

// select_in_piece_body as one out-of-line copy (the draw kernel calls it from
// several places); the selection kernel inlines the body instead, keeping
// its short code contiguous.
template <typename T>
__device__ __noinline__ int select_in_piece(const WeightRow r, const float* seg, const unsigned char* tbuf,
                                            const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0, int n,
                                            float target) {
    return select_in_piece_body<T>(r, seg, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, target);
}

// A queued draw, read through L2 (another kernel wrote it).
__device__ __forceinline__ DrawReq load_req(const DrawReq* src) {
    DrawReq r;
    const int4* s4 = reinterpret_cast<const int4*>(src);
    int4* d4 = reinterpret_cast<int4*>(&r);
#pragma unroll
    for (int i = 0; i < int(sizeof(DrawReq) / 16); ++i) d4[i] = __ldcg(s4 + i);
    return r;
}

// Warp 0: piece weights w[c] (c < P) held in s_pw -> total and the piece that
// holds ustar * total (-1 if none has positive weight); lane 0 stores them.
__device__ __forceinline__ void pick_piece(const float* s_pw, int P, float ustar, int* s_pick, float* s_target,
                                           float* s_W) {
    const int lane = threadIdx.x & 31;
    const int cps = (P + 31) / 32;
    float w[kMaxPiecesPerLane];
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPiecesPerLane; ++k) {
        const int c = lane * cps + k;
        w[k] = (k < cps && c < P) ? s_pw[c] : 0.f;
        tot += w[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    float local = INFINITY;
    const int pstar = tot > 0.f ? warp_pick<kMaxPiecesPerLane>(w, P, ustar * tot, &local) : -1;
    if (lane == 0) {
        *s_pick = pstar;
        *s_target = local;
        *s_W = tot;
    }
}

// Task numbering: CTA x of G runs tasks x, x + G, x + 2G, ...  The first
// n1 = min(#single, W) single-piece draws (bonus, one-hot: the tasks with the
// longest chain) go to the last CTAs of the first round, one each, counting
// down from CTA W - 1 (W = min(G, #tasks)), so that no CTA runs one after
// another task; residual pieces fill the other tasks in queue order, and any
// further single-piece draws come last.
struct TaskMap {
    int n_res_tasks, ntask, W, n1;   // < B * (P + 1) <= 2^31 - 1
    // residual piece index (>= 0: draw index / P, piece index % P), or
    // -(1 + single-piece draw index)
    __device__ __forceinline__ int decode(int t) const {
        if (t < W) {
            const int d = W - 1 - t;
            return d < n1 ? -(1 + d) : t;
        }
        const int q = t - n1;
        return q < n_res_tasks ? q : -(1 + n1 + (q - n_res_tasks));
    }
};

// The queue entry of task code e (TaskMap::decode).
__device__ __forceinline__ DrawReq task_req(const DrawParams& p, int e) {
    return e >= 0 ? load_req(p.res_req + e / p.P) : load_req(p.one_req + (-e - 1));
}

template <typename T>
__global__ void __launch_bounds__(kDrawThreads, kDrawCtasPerSm)
verify_draw_kernel(const DrawParams p) {
    extern __shared__ __align__(1024) unsigned char draw_dsm[];
    __shared__ __align__(8) uint64_t s_bar[2];
    __shared__ float s_seg[kSegsPerPiece];
    __shared__ float s_pw[kMaxPieces];
    __shared__ DrawReq s_req[2];
    __shared__ int s_pick;
    __shared__ float s_target, s_W;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = p.k_max;
    const int P = p.P;
    const int64_t esz = Logit<T>::kSize;
    const bool vec_ok = p.rows_aligned != 0;

    // the selection kernel may be launched now; it waits for this grid
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");
    // the scan kernel's queue (this kernel is a programmatic dependent of it);
    // thread 0 reads the two entries its first task can have when there are
    // at least G tasks (residual piece x, or single-piece draw G - 1 - x)
    // together with the queue lengths
    asm volatile("griddepcontrol.wait;" ::: "memory");
    DrawReq first, first_one;
    if (tid == 0) {
        first = load_req(p.res_req + min(int(blockIdx.x / P), p.B - 1));
        first_one = load_req(p.one_req + min(int(gridDim.x - 1 - blockIdx.x), p.B - 1));
    }
    const int nres = __ldcg(p.ctrl + 0);
    const int none = __ldcg(p.ctrl + 1);
    TaskMap tm;
    tm.n_res_tasks = nres * P;
    tm.ntask = tm.n_res_tasks + none;
    tm.W = min(int(gridDim.x), tm.ntask);
    tm.n1 = min(none, tm.W);
    const int ntask = tm.ntask;
    if (blockIdx.x >= ntask) return;
    if (tid == 0) {
        mbar_init(&s_bar[0], 1);
        mbar_init(&s_bar[1], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto trow_of = [&](const DrawReq& r) { return p.target + (int64_t(r.b) * (K + 1) + r.j) * p.row_stride * esz; };
    auto drow_of = [&](const DrawReq& r) { return p.draft + (int64_t(r.b) * K + r.j) * p.row_stride * esz; };
    auto piece_n = [&](int pc) { return min(p.V - pc * p.PE, p.PE); };
    // bytes of piece pc that a bulk copy delivers (the ragged end of the row
    // is read from global memory); 0 for rows that are not 16-byte aligned
    auto staged_bytes = [&](int pc) { return vec_ok ? (piece_n(pc) * int(esz)) & ~15 : 0; };
    auto part_row = [&](const DrawReq& r) { return p.partials + (int64_t(r.b) * (2 * K + 1) + r.j) * P; };

    // Barrier bookkeeping, identical in every thread: buffer x's next
    // completion has parity ph_x; pend_x says a copy (or arrival) into it was
    // issued and not yet waited for successfully.
    uint32_t ph0 = 0u, ph1 = 0u;
    bool pend0 = false, pend1 = false;
    bool failed = false;  // a wait ran out: every later draw of this CTA is reported -2

    // Thread 0 only: store task t's draw r in s_req[buf] and issue the copies
    // of its first piece into buffer buf (completing on s_bar[buf]).
    auto issue = [&](int t, const DrawReq& r, int buf) {
        const int e = tm.decode(t);
        const bool resid = e >= 0;
        const int pc = resid ? static_cast<int>(e % P) : (r.mode == kBonus ? r.piece : r.x / p.PE);
        s_req[buf] = r;
        if (r.b == p.lost_draw_b && pc == (resid ? 0 : pc)) return;  // injected fault: nothing completes the wait
        unsigned char* dst = draw_dsm + size_t(buf) * kDrawBufBytes;
        const uint32_t nb = static_cast<uint32_t>(staged_bytes(pc));
        if (nb == 0) {
            mbar_arrive(&s_bar[buf]);
            return;
        }
        mbar_arrive_expect_tx(&s_bar[buf], resid ? 2 * nb : nb);
        const int64_t off = int64_t(pc) * p.PE * esz;
        // default L2 policy: the selection kernel re-reads one segment of the
        // chosen piece right after this kernel, and finds it in L2
        bulk_copy_g2s(dst, trow_of(r) + off, nb, &s_bar[buf]);
        if (resid) bulk_copy_g2s(dst + kPieceBytes, drow_of(r) + off, nb, &s_bar[buf]);
    };
    // All threads: wait for buffer buf's pending completion (bounded);
    // block-uniform result.  On success the parity moves on; on a timeout it
    // stays, so the final drain waits for the same completion.
    auto wait_buf = [&](int buf) {
        const uint32_t ph = buf ? ph1 : ph0;
        bool ok = mbar_wait_bounded(&s_bar[buf], ph, p.timeout_ns);
        ok = __syncthreads_and(ok);
        if (ok) {
            if (buf) { ph1 ^= 1u; pend1 = false; } else { ph0 ^= 1u; pend0 = false; }
        }
        return ok;
    };
    // A lost draw: the request reports -2; a residual draw is also marked so
    // that the selection kernel leaves it alone.
    auto fail_request = [&](const DrawReq& r, int t) {
        int32_t* tok = p.out_tokens + int64_t(r.b) * (K + 1);
        for (int i = tid; i <= K; i += kDrawThreads) tok[i] = -1;
        if (tid == 0) {
            p.out_len[r.b] = -2;
            const int e = tm.decode(t);
            if (e >= 0) p.res_lost[e / P] = 1;
        }
    };

    // Thread 0 keeps the queue entry of the task after the next one in
    // registers, loaded one iteration ahead of its use.
    DrawReq ahead;
    if (tid == 0) {
        const int x = blockIdx.x;
        const int e = tm.decode(x);
        if (e < 0 && -e - 1 == int(gridDim.x) - 1 - x) first = first_one;
        else if (!(e >= 0 && e / P == x / P)) first = task_req(p, e);
        issue(blockIdx.x, first, 0);
        if (blockIdx.x + gridDim.x < ntask) ahead = task_req(p, tm.decode(blockIdx.x + gridDim.x));
    }
    pend0 = true;
    int it = 0;
    for (int t = blockIdx.x; t < ntask; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const int tn = t + int(gridDim.x);
        __syncthreads();  // s_req[buf] is written; buffer buf ^ 1 is free again
        const DrawReq r = s_req[buf];
        if (tn < ntask) {
            if (tid == 0) {
                if (failed) s_req[buf ^ 1] = ahead;   // no more copies: only the entry is passed on
                else issue(tn, ahead, buf ^ 1);
                if (tn + gridDim.x < ntask) ahead = task_req(p, tm.decode(tn + gridDim.x));
            }
            if (!failed) {
                if (buf) pend0 = true; else pend1 = true;
            }
        }
        if (failed) {
            fail_request(r, t);
            continue;
        }
        if (!wait_buf(buf)) {
            failed = true;
            fail_request(r, t);
            continue;
        }
        unsigned char* tbuf = draw_dsm + size_t(buf) * kDrawBufBytes;
        unsigned char* dbuf = tbuf + kPieceBytes;
        WeightRow wr;
        wr.trow = trow_of(r);
        wr.drow = r.mode == kResidual ? drow_of(r) : nullptr;
        wr.scale = p.scale;
        wr.lse_p = r.lse_p;
        wr.lse_q = r.lse_q;
        wr.mode = r.mode;
        wr.zero_at = r.mode == kOneHot ? r.x : -1;
        int32_t* out_tok = p.out_tokens + int64_t(r.b) * (K + 1) + r.j;
        int pc_loaded = -1;   // piece of target row j staged in tbuf with s_seg holding its p-based segment sums

        const int code = tm.decode(t);
        if (code >= 0) {
            // residual piece: its segment sums go to the selection kernel
            const int slot = static_cast<int>(code / P);
            const int pc = static_cast<int>(code % P);
            piece_segments<T>(wr, tbuf, dbuf, staged_bytes(pc) / 16, vec_ok, pc * p.PE, piece_n(pc), s_seg);
            if (warp == 0) p.seg[(int64_t(slot) * P + pc) * kSegsPerPiece + lane] = s_seg[lane];
            continue;
        }
        if (r.mode == kBonus) {
            // ------------------ bonus: the scan kernel chose the piece ------------------
            piece_segments<T>(wr, tbuf, nullptr, staged_bytes(r.piece) / 16, vec_ok, r.piece * p.PE,
                              piece_n(r.piece), s_seg);
            if (warp == 0) {
                const int tok = select_in_piece<T>(wr, s_seg, tbuf, nullptr, staged_bytes(r.piece) / 16, vec_ok,
                                                   r.piece * p.PE, piece_n(r.piece), r.target);
                if (lane == 0) s_pick = tok;
            }
            __syncthreads();
            if (s_pick >= 0) {
                if (tid == 0) *out_tok = s_pick;
                continue;
            }
            // no positive weight where the partials put u*W: pick again below
            pc_loaded = r.piece;
        } else {
            // --------- one-hot: exact weight of the drafted id's piece (staged) ---------
            const int px = r.x / p.PE;
            piece_segments<T>(wr, tbuf, nullptr, staged_bytes(px) / 16, vec_ok, px * p.PE, piece_n(px), s_seg);
            pc_loaded = px;
        }

        // ----- piece weights of row j: s * 2^(m - lse) from the partials; the one-hot
        // ----- draw's own piece gets its exact residual weight from s_seg
        {
            const float2* part_j = part_row(r);
            for (int c = tid; c < P; c += kDrawThreads) {
                const float2 pp = part_j[c];
                s_pw[c] = pp.y * exp2f(pp.x - wr.lse_p);
            }
            __syncthreads();
            if (warp == 0) {
                if (wr.mode == kOneHot) {
                    float wx = s_seg[lane];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) wx += __shfl_xor_sync(0xffffffffu, wx, o);
                    if (lane == 0) s_pw[pc_loaded] = wx;
                    __syncwarp();
                }
                pick_piece(s_pw, P, r.ustar, &s_pick, &s_target, &s_W);
            }
            __syncthreads();
            if (!(s_W > 0.f) && wr.mode == kOneHot) {
                // zero one-hot residual mass (p(x) == 1 numerically): draw from p_j
                wr.mode = kBonus;
                wr.zero_at = -1;
                pc_loaded = -1;
                for (int c = tid; c < P; c += kDrawThreads) {
                    const float2 pp = part_j[c];
                    s_pw[c] = pp.y * exp2f(pp.x - wr.lse_p);
                }
                __syncthreads();
                if (warp == 0) pick_piece(s_pw, P, r.ustar, &s_pick, &s_target, &s_W);
                __syncthreads();
            }
        }
        int pstar = s_pick;
        float target = s_target;
        int tok = -1;
        // At most two attempts: the chosen piece, then (if rounding left it
        // without positive weight) the last positive element of the heaviest
        // other piece.
        for (int attempt = 0; attempt < 2 && pstar >= 0 && !failed; ++attempt) {
            if (pstar != pc_loaded) {
                __syncthreads();  // nobody reads tbuf / s_seg any more
                if (tid == 0) {
                    const uint32_t nb = static_cast<uint32_t>(staged_bytes(pstar));
                    if (nb == 0) {
                        mbar_arrive(&s_bar[buf]);
                    } else {
                        mbar_arrive_expect_tx(&s_bar[buf], nb);
                        bulk_copy_g2s(tbuf, wr.trow + int64_t(pstar) * p.PE * esz, nb, &s_bar[buf]);
                    }
                }
                if (buf) pend1 = true; else pend0 = true;
                if (!wait_buf(buf)) {
                    failed = true;
                    break;
                }
                piece_segments<T>(wr, tbuf, nullptr, staged_bytes(pstar) / 16, vec_ok, pstar * p.PE,
                                  piece_n(pstar), s_seg);
                pc_loaded = pstar;
            }
            if (warp == 0) {
                const int e = select_in_piece<T>(wr, s_seg, tbuf, nullptr, staged_bytes(pstar) / 16, vec_ok,
                                                 pstar * p.PE, piece_n(pstar), target);
                if (lane == 0) s_pick = e;
            }
            __syncthreads();
            tok = s_pick;
            if (tok >= 0) break;
            if (warp == 0) {
                float best = 0.f;
                int bi = -1;
                for (int c = lane; c < P; c += 32)
                    if (c != pstar && s_pw[c] > best) { best = s_pw[c]; bi = c; }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (ob > best || (ob == best && oi >= 0 && (bi < 0 || oi < bi))) { best = ob; bi = oi; }
                }
                if (lane == 0) s_pick = bi;
            }
            __syncthreads();
            pstar = s_pick;
            target = INFINITY;
        }
        if (tok >= 0) {
            if (tid == 0) *out_tok = tok;
        } else {
            fail_request(r, t);
        }
    }
    // A copy issued into a buffer that was never (successfully) waited for
    // must land before the CTA exits.
    __syncthreads();
    if (tid == 0) {
        if (pend0) (void)mbar_wait_bounded(&s_bar[0], ph0, p.timeout_ns);
        if (pend1) (void)mbar_wait_bounded(&s_bar[1], ph1, p.timeout_ns);
    }
}

// A staged copy of a residual piece: target and draft bytes (generic
// addresses) and the 16-byte vectors they hold; tbuf == nullptr: none.
struct StagedPiece {
    const unsigned char* tbuf;
    const unsigned char* dbuf;
    int nvec;
};

// One warp: the residual draw r from its piece totals w (lane l holding
// pieces [l*cps, l*cps + cps)): the piece and the segment holding u*W, then
// the vector and the element, re-reading that segment of both rows
// (seg_of(c) returns piece c's 32 segment sums where the whole warp can read
// them; stage_of(c) the piece's staged copy when one is still held, whose
// vectors are then read instead of global memory).  Zero residual mass (p == q numerically) draws from p_j instead:
// the piece from the partials, its segment sums computed here by the warp
// into s_tmp (32 floats).  Returns the token, or -1 when no positive weight
// is found (not reached with finite logits).  Used by the cluster kernel;
// the selection kernel below takes the same steps inline, interleaved with
// its loads (0.7 us per step faster on the largest workload than calling
// this function).  Their picks are identical.
template <typename T, typename Params, typename SegOf, typename StageOf>
__device__ __forceinline__ int select_residual_warp(const Params& p, const DrawReq& r,
                                                    const float (&w)[kMaxPiecesPerLane], SegOf seg_of,
                                                    StageOf stage_of, float* s_tmp) {
    constexpr int PV = Logit<T>::kPerVec;
    const int lane = threadIdx.x & 31;
    const int K = p.k_max;
    const int P = p.P;
    const int64_t esz = Logit<T>::kSize;
    const bool vec_ok = p.rows_aligned != 0;
    const int cps = (P + 31) / 32;
    WeightRow wr;
    wr.trow = p.target + (int64_t(r.b) * (K + 1) + r.j) * p.row_stride * esz;
    wr.drow = p.draft + (int64_t(r.b) * K + r.j) * p.row_stride * esz;
    wr.scale = p.scale;
    wr.lse_p = r.lse_p;
    wr.lse_q = r.lse_q;
    wr.mode = kResidual;
    wr.zero_at = -1;
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPiecesPerLane; ++k) tot += w[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    float local = INFINITY;
    int pstar = -1;
    const float* segp = nullptr;
    if (tot > 0.f) {
        pstar = warp_pick<kMaxPiecesPerLane>(w, P, r.ustar * tot, &local);
        if (pstar >= 0) segp = seg_of(pstar);
    } else {
        wr.mode = kBonus;
        wr.drow = nullptr;
        const float2* part_j = p.partials + (int64_t(r.b) * (2 * K + 1) + r.j) * P;
        float pw[kMaxPiecesPerLane];
        float ptot = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxPiecesPerLane; ++k) {
            const int c = lane * cps + k;
            pw[k] = 0.f;
            if (k < cps && c < P) {
                const float2 pp = part_j[c];
                pw[k] = pp.y * exp2f(pp.x - wr.lse_p);
            }
            ptot += pw[k];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ptot += __shfl_xor_sync(0xffffffffu, ptot, o);
        if (ptot > 0.f) pstar = warp_pick<kMaxPiecesPerLane>(pw, P, r.ustar * ptot, &local);
        if (pstar >= 0) {
            const int e0 = pstar * p.PE, n = min(p.V - e0, p.PE);
            const int nvec = (n + PV - 1) / PV;
            for (int sg = 0; sg < kSegsPerPiece; ++sg) {
                const int v = sg * kSegVecs + lane;
                float wv[PV];
                float sum = v < nvec ? piece_vec_weights<T>(wr, nullptr, nullptr, 0, vec_ok, e0, n, v, wv) : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) s_tmp[sg] = sum;
            }
            __syncwarp();
            segp = s_tmp;
        }
    }
    if (pstar < 0) return -1;
    if (wr.mode == kResidual) {
        // the piece's staged copy, where it is still held (a generic address)
        const StagedPiece sp = stage_of(pstar);
        if (sp.tbuf)
            return select_in_piece_body<T, true>(wr, segp, sp.tbuf, sp.dbuf, sp.nvec, vec_ok, pstar * p.PE,
                                                 min(p.V - pstar * p.PE, p.PE), local);
    }
    return select_in_piece_body<T>(wr, segp, nullptr, nullptr, 0, vec_ok, pstar * p.PE,
                                   min(p.V - pstar * p.PE, p.PE), local);
}

// ============================================================================
// K2c: selection of the residual draws, one warp per queued residual draw.

constexpr int kSelectThreads = 256;
constexpr int kSelectWarps = kSelectThreads / 32;

struct SelectParams {
    int32_t B;
    const unsigned char* target;
    const unsigned char* draft;
    const float2* partials;
    const int32_t* ctrl;
    const DrawReq* res_req;
    const float* seg;            // [B][P][32] segment sums written by K2b
    const int32_t* res_lost;     // [B] residual draws K2b lost to a timeout (already reported -2)
    int32_t* out_len;
    int32_t* out_tokens;
    int32_t k_max;
    int32_t V;
    int64_t row_stride;
    int32_t P;
    int32_t PE;
    float scale;
    int32_t rows_aligned;
};

template <typename T>
__global__ void __launch_bounds__(kSelectThreads)
verify_select_kernel(const SelectParams p) {
    constexpr int PV = Logit<T>::kPerVec;
    // per warp: the segment sums of the draw's pieces as loaded (one row of
    // 33 floats per lane, so the lanes' stores hit distinct banks), kept when
    // every lane holds one piece (P <= 32) so that the chosen piece's sums
    // need no second load; the zero-mass path reuses the first row
    __shared__ float s_segs[kSelectWarps][32 * (kSegsPerPiece + 1)];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the next call's first kernel may be launched now; it waits for this grid
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // slot < B: every load below stays inside the workspace, so the queue
    // length, the loss mark, the entry and the segment sums are read at once
    const int slot = blockIdx.x * kSelectWarps + warp;
    if (slot >= p.B) return;
    const int K = p.k_max;
    const int P = p.P;
    const int64_t esz = Logit<T>::kSize;
    const bool vec_ok = p.rows_aligned != 0;
    const int nres = __ldcg(p.ctrl + 0);
    const int lost = __ldcg(p.res_lost + slot);
    const DrawReq r = load_req(p.res_req + slot);
    WeightRow wr;
    wr.trow = p.target + (int64_t(r.b) * (K + 1) + r.j) * p.row_stride * esz;
    wr.drow = p.draft + (int64_t(r.b) * K + r.j) * p.row_stride * esz;
    wr.scale = p.scale;
    wr.lse_p = r.lse_p;
    wr.lse_q = r.lse_q;
    wr.mode = kResidual;
    wr.zero_at = -1;
    const float* seg = p.seg + int64_t(slot) * P * kSegsPerPiece;
    // piece totals: lane l sums the 32 segment sums of its pieces [l*cps, l*cps + cps)
    const int cps = (P + 31) / 32;
    float w[kMaxPiecesPerLane];
#pragma unroll
    for (int k = 0; k < kMaxPiecesPerLane; ++k) {
        const int c = lane * cps + k;
        float t = 0.f;
        if (k < cps && c < P) {
            const float4* s4 = reinterpret_cast<const float4*>(seg + int64_t(c) * kSegsPerPiece);
            float* keep = &s_segs[warp][lane * (kSegsPerPiece + 1)];
#pragma unroll
            for (int q = 0; q < kSegsPerPiece / 4; ++q) {
                const float4 v = s4[q];
                t += (v.x + v.y) + (v.z + v.w);
                if (cps == 1) {
                    keep[4 * q] = v.x;
                    keep[4 * q + 1] = v.y;
                    keep[4 * q + 2] = v.z;
                    keep[4 * q + 3] = v.w;
                }
            }
        }
        w[k] = t;
    }
    __syncwarp();
    if (slot >= nres || lost != 0) return;
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPiecesPerLane; ++k) tot += w[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    float local = INFINITY;
    int pstar = -1;
    const float* segp = nullptr;
    if (tot > 0.f) {
        pstar = warp_pick<kMaxPiecesPerLane>(w, P, r.ustar * tot, &local);
        segp = cps == 1 ? &s_segs[warp][pstar * (kSegsPerPiece + 1)] : seg + int64_t(pstar) * kSegsPerPiece;
    } else {
        // zero residual mass (p == q numerically): draw from p_j -- the piece
        // from the partials, its segment sums computed here by the warp
        wr.mode = kBonus;
        wr.drow = nullptr;
        const float2* part_j = p.partials + (int64_t(r.b) * (2 * K + 1) + r.j) * P;
        float pw[kMaxPiecesPerLane];
        float ptot = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxPiecesPerLane; ++k) {
            const int c = lane * cps + k;
            pw[k] = 0.f;
            if (k < cps && c < P) {
                const float2 pp = part_j[c];
                pw[k] = pp.y * exp2f(pp.x - wr.lse_p);
            }
            ptot += pw[k];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ptot += __shfl_xor_sync(0xffffffffu, ptot, o);
        if (ptot > 0.f) pstar = warp_pick<kMaxPiecesPerLane>(pw, P, r.ustar * ptot, &local);
        if (pstar >= 0) {
            const int e0 = pstar * p.PE, n = min(p.V - e0, p.PE);
            const int nvec = (n + PV - 1) / PV;
            for (int sg = 0; sg < kSegsPerPiece; ++sg) {
                const int v = sg * kSegVecs + lane;
                float wv[PV];
                float sum = v < nvec ? piece_vec_weights<T>(wr, nullptr, nullptr, 0, vec_ok, e0, n, v, wv) : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) s_segs[warp][sg] = sum;
            }
            __syncwarp();
            segp = s_segs[warp];
        }
    }
    int tok = -1;
    if (pstar >= 0)
        tok = select_in_piece_body<T>(wr, segp, nullptr, nullptr, 0, vec_ok, pstar * p.PE,
                                      min(p.V - pstar * p.PE, p.PE), local);
    if (tok >= 0) {
        if (lane == 0) p.out_tokens[int64_t(r.b) * (K + 1) + r.j] = tok;
    } else {
        // no positive weight anywhere the draw could land (not reached with
        // finite logits): the request is reported as lost
        int32_t* out = p.out_tokens + int64_t(r.b) * (K + 1);
        for (int i = lane; i <= K; i += 32) out[i] = -1;
        if (lane == 0) p.out_len[r.b] = -2;
    }
}

}  // namespace sv
