// sv_verify_draw.cuh -- K2b, the final draw (residual / bonus / one-hot).
//
// The scan kernel queued one draw per sampling request: a residual draw
// (rejection with draft logits) as P tasks, one per piece of the row pair,
// and a bonus or one-hot draw as one task.  This kernel is a persistent grid
// of resident CTAs; CTA x takes tasks x, x + G, x + 2G, ... (residual tasks
// first, ordered slot-major, so one draw's pieces run on P different CTAs at
// once).  Each task stages its piece(s) in shared memory with 1-D bulk copies
// (double-buffered: the next task's copies are in flight while the current
// one is computed) and computes the draw weights
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
//   * residual: each task stores its piece's 32 segment sums and counts the
//     piece as done (atomic add after a fence); the CTA that finishes the
//     last piece picks the piece and segment from the stored sums, re-reads
//     that one segment of both rows (one vector per lane) and picks the
//     vector and element.  Nothing waits on another CTA.
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
// Waits: only on this CTA's own bulk copies, bounded by timeout_ns; after a
// timeout the CTA reports its remaining draws with out_accept_len = -2.
#pragma once

#include "sv_common.cuh"
#include "sv_verify_scan.cuh"

#ifndef SV_DRAW_CTAS_PER_SM
#define SV_DRAW_CTAS_PER_SM 3
#endif

namespace sv {

struct DrawParams {
    const unsigned char* target;
    const unsigned char* draft;
    const float2* partials;      // [B][2k+1][P] row-statistics partials
    const int32_t* ctrl;         // [0] residual draws, [1] single-piece draws
    const DrawReq* res_req;
    const DrawReq* one_req;
    int32_t* res_cnt;            // [B] pieces finished per residual draw
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
template <typename T>
__device__ __forceinline__ void load_vec(const unsigned char* sm, const unsigned char* row, int idx0, int count,
                                         bool vec_ok, float (&z)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    if (sm) {
        Logit<T>::unpack(ld_shared_v4(sm), z);
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
template <typename T>
__device__ __forceinline__ float piece_vec_weights(const WeightRow& r, const unsigned char* tbuf,
                                                   const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0,
                                                   int n, int v, float (&w)[Logit<T>::kPerVec]) {
    constexpr int PV = Logit<T>::kPerVec;
    const int idx0 = e0 + v * PV;
    const int count = min(PV, n - v * PV);
    float z[PV], y[PV];
    const bool staged = v < nstaged_vec;
    load_vec<T>(staged ? tbuf + 16 * v : nullptr, r.trow, idx0, count, vec_ok, z);
    if (r.mode == kResidual) load_vec<T>(staged ? dbuf + 16 * v : nullptr, r.drow, idx0, count, vec_ok, y);
#pragma unroll
    for (int i = 0; i < PV; ++i)
        if (r.mode != kResidual) y[i] = 0.f;
    return vec_weights<T>(r, z, y, idx0, count, w);
}

// All threads: the 32 segment sums of one piece into s_seg (ends with
// __syncthreads).  Thread t handles vectors t + 256 k, so warp w at step k
// covers segment w + 8 k.
template <typename T>
__device__ __forceinline__ void piece_segments(const WeightRow& r, const unsigned char* tbuf,
                                               const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0,
                                               int n, float* s_seg) {
    constexpr int PV = Logit<T>::kPerVec;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = (n + PV - 1) / PV;
#pragma unroll
    for (int k = 0; k < kVecsPerThread; ++k) {
        const int v = threadIdx.x + k * kDrawThreads;
        float w[PV];
        float sum = v < nvec ? piece_vec_weights<T>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, v, w) : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) s_seg[warp + kDrawWarps * k] = sum;
    }
    __syncthreads();
}

// One warp: inside a piece (elements [e0, e0 + n) of row j) whose segment
// sums are seg[0..32), the element at which the running weight first exceeds
// `target` -- segment (scan over lanes), vector (one vector per lane, a scan
// over lanes) and element.  Returns the row index (same in every lane), or -1
// when the piece has no positive weight.
template <typename T>
__device__ __noinline__ int select_in_piece(const WeightRow r, const float* seg, const unsigned char* tbuf,
                                            const unsigned char* dbuf, int nstaged_vec, bool vec_ok, int e0, int n,
                                            float target) {
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
    if (v < nvec) sum = piece_vec_weights<T>(r, tbuf, dbuf, nstaged_vec, vec_ok, e0, n, v, w);
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

template <typename T>
__global__ void __launch_bounds__(kDrawThreads, kDrawCtasPerSm)
verify_draw_kernel(const DrawParams p) {
    extern __shared__ __align__(1024) unsigned char draw_dsm[];
    __shared__ __align__(8) uint64_t s_bar[2];
    __shared__ float s_seg[kSegsPerPiece];
    __shared__ float s_pw[kMaxPieces];
    __shared__ DrawReq s_req[2];
    __shared__ int s_last, s_pick;
    __shared__ float s_target, s_W;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = p.k_max;
    const int P = p.P;
    const int64_t esz = Logit<T>::kSize;
    const bool vec_ok = p.rows_aligned != 0;

    // the scan kernel's queue (this kernel is a programmatic dependent of it)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int nres = __ldcg(p.ctrl + 0);
    const int none = __ldcg(p.ctrl + 1);
    const int64_t n_res_tasks = int64_t(nres) * P;
    const int64_t ntask = n_res_tasks + none;
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

    // Thread 0 only: read task t's draw into s_req[buf] and issue the copies
    // of its first piece into buffer buf (completing on s_bar[buf]).
    auto issue = [&](int64_t t, int buf) {
        DrawReq r;
        int pc;
        bool resid;
        if (t < n_res_tasks) {
            r = load_req(p.res_req + t / P);
            pc = static_cast<int>(t % P);
            resid = true;
        } else {
            r = load_req(p.one_req + (t - n_res_tasks));
            pc = r.mode == kBonus ? r.piece : r.x / p.PE;
            resid = false;
        }
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
    auto fail_request = [&](const DrawReq& r) {
        int32_t* tok = p.out_tokens + int64_t(r.b) * (K + 1);
        for (int i = tid; i <= K; i += kDrawThreads) tok[i] = -1;
        if (tid == 0) p.out_len[r.b] = -2;
    };

    if (tid == 0) issue(blockIdx.x, 0);
    pend0 = true;
    int it = 0;
    for (int64_t t = blockIdx.x; t < ntask; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const int64_t tn = t + gridDim.x;
        __syncthreads();  // s_req[buf] is written; buffer buf ^ 1 is free again
        const DrawReq r = s_req[buf];
        if (failed) {
            fail_request(r);
            if (tn < ntask && tid == 0) s_req[buf ^ 1] = t + gridDim.x < n_res_tasks
                                                             ? load_req(p.res_req + tn / P)
                                                             : load_req(p.one_req + (tn - n_res_tasks));
            continue;
        }
        if (tn < ntask) {
            if (tid == 0) issue(tn, buf ^ 1);
            if (buf) pend0 = true; else pend1 = true;
        }
        if (!wait_buf(buf)) {
            failed = true;
            fail_request(r);
            if (tn < ntask && tid == 0) {
                // the next task's draw is already in s_req[buf ^ 1]; its copy is
                // pending and drained at the end
            }
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

        if (t < n_res_tasks) {
            // ---------------------------- residual piece ----------------------------
            const int slot = static_cast<int>(t / P);
            const int pc = static_cast<int>(t % P);
            piece_segments<T>(wr, tbuf, dbuf, staged_bytes(pc) / 16, vec_ok, pc * p.PE, piece_n(pc), s_seg);
            float* seg_out = p.seg + (int64_t(slot) * P + pc) * kSegsPerPiece;
            if (warp == 0) {
                seg_out[lane] = s_seg[lane];
                __threadfence();  // the sums are visible before the piece is counted
            }
            __syncthreads();
            if (tid == 0) {
                s_last = atomicAdd(p.res_cnt + slot, 1) == P - 1;
                __threadfence();
            }
            __syncthreads();
            if (!s_last) continue;
            // The last piece of this draw: piece totals from every task's
            // segment sums, then piece, segment (sums re-read into s_seg) and
            // element (one vector per lane re-read from the rows).
            const float* seg_all = p.seg + int64_t(slot) * P * kSegsPerPiece;
            for (int c = warp; c < P; c += kDrawWarps) {
                float v = __ldcg(seg_all + int64_t(c) * kSegsPerPiece + lane);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) s_pw[c] = v;
            }
            __syncthreads();
            if (warp == 0) pick_piece(s_pw, P, r.ustar, &s_pick, &s_target, &s_W);
            __syncthreads();
            if (s_W > 0.f) {
                const int pstar = s_pick;
                if (warp == 0) {
                    s_seg[lane] = __ldcg(seg_all + int64_t(pstar) * kSegsPerPiece + lane);
                    __syncwarp();
                    const int tok = select_in_piece<T>(wr, s_seg, nullptr, nullptr, 0, vec_ok, pstar * p.PE,
                                                       piece_n(pstar), s_target);
                    if (lane == 0) s_pick = tok;
                }
                __syncthreads();
                if (s_pick >= 0) {
                    if (tid == 0) *out_tok = s_pick;
                } else {
                    fail_request(r);
                }
                continue;
            }
            // zero residual mass (p == q numerically): the draw uses p_j
            wr.mode = kBonus;
            wr.drow = nullptr;
        } else if (r.mode == kBonus) {
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
            fail_request(r);
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

}  // namespace sv
