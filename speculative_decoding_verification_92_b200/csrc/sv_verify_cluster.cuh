// sv_verify_cluster.cuh -- the scan and the final draw of a small batch in
// one kernel: one thread-block cluster of C CTAs per request.
//
// Used for sampling calls whose B clusters all fit on the GPU at once (the
// long-tail phase: a few long requests).  It replaces the scan kernel, the
// draw kernel and the selection kernel, and with them two grid boundaries
// and the draw queue:
//   1. CTA 0 runs the scan of the request (scan_request: merge of the row
//      partials, p and q at the drafted ids, the first rejection j, the
//      outputs, and the draw they imply) and stores the draw into every
//      CTA's shared memory before a cluster barrier;
//   2. residual draw (rejection with draft logits): CTA r stages pieces
//      r, r + C, ... of the row pair j (1-D bulk copies, double-buffered) and
//      keeps each piece's 32 segment sums and total in its shared memory;
//      after a cluster barrier CTA 0 reads every piece total through
//      distributed shared memory, picks the piece and the segment holding
//      u*W, reads that segment of both rows (from the staging buffer of the
//      CTA that holds the piece when it still holds it, else from global
//      memory) and picks the vector and the element (select_residual_warp:
//      the selection kernel's steps);
//   3. bonus and one-hot draws: CTA 0 alone, as one task of the draw kernel.
// The weights, the selection order and the fallbacks are the draw kernel's
// ("AI 开始抄自己的作业——而且抄得理直气壮", section "⚡ 投机解码：让草稿先跑，考官殿后").
// Waits: only on a CTA's own bulk copies (bounded); a timeout reports the
// request with out_accept_len = -2.  Every CTA of a cluster passes the same
// cluster barriers, whatever happened to its copies.
#pragma once

#include <cooperative_groups.h>

#include "sv_verify_draw.cuh"

namespace sv {

// CTAs per cluster: min(P, cmax) with cmax = 16 (a non-portable cluster
// size, used where the GPU can place such clusters) or else 8 (portable).
constexpr int kClusterMaxCtas = 16;
constexpr int kClusterPortableCtas = 8;
// pieces per CTA: at most ceil(P / 8)
constexpr int kClusterMaxPerCta = (kMaxPieces + kClusterPortableCtas - 1) / kClusterPortableCtas;
constexpr size_t kClusterBufBytes = kDrawBufBytes;        // one staging buffer: a target and a draft piece

__host__ __device__ inline int cluster_ctas(int P, int cmax) { return P < cmax ? (P < 1 ? 1 : P) : cmax; }

// Dynamic shared memory of the cluster kernel: the scan's area, then two
// staging buffers.
__host__ __device__ inline size_t cluster_scan_area(int k_max, int P) {
    return (scan_smem_bytes(k_max, P) + 1023) & ~size_t(1023);
}
__host__ __device__ inline size_t cluster_smem_bytes(int k_max, int P) {
    return cluster_scan_area(k_max, P) + 2 * kClusterBufBytes;
}

template <typename T>
__global__ void __launch_bounds__(kScanThreads)
verify_cluster_kernel(const ScanParams sp, const DrawParams p) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(1024) unsigned char cl_dsm[];
    __shared__ ScanShared ss;
    __shared__ __align__(8) uint64_t s_bar[2];
    __shared__ float s_seg[kSegsPerPiece];
    __shared__ float s_ptot[kClusterMaxPerCta];
    __shared__ float s_pseg[kClusterMaxPerCta][kSegsPerPiece];
    __shared__ float s_sel[kSegsPerPiece];
    __shared__ float s_pw[kMaxPieces];
    __shared__ int s_lost, s_pick;
    __shared__ float s_target, s_W;

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int b = static_cast<int>(blockIdx.x) / C;  // clusters are consecutive runs of C blocks
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the next call's first kernel may be launched now; it waits for this grid
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;");

    // CTA 0 scans the request and hands the outcome to every CTA of the
    // cluster (stores into their shared memory, made visible by the cluster
    // barrier), so all of them take the same path through the barriers below.
    __shared__ int s_go;
    __shared__ DrawReq s_draw;
    if (rank == 0) {
        const bool go = scan_request<T>(sp, b, cl_dsm, &ss, true, false);
        if (tid < C) {
            *cluster.map_shared_rank(&s_go, tid) = go ? 1 : 0;
            if (go) *cluster.map_shared_rank(&s_draw, tid) = ss.draw;
        }
    }
    cluster.sync();
    if (!s_go) return;
    const DrawReq r = s_draw;

    const int K = p.k_max;
    const int P = p.P;
    const int64_t esz = Logit<T>::kSize;
    const bool vec_ok = p.rows_aligned != 0;
    unsigned char* bufs = cl_dsm + cluster_scan_area(K, P);
    const unsigned char* trow = p.target + (int64_t(r.b) * (K + 1) + r.j) * p.row_stride * esz;
    const unsigned char* drow = r.mode == kResidual ? p.draft + (int64_t(r.b) * K + r.j) * p.row_stride * esz : nullptr;
    auto piece_n = [&](int pc) { return min(p.V - pc * p.PE, p.PE); };
    auto staged_bytes = [&](int pc) { return vec_ok ? (piece_n(pc) * int(esz)) & ~15 : 0; };
    WeightRow wr;
    wr.trow = trow;
    wr.drow = drow;
    wr.scale = p.scale;
    wr.lse_p = r.lse_p;
    wr.lse_q = r.lse_q;
    wr.mode = r.mode;
    wr.zero_at = r.mode == kOneHot ? r.x : -1;
    int32_t* out = p.out_tokens + int64_t(r.b) * (K + 1);

    if (tid == 0) {
        mbar_init(&s_bar[0], 1);
        mbar_init(&s_bar[1], 1);
        fence_mbar_init();
        s_lost = 0;
    }
    __syncthreads();
    // Buffer x's next completion has parity ph[x]; pend[x]: a copy into it was
    // issued and not yet waited for successfully (same in every thread).
    uint32_t ph[2] = {0u, 0u};
    bool pend[2] = {false, false};
    bool injected = r.b == p.lost_draw_b;  // test fault injection: the first staging is never issued
    // Thread 0: stage piece pc of the target row (and of the draft row, `both`)
    // into buffer x.
    auto issue = [&](int pc, bool both, int x) {
        const bool skip = injected;  // same in every thread
        injected = false;
        if (skip) return;            // nothing completes buffer x's wait
        pend[x] = true;
        if (tid == 0) {
            unsigned char* dst = bufs + size_t(x) * kClusterBufBytes;
            const uint32_t nb = static_cast<uint32_t>(staged_bytes(pc));
            if (nb == 0) {
                mbar_arrive(&s_bar[x]);
                return;
            }
            mbar_arrive_expect_tx(&s_bar[x], both ? 2 * nb : nb);
            const int64_t off = int64_t(pc) * p.PE * esz;
            bulk_copy_g2s(dst, trow + off, nb, &s_bar[x]);
            if (both) bulk_copy_g2s(dst + kPieceBytes, drow + off, nb, &s_bar[x]);
        }
    };
    // All threads: wait for buffer x (bounded); block-uniform result.
    auto wait_buf = [&](int x) {
        bool ok = mbar_wait_bounded(&s_bar[x], ph[x], p.timeout_ns);
        ok = __syncthreads_and(ok);
        if (ok) {
            ph[x] ^= 1u;
            pend[x] = false;
        }
        return ok;
    };
    auto report_lost = [&]() {  // one warp
        for (int i = lane; i <= K; i += 32) out[i] = -1;
        if (lane == 0) p.out_len[r.b] = -2;
    };
    auto drain = [&]() {
        __syncthreads();
        if (tid == 0) {
            if (pend[0]) (void)mbar_wait_bounded(&s_bar[0], ph[0], p.timeout_ns);
            if (pend[1]) (void)mbar_wait_bounded(&s_bar[1], ph[1], p.timeout_ns);
        }
    };

    if (r.mode == kResidual) {
        // ---- pieces rank, rank + C, ... of the row pair: segment sums and totals ----
        const int npc = rank < P ? (P - 1 - rank) / C + 1 : 0;
        if (npc > 0) issue(rank, true, 0);
        for (int k = 0; k < npc; ++k) {
            const int x = k & 1;
            const int pc = rank + k * C;
            if (k + 1 < npc) issue(pc + C, true, x ^ 1);
            if (!wait_buf(x)) {
                if (tid == 0) s_lost = 1;
                break;
            }
            unsigned char* tb = bufs + size_t(x) * kClusterBufBytes;
            piece_segments<T>(wr, tb, tb + kPieceBytes, staged_bytes(pc) / 16, vec_ok, pc * p.PE, piece_n(pc),
                              s_seg);
            if (warp == 0) {
                s_pseg[k][lane] = s_seg[lane];
                if (lane == 0) {
                    // the piece total, added in the selection kernel's order
                    float t = 0.f;
#pragma unroll
                    for (int q = 0; q < kSegsPerPiece / 4; ++q)
                        t += (s_seg[4 * q] + s_seg[4 * q + 1]) + (s_seg[4 * q + 2] + s_seg[4 * q + 3]);
                    s_ptot[k] = t;
                }
            }
            __syncthreads();  // buffer x is free for piece k + 2
        }
        drain();
        cluster.sync();  // every CTA's sums are complete and visible to the cluster
        if (rank == 0 && warp == 0) {
            int lost = 0;
            if (lane < C) lost = *cluster.map_shared_rank(&s_lost, lane);
            if (__any_sync(0xffffffffu, lost != 0)) {
                report_lost();
            } else {
                // piece totals: lane l holds pieces [l*cps, l*cps + cps); piece c
                // lives in CTA c % C, slot c / C
                const int cps = (P + 31) / 32;
                float w[kMaxPiecesPerLane];
#pragma unroll
                for (int k = 0; k < kMaxPiecesPerLane; ++k) {
                    const int c = lane * cps + k;
                    w[k] = (k < cps && c < P) ? *cluster.map_shared_rank(&s_ptot[c / C], c % C) : 0.f;
                }
                auto seg_of = [&](int c) -> const float* {
                    s_sel[lane] = *cluster.map_shared_rank(&s_pseg[c / C][lane], c % C);
                    __syncwarp();
                    return s_sel;
                };
                // a CTA with at most two pieces still holds both in its buffers
                // (piece k in buffer k): the selection reads the chosen one there
                auto stage_of = [&](int c) -> StagedPiece {
                    const int owner = c % C, k = c / C;
                    if ((P - 1 - owner) / C + 1 > 2) return StagedPiece{nullptr, nullptr, 0};
                    const unsigned char* tb = cluster.map_shared_rank(bufs + size_t(k) * kClusterBufBytes, owner);
                    return StagedPiece{tb, tb + kPieceBytes, staged_bytes(c) / 16};
                };
                const int tok = select_residual_warp<T>(p, r, w, seg_of, stage_of, s_sel);
                if (tok >= 0) {
                    if (lane == 0) out[r.j] = tok;
                } else {
                    report_lost();
                }
            }
        }
        cluster.sync();  // nobody leaves while CTA 0 reads its shared memory
        return;
    }

    if (rank != 0) return;
    // ---- bonus / one-hot: this CTA alone ----
    unsigned char* tb = bufs;
    int pc_loaded = -1;  // piece of target row j staged in tb with s_seg holding its segment sums
    bool ok = true;
    if (r.mode == kBonus) {
        issue(r.piece, false, 0);
        ok = wait_buf(0);
        if (ok) {
            piece_segments<T>(wr, tb, nullptr, staged_bytes(r.piece) / 16, vec_ok, r.piece * p.PE,
                              piece_n(r.piece), s_seg);
            if (warp == 0) {
                const int tok = select_in_piece<T>(wr, s_seg, tb, nullptr, staged_bytes(r.piece) / 16, vec_ok,
                                                   r.piece * p.PE, piece_n(r.piece), r.target);
                if (lane == 0) s_pick = tok;
            }
            __syncthreads();
            if (s_pick >= 0) {
                if (tid == 0) out[r.j] = s_pick;
                drain();
                return;
            }
            pc_loaded = r.piece;  // no positive weight where the partials put u*W: pick again below
        }
    } else {
        const int px = r.x / p.PE;  // exact weight of the drafted id's piece
        issue(px, false, 0);
        ok = wait_buf(0);
        if (ok) {
            piece_segments<T>(wr, tb, nullptr, staged_bytes(px) / 16, vec_ok, px * p.PE, piece_n(px), s_seg);
            pc_loaded = px;
        }
    }
    if (ok) {
        // piece weights of row j from the partials; the one-hot draw's own piece
        // gets its exact residual weight from s_seg
        const float2* part_j = p.partials + (int64_t(r.b) * (2 * K + 1) + r.j) * P;
        for (int c = tid; c < P; c += kScanThreads) {
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
            for (int c = tid; c < P; c += kScanThreads) {
                const float2 pp = part_j[c];
                s_pw[c] = pp.y * exp2f(pp.x - wr.lse_p);
            }
            __syncthreads();
            if (warp == 0) pick_piece(s_pw, P, r.ustar, &s_pick, &s_target, &s_W);
            __syncthreads();
        }
    }
    int pstar = ok ? s_pick : -1;
    float target = ok ? s_target : INFINITY;
    int tok = -1;
    // At most two attempts: the chosen piece, then (if rounding left it
    // without positive weight) the last positive element of the heaviest
    // other piece.
    for (int attempt = 0; attempt < 2 && pstar >= 0 && ok; ++attempt) {
        if (pstar != pc_loaded) {
            __syncthreads();  // nobody reads tb / s_seg any more
            issue(pstar, false, 0);
            if (!(ok = wait_buf(0))) break;
            piece_segments<T>(wr, tb, nullptr, staged_bytes(pstar) / 16, vec_ok, pstar * p.PE, piece_n(pstar),
                              s_seg);
            pc_loaded = pstar;
        }
        if (warp == 0) {
            const int e = select_in_piece<T>(wr, s_seg, tb, nullptr, staged_bytes(pstar) / 16, vec_ok, pstar * p.PE,
                                             piece_n(pstar), target);
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
        if (tid == 0) out[r.j] = tok;
    } else if (warp == 0) {
        report_lost();
    }
    drain();
}

}  // namespace sv
