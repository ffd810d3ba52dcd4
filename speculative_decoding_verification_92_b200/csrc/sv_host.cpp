// sv_host.cpp -- host-side components declared in include/sv_host.h: the
// per-prompt n-gram drafter, the suffix drafter with frequency scoring, the
// fan-out prefetch budget, the draft-length controller, the speculation
// switch and the length-aware budgets.  Plain C++17 on host memory; nothing
// here touches a GPU.  The rules each function follows are stated in the
// header, with the page and section they come from.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <deque>
#include <limits>
#include <new>
#include <numeric>
#include <thread>
#include <unordered_map>
#include <utility>
#include <vector>

#include "spec_verify.h"
#include "sv_host.h"

namespace {

// 64-bit FNV-1a over a run of token ids (n-gram / context keys; every hit is
// confirmed by comparing the tokens, so collisions cost time, never results).
uint64_t hash_tokens(const int32_t* t, int64_t n) {
    uint64_t h = 1469598103934665603ull ^ static_cast<uint64_t>(n);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t v = static_cast<uint32_t>(t[i]);
        for (int b = 0; b < 4; ++b) {
            h ^= (v >> (8 * b)) & 0xffu;
            h *= 1099511628211ull;
        }
    }
    return h;
}

}  // namespace

// ===========================================================================
// Per-prompt n-gram drafter.
//
// One index per prompt maps every n-gram (n = 1..max_n) of its retained
// rollouts to its occurrences, each stored as (rollout sequence number,
// continuation start) in 8 bytes.  Rollouts get consecutive sequence numbers
// in the order they are added, so every occurrence list is sorted oldest
// first and the most recent occurrence is found from its back; a lookup costs
// one hash probe per n whatever the number of rollouts.  Evicting a step's
// rollouts cuts the same prefix off every list.

struct sv_ngram {
    struct Rollout {
        int64_t step;
        std::vector<int32_t> tok;
    };
    struct Occ {
        int32_t seq;  // rollout sequence number within the prompt
        int32_t p;    // continuation start: the n-gram is tok[p-n .. p), tok[p] exists
    };
    struct Prompt {
        std::deque<Rollout> rollouts;  // oldest first; rollouts[i] has sequence number first_seq + i
        int32_t first_seq = 0;
        std::unordered_map<uint64_t, std::vector<Occ>> index;  // n-gram key -> occurrences, oldest first
        const Rollout& rollout(int32_t seq) const { return rollouts[static_cast<size_t>(seq - first_seq)]; }
    };
    int32_t max_n = 6;
    int32_t window = 4;
    int64_t step = 0;
    bool started = false;
    std::unordered_map<int64_t, Prompt> prompts;
};

namespace {

struct Occurrence {
    const sv_ngram::Rollout* r = nullptr;
    int64_t p = -1;  // continuation start
};

// Whether occurrence q of the list under key's hash really is the n-gram
// key[0..n) (a hash collision, with another n-gram or another n, is not).
bool occ_matches(const sv_ngram::Prompt& pr, const sv_ngram::Occ& q, const int32_t* key, int32_t n) {
    if (q.p < n) return false;
    const sv_ngram::Rollout& r = pr.rollout(q.seq);
    return std::memcmp(r.tok.data() + q.p - n, key, sizeof(int32_t) * n) == 0;
}

// Longest n whose last n context tokens occur followed by a token; fills the
// most recent occurrence (latest step, then latest rollout, then latest
// position: the back of the sorted list).
int32_t longest_match(const sv_ngram& t, const sv_ngram::Prompt& pr, const int32_t* ctx, int64_t n_ctx,
                      Occurrence* occ) {
    const int32_t top = static_cast<int32_t>(std::min<int64_t>(t.max_n, n_ctx));
    for (int32_t n = top; n >= 1; --n) {
        const int32_t* key = ctx + n_ctx - n;
        auto it = pr.index.find(hash_tokens(key, n));
        if (it == pr.index.end()) continue;
        const std::vector<sv_ngram::Occ>& v = it->second;
        for (auto q = v.rbegin(); q != v.rend(); ++q)
            if (occ_matches(pr, *q, key, n)) {
                occ->r = &pr.rollout(q->seq);
                occ->p = q->p;
                return n;
            }
    }
    return 0;
}

}  // namespace

extern "C" {

sv_ngram* sv_ngram_create(int32_t max_n, int32_t window) {
    if (max_n < 1 || max_n > 16 || window < 1) return nullptr;
    sv_ngram* t = new (std::nothrow) sv_ngram;
    if (!t) return nullptr;
    t->max_n = max_n;
    t->window = window;
    return t;
}

void sv_ngram_destroy(sv_ngram* t) { delete t; }

void sv_ngram_begin_step(sv_ngram* t) {
    if (!t) return;
    if (t->started) ++t->step;
    t->started = true;
    for (auto it = t->prompts.begin(); it != t->prompts.end();) {
        sv_ngram::Prompt& pr = it->second;
        const int32_t before = pr.first_seq;
        while (!pr.rollouts.empty() && pr.rollouts.front().step <= t->step - t->window) {
            pr.rollouts.pop_front();
            ++pr.first_seq;
        }
        if (pr.rollouts.empty()) {
            it = t->prompts.erase(it);
            continue;
        }
        if (pr.first_seq != before) {
            // the evicted rollouts are the oldest: a prefix of every list
            for (auto e = pr.index.begin(); e != pr.index.end();) {
                std::vector<sv_ngram::Occ>& v = e->second;
                auto keep = std::lower_bound(v.begin(), v.end(), pr.first_seq,
                                             [](const sv_ngram::Occ& q, int32_t s) { return q.seq < s; });
                v.erase(v.begin(), keep);
                if (v.empty()) e = pr.index.erase(e);
                else ++e;
            }
        }
        ++it;
    }
}

int32_t sv_ngram_add(sv_ngram* t, int64_t prompt_id, const int32_t* tokens, int64_t n) {
    if (!t || n < 0 || (n > 0 && !tokens) || n > std::numeric_limits<int32_t>::max()) return -1;
    if (!t->started) sv_ngram_begin_step(t);
    try {
        sv_ngram::Prompt& pr = t->prompts[prompt_id];
        if (pr.first_seq + static_cast<int64_t>(pr.rollouts.size()) >= std::numeric_limits<int32_t>::max())
            return -1;
        const int32_t seq = pr.first_seq + static_cast<int32_t>(pr.rollouts.size());
        pr.rollouts.push_back(sv_ngram::Rollout{t->step, std::vector<int32_t>(tokens, tokens + n)});
        // n-grams that some token follows: continuation starts p = 1 .. n-1
        for (int64_t p = 1; p < n; ++p)
            for (int32_t k = 1; k <= t->max_n && k <= p; ++k)
                pr.index[hash_tokens(tokens + p - k, k)].push_back({seq, static_cast<int32_t>(p)});
        return 0;
    } catch (...) {
        return -1;
    }
}

int32_t sv_ngram_draft(const sv_ngram* t, int64_t prompt_id, const int32_t* context, int64_t n, int32_t k,
                       int32_t* out) {
    if (!t || n < 0 || (n > 0 && !context) || k < 0 || (k > 0 && !out)) return -1;
    auto it = t->prompts.find(prompt_id);
    if (it == t->prompts.end() || n == 0 || k == 0) return 0;
    Occurrence occ;
    if (longest_match(*t, it->second, context, n, &occ) == 0) return 0;
    const int64_t avail = static_cast<int64_t>(occ.r->tok.size()) - occ.p;
    const int32_t m = static_cast<int32_t>(std::min<int64_t>(k, avail));
    std::memcpy(out, occ.r->tok.data() + occ.p, sizeof(int32_t) * m);
    return m;
}

int32_t sv_ngram_candidates(const sv_ngram* t, int64_t prompt_id, const int32_t* context, int64_t n, int32_t f,
                            int32_t* out) {
    if (!t || n < 0 || (n > 0 && !context) || f < 0 || (f > 0 && !out)) return -1;
    auto it = t->prompts.find(prompt_id);
    if (it == t->prompts.end() || n == 0 || f == 0) return 0;
    const sv_ngram::Prompt& pr = it->second;
    Occurrence occ;
    const int32_t nm = longest_match(*t, pr, context, n, &occ);
    if (nm == 0) return 0;
    // every occurrence of the matched n-gram, newest first: count followers
    // and remember the order of their most recent occurrence
    const int32_t* key = context + n - nm;
    struct Cand { int32_t tok; int64_t count; int64_t first_seen; };
    try {
        std::vector<Cand> cands;
        std::unordered_map<int32_t, size_t> slot;
        int64_t order = 0;
        const std::vector<sv_ngram::Occ>& v = pr.index.find(hash_tokens(key, nm))->second;
        for (auto q = v.rbegin(); q != v.rend(); ++q) {
            if (!occ_matches(pr, *q, key, nm)) continue;
            const int32_t nxt = pr.rollout(q->seq).tok[static_cast<size_t>(q->p)];
            auto s = slot.find(nxt);
            if (s == slot.end()) {
                slot.emplace(nxt, cands.size());
                cands.push_back({nxt, 1, order});
            } else {
                ++cands[s->second].count;
            }
            ++order;
        }
        std::stable_sort(cands.begin(), cands.end(), [](const Cand& a, const Cand& b) {
            return a.count != b.count ? a.count > b.count : a.first_seen < b.first_seen;
        });
        const int32_t m = static_cast<int32_t>(std::min<size_t>(f, cands.size()));
        for (int32_t i = 0; i < m; ++i) out[i] = cands[i].tok;
        return m;
    } catch (...) {
        return -1;
    }
}

int64_t sv_ngram_rollouts(const sv_ngram* t) {
    if (!t) return -1;
    int64_t n = 0;
    for (const auto& kv : t->prompts) n += static_cast<int64_t>(kv.second.rollouts.size());
    return n;
}

int64_t sv_ngram_tokens(const sv_ngram* t) {
    if (!t) return -1;
    int64_t n = 0;
    for (const auto& kv : t->prompts)
        for (const auto& r : kv.second.rollouts) n += static_cast<int64_t>(r.tok.size());
    return n;
}

}  // extern "C"

// ===========================================================================
// Suffix drafter with frequency scoring.
//
// Every distinct context (the d <= max_depth tokens before some position of a
// trajectory) is one 32-byte entry that points at its first occurrence in a
// trajectory instead of copying it, and keeps its first follower inline; the
// rare further followers go to a side list.  A hash of the context selects a
// chain of entries; a context is confirmed by comparing its tokens.

struct sv_suffix {
    struct Entry {
        int32_t traj;   // trajectory holding the context's first occurrence
        int32_t end;    // the context is that trajectory's tokens [end - d, end)
        int32_t d;
        int32_t chain;  // next entry under the same hash, or -1
        int64_t cnt0;   // count of the first follower seen
        int32_t tok0;   // that follower
        int32_t more;   // index of the list of further followers, or -1
    };
    struct Problem {
        std::unordered_map<int64_t, int32_t> slot;                    // seq_id -> trajectory index
        std::vector<std::vector<int32_t>> trajs;
        std::unordered_map<uint64_t, int32_t> head;                   // context hash -> first entry
        std::vector<Entry> entries;
        std::vector<std::vector<std::pair<int32_t, int64_t>>> extra;  // followers beyond the first
    };
    int32_t max_depth = 8;
    std::unordered_map<int64_t, Problem> problems;
};

namespace {

const sv_suffix::Entry* find_context(const sv_suffix::Problem& pb, const int32_t* c, int32_t d) {
    auto it = pb.head.find(hash_tokens(c, d));
    if (it == pb.head.end()) return nullptr;
    for (int32_t i = it->second; i >= 0; i = pb.entries[static_cast<size_t>(i)].chain) {
        const sv_suffix::Entry& e = pb.entries[static_cast<size_t>(i)];
        if (e.d == d &&
            std::memcmp(pb.trajs[static_cast<size_t>(e.traj)].data() + e.end - d, c, sizeof(int32_t) * d) == 0)
            return &e;
    }
    return nullptr;
}

// Longest d <= max_depth with a count table for the last d tokens of c[0..n).
const sv_suffix::Entry* longest_context(const sv_suffix& t, const sv_suffix::Problem& pb, const int32_t* c,
                                        int64_t n) {
    const int32_t top = static_cast<int32_t>(std::min<int64_t>(t.max_depth, n));
    for (int32_t d = top; d >= 1; --d) {
        const sv_suffix::Entry* e = find_context(pb, c + n - d, d);
        if (e) return e;
    }
    return nullptr;
}

// Every follower of e with its count, in no particular order.
std::vector<std::pair<int32_t, int64_t>> followers(const sv_suffix::Problem& pb, const sv_suffix::Entry& e) {
    std::vector<std::pair<int32_t, int64_t>> c{{e.tok0, e.cnt0}};
    if (e.more >= 0) {
        const auto& x = pb.extra[static_cast<size_t>(e.more)];
        c.insert(c.end(), x.begin(), x.end());
    }
    return c;
}

// Most frequent follower, ties to the lowest id.
int32_t top_follower(const sv_suffix::Problem& pb, const sv_suffix::Entry& e) {
    int32_t best = e.tok0;
    int64_t best_n = e.cnt0;
    if (e.more >= 0)
        for (const auto& kv : pb.extra[static_cast<size_t>(e.more)])
            if (kv.second > best_n || (kv.second == best_n && kv.first < best)) {
                best = kv.first;
                best_n = kv.second;
            }
    return best;
}

}  // namespace

extern "C" {

sv_suffix* sv_suffix_create(int32_t max_depth) {
    if (max_depth < 1 || max_depth > 64) return nullptr;
    sv_suffix* t = new (std::nothrow) sv_suffix;
    if (!t) return nullptr;
    t->max_depth = max_depth;
    return t;
}

void sv_suffix_destroy(sv_suffix* t) { delete t; }

void sv_suffix_clear(sv_suffix* t) {
    if (t) t->problems.clear();
}

int32_t sv_suffix_append(sv_suffix* t, int64_t problem_id, int64_t seq_id, const int32_t* tokens, int64_t m) {
    if (!t || m < 0 || (m > 0 && !tokens)) return -1;
    try {
        sv_suffix::Problem& pb = t->problems[problem_id];
        auto sl = pb.slot.find(seq_id);
        if (sl == pb.slot.end()) {
            if (pb.trajs.size() >= static_cast<size_t>(std::numeric_limits<int32_t>::max())) return -1;
            sl = pb.slot.emplace(seq_id, static_cast<int32_t>(pb.trajs.size())).first;
            pb.trajs.emplace_back();
        }
        const int32_t ti = sl->second;
        std::vector<int32_t>& seq = pb.trajs[static_cast<size_t>(ti)];
        if (static_cast<int64_t>(seq.size()) + m > std::numeric_limits<int32_t>::max()) return -1;
        for (int64_t i = 0; i < m; ++i) {
            const int32_t tok = tokens[i];
            const int32_t n = static_cast<int32_t>(seq.size());
            for (int32_t d = 1; d <= t->max_depth && d <= n; ++d) {
                const int32_t* c = seq.data() + n - d;
                const sv_suffix::Entry* found = find_context(pb, c, d);
                if (!found) {
                    if (pb.entries.size() >= static_cast<size_t>(std::numeric_limits<int32_t>::max())) return -1;
                    const int32_t idx = static_cast<int32_t>(pb.entries.size());
                    int32_t& h = pb.head.try_emplace(hash_tokens(c, d), -1).first->second;
                    pb.entries.push_back(sv_suffix::Entry{ti, n, d, h, 1, tok, -1});
                    h = idx;
                    continue;
                }
                sv_suffix::Entry& e = pb.entries[static_cast<size_t>(found - pb.entries.data())];
                if (e.tok0 == tok) {
                    ++e.cnt0;
                    continue;
                }
                if (e.more < 0) {
                    e.more = static_cast<int32_t>(pb.extra.size());
                    pb.extra.emplace_back();
                }
                auto& x = pb.extra[static_cast<size_t>(e.more)];
                auto f = std::find_if(x.begin(), x.end(), [tok](const auto& kv) { return kv.first == tok; });
                if (f == x.end()) x.emplace_back(tok, 1);
                else ++f->second;
            }
            seq.push_back(tok);
        }
        return 0;
    } catch (...) {
        return -1;
    }
}

int32_t sv_suffix_draft(const sv_suffix* t, int64_t problem_id, const int32_t* context, int64_t n, int32_t k,
                        int32_t* out) {
    if (!t || n < 0 || (n > 0 && !context) || k < 0 || (k > 0 && !out)) return -1;
    auto it = t->problems.find(problem_id);
    if (it == t->problems.end() || k == 0) return 0;
    try {
        // the draft extends the context: keep the last max_depth tokens of both
        std::vector<int32_t> ctx(context + std::max<int64_t>(0, n - t->max_depth), context + n);
        int32_t m = 0;
        while (m < k) {
            const sv_suffix::Entry* e =
                longest_context(*t, it->second, ctx.data(), static_cast<int64_t>(ctx.size()));
            if (!e) break;
            const int32_t tok = top_follower(it->second, *e);
            out[m++] = tok;
            ctx.push_back(tok);
            if (static_cast<int32_t>(ctx.size()) > t->max_depth) ctx.erase(ctx.begin());
        }
        return m;
    } catch (...) {
        return -1;
    }
}

int32_t sv_suffix_candidates(const sv_suffix* t, int64_t problem_id, const int32_t* context, int64_t n, int32_t f,
                             int32_t* out) {
    if (!t || n < 0 || (n > 0 && !context) || f < 0 || (f > 0 && !out)) return -1;
    auto it = t->problems.find(problem_id);
    if (it == t->problems.end() || f == 0) return 0;
    const sv_suffix::Entry* e = longest_context(*t, it->second, context, n);
    if (!e) return 0;
    try {
        std::vector<std::pair<int32_t, int64_t>> c = followers(it->second, *e);
        std::sort(c.begin(), c.end(), [](const auto& a, const auto& b) {
            return a.second != b.second ? a.second > b.second : a.first < b.first;
        });
        const int32_t m = static_cast<int32_t>(std::min<size_t>(f, c.size()));
        for (int32_t i = 0; i < m; ++i) out[i] = c[i].first;
        return m;
    } catch (...) {
        return -1;
    }
}

}  // extern "C"

// ===========================================================================
// Batched drafting into spec_verify's drafted-id and length arrays.

namespace {

// Below this many requests per thread, starting a thread costs more than the
// lookups it takes over (a lookup takes ~0.1-0.2 us, a thread start tens of
// microseconds).
constexpr int32_t kMinRequestsPerThread = 512;

bool batch_args_ok(const void* t, int32_t B, const int64_t* ids, const int32_t* ctx, const int64_t* ctx_off,
                   int32_t k_max, const int32_t* max_lens, int32_t n_threads, const int32_t* out_tokens,
                   const int32_t* out_lens) {
    if (!t || B < 0 || k_max < 0 || k_max > SV_MAX_K || n_threads < 0) return false;
    if (B == 0) return true;
    if (!ids || !ctx_off || !out_lens || (k_max > 0 && !out_tokens)) return false;
    if (ctx_off[0] < 0) return false;
    for (int32_t b = 0; b < B; ++b) {
        if (ctx_off[b + 1] < ctx_off[b]) return false;
        if (max_lens && max_lens[b] < 0) return false;
    }
    return ctx || ctx_off[B] == ctx_off[0];
}

// Fill row b of out_tokens / out_lens with draft_one(b, cap, row) for every
// b, on up to n_threads threads over contiguous blocks of requests.  A thread
// that cannot be started leaves its block to the calling thread, so the
// result never depends on the thread count.
template <typename DraftOne>
void draft_batch(int32_t B, int32_t k_max, const int32_t* max_lens, int32_t n_threads, int32_t* out_tokens,
                 int32_t* out_lens, const DraftOne& draft_one) {
    auto run = [&](int32_t lo, int32_t hi) {
        for (int32_t b = lo; b < hi; ++b) {
            int32_t* row = out_tokens ? out_tokens + static_cast<int64_t>(b) * k_max : nullptr;
            const int32_t cap = max_lens ? std::min(k_max, max_lens[b]) : k_max;
            int32_t m = cap > 0 ? draft_one(b, cap, row) : 0;
            m = std::max(m, 0);
            for (int32_t i = m; i < k_max; ++i) row[i] = -1;
            out_lens[b] = m;
        }
    };
    int32_t nt = n_threads;
    if (nt == 0) nt = static_cast<int32_t>(std::max(1u, std::thread::hardware_concurrency()));
    nt = std::max<int32_t>(1, std::min<int32_t>(nt, B / kMinRequestsPerThread));
    auto block = [&](int32_t i) { return static_cast<int32_t>(static_cast<int64_t>(B) * i / nt); };
    std::vector<std::thread> pool;
    std::vector<std::pair<int32_t, int32_t>> left;  // blocks whose thread did not start
    for (int32_t i = 1; i < nt; ++i) {
        try {
            pool.emplace_back(run, block(i), block(i + 1));
        } catch (...) {
            try {
                left.emplace_back(block(i), block(i + 1));
            } catch (...) {
                run(block(i), block(i + 1));
            }
        }
    }
    run(0, block(1));
    for (const auto& r : left) run(r.first, r.second);
    for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

int32_t sv_ngram_draft_batch(const sv_ngram* t, int32_t B, const int64_t* ids, const int32_t* ctx,
                             const int64_t* ctx_off, int32_t k_max, const int32_t* max_lens, int32_t n_threads,
                             int32_t* out_tokens, int32_t* out_lens) {
    if (!batch_args_ok(t, B, ids, ctx, ctx_off, k_max, max_lens, n_threads, out_tokens, out_lens)) return -1;
    draft_batch(B, k_max, max_lens, n_threads, out_tokens, out_lens, [&](int32_t b, int32_t cap, int32_t* row) {
        const int64_t n = ctx_off[b + 1] - ctx_off[b];
        return sv_ngram_draft(t, ids[b], n > 0 ? ctx + ctx_off[b] : nullptr, n, cap, row);
    });
    return 0;
}

int32_t sv_suffix_draft_batch(const sv_suffix* t, int32_t B, const int64_t* ids, const int32_t* ctx,
                              const int64_t* ctx_off, int32_t k_max, const int32_t* max_lens, int32_t n_threads,
                              int32_t* out_tokens, int32_t* out_lens) {
    if (!batch_args_ok(t, B, ids, ctx, ctx_off, k_max, max_lens, n_threads, out_tokens, out_lens)) return -1;
    draft_batch(B, k_max, max_lens, n_threads, out_tokens, out_lens, [&](int32_t b, int32_t cap, int32_t* row) {
        const int64_t n = ctx_off[b + 1] - ctx_off[b];
        return sv_suffix_draft(t, ids[b], n > 0 ? ctx + ctx_off[b] : nullptr, n, cap, row);
    });
    return 0;
}

}  // extern "C"

// ===========================================================================
// Fan-out prefetch budget.

struct sv_prefetch {
    int32_t k = 0, fmax = 1, window = 1;
    std::deque<std::pair<int32_t, int32_t>> obs;  // (j, rank), oldest first
};

namespace {

// P(j) and c_j(f) over the window; returns the observation count.
int32_t estimates(const sv_prefetch& p, std::vector<double>* P, std::vector<double>* cov) {
    const int32_t K1 = p.k + 1, F1 = p.fmax + 1;
    P->assign(K1, 0.0);
    cov->assign(size_t(K1) * F1, 0.0);
    const int32_t n = static_cast<int32_t>(p.obs.size());
    if (n == 0) return 0;
    std::vector<int64_t> cnt(K1, 0), hits(size_t(K1) * F1, 0), pooled(F1, 0);
    for (const auto& o : p.obs) {
        ++cnt[o.first];
        for (int32_t f = 1; f <= p.fmax; ++f)
            if (o.second >= 0 && o.second < f) {
                ++hits[size_t(o.first) * F1 + f];
                ++pooled[f];
            }
    }
    for (int32_t j = 0; j < K1; ++j) {
        (*P)[j] = double(cnt[j]) / n;
        for (int32_t f = 1; f <= p.fmax; ++f)
            (*cov)[size_t(j) * F1 + f] = cnt[j] ? double(hits[size_t(j) * F1 + f]) / cnt[j] : double(pooled[f]) / n;
    }
    return n;
}

}  // namespace

extern "C" {

sv_prefetch* sv_prefetch_create(int32_t k, int32_t fmax, int32_t window) {
    if (k < 0 || fmax < 1 || window < 1) return nullptr;
    sv_prefetch* p = new (std::nothrow) sv_prefetch;
    if (!p) return nullptr;
    p->k = k;
    p->fmax = fmax;
    p->window = window;
    return p;
}

void sv_prefetch_destroy(sv_prefetch* p) { delete p; }

int32_t sv_prefetch_observe(sv_prefetch* p, int32_t j, int32_t b_rank) {
    if (!p || j < 0 || j > p->k || b_rank < -1) return -1;
    p->obs.emplace_back(j, b_rank >= p->fmax ? -1 : b_rank);
    while (static_cast<int32_t>(p->obs.size()) > p->window) p->obs.pop_front();
    return 0;
}

int32_t sv_prefetch_estimates(const sv_prefetch* p, double* P_j, double* coverage) {
    if (!p) return -1;
    std::vector<double> P, cov;
    const int32_t n = estimates(*p, &P, &cov);
    if (P_j) std::copy(P.begin(), P.end(), P_j);
    if (coverage) std::copy(cov.begin(), cov.end(), coverage);
    return n;
}

double sv_prefetch_allocate(const sv_prefetch* p, int32_t budget, int32_t* out_f) {
    if (!p || !out_f) return -1.0;
    const int32_t K1 = p->k + 1, F1 = p->fmax + 1;
    std::fill(out_f, out_f + K1, 0);
    std::vector<double> P, cov;
    if (estimates(*p, &P, &cov) == 0) return 0.0;
    double total = 0.0;
    for (int32_t spent = 0; spent < budget; ++spent) {
        int32_t best = -1;
        double best_gain = 0.0;
        for (int32_t j = 0; j < K1; ++j) {
            if (out_f[j] >= p->fmax) continue;
            const double g = P[j] * (cov[size_t(j) * F1 + out_f[j] + 1] - cov[size_t(j) * F1 + out_f[j]]);
            if (g > best_gain) {  // strict: ties keep the lower j
                best_gain = g;
                best = j;
            }
        }
        if (best < 0) break;
        ++out_f[best];
        total += best_gain;
    }
    return total;
}

// ---------------------------------------------------------------------------
// Fan-out prefetch of the next draft: for every covered outcome (j, b), the
// draft that follows context + d[0..j) + b, computed ahead of the outcome.

int32_t sv_ngram_prefetch(const sv_ngram* t, int64_t prompt_id, const int32_t* context, int64_t n,
                          const int32_t* draft, int32_t L, const int32_t* f, int32_t k, int32_t max_entries,
                          int32_t* out_j, int32_t* out_b, int32_t* out_tokens, int32_t* out_lens) {
    if (!t || n < 0 || (n > 0 && !context) || L < 0 || L > SV_MAX_K || (L > 0 && !draft) || !f || k < 0 ||
        k > SV_MAX_K || max_entries < 0)
        return -1;
    for (int32_t j = 0; j <= L; ++j)
        if (f[j] < 0) return -1;
    if (max_entries > 0 && (!out_j || !out_b || !out_lens || (k > 0 && !out_tokens))) return -1;
    try {
        std::vector<int32_t> ctx;  // context + d[0..j), then + b while drafting
        ctx.reserve(static_cast<size_t>(n) + L + 1);
        ctx.assign(context, context + n);
        std::vector<int32_t> cand;
        int32_t e = 0;
        for (int32_t j = 0; j <= L && e < max_entries; ++j) {
            if (j > 0) ctx.push_back(draft[j - 1]);
            const int32_t want = std::min(f[j], max_entries - e);
            if (want == 0) continue;
            cand.resize(static_cast<size_t>(want));
            const int32_t nc = sv_ngram_candidates(t, prompt_id, ctx.data(), static_cast<int64_t>(ctx.size()), want,
                                                   cand.data());
            for (int32_t r = 0; r < nc; ++r, ++e) {
                ctx.push_back(cand[r]);
                int32_t* row = k > 0 ? out_tokens + static_cast<int64_t>(e) * k : nullptr;
                int32_t m = k > 0 ? sv_ngram_draft(t, prompt_id, ctx.data(), static_cast<int64_t>(ctx.size()), k, row)
                                  : 0;
                m = std::max(m, 0);
                for (int32_t i = m; i < k; ++i) row[i] = -1;
                ctx.pop_back();
                out_j[e] = j;
                out_b[e] = cand[r];
                out_lens[e] = m;
            }
        }
        return e;
    } catch (...) {  // allocation failure: nothing may cross the C boundary
        return -1;
    }
}

int32_t sv_prefetch_find(const int32_t* out_j, const int32_t* out_b, int32_t count, int32_t j, int32_t b) {
    if (!out_j || !out_b) return -1;
    for (int32_t e = 0; e < count; ++e)
        if (out_j[e] == j && out_b[e] == b) return e;
    return -1;
}

// ===========================================================================
// Draft-length controller, block efficiency, speculation switch.

}  // extern "C"

struct sv_draft_len {
    std::vector<int32_t> lengths;
    double up = 0.7, down = 0.4;
    int32_t patience = 2;
    int32_t idx = 0, up_run = 0, down_run = 0;
};

extern "C" {

sv_draft_len* sv_draft_len_create(const int32_t* lengths, int32_t n_lengths, double up_frac, double down_frac,
                                  int32_t patience) {
    if (!lengths || n_lengths < 1 || n_lengths > 64 || patience < 1) return nullptr;
    if (!(down_frac >= 0.0 && down_frac <= up_frac && up_frac <= 1.0)) return nullptr;
    for (int32_t i = 0; i < n_lengths; ++i)
        if (lengths[i] < 1 || (i > 0 && lengths[i] <= lengths[i - 1])) return nullptr;
    sv_draft_len* c = new (std::nothrow) sv_draft_len;
    if (!c) return nullptr;
    c->lengths.assign(lengths, lengths + n_lengths);
    c->up = up_frac;
    c->down = down_frac;
    c->patience = patience;
    return c;
}

void sv_draft_len_destroy(sv_draft_len* c) { delete c; }

int32_t sv_draft_len_current(const sv_draft_len* c) { return c ? c->lengths[c->idx] : -1; }

int32_t sv_draft_len_update(sv_draft_len* c, double tau) {
    if (!c) return -1;
    const double r = tau / double(c->lengths[c->idx] + 1);
    // NaN (no valid request this step) extends neither streak
    c->up_run = r >= c->up ? c->up_run + 1 : 0;
    c->down_run = r < c->down ? c->down_run + 1 : 0;
    if (c->up_run >= c->patience && c->idx + 1 < static_cast<int32_t>(c->lengths.size())) {
        ++c->idx;
        c->up_run = c->down_run = 0;
    } else if (c->down_run >= c->patience && c->idx > 0) {
        --c->idx;
        c->up_run = c->down_run = 0;
    }
    return c->lengths[c->idx];
}

double sv_block_efficiency(const int32_t* accept_len, int64_t n) {
    if (!accept_len || n <= 0) return std::numeric_limits<double>::quiet_NaN();
    double s = 0.0;
    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i)
        if (accept_len[i] >= 0) {
            s += double(accept_len[i]) + 1.0;
            ++m;
        }
    return m ? s / double(m) : std::numeric_limits<double>::quiet_NaN();
}

int32_t sv_spec_switch(int32_t* state, double predicted_speedup, double threshold) {
    if (!state) return -1;
    if (*state == 0 && predicted_speedup > threshold) *state = 1;
    return *state != 0 ? 1 : 0;
}

// ===========================================================================
// Length-aware budgets.

}  // extern "C"

namespace {

std::vector<int64_t> longest_first(const double* len, int64_t n) {
    std::vector<int64_t> order(static_cast<size_t>(n));
    std::iota(order.begin(), order.end(), int64_t(0));
    std::stable_sort(order.begin(), order.end(), [len](int64_t a, int64_t b) { return len[a] > len[b]; });
    return order;
}

}  // namespace

extern "C" {

int32_t sv_length_classes(const double* predicted_len, int64_t n, const int32_t budgets[3], int32_t* out_class,
                          int32_t* out_budget) {
    if (n < 0 || (n > 0 && (!predicted_len || !budgets || !out_class || !out_budget))) return -1;
    for (int64_t i = 0; i < n; ++i)
        if (std::isnan(predicted_len[i])) return -1;
    const std::vector<int64_t> order = longest_first(predicted_len, n);
    const int64_t third = n / 3;
    for (int64_t r = 0; r < n; ++r) {
        const int64_t i = order[static_cast<size_t>(r)];
        const int32_t cls = r < third ? 2 : (r >= n - third ? 0 : 1);
        out_class[i] = cls;
        out_budget[i] = budgets[cls];
    }
    return 0;
}

int32_t sv_interleave_ranks(const double* predicted_len, int64_t n, int32_t world_size, int32_t* out_rank) {
    if (n < 0 || world_size < 1 || (n > 0 && (!predicted_len || !out_rank))) return -1;
    for (int64_t i = 0; i < n; ++i)
        if (std::isnan(predicted_len[i])) return -1;
    const std::vector<int64_t> order = longest_first(predicted_len, n);
    for (int64_t r = 0; r < n; ++r) out_rank[order[static_cast<size_t>(r)]] = static_cast<int32_t>(r % world_size);
    return 0;
}

}  // extern "C"

// ===========================================================================
// Roofline predictor behind the switch.

namespace {

bool arch_ok(const sv_arch* a) {
    return a && std::isfinite(a->params) && a->params > 0.0 && std::isfinite(a->weight_bytes) &&
           a->weight_bytes > 0.0 && a->layers > 0 && a->width > 0 && a->kv_heads > 0 && a->head_dim > 0 &&
           std::isfinite(a->kv_bytes) && a->kv_bytes > 0.0;
}

bool roofline_ok(const sv_roofline* r) {
    return r && std::isfinite(r->flops_per_s) && r->flops_per_s > 0.0 && std::isfinite(r->bytes_per_s) &&
           r->bytes_per_s > 0.0 && std::isfinite(r->overhead_s) && r->overhead_s >= 0.0;
}

bool count_ok(double x) { return std::isfinite(x) && x >= 0.0; }

void step_work(const sv_arch& a, double B, double q, double n, double* flops, double* bytes) {
    *flops = 2.0 * a.params * B * q + 4.0 * a.layers * static_cast<double>(a.width) * B * q * n;
    *bytes = a.params * a.weight_bytes +
             2.0 * a.layers * static_cast<double>(a.kv_heads) * a.head_dim * a.kv_bytes * B * n;
}

double step_time(const sv_roofline& r, double flops, double bytes) {
    return std::max(flops / r.flops_per_s, bytes / r.bytes_per_s) + r.overhead_s;
}

// Sum of squared relative errors of the fit (pi, beta) with its best tau >= 0,
// which is written to *tau: d/dtau sum ((m_i + tau - t_i) / t_i)^2 = 0 gives
// tau = sum (t_i - m_i) / t_i^2 / sum 1 / t_i^2, clipped at 0 (the error is a
// parabola in tau, so the clip is the constrained optimum).
double fit_error(const std::vector<double>& F, const std::vector<double>& M, const double* t, double pi,
                 double beta, double* tau) {
    double num = 0.0, den = 0.0;
    for (size_t i = 0; i < F.size(); ++i) {
        const double m = std::max(F[i] / pi, M[i] / beta);
        const double w = 1.0 / (t[i] * t[i]);
        num += (t[i] - m) * w;
        den += w;
    }
    const double tt = std::max(0.0, num / den);
    double e = 0.0;
    for (size_t i = 0; i < F.size(); ++i) {
        const double d = (std::max(F[i] / pi, M[i] / beta) + tt - t[i]) / t[i];
        e += d * d;
    }
    *tau = tt;
    return e;
}

}  // namespace

extern "C" {

int32_t sv_roofline_work(const sv_arch* a, double B, double q, double n, double* flops, double* bytes) {
    if (!arch_ok(a) || !count_ok(B) || !count_ok(q) || !count_ok(n) || !flops || !bytes) return -1;
    step_work(*a, B, q, n, flops, bytes);
    return 0;
}

double sv_roofline_time(const sv_arch* a, const sv_roofline* r, double B, double q, double n) {
    if (!arch_ok(a) || !roofline_ok(r) || !count_ok(B) || !count_ok(q) || !count_ok(n))
        return std::numeric_limits<double>::quiet_NaN();
    double F, M;
    step_work(*a, B, q, n, &F, &M);
    return step_time(*r, F, M);
}

int32_t sv_roofline_fit(const sv_arch* a, int32_t m, const double* B, const double* q, const double* n,
                        const double* seconds, sv_roofline* out, double* rms_rel) {
    if (!arch_ok(a) || m < 3 || !B || !q || !n || !seconds || !out) return -1;
    try {
        std::vector<double> F(static_cast<size_t>(m)), M(static_cast<size_t>(m));
        double f_rate = 0.0, m_rate = 0.0;  // the largest flops and bytes per measured second
        for (int32_t i = 0; i < m; ++i) {
            if (!count_ok(B[i]) || !count_ok(q[i]) || !count_ok(n[i]) || !std::isfinite(seconds[i]) ||
                !(seconds[i] > 0.0))
                return -1;
            step_work(*a, B[i], q[i], n[i], &F[i], &M[i]);
            f_rate = std::max(f_rate, F[i] / seconds[i]);
            m_rate = std::max(m_rate, M[i] / seconds[i]);
        }
        if (!(f_rate > 0.0) || !(m_rate > 0.0)) return -1;
        // log10 grids: each rate lies at or above the fastest the data shows,
        // so start from a decade below it to three above, 41 x 41 points;
        // then re-grid +-2 steps around the best point, seven times
        constexpr int kGrid = 41;
        double lp0 = std::log10(f_rate) - 1.0, lb0 = std::log10(m_rate) - 1.0;
        double step = 4.0 / (kGrid - 1);
        double best_e = std::numeric_limits<double>::infinity(), best_lp = lp0, best_lb = lb0, best_tau = 0.0;
        for (int round = 0; round < 8; ++round) {
            const double cp = best_lp, cb = best_lb;
            for (int i = 0; i < kGrid; ++i)
                for (int j = 0; j < kGrid; ++j) {
                    const double lp = round == 0 ? lp0 + i * step : cp + (i - kGrid / 2) * step;
                    const double lb = round == 0 ? lb0 + j * step : cb + (j - kGrid / 2) * step;
                    double tau;
                    const double e = fit_error(F, M, seconds, std::pow(10.0, lp), std::pow(10.0, lb), &tau);
                    if (e < best_e) {
                        best_e = e;
                        best_lp = lp;
                        best_lb = lb;
                        best_tau = tau;
                    }
                }
            step = 4.0 * step / (kGrid - 1);  // the next grid spans +-2 steps of this one
        }
        out->flops_per_s = std::pow(10.0, best_lp);
        out->bytes_per_s = std::pow(10.0, best_lb);
        out->overhead_s = best_tau;
        if (rms_rel) *rms_rel = std::sqrt(best_e / m);
        return 0;
    } catch (...) {
        return -1;
    }
}

double sv_spec_speedup(const sv_arch* target, const sv_roofline* rt, const sv_arch* draft, const sv_roofline* rd,
                       double B, int32_t k, double alpha, double n) {
    const double nan = std::numeric_limits<double>::quiet_NaN();
    if (!arch_ok(target) || !roofline_ok(rt) || !arch_ok(draft) || !roofline_ok(rd) || !(B > 0.0) ||
        !std::isfinite(B) || k < 1 || !(alpha >= 0.0 && alpha <= 1.0) || !count_ok(n))
        return nan;
    const double E = alpha >= 1.0 ? k + 1.0 : (1.0 - std::pow(alpha, k + 1.0)) / (1.0 - alpha);
    const double t1 = sv_roofline_time(target, rt, B, 1.0, n);
    const double tk = sv_roofline_time(target, rt, B, k + 1.0, n);
    const double d1 = sv_roofline_time(draft, rd, B, 1.0, n);
    return E * t1 / (k * d1 + tk);
}

}  // extern "C"
