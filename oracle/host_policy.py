"""Plain-Python oracle of the host-side components (TEST INFRASTRUCTURE ONLY).

Slow, obviously correct restatements of the rules in ``include/sv_host.h``,
written from the pages with brute-force scans instead of indexes; the C++
implementation (``csrc/sv_host.cpp``) is compared against them in
``tests/test_host_policy.py``.  Nothing on the product path imports this.

Sources (by page title and section):
* "AI 开始抄自己的作业——而且抄得理直气壮", sections "📓 NgramRL：每道题配一本活页草稿本"
  (per-prompt n-gram table, n <= 6, k = 16 drafted tokens, rollouts of the
  last W steps) and "🚰 真正的瓶颈不在算法，在流水线" (fan-out prefetch: causal
  window statistics P(j) and c_j(f), greedy budget of N candidates);
* "distribution-aware speculative decoding" (Together AI blog), sections
  "Adaptive suffix tree drafter" (frequency-scored continuation of the
  longest match, verified tokens inserted at once) and "Length-aware
  scheduling" (Long / Medium / Short budgets, long requests interleaved
  across ranks);
* the EfficientRollout article (qunfachuanzhen.com), sections
  "四、自适应草稿长度" (lengths 5/7/9/11, two-step hysteresis on the block
  efficiency) and "三、聪明的开关" (switch on above a 1.05x predicted speedup,
  then stay on).
"""
from __future__ import annotations

import math


# --------------------------------------------------------------------------
# n-gram drafter

class NgramOracle:
    def __init__(self, max_n=6, window=4):
        self.max_n, self.window = max_n, window
        self.step = -1
        self.rollouts = {}   # prompt -> list of (step, tokens), oldest first

    def begin_step(self):
        self.step += 1
        for pid in list(self.rollouts):
            kept = [(s, t) for s, t in self.rollouts[pid] if s > self.step - self.window]
            if kept:
                self.rollouts[pid] = kept
            else:
                del self.rollouts[pid]

    def add(self, pid, tokens):
        if self.step < 0:
            self.begin_step()
        self.rollouts.setdefault(pid, []).append((self.step, [int(x) for x in tokens]))

    def _occurrences(self, pid, key):
        """Positions p right after an occurrence of key that some token
        follows, newest first (newest rollout, then latest position)."""
        n = len(key)
        for _, r in reversed(self.rollouts.get(pid, [])):
            for p in range(len(r) - 1, n - 1, -1):
                if r[p - n:p] == key:
                    yield r, p

    def _longest(self, pid, ctx):
        ctx = [int(x) for x in ctx]
        for n in range(min(self.max_n, len(ctx)), 0, -1):
            occ = list(self._occurrences(pid, ctx[-n:]))
            if occ:
                return n, occ
        return 0, []

    def draft(self, pid, ctx, k=16):
        n, occ = self._longest(pid, ctx)
        if n == 0 or k == 0:
            return []
        r, p = occ[0]
        return r[p:p + k]

    def candidates(self, pid, ctx, f):
        n, occ = self._longest(pid, ctx)
        if n == 0 or f == 0:
            return []
        count, first = {}, {}
        for order, (r, p) in enumerate(occ):
            t = r[p]
            count[t] = count.get(t, 0) + 1
            first.setdefault(t, order)
        ranked = sorted(count, key=lambda t: (-count[t], first[t]))
        return ranked[:f]


# --------------------------------------------------------------------------
# suffix drafter

class SuffixOracle:
    def __init__(self, max_depth=8):
        self.max_depth = max_depth
        self.seqs = {}   # problem -> {seq_id: tokens}

    def clear(self):
        self.seqs = {}

    def append(self, pid, sid, tokens):
        self.seqs.setdefault(pid, {}).setdefault(sid, []).extend(int(x) for x in tokens)

    def _followers(self, pid, ctx):
        """Counts of the tokens that follow each occurrence of ctx."""
        d = len(ctx)
        cnt = {}
        for s in self.seqs.get(pid, {}).values():
            for p in range(d, len(s)):
                if s[p - d:p] == ctx:
                    cnt[s[p]] = cnt.get(s[p], 0) + 1
        return cnt

    def _longest(self, pid, ctx):
        for d in range(min(self.max_depth, len(ctx)), 0, -1):
            cnt = self._followers(pid, ctx[-d:])
            if cnt:
                return cnt
        return {}

    def draft(self, pid, ctx, k=16):
        ctx = [int(x) for x in ctx]
        out = []
        while len(out) < k:
            cnt = self._longest(pid, ctx)
            if not cnt:
                break
            t = min(cnt, key=lambda x: (-cnt[x], x))
            out.append(t)
            ctx.append(t)
        return out

    def candidates(self, pid, ctx, f):
        cnt = self._longest(pid, [int(x) for x in ctx])
        return sorted(cnt, key=lambda x: (-cnt[x], x))[:f]


# --------------------------------------------------------------------------
# fan-out prefetch budget

def prefetch_estimates(obs, k, fmax, window):
    """P(j) and c_j(f) from the last `window` (j, rank) observations."""
    w = obs[-window:]
    n = len(w)
    P = [0.0] * (k + 1)
    cov = [[0.0] * (fmax + 1) for _ in range(k + 1)]
    if n == 0:
        return n, P, cov
    for j in range(k + 1):
        mine = [r for (jj, r) in w if jj == j]
        P[j] = len(mine) / n
        for f in range(1, fmax + 1):
            if mine:
                cov[j][f] = sum(1 for r in mine if 0 <= r < f) / len(mine)
            else:
                cov[j][f] = sum(1 for (_, r) in w if 0 <= r < f) / n
    return n, P, cov


def prefetch_allocate(obs, k, fmax, window, budget):
    n, P, cov = prefetch_estimates(obs, k, fmax, window)
    f = [0] * (k + 1)
    if n == 0:
        return f, 0.0
    total = 0.0
    for _ in range(budget):
        best, gain = -1, 0.0
        for j in range(k + 1):
            if f[j] >= fmax:
                continue
            g = P[j] * (cov[j][f[j] + 1] - cov[j][f[j]])
            if g > gain:
                best, gain = j, g
        if best < 0:
            break
        f[best] += 1
        total += gain
    return f, total


def expected_coverage(P, cov, f):
    return sum(P[j] * cov[j][f[j]] for j in range(len(f)))


def prefetch_drafts(drafter, pid, ctx, draft, f, k):
    """Fan-out prefetch ("🚰 真正的瓶颈不在算法，在流水线"): for each branch j (j drafts
    accepted) and each of its f[j] best-ranked candidates b for the next
    token, the draft that would follow context + draft[:j] + [b], computed
    before the outcome is known.  Returns {(j, b): draft}."""
    ctx, draft = [int(x) for x in ctx], [int(x) for x in draft]
    out = {}
    for j in range(len(draft) + 1):
        branch = ctx + draft[:j]
        for b in drafter.candidates(pid, branch, f[j]):
            out[(j, int(b))] = [int(x) for x in drafter.draft(pid, branch + [int(b)], k)]
    return out


# --------------------------------------------------------------------------
# draft length, block efficiency, switch, budgets

def draft_length_trajectory(lengths, taus, up=0.7, down=0.4, patience=2):
    """Lengths used at every step (the first is lengths[0]) and the one after
    the last report."""
    idx, up_run, down_run = 0, 0, 0
    used = []
    for tau in taus:
        used.append(lengths[idx])
        r = tau / (lengths[idx] + 1)
        up_run = up_run + 1 if r >= up else 0
        down_run = down_run + 1 if r < down else 0
        if up_run >= patience and idx + 1 < len(lengths):
            idx, up_run, down_run = idx + 1, 0, 0
        elif down_run >= patience and idx > 0:
            idx, up_run, down_run = idx - 1, 0, 0
    return used, lengths[idx]


def block_efficiency(accept_len):
    v = [a + 1 for a in accept_len if a >= 0]
    return sum(v) / len(v) if v else math.nan


def spec_switch(predictions, threshold=1.05):
    on, out = 0, []
    for s in predictions:
        if not on and s > threshold:
            on = 1
        out.append(on)
    return out


def length_classes(pred, budgets=(0, 8, 16)):
    order = sorted(range(len(pred)), key=lambda i: (-pred[i], i))
    third = len(pred) // 3
    cls = [0] * len(pred)
    for r, i in enumerate(order):
        cls[i] = 2 if r < third else (0 if r >= len(pred) - third else 1)
    return cls, [budgets[c] for c in cls]


def interleave_ranks(pred, world):
    order = sorted(range(len(pred)), key=lambda i: (-pred[i], i))
    ranks = [0] * len(pred)
    for r, i in enumerate(order):
        ranks[i] = r % world
    return ranks


# --------------------------------------------------------------------------
# roofline predictor behind the switch (EfficientRollout article, section
# "三、聪明的开关": each step bound by compute or by memory bandwidth,
# calibrated on measured run times; the terms are this oracle's reading)

def roofline_work(a, B, q, n):
    """flops and bytes of one decoder step: every weight used twice per new
    token (multiply and add) and read once; attention scores and values over
    n cached positions (two width x n products per new token per layer); the
    K and V cache read once."""
    flops = 2.0 * a["params"] * B * q + 4.0 * a["layers"] * a["width"] * B * q * n
    nbytes = a["params"] * a["weight_bytes"] + 2.0 * a["layers"] * a["kv_heads"] * a["head_dim"] * a["kv_bytes"] * B * n
    return flops, nbytes


def roofline_time(a, r, B, q, n):
    f, m = roofline_work(a, B, q, n)
    return max(f / r["flops_per_s"], m / r["bytes_per_s"]) + r["overhead_s"]


def accepted_per_cycle(alpha, k):
    """Expected tokens per draft-verify cycle with i.i.d. acceptance alpha:
    the accepted prefix plus the one drawn token, summed term by term."""
    return sum(alpha ** i for i in range(k + 1))


def spec_speedup(target, rt, draft, rd, B, k, alpha, n):
    cycle = k * roofline_time(draft, rd, B, 1, n) + roofline_time(target, rt, B, k + 1, n)
    return accepted_per_cycle(alpha, k) * roofline_time(target, rt, B, 1, n) / cycle


def roofline_fit(a, B, q, n, seconds, starts=12):
    """Least squared relative error over (pi, beta, tau >= 0) by Nelder-Mead
    from many starts in log space, tau by bounded scalar minimisation inside
    (slow, and independent of the C++ grid search)."""
    import numpy as np
    from scipy import optimize
    work = [roofline_work(a, b, qq, nn) for b, qq, nn in zip(B, q, n)]
    t = [float(x) for x in seconds]

    def err(lp, lb, tau):
        pi, beta = 10.0 ** lp, 10.0 ** lb
        return sum(((max(f / pi, m / beta) + tau - ti) / ti) ** 2 for (f, m), ti in zip(work, t))

    def err2(x):
        res = optimize.minimize_scalar(lambda tau: err(x[0], x[1], tau), bounds=(0.0, max(t)), method="bounded",
                                       options={"xatol": 1e-15})
        return min(res.fun, err(x[0], x[1], 0.0))

    fr = max(f / ti for (f, _), ti in zip(work, t))
    mr = max(m / ti for (_, m), ti in zip(work, t))
    rng = np.random.default_rng(0)
    best = None
    for _ in range(starts):
        x0 = [np.log10(fr) + rng.uniform(-1, 3), np.log10(mr) + rng.uniform(-1, 3)]
        r = optimize.minimize(err2, x0, method="Nelder-Mead", options={"xatol": 1e-9, "fatol": 1e-16, "maxiter": 4000})
        if best is None or r.fun < best.fun:
            best = r
    lp, lb = best.x
    res = optimize.minimize_scalar(lambda tau: err(lp, lb, tau), bounds=(0.0, max(t)), method="bounded",
                                   options={"xatol": 1e-15})
    tau = res.x if res.fun < err(lp, lb, 0.0) else 0.0
    return {"flops_per_s": 10.0 ** lp, "bytes_per_s": 10.0 ** lb, "overhead_s": tau}, err(lp, lb, tau)
